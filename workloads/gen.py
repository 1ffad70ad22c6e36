"""Counter-based random values, host side (numpy).

Definition (shared with ``csrc/gen.cu``; both implement it independently):

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014; constants of Vigna's reference version):
  ``mix(z)``: z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
  z *= 0x94D049BB133111EB; z ^= z >> 31 (all mod 2^64).
  ``word(key, c) = mix(key + (c + 1) * GAMMA)`` with GAMMA = 0x9E3779B97F4A7C15,
  i.e. output number c of the SplitMix64 stream seeded with ``key``.
* stream keys: ``key = mix((seed+1)*G); key = mix(key ^ (tensor+1)*G);
  key = mix(key ^ (step+1)*G); key = mix(key ^ (kind+1)*G)``.
* unit normal number j of element i (J normals per element): Irwin-Hall sum
  of the eight 16-bit fields of words 2(J*i+j) and 2(J*i+j)+1; the integer
  ``2*S - 8*65535`` (odd, |.| < 2^20, exact in binary32) is multiplied in
  binary32 by a binary32 constant ``c``; ``c = f32(sigma / SD)`` with
  ``SD = sqrt(8 * (2^32 - 1) / 3)``, the standard deviation of that integer.
  Support is +-4.9 sigma.
* Student-t with 3 degrees of freedom: ``z0 / sqrt((z1*z1 + z2*z2 + z3*z3)/3)``
  from four unit normals, left to right in binary32, then times ``scale``.
* outliers: element i is multiplied by 100 when ``word(key_o, i) % 100 == 0``,
  ``key_o`` the stream of kind OUTLIER.

Everything after the integer sum is one correctly rounded binary32
operation at a time (numpy float32 ufuncs), so the device generator gives
identical bits.
"""
from __future__ import annotations

import math

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB
MASK = (1 << 64) - 1

SD_IH8 = math.sqrt(8.0 * (2.0 ** 32 - 1.0) / 3.0)

# stream kinds
KIND_MASTER = 1
KIND_GRAD = 2
KIND_OUTLIER = 3
KIND_STATE = 4


def _mix_int(z: int) -> int:
    z &= MASK
    z = ((z ^ (z >> 30)) * M1) & MASK
    z = ((z ^ (z >> 27)) * M2) & MASK
    return z ^ (z >> 31)


def stream_key(seed: int, tensor: int, step: int, kind: int) -> int:
    seed, tensor, step, kind = int(seed), int(tensor), int(step), int(kind)
    k = _mix_int((seed + 1) * GAMMA)
    k = _mix_int(k ^ (((tensor + 1) * GAMMA) & MASK))
    k = _mix_int(k ^ (((step + 1) * GAMMA) & MASK))
    k = _mix_int(k ^ (((kind + 1) * GAMMA) & MASK))
    return k


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(M1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(M2)
    return z ^ (z >> np.uint64(31))


def words(key: int, counters: np.ndarray) -> np.ndarray:
    c = np.asarray(counters, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(np.uint64(key) + (c + np.uint64(1)) * np.uint64(GAMMA))


def _ih8_int(key: int, idx: np.ndarray, j: int, J: int) -> np.ndarray:
    base = (idx.astype(np.uint64) * np.uint64(J) + np.uint64(j)) * np.uint64(2)
    s = np.zeros(idx.shape, np.int64)
    for off in (0, 1):
        w = words(key, base + np.uint64(off))
        for sh in (0, 16, 32, 48):
            s += ((w >> np.uint64(sh)) & np.uint64(0xFFFF)).astype(np.int64)
    return (2 * s - 8 * 65535).astype(np.int32)


def normal_scale(sigma: float) -> np.float32:
    """binary32 multiplier that turns the Irwin-Hall integer into N(0, sigma)."""
    return np.float32(sigma / SD_IH8)


def normal(key: int, idx: np.ndarray, sigma: float, j: int = 0, J: int = 1) -> np.ndarray:
    zi = _ih8_int(key, np.asarray(idx), j, J)
    return zi.astype(np.float32) * normal_scale(sigma)


def student_t3(key: int, idx: np.ndarray, scale: float) -> np.ndarray:
    idx = np.asarray(idx)
    one = 1.0
    z0 = normal(key, idx, one, 0, 4)
    z1 = normal(key, idx, one, 1, 4)
    z2 = normal(key, idx, one, 2, 4)
    z3 = normal(key, idx, one, 3, 4)
    s = z1 * z1
    s = s + z2 * z2
    s = s + z3 * z3
    s = s / np.float32(3.0)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = z0 / np.sqrt(s)
    return t * np.float32(scale)


def outlier_mask(key_o: int, idx: np.ndarray) -> np.ndarray:
    return (words(key_o, np.asarray(idx)) % np.uint64(100)) == np.uint64(0)


def to_16bit(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round-to-nearest-even cast of float32 values to bf16/fp16 bit patterns
    (library casts: torch for bf16, numpy for fp16)."""
    if dtype == "fp16":
        return np.asarray(x, np.float32).astype(np.float16).view(np.uint16)
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)
