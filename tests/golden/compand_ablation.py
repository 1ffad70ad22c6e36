"""Synthetic ablation of the 8-bit state codecs: companded (the method's
softsign-like momentum and square-root variance codes) against plain linear
8-bit codes with the same group of 32 and the same kind of per-group scale,
on heavy-tailed gradients (Student-t with 3 degrees of freedom, scaled by
1e-4, as in the Llama-3.1-8B workload).  No training run: it measures the
quantisation error of the states and of the AdamW update direction they give.

"FlashOptim: Breaking the Memory Wall with 24-bit Weights and Companded
States", section "2. Companded Quantization": linear 8-bit quantisation of the
optimizer states loses the small entries (the variance in particular), which
the companding functions are there to keep; Davis Blalock's release thread
reports the resulting divergence of a linear-8-bit GPT-2 run.

Run as a script to rewrite compand_ablation.txt; the test imports study().
Only the oracle (test infrastructure) and numpy are used.
"""
from __future__ import annotations

import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402

B1, B2, EPS = 0.9, 0.999, 1e-8
M, V = 0, 1


def _fp16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def _group_scale(a):
    """fp16 scale rounded up per group of 32 (the method's scale rule)."""
    g = np.abs(a).reshape(-1, 32).max(axis=1).astype(np.float32)
    return np.repeat(_fp16(oracle.scale_fp16(g)), 32)


def compand_m(m):
    q, s = oracle.quantize_state(m.astype(np.float32), M)
    return oracle.dequantize_state(q, s, M).astype(np.float64)


def compand_v(v):
    q, s = oracle.quantize_state(np.sqrt(v).astype(np.float32), V)
    return oracle.dequantize_state(q, s, V).astype(np.float64)


def linear_m(m):
    S = _group_scale(m)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(S > 0, np.clip(np.rint(m / S * 127), -127, 127), 0)
    return q * S / 127


def linear_v(v, f32_scale=False):
    if f32_scale:
        S = np.repeat(v.reshape(-1, 32).max(axis=1), 32)
    else:
        S = _group_scale(v)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(S > 0, np.clip(np.rint(v / S * 255), 0, 255), 0)
    return q * S / 255


def study(n_groups=8192, steps=20, seed=0):
    """Moments after `steps` AdamW updates on fresh Student-t(3) x 1e-4
    gradients, kept exactly (f64) and through each codec (stored quantised
    after every step, as the fused step does)."""
    rng = np.random.default_rng(seed)
    n = 32 * n_groups
    m = np.zeros(n)
    v = np.zeros(n)
    cm = np.zeros(n)
    cv = np.zeros(n)
    lm = np.zeros(n)
    lv16 = np.zeros(n)
    lv32 = np.zeros(n)
    for _ in range(steps):
        g = rng.standard_t(3, n) * 1e-4
        m = B1 * m + (1 - B1) * g
        v = B2 * v + (1 - B2) * g * g
        cm = compand_m(B1 * cm + (1 - B1) * g)
        cv = compand_v(B2 * cv + (1 - B2) * g * g)
        lm = linear_m(B1 * lm + (1 - B1) * g)
        lv16 = linear_v(B2 * lv16 + (1 - B2) * g * g)
        lv32 = linear_v(B2 * lv32 + (1 - B2) * g * g, f32_scale=True)
    bc1, bc2 = 1 - B1 ** steps, 1 - B2 ** steps

    def upd(mm, vv):
        return (mm / bc1) / (np.sqrt(vv / bc2) + EPS)

    u = upd(m, v)
    rms_u = float(np.sqrt(np.mean(u * u)))
    small_m = np.abs(m) < np.median(np.abs(m))
    small_v = v < np.median(v)
    rows = {}
    for name, mm, vv in (("companded m, companded v", cm, cv),
                         ("linear m, linear v (fp16 scale)", lm, lv16),
                         ("linear m, linear v (f32 scale)", lm, lv32)):
        du = np.abs(upd(mm, vv) - u) / rms_u
        rows[name] = dict(
            m_err_small=float(np.mean(np.abs(mm - m)[small_m]) / np.mean(np.abs(m)[small_m])),
            m_zero=float(np.mean((mm == 0) & (m != 0))),
            v_err_small=float(np.mean(np.abs(vv - v)[small_v]) / np.mean(v[small_v])),
            v_zero=float(np.mean((vv == 0) & (v != 0))),
            upd_med=float(np.median(du)),
            upd_p99=float(np.quantile(du, 0.99)),
            upd_max=float(du.max()),
            upd_gt_rms=float(np.mean(du > 1.0)),
        )
    return rows


def report(rows) -> str:
    cols = ("m_err_small", "m_zero", "v_err_small", "v_zero", "upd_med", "upd_p99", "upd_max", "upd_gt_rms")
    lines = ["# Synthetic compand ablation (tests/golden/compand_ablation.py): 8192 groups of 32,",
             "# 20 AdamW moment updates on Student-t(3) x 1e-4 gradients, states stored through",
             "# each codec after every update; errors against the exact f64 moments.",
             "# m_err_small / v_err_small: mean |error| / mean |value| over the smaller half;",
             "# m_zero / v_zero: fraction of nonzero entries stored as 0; upd_*: error of the",
             "# update direction m/(sqrt(v)+eps) (bias-corrected, eps 1e-8) in units of its RMS:",
             "# median, 99th percentile, max, and the fraction of entries whose error exceeds the RMS.",
             "codec\t" + "\t".join(cols)]
    for name, r in rows.items():
        lines.append(name + "\t" + "\t".join(f"{r[c]:.4g}" for c in cols))
    return "\n".join(lines) + "\n"


if __name__ == "__main__":
    out = os.path.join(HERE, "compand_ablation.txt")
    with open(out, "w") as f:
        f.write(report(study()))
    print(open(out).read())
