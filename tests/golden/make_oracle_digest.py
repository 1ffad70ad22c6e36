"""Write tests/golden/oracle_digest.txt: SHA-256 digests of the oracle's
output bytes for a small fixed workload (the flat-group recipe at 4096+13
parameters, 10 AdamW steps; and 3 SGD-momentum steps with fp16 masters).

Run from the repository root:  python tests/golden/make_oracle_digest.py
It calls only the oracle and the input generator.  A change of these
digests means the oracle's arithmetic changed; the commit that updates the
file must say which passage of the pages (or which reading of it) justifies
the change.
"""
import hashlib
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from workloads import gen  # noqa: E402

N = 4096 + 13
OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_digest.txt")


def digest(st):
    h = hashlib.sha256()
    for a in (st.w, st.ecc, st.mq, st.ms, st.vq, st.vs):
        if a is not None:
            h.update(a.tobytes())
    return h.hexdigest()


def lines():
    idx = np.arange(N)
    x = gen.normal(gen.stream_key(0, 0, 0, gen.KIND_MASTER), idx, 0.02)
    w, e = oracle.encode_master(x, 0, 8)
    st = oracle.State.zeros_like_master(w, e, adam=True)
    out = [f"adamw_bf16_ecc8 step 0 {digest(st)}"]
    for t in range(1, 11):
        g = gen.to_16bit(gen.normal(gen.stream_key(0, 0, t, gen.KIND_GRAD), idx, 1e-3), "bf16")
        oracle.adamw_step(st, g, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, step=t)
        out.append(f"adamw_bf16_ecc8 step {t} {digest(st)}")
    w, e = oracle.encode_master(x, 1, 8)
    st = oracle.State.zeros_like_master(w, e, adam=False)
    for t in range(1, 4):
        g = gen.to_16bit(gen.normal(gen.stream_key(0, 0, t, gen.KIND_GRAD), idx, 1e-2), "fp16")
        oracle.sgdm_step(st, g, lr=0.1, momentum=0.9, weight_decay=1e-4, step=t, wdt=1, gdt=1)
        out.append(f"sgdm_fp16_ecc8 step {t} {digest(st)}")
    w, e = oracle.encode_master(x, 0, 16)
    st = oracle.State.zeros_like_master(w, e, adam=True)
    for t in range(1, 4):
        g = gen.to_16bit(gen.normal(gen.stream_key(0, 0, t, gen.KIND_GRAD), idx, 1e-3), "bf16")
        oracle.adamw_step(st, g, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01,
                          step=t, ecc_bits=16)
        out.append(f"adamw_bf16_ecc16 step {t} {digest(st)}")
    return out


if __name__ == "__main__":
    with open(OUT, "w") as f:
        f.write("# written by tests/golden/make_oracle_digest.py (oracle only)\n")
        for l in lines():
            f.write(l + "\n")
    print(open(OUT).read())
