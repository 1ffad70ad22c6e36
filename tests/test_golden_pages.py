"""Checks of the numbers printed on the pages (tests/golden/pages_numbers.txt)
against the storage layout this library uses."""
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    out = {}
    with open(os.path.join(HERE, "golden", "pages_numbers.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = line.split()
                out[k] = float(v)
    return out


def test_baseline_accounting_adds_up():
    g = _golden()
    assert g["master_bytes_baseline"] + g["grad_bytes_baseline"] + g["adam_state_bytes_baseline"] \
        == g["adamw_bytes_per_param_baseline"]
    # an 8.03e9-parameter Llama-3.1-8B list at 16 bytes/param
    from workloads import workload
    n = workload("llama3.1-8b").numel
    assert abs(n * g["adamw_bytes_per_param_baseline"] / 1e9 - g["llama3_8b_gb_at_16_bytes"]) < 1.0


def test_layout_bytes_per_param_is_seven_plus_scales(orc):
    """bf16 theta' (2) + 8-bit rho (1) + bf16 grad (2) + int8 m (1) + uint8 v (1)
    = 7 bytes; the two fp16 scales per 32 elements add 0.125."""
    g = _golden()
    n = 32 * 1000
    x = np.zeros(n, np.float32)
    w, e = orc.encode_master(x, 0, 8)
    st = orc.State.zeros_like_master(w, e, adam=True)
    grad = np.zeros(n, np.uint16)
    per = (st.w.nbytes + st.ecc.nbytes + grad.nbytes + st.mq.nbytes + st.vq.nbytes) / n
    scales = (st.ms.nbytes + st.vs.nbytes) / n
    assert per == g["adamw_bytes_per_param_flashoptim"]
    assert scales == 2 * (g["scale_bits"] / 8) / g["group_size"]
    assert (st.w.itemsize + st.ecc.itemsize) * 8 == g["effective_master_bits"]
    assert st.w.itemsize * 8 == g["base_weight_bits"] == g["downcast_bits_24bit_master"]
    assert st.ecc.itemsize * 8 == g["correction_bits"] == g["master_bits"] - 24
    assert st.mq.itemsize * 8 == st.vq.itemsize * 8 == g["state_bits"]
    assert 2 ** (st.mq.itemsize * 8) == g["state_bins"]
