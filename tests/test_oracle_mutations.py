"""The oracle's pins must catch plausible mistakes.

Each case copies fo_oracle.c, plants one mistake (a dropped term, a wrong
sign, a wrong constant, a swapped operand, a wrong rounding direction),
builds the copy on the CPU and runs one pin test against it: the pin must
fail.  The oracle itself is never modified.
"""
import ctypes
import os

import pytest

import oracle
from oracle.build import SRC, build

import test_oracle_ecc as T_ecc
import test_oracle_nonfinite as T_nf
import test_oracle_states as T_st
import test_oracle_update as T_up

MUTATIONS = [
    ("drop AdamW bias correction", "s.step = (float)(lr / bc1);", "s.step = (float)(lr);",
     lambda o: T_up.test_adamw_step1_matches_torch(o)),
    ("drop second-moment bias correction", "s.ibc2 = (float)(1.0 / sqrt(bc2));", "s.ibc2 = 1.0f;",
     lambda o: T_up.test_adamw_step1_matches_torch(o)),
    ("momentum update reads v", "float vn = fmaf(s->b2, v, s->omb2 * (gr * gr));",
     "float vn = fmaf(s->b2, m, s->omb2 * (gr * gr));",
     lambda o: T_up.test_adamw_ten_steps_track_torch(o)),
    ("ECC ignores the sign of x'", "double e = iv.s * ((double)x - xp);", "double e = ((double)x - xp);",
     lambda o: T_ecc.test_bf16_encode_matches_integer_closed_form(o, 8)),
    ("inward spacing not halved at powers of two",
     "iv.u_in = (pow2 && E > f.emin) ? iv.u_out / 2 : iv.u_out;", "iv.u_in = iv.u_out;",
     lambda o: T_ecc.test_bf16_encode_matches_integer_closed_form(o, 16)),
    ("ECC rounds by truncation", "double r = nearbyint(t);", "double r = trunc(t);",
     lambda o: T_ecc.test_fp16_code_is_nearest_and_rounds_back(o, 8)),
    ("softsign without the factor 2", "float num = 2.0f * y;", "float num = y;",
     lambda o: T_st.test_momentum_compander_is_scaled_softsign(o)),
    ("scale rounded to nearest", "double k = ceil(a / ulp);", "double k = nearbyint(a / ulp);",
     lambda o: T_st.test_scale_is_fp16_round_up(o)),
    ("variance code without the sqrt domain", "        float t = sv[i] * k;",
     "        float t = sv[i] * sv[i] * k;",
     lambda o: T_st.test_variance_compander_is_sqrt(o)),
    ("inf kept in the group maximum", "        if (finite_f(z[i])) A = fmaxf(A, fabsf(z[i]));",
     "        if (!isnan(z[i])) A = fmaxf(A, fabsf(z[i]));",
     lambda o: T_nf.test_nonfinite_state_values_stay_out_of_the_scale(o, 0)),
    ("NaN downcast keeps its sign", "    if (isnan(x)) return fmt_qnan_bits(f);",
     "    if (isnan(x)) return (uint16_t)(sign | fmt_qnan_bits(f));",
     lambda o: T_nf.test_adamw_nonfinite_gradient_poisons_only_its_element(o, 0, 0, 8)),
    ("SGD weight decay with the wrong sign", "float g1 = fmaf(J->wd, x, gr);", "float g1 = fmaf(-J->wd, x, gr);",
     lambda o: T_up.test_sgdm_matches_torch(o, 0.0, False)),
]


@pytest.mark.parametrize("name,old,new,pin", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pin_catches_mutation(tmp_path, name, old, new, pin):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {old!r}"
    mpath = os.path.join(tmp_path, "mutant.c")
    with open(mpath, "w") as f:
        f.write(src.replace(old, new))
    so = build(force=True, src=mpath, out=os.path.join(tmp_path, "libmutant.so"))
    saved = oracle._lib
    oracle._lib = oracle.bind(ctypes.CDLL(so))
    try:
        with pytest.raises(AssertionError):
            pin(oracle)
    finally:
        oracle._lib = saved
