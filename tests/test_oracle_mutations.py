"""Plant plausible mistakes in a copy of the oracle's C source, on the CPU,
and check that the pins catch every one of them."""
import os
import subprocess

import pytest

import oracle
from tests import oracle_pins

MUTATIONS = {
    "scale_dropped": ("s *= scale;", "s *= 1.0;"),
    "lse_log2": ("return m + log(l);", "return m + log2(l);"),
    "softmax_not_normalised": ("for (int j = 0; j <= i; ++j) p[j] /= l;", ""),
    "pv_wrong_value_row": ("acc += p[j] * vh[(int64_t)j * D + d];\n                    oh[",
                           "acc += p[j] * vh[(int64_t)i * D + d];\n                    oh["),
    "decode_pv_wrong_value_row": ("acc += p[j] * vh[(int64_t)j * D + d];\n                    o[(bh",
                                  "acc += p[j] * vh[(int64_t)r * D + d];\n                    o[(bh"),
    "dv_transposed_p": ("acc += Z[(int64_t)i * T + j] * gh[(int64_t)i * D + d];",
                        "acc += Z[(int64_t)j * T + i] * gh[(int64_t)i * D + d];"),
    "ds_sign_flipped": ("keep_factor(dr, bh, i, j) * dp - delta)", "delta - keep_factor(dr, bh, i, j) * dp)"),
    "ds_delta_dropped": ("keep_factor(dr, bh, i, j) * dp - delta)", "keep_factor(dr, bh, i, j) * dp)"),
    "dk_uses_k": ("acc += dS[(int64_t)i * T + j] * qh[(int64_t)i * D + d];",
                  "acc += dS[(int64_t)i * T + j] * kh[(int64_t)i * D + d];"),
    "dq_scale_dropped": ("dqh[(int64_t)i * D + d] = scale * acc;", "dqh[(int64_t)i * D + d] = acc;"),
    "dq_transposed_ds": ("acc += dS[(int64_t)i * T + j] * kh[(int64_t)j * D + d];",
                         "acc += dS[(int64_t)j * T + i] * kh[(int64_t)j * D + d];"),
    "nc_keeps_mask": ("return causal ? i : T - 1;", "return i;"),
    "nc_bwd_sums_keep_mask": ("return causal ? j : 0;", "return j;"),
    "nc_misses_last_key": ("return causal ? i : T - 1;", "return causal ? i : T - 2;"),
    "philox_wrong_key_bump": ("k1 += PHILOX_W1;", "k1 += PHILOX_W0;"),
    "philox_swapped_products": ("c1 = lo1;", "c1 = lo0;"),
    "dropout_scale_dropped": ("return 65536.0 / (65536.0 - (double)t);", "return 1.0;"),
    "dropout_threshold_flipped": ("return u >= t;", "return u < t;"),
    "dropout_counter_ignores_head": ("{(uint32_t)i, (uint32_t)j >> 3, (uint32_t)bh, offset}",
                                     "{(uint32_t)i, (uint32_t)j >> 3, 0u, offset}"),
    "dropout_counter_ignores_offset": ("{(uint32_t)i, (uint32_t)j >> 3, (uint32_t)bh, offset}",
                                       "{(uint32_t)i, (uint32_t)j >> 3, (uint32_t)bh, 0u}"),
    "dropout_wrong_half_word": ("(16 * (j & 1))", "(16 * ((j >> 1) & 1))"),
    "dropout_dv_uses_p": ("acc += Z[(int64_t)i * T + j] * gh[(int64_t)i * D + d];",
                          "acc += P[(int64_t)i * T + j] * gh[(int64_t)i * D + d];"),
    "dropout_ds_ignores_mask": ("(keep_factor(dr, bh, i, j) * dp - delta)", "(dp - delta)"),
    "decode_sees_one_key_too_few": ("const int last = Tk - Tq + r;", "const int last = Tk - Tq + r - 1;"),
    "decode_wrong_query_row": ("const double *qr = q + (bh * Tq + r) * (int64_t)D;",
                               "const double *qr = q + (bh * Tq) * (int64_t)D;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(oracle.source_path()).read()
    assert src.count(old) == 1, f"mutation anchor for {name} must be unique"
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / f"libmut_{name}.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(lib),
                           str(path), "-lm"])
    impl = oracle.OracleLib(str(lib))
    caught = None
    for check in oracle_pins.ALL_PINS:
        try:
            check(impl)
        except AssertionError:
            caught = check.__name__
            break
    assert caught, f"no pin caught the planted mistake {name}"
