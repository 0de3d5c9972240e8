"""Plant a plausible mistake in a copy of the oracle (on the CPU) and check
that at least one pin catches it: the pins must be able to tell a wrong
oracle from a right one, or they pin nothing."""

import os

import pytest

import oracle
import oracle_pins

# (name, text in oracle.c, replacement): a dropped term, a wrong sign, a wrong
# index, a transposed operand, a wrong head mapping, a missing rescale ...
MUTANTS = [
    ("lse_drops_log_l", "lseh[i] = m + log(l);", "lseh[i] = m;"),
    ("causal_mask_off_by_one", "(P->causal && j > i)", "(P->causal && j >= i)"),
    ("softmax_max_not_subtracted", "s[j] = exp(s[j] - m) / l;", "s[j] = exp(s[j]) / l;"),
    ("dS_wrong_sign", "Pm[i * N + j] * (dP[i * N + j] - D)", "Pm[i * N + j] * (D - dP[i * N + j])"),
    ("dP_transposed", "dP[i * N + j] = dot(doh + i * d, vh + j * d, d);",
     "dP[i * N + j] = dot(doh + j * d, vh + i * d, d);"),
    ("dQ_missing_scale", "dqi[c] += P->scale * ds * kj[c];", "dqi[c] += ds * kj[c];"),
    ("gqa_interleaved_heads", "g = h / group;", "g = h % P->Hkv;"),
    ("D_without_P", "D += Pm[i * N + j] * dP[i * N + j];", "D += dP[i * N + j];"),
    ("dV_from_dS", "dvj[c] += p * doi[c];", "dvj[c] += ds * doi[c];"),
    ("dK_from_k", "dkj[c] += P->scale * ds * qi[c];", "dkj[c] += P->scale * ds * kj[c];"),
    ("online_no_rescale", "acc[c] *= corr;", "acc[c] *= 1.0;"),
    ("rows_D_from_wrong_row", "dp[j] = dot(doi, vh + j * d, d);", "dp[j] = dot(qi, vh + j * d, d);"),
    ("cols_missing_group_sum", "for (i64 t = 0; t < C->group; ++t) {", "for (i64 t = 0; t < 1; ++t) {"),
    ("window_edge_off_by_one", "j <= i - P->window", "j < i - P->window"),
    ("philox_wrong_multiplier", "M1 = 0xCD9E8D57u", "M1 = 0xCD9E8D59u"),
    ("decode_sees_one_key_too_few", "const i64 n_vis = L - D->Nq + t + 1;", "const i64 n_vis = L - D->Nq + t;"),
    ("decode_slot_from_wrong_head", "((page * D->Hkv + g) * D->P + slot) * d;\n        s[kk]", "((page * D->Hkv + 0) * D->P + slot) * d;\n        s[kk]"),
    ("dropout_no_rescale", "256.0 / (256.0 - P->drop_t) : 0.0", "1.0 : 0.0"),
    ("dropout_word_byte_swapped", "(x[i & 3] >> (8 * (j & 3)))", "(x[j & 3] >> (8 * (i & 3)))"),
    ("dropout_dV_undropped_in_columns", "dvj[c] += p * f * doh[i * d + c];", "dvj[c] += p * doh[i * d + c];"),
    ("window_ignored_in_columns", "            if (hidden(P, S->h, i, j)) continue;", "            if (P->causal && j > i) continue;"),
    ("e4m3_exponent_bias_8", "ldexp(1.0 + (double)f / 8.0, e - 7)", "ldexp(1.0 + (double)f / 8.0, e - 8)"),
    ("e4m3_subnormal_as_normal", "mag = ldexp((double)f / 8.0, -6);", "mag = ldexp(1.0 + (double)f / 8.0, -6);"),
    ("e4m3_no_nan_code", "if (e == 15 && f == 7)\n        return NAN;", "if (0)\n        return NAN;"),
    ("e4m3_sign_dropped", "return sign ? -mag : mag;", "return mag;"),
    # block masks (every planted index stays inside the mask array)
    ("block_mask_of_head_0_for_all", "!P->bmask[h * P->bm_hstride +", "!P->bmask[0 * P->bm_hstride +"),
    ("block_mask_ignored_in_columns", "            if (hidden(P, S->h, i, j)) continue;",
     "            if ((P->causal && j > i) || (P->window > 0 && j <= i - P->window)) continue;"),
    ("empty_row_not_zeroed", "    if (m == -INFINITY) {\n        for (i64 j = 0; j < N; ++j) s[j] = 0.0;",
     "    if (0) {\n        for (i64 j = 0; j < N; ++j) s[j] = 0.0;"),
    ("online_empty_row_divides_by_zero", "if (l == 0.0) { /* no visible key", "if (0) { /* no visible key"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new):
    src = open(oracle.SOURCE).read()
    assert old in src, f"mutation site for {name} not found in oracle.c"
    mutant_src = tmp_path / "oracle_mutant.c"
    mutant_src.write_text(src.replace(old, new))
    lib = oracle.build(force=True, src=str(mutant_src), out=str(tmp_path / f"lib_{name}.so"))
    orc = oracle.Oracle(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError, FloatingPointError) as e:
            caught.append((pin.__name__, str(e)[:80]))
            break
    assert caught, f"no pin caught the planted mistake {name}"


# Mistakes in the numpy-side wiring of the FP8 forward (the per-tensor
# factors), planted in a subclass of the oracle.
def _dequant_q_v_swapped(self, q8, k8, v8, descale):
    dq, dk, dv = (float(x) for x in descale)
    return self.e4m3_decode(q8) * dv, self.e4m3_decode(k8) * dk, self.e4m3_decode(v8) * dq


def _dequant_no_value_factor(self, q8, k8, v8, descale):
    dq, dk, dv = (float(x) for x in descale)
    return self.e4m3_decode(q8) * dq, self.e4m3_decode(k8) * dk, self.e4m3_decode(v8)


def _dequant_key_factor_twice(self, q8, k8, v8, descale):
    dq, dk, dv = (float(x) for x in descale)
    return self.e4m3_decode(q8) * dk, self.e4m3_decode(k8) * dk, self.e4m3_decode(v8) * dv


PY_MUTANTS = [("fp8_q_v_factors_swapped", _dequant_q_v_swapped),
              ("fp8_value_factor_dropped", _dequant_no_value_factor),
              ("fp8_key_factor_for_queries", _dequant_key_factor_twice)]


@pytest.mark.parametrize("name,dequant", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_pins_catch_planted_fp8_wiring_mistake(name, dequant):
    mutant = type("MutantOracle", (oracle.Oracle,), {"_dequant": dequant})(oracle.build())
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError, FloatingPointError) as e:
            caught.append((pin.__name__, str(e)[:80]))
            break
    assert caught, f"no pin caught the planted mistake {name}"
