"""Planted mistakes: each pin of the oracle must fail when the step it guards
is wrong.

Every case below plants one plausible slip in a copy of oracle.c (a wrong tie
rule, a dropped sign or factor, an off-by-one, a transposed operand, the wrong
flag bit, a reading of the method other than the one taken), compiles it into
a temporary library, routes the oracle through it and runs the pin that
guards that step: the pin must fail.  The unmodified oracle passes the same
pins in tests/test_oracle_pins.py.

One slip cannot be planted observably: the ties-to-even rule of the bf16
rounding of the global-scale format's values E2M1 * s_b / G is unreachable.
E2M1 * s_b has at most 6 significant bits, so whenever the exact quotient by G
is a dyadic rational it has at most 6 significant bits too and is exact in
bf16; otherwise it cannot lie on a midpoint.  A different tie rule there gives
the same results on every input."""
import pytest

import oracle
from tests import test_oracle_pins as pins

Q, K, V, ALL = oracle.QUANT_Q, oracle.QUANT_K, oracle.QUANT_V, oracle.QUANT_ALL

# (name, text in oracle.c, replacement, pin, pin arguments)
MUTANTS = [
    ("e4m3 ties away from even",
     "        return k + 1;\n    return (k % 2 == 0) ? k : k + 1;\n}\n\n/* Round |x|/s",
     "        return k + 1;\n    return k + 1;\n}\n\n/* Round |x|/s",
     "test_e4m3_scale_exhaustive_vs_torch_float8", {}),
    ("e4m3 scale from amax/4",
     "while (k < 126 && 6.0 * oracle_e4m3_value(k + 1) <= a)",
     "while (k < 126 && 4.0 * oracle_e4m3_value(k + 1) <= a)",
     "test_e4m3_scale_exhaustive_vs_torch_float8", {}),
    ("e4m3 subnormal exponent",
     "return ldexp((double)mant, -9);", "return ldexp((double)mant, -10);",
     "test_e4m3_value_table_matches_torch", {}),
    ("e4m3 normal exponent",
     "return ldexp((double)(8 + mant), e - 10);", "return ldexp((double)(8 + mant), e - 9);",
     "test_e4m3_value_table_matches_torch", {}),
    ("e4m3 saturates below 448",
     "    if (a >= 6.0 * 448.0)\n        return 126;", "    if (a >= 6.0 * 448.0)\n        return 125;",
     "test_e4m3_scale_exhaustive_vs_torch_float8", {}),
    ("e2m1 ties down",
     "        return k + 1;\n    return (k % 2 == 0) ? k : k + 1;\n}\n\n/* Element-wise",
     "        return k + 1;\n    return k;\n}\n\n/* Element-wise",
     "test_e2m1_exhaustive_all_bf16_times_all_scales", {}),
    ("e2m1 grid value",
     "{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0}", "{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 5.0, 6.0}",
     "test_e2m1_exhaustive_all_bf16_times_all_scales", {}),
    ("fq drops the sign",
     "y[i * ys] = neg ? -mag : mag;", "y[i * ys] = mag;",
     "test_block_quantizer_vs_exact_rationals", {}),
    ("block amax misses the last element",
     "    for (long i = 0; i < n; i++) {\n        double ax = fabs(x[i * xs]);",
     "    for (long i = 0; i < n - 1; i++) {\n        double ax = fabs(x[i * xs]);",
     "test_block_quantizer_vs_exact_rationals", {}),
    ("sign bit from x < 0 (loses the sign of zero)",
     "        int neg = signbit(xi) ? 1 : 0;", "        int neg = (xi < 0) ? 1 : 0;",
     "test_block_quantizer_vs_exact_rationals", {}),
    ("code nibbles swapped",
     "(uint8_t)(cb[i] | (cb[i + 1] << 4));\n            if (deq)\n                for",
     "(uint8_t)(cb[i + 1] | (cb[i] << 4));\n            if (deq)\n                for",
     "test_block_quantizer_vs_exact_rationals", {}),
    ("fq(Q) keyed to the K flag",
     "    if (flags & ORACLE_QUANT_Q)\n        for (long r = 0; r < Lq; r++)",
     "    if (flags & ORACLE_QUANT_K)\n        for (long r = 0; r < Lq; r++)",
     "test_single_quantizer_equals_quantizing_that_operand_first", {"flag": Q}),
    ("fq(V) blocked along channels",
     "        for (long d = 0; d < D; d++)\n            for (long t0 = 0; t0 < Lk; t0 += BLOCK) {\n"
     "                long n = Lk - t0 < BLOCK ? Lk - t0 : BLOCK;\n"
     "                fq_block(Vh + t0 * D + d, n, D, Vh + t0 * D + d, D, NULL, NULL);\n            }",
     "        for (long r = 0; r < Lk; r++)\n            for (long b = 0; b < D / BLOCK; b++)\n"
     "                fq_block(Vh + r * D + b * BLOCK, BLOCK, 1, Vh + r * D + b * BLOCK, 1, NULL, NULL);",
     "test_single_quantizer_equals_quantizing_that_operand_first", {"flag": V}),
    ("row max over the first 16 keys only",
     "        if (selected(flags, sel, T, nkt, i, j) && S[j] > m)",
     "        if (selected(flags, sel, T, nkt, i, j) && S[j] > m && j < 16)",
     "test_unquantized_forward_matches_sdpa_and_softmax", {}),
    ("l summed over fq(P~)",
     "    *m_out = m;\n    *l_out = l;",
     "    l = 0.0;\n    for (long j = 0; j < Lk; j++)\n        l += Phat[j];\n    *m_out = m;\n    *l_out = l;",
     "test_identical_keys_closed_form", {}),
    ("fq(P~) in blocks of 32 keys",
     "        for (long t0 = 0; t0 < Lk; t0 += BLOCK) {\n            long n = Lk - t0 < BLOCK ? Lk - t0 : BLOCK;\n"
     "            fq_block(Pt + t0, n, 1, Phat + t0, 1, NULL, NULL);",
     "        for (long t0 = 0; t0 < Lk; t0 += 32) {\n            long n = Lk - t0 < 32 ? Lk - t0 : 32;\n"
     "            fq_block(Pt + t0, n, 1, Phat + t0, 1, NULL, NULL);",
     "test_ragged_lk_zero_padding_equivalence", {}),
    ("O from the unquantized P~",
     "                    acc[d] += Ph[j] * Vh[j * D + d];", "                    acc[d] += Pt[j] * Vh[j * D + d];",
     "test_identical_keys_closed_form", {}),
    ("O not divided by l",
     "                acc[d] = li > 0.0 ? acc[d] / li : 0.0;", "                acc[d] = li > 0.0 ? acc[d] : 0.0;",
     "test_unquantized_forward_matches_sdpa_and_softmax", {}),
    ("LSE without m",
     "            lse[t] = li > 0.0 ? mi + log(li) : -INFINITY;", "            lse[t] = li > 0.0 ? log(li) : -INFINITY;",
     "test_unquantized_forward_matches_sdpa_and_softmax", {}),
    ("Delta from the wrong row of O",
     "            s += oracle_bf16_value(dO[i * D + d]) * O[i * D + d];",
     "            s += oracle_bf16_value(dO[i * D + d]) * O[d];",
     "test_unquantized_gradients_match_autograd", {}),
    ("dQ without sm_scale",
     "            for (long d = 0; d < D; d++)\n                dQ[t * D + d] *= c;",
     "            for (long d = 0; d < D; d++)\n                dQ[t * D + d] *= 1.0;",
     "test_unquantized_gradients_match_autograd", {}),
    ("dK without sm_scale",
     "            dKt[x] *= c;", "            dKt[x] *= 1.0;",
     "test_unquantized_gradients_match_autograd", {}),
    ("dS with the wrong sign in dQ",
     "                double dS = P * (dP - delta[i]);\n                for (long d = 0; d < D; d++)\n"
     "                    dQ[t * D + d] += dS * Kh[j * D + d];",
     "                double dS = P * (delta[i] - dP);\n                for (long d = 0; d < D; d++)\n"
     "                    dQ[t * D + d] += dS * Kh[j * D + d];",
     "test_unquantized_gradients_match_autograd", {}),
    ("dK from K instead of Q",
     "                    dKt[jj * D + d] += dS * Qh[i * D + d];",
     "                    dKt[jj * D + d] += dS * Kh[(j0 + jj) * D + d];",
     "test_unquantized_gradients_match_autograd", {}),
    ("dP misses the last channel",
     "                double dP = dot(dOi, Vh + (j0 + jj) * D, D);",
     "                double dP = dot(dOi, Vh + (j0 + jj) * D, D - 1);",
     "test_unquantized_gradients_match_autograd", {}),
    ("dV weight not divided by l",
     "                for (long jj = 0; jj < n; jj++)\n                    w[jj] = Ph[jj] / l[i];",
     "                for (long jj = 0; jj < n; jj++)\n                    w[jj] = Ph[jj];",
     "test_quantized_gradients_match_ste_surrogate", {"flags": ALL}),
    ("dV from the unquantized P~",
     "                fq_block(Pt, n, 1, Ph, 1, NULL, NULL);\n                for (long jj = 0; jj < n; jj++)\n"
     "                    w[jj] = Ph[jj] / l[i];",
     "                fq_block(Pt, n, 1, Ph, 1, NULL, NULL);\n                for (long jj = 0; jj < n; jj++)\n"
     "                    w[jj] = Pt[jj] / l[i];",
     "test_quantized_gradients_match_ste_surrogate", {"flags": ALL}),
    ("causal mask off by one",
     "    if ((flags & ORACLE_CAUSAL) && j > i)", "    if ((flags & ORACLE_CAUSAL) && j >= i)",
     "test_causal_quantizers_off_vs_torch_sdpa", {}),
    ("tile mask inverted",
     "    return sel == NULL || sel[(i / T) * nkt + j / T] != 0;",
     "    return sel == NULL || sel[(i / T) * nkt + j / T] == 0;",
     "test_sparse_all_tiles_selected_is_dense", {}),
    ("dQ over unselected keys",
     "                if (!(l[i] > 0.0) || !selected(flags, sel, T, nkt, i, j))\n                    continue;",
     "                if (!(l[i] > 0.0))\n                    continue;",
     "test_sparse_equals_dense_attention_on_the_gathered_tiles", {"flags": ALL}),
    ("selection ties to the higher tile",
     "(best < 0 || sc[j] > sc[best])", "(best < 0 || sc[j] >= sc[best])",
     "test_vsa_select_ties_go_to_the_lower_tile_and_topk_bounds", {}),
    ("ragged tile mean over T rows",
     "            mean[t * D + d] = s / (float)(r1 - r0);", "            mean[t * D + d] = s / (float)T;",
     "test_vsa_select_agrees_with_float64_ranking", {}),
    ("global scale 448 / amax",
     "    volatile float num = 2688.0f;", "    volatile float num = 448.0f;",
     "test_global_scale_format_vs_exact_rationals", {"seed": 1, "mag": 1.0}),
    ("global-scale value not divided by G",
     "bf16_of_quotient(E2M1_GRID[c] * sb, g);", "bf16_of_quotient(E2M1_GRID[c] * sb, 1.0);",
     "test_global_scale_format_vs_exact_rationals", {"seed": 1, "mag": 1.0}),
    ("global amax misses the last column",
     "        for (long j = 0; j < cols; j++) {\n            double a = fabs(oracle_bf16_value(x[r * srow + j * scol]));",
     "        for (long j = 0; j < cols - 1; j++) {\n            double a = fabs(oracle_bf16_value(x[r * srow + j * scol]));",
     "test_global_scale_sees_every_element", {}),
    ("global-scale block scale without G",
     "int k = oracle_e4m3_round_div6(ab * g);", "int k = oracle_e4m3_round_div6(ab);",
     "test_global_scale_format_vs_exact_rationals", {"seed": 1, "mag": 1.0}),
    ("global-scale code without G",
     "oracle_e2m1_round(fabs(xb[i]) * g, sb)", "oracle_e2m1_round(fabs(xb[i]), sb)",
     "test_global_scale_format_vs_exact_rationals", {"seed": 1, "mag": 1.0}),
    ("global scale overflow to 1",
     "    if (isinf(g))\n        g = 3.40282347e38f;", "    if (isinf(g))\n        g = 1.0f;",
     "test_global_scale_special_cases", {}),
    ("global scale of an all-zero tensor 0",
     "    if (!(amax > 0.0))\n        return 1.0f;", "    if (!(amax > 0.0))\n        return 0.0f;",
     "test_global_scale_special_cases", {}),
    ("scores without sm_scale",
     "        S[j] = c * dot(Qi, Kh + j * D, D);", "        S[j] = dot(Qi, Kh + j * D, D);",
     "test_unquantized_forward_matches_sdpa_and_softmax", {}),
    ("dK/dV ignore the mask",
     "                Pt[jj] = selected(flags, sel, T, nkt, i, j0 + jj) ? exp(S[jj] - m[i]) : 0.0;",
     "                Pt[jj] = exp(S[jj] - m[i]);",
     "test_causal_rows_equal_dense_attention_on_their_prefix", {}),
    ("dK/dV keep rows that select no key",
     "            if (!(l[i] > 0.0))\n                continue; /* no selected key: the row adds nothing */",
     "            if (!(l[i] > 0.0) && 0)\n                continue; /* no selected key: the row adds nothing */",
     "test_sparse_equals_dense_attention_on_the_gathered_tiles", {"flags": ALL}),
    ("literal dV reading without the division by l",
     "                    Pn[jj] = Pt[jj] / l[i];", "                    Pn[jj] = Pt[jj];",
     "test_dv_literal_reading_zeroes_normalised_blocks", {}),
    ("sampled forward rows ignored",
     "            long i = rows[t];\n            double mi, li;\n            prob_row(Qh + i * D, i, Kh, Lk, D, c, flags, sel, T, S, Pt, Ph, &mi,\n                     &li);\n            /* O_d",
     "            long i = t;\n            double mi, li;\n            prob_row(Qh + i * D, i, Kh, Lk, D, c, flags, sel, T, S, Pt, Ph, &mi,\n                     &li);\n            /* O_d",
     "test_sampled_rows_equal_full_computation", {}),
    ("sampled key blocks ignored",
     "        long j0 = blocks[t] * BLOCK;", "        long j0 = t * BLOCK;",
     "test_sampled_rows_equal_full_computation", {}),
    ("tile mask indexed with 128-token tiles whatever the tile",
     "    return sel == NULL || sel[(i / T) * nkt + j / T] != 0;",
     "    return sel == NULL || sel[(i / 128) * nkt + j / 128] != 0;",
     "test_sparse_equals_dense_attention_on_the_gathered_tiles", {"flags": ALL}),
]


@pytest.mark.parametrize("name,old,new,pin,kwargs", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_its_pin(tmp_path, name, old, new, pin, kwargs):
    src = open(oracle.SRC).read()
    assert src.count(old) == 1, "the planted text must occur once in oracle.c"
    mutant = tmp_path / "oracle_mutant.c"
    mutant.write_text(src.replace(old, new))
    lib = oracle.compile_library(str(mutant), str(tmp_path / "liboracle_mutant.so"))
    with oracle.library(lib):
        with pytest.raises(AssertionError):
            getattr(pins, pin)(**kwargs)
