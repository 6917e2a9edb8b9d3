"""Planted mistakes: each case rebuilds the oracle from its own source with
one plausible error (a dropped term, a wrong sign, index or threshold, a
swapped operand) and checks that the pin written for that step fails on it.
The mistakes are planted in the CPU oracle only, in a temporary copy of its
source; the committed oracle is untouched."""
import numpy as np
import pytest

import oracle
from oracle import build as oracle_build
import test_oracle_mx_pins as MXP
import test_oracle_pins as P
import test_oracle_vector_scales as VSP
from test_oracle_pins import aten_philox, pr1  # noqa: F401  (fixtures)
from nvfp4_block_quantization_amax_b200 import synthetic

SOURCE = open(oracle_build.SRC).read()


def _ms_eden_inner_product_unbiased(n=300):
    """Light form of the MS-EDEN unbiasedness pin (Quartet II §一): the mean of
    <r, dequant> / ||r||^2 over seeds stays within 5 standard errors of 1 for
    every block whose scale never saturates at 448 (the unbiasing value is
    clipped there, so the identity holds only below it)."""
    import scipy.linalg
    H = scipy.linalg.hadamard(16).astype(np.float64)
    x = synthetic.bf16_bits(synthetic.normal_with_entry_outliers(16, 64, seed=33))
    xb = P.f32(x).astype(np.float64).reshape(-1, 16)
    ratios = []
    saturated = np.zeros(xb.shape[0], bool)
    for seed in range(n):
        out = oracle.quantize(x, oracle.MS_EDEN, oracle.ROWWISE, seed=seed)
        saturated |= out["scales_row"].reshape(-1) == 0x7E
        dq = oracle.dequantize(out["codes_row"], out["scales_row"], out["alpha_row"], 16, 64, 0, seed)
        s = oracle.sign_bits(seed)
        d = np.array([-1.0 if (s >> i) & 1 else 1.0 for i in range(16)])
        r = 0.25 * (xb * d) @ H.T
        ratios.append((r * dq.reshape(-1, 16)).sum(1) / (r ** 2).sum(1))
    ratios = np.array(ratios)
    z = (ratios.mean(0) - 1) / np.maximum(ratios.std(0) / np.sqrt(n), 1e-12)
    assert saturated.sum() <= 2            # only the blocks holding the tensor maximum
    assert np.max(np.abs(z[~saturated])) < 5.0


# (name, text in the oracle source, planted replacement, pin that must fail)
MUTATIONS = [
    ("alpha divisor", "{ return amax / 2688.0f; }", "{ return amax / 2687.0f; }",
     lambda f: P.test_alpha_is_eq1(f("pr1"))),
    ("headroom divisor", "return amax / 1792.0f;", "return amax / 1793.0f;",
     lambda f: P.test_headroom_alpha_keeps_the_four_candidate_in_range()),
    ("Philox rounds", "for (int round = 0; round < 10; ++round)", "for (int round = 0; round < 9; ++round)",
     lambda f: P.test_philox_matches_aten_engine(f("aten_philox"))),
    ("sign vector word", "return w[0] & 0xFFFFu;", "return w[1] & 0xFFFFu;",
     lambda f: P.test_sign_vector_is_first_word_of_tag3(f("aten_philox"))),
    ("E4M3 tie to even", "return (lo & 1) ? hi : lo; /* tie: even mantissa */", "return hi;",
     lambda f: P.test_e4m3_rne_matches_library_casts()),
    ("E4M3 ceil of an exact value", "  if (oracle_e4m3_value(lo) == v) return lo;\n  return (uint8_t)(lo + 1);",
     "  return (uint8_t)(lo + 1);", lambda f: P.test_e4m3_ceil_is_smallest_value_not_below()),
    ("E4M3 SR threshold", "((float)u24 < f * 16777216.0f)", "((float)u24 <= f * 16777216.0f)",
     lambda f: P.test_e4m3_sr_threshold_and_expectation()),
    ("E2M1 grid value", "{0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f}",
     "{0.0f, 0.5f, 1.0f, 1.25f, 2.0f, 3.0f, 4.0f, 6.0f}", lambda f: P.test_e2m1_decode_matches_ml_dtypes()),
    ("E2M1 tie to even", "(i & 1) == 0 && (best & 1) == 1", "(i & 1) == 1 && (best & 1) == 0",
     lambda f: P.test_e2m1_rne_all_bf16_in_range_eq3_and_ml_dtypes()),
    ("E2M1 SR threshold", "int up = (float)u16 < f * 65536.0f;", "int up = (float)u16 <= f * 65536.0f;",
     lambda f: P.test_e2m1_sr_threshold()),
    ("hardware SR threshold", "* 65536.0 >= (65536.0 - (double)r16) * gap;",
     "* 65536.0 > (65536.0 - (double)r16) * gap;", lambda f: P.test_e2m1_sr_hw_threshold_and_expectation()),
    ("rotation butterfly sign", "        v[i + h] = a - b;\n      }\n  for (int i = 0; i < 16; ++i) r[i]",
     "        v[i + h] = b - a;\n      }\n  for (int i = 0; i < 16; ++i) r[i]",
     lambda f: P.test_rht_exact_on_integers()),
    ("4/6 tie rule", "*out = (err4 < err6) ? b4 : b6;", "*out = (err4 <= err6) ? b4 : b6;",
     lambda f: P.test_four_six_exact_tie_keeps_six()),
    ("4/6 error in the scaled domain", "float xhat = oracle_e2m1_value(b->code[i]) * s;",
     "float xhat = oracle_e2m1_value(b->code[i]);",
     lambda f: P.test_four_six_keeps_the_lower_error_candidate(f("pr1"))),
    ("MS-EDEN drops alpha", "float den = alpha * sum16(rq);", "float den = sum16(rq);",
     lambda f: _ms_eden_inner_product_unbiased()),
    ("row nibble order", "(uint8_t)(q.code[2 * j] | (q.code[2 * j + 1] << 4));",
     "(uint8_t)(q.code[2 * j + 1] | (q.code[2 * j] << 4));",
     lambda f: P.test_rtn_rows_match_library_encoders(f("pr1"))),
    ("2D column packing", "(uint8_t)(cand_code[pick][i][j] | (cand_code[pick][i + 1][j] << 4));",
     "(uint8_t)(cand_code[pick][i][j] | (cand_code[pick][i][j + 1] << 4));",
     lambda f: P.test_2d_blocks_consistent_across_orientations(f("pr1"))),
    ("dequant drops alpha", "        v[k] = oracle_e2m1_value(q) * s;\n      }\n      if (flags & OR_INVERSE_RHT) {\n"
     "        float t[16];\n        oracle_irht16(v, signs, t);\n        memcpy(v, t, sizeof t);\n      }\n"
     "      for (int k = 0; k < 16; ++k) y[r * C + 16 * b + k] = v[k];\n    }\n  return OR_OK;\n}\n\n/* GEMM",
     "        v[k] = oracle_e2m1_value(q) * oracle_e4m3_value(sb);\n      }\n      if (flags & OR_INVERSE_RHT) {\n"
     "        float t[16];\n        oracle_irht16(v, signs, t);\n        memcpy(v, t, sizeof t);\n      }\n"
     "      for (int k = 0; k < 16; ++k) y[r * C + 16 * b + k] = v[k];\n    }\n  return OR_OK;\n}\n\n/* GEMM",
     lambda f: P.test_dequant_matches_library_decode(f("pr1"))),
    ("GEMM drops a tensor scale", "D[i * ncols + j] = acc * (double)alphaA * (double)alphaB;",
     "D[i * ncols + j] = acc * (double)alphaA;", lambda f: P.test_gemm_f64_matches_numpy_matmul()),
    ("vector scales from one vector's amax",
     "float a = (flags & OR_HEADROOM) ? oracle_alpha_headroom(av[i]) : oracle_alpha_from_amax(av[i]);",
     "float a = (flags & OR_HEADROOM) ? oracle_alpha_headroom(av[0]) : oracle_alpha_from_amax(av[0]);",
     lambda f: VSP.test_vector_alpha_is_eq1_per_vector(VSP.x.__wrapped__(), False)),
    ("vector-scaled GEMM column scale", "D[i * ncols + j] *= (double)alphaA[m] * (double)alphaB[n];",
     "D[i * ncols + j] *= (double)alphaA[m] * (double)alphaA[n];",
     lambda f: VSP.test_gemm_f64_vector_scales_matches_numpy()),
    ("MX shared exponent", "int e = (k - 1) - 2;", "int e = (k - 1) - 1;",
     lambda f: MXP.test_shared_exponent_puts_block_max_in_4_to_8()),
    ("MX nibble order", "(uint8_t)(q[2 * k] | (q[2 * k + 1] << 4));", "(uint8_t)(q[2 * k + 1] | (q[2 * k] << 4));",
     lambda f: MXP.test_codes_and_scales_match_library_casts((64, 128))),
    ("MX GEMM scale index", "oracle_e8m0_value(sB[n * (K / 32) + k / 32]);",
     "oracle_e8m0_value(sB[n * (K / 32) + k / 64]);",
     lambda f: MXP.test_mx_gemm_matches_numpy_on_library_decoded_operands()),
]


@pytest.mark.parametrize("name,old,new,pin", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_fails_its_pin(name, old, new, pin, tmp_path, request):
    assert SOURCE.count(old) == 1, f"mutation site for '{name}' not unique in the oracle source"
    path = oracle_build.build_variant(SOURCE.replace(old, new), str(tmp_path))
    with oracle.use_library(path):
        with pytest.raises((AssertionError, oracle.OracleError)):
            pin(request.getfixturevalue)


def test_unmodified_source_passes_the_same_pins(tmp_path, request):
    """The same harness on an unmodified copy: every pin above passes, so a
    failure under a mutation comes from the planted mistake."""
    path = oracle_build.build_variant(SOURCE, str(tmp_path))
    with oracle.use_library(path):
        for _, _, _, pin in MUTATIONS:
            pin(request.getfixturevalue)
