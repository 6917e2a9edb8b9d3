"""Pins of the oracle's MXFP4 path (32-element blocks, power-of-two UE8M0
scales, E2M1 values; NVFP4 write-up §一 and §五, AMD MI355X write-up 01-02
for the fixed rotation) against library types, closed forms and brute force.
CPU only."""
import ml_dtypes
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from nvfp4_block_quantization_amax_b200 import synthetic

ROW, COL, RHT, INV = oracle.ROWWISE, oracle.COLWISE, oracle.RHT, oracle.INVERSE_RHT
H16 = scipy.linalg.hadamard(16).astype(np.float64)


def f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def nibbles(codes):
    """[n, m/2] packed bytes -> [n, m] codes, element 2j in the low nibble."""
    c = np.asarray(codes, np.uint8)
    out = np.empty(c.shape[:-1] + (2 * c.shape[-1],), np.uint8)
    out[..., 0::2] = c & 0xF
    out[..., 1::2] = c >> 4
    return out


def e2m1_lib_value(codes):
    return np.asarray(codes, np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float32)


def e8m0_lib_value(b):
    return np.asarray(b, np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)


def test_e8m0_decode_matches_library_types():
    b = np.arange(256, dtype=np.uint8)
    ours = np.array([oracle.e8m0_value(v) for v in b], np.float64)
    lib = e8m0_lib_value(b)
    tch = torch.from_numpy(b.copy()).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    assert np.array_equal(ours[:255], lib[:255]) and np.array_equal(ours[:255], tch[:255])
    assert np.isnan(ours[255]) and np.isnan(lib[255])


def test_shared_exponent_puts_block_max_in_4_to_8():
    """The exponent is the unique integer e with amax / 2^e in [4, 8) (largest
    E2M1 exponent 2), clamped to the UE8M0 range; zero blocks take -127."""
    rng = np.random.default_rng(0)
    vals = np.concatenate([np.exp(rng.uniform(-80, 80, 3000)),
                           2.0 ** np.arange(-120, 120), np.nextafter(2.0 ** np.arange(-120, 120), 0)])
    for a in vals.astype(np.float32):
        if not np.isfinite(a) or a == 0:
            continue
        e = oracle.mx_exponent(a)
        q = float(a) / 2.0 ** e
        if e > -127:
            assert 4.0 <= q < 8.0, (a, e)
        else:
            assert q < 8.0
    assert oracle.mx_exponent(0.0) == -127
    assert oracle.mx_exponent(np.float32(1e-40)) == -127            # subnormal maximum: clamped
    assert oracle.mx_exponent(np.float32(3.0e38)) == 125


@pytest.mark.parametrize("shape", [(64, 128), (96, 64)])
def test_codes_and_scales_match_library_casts(shape):
    """Rows: scale byte = e + 127 with e from the block max; codes = the
    library's saturating E2M1 cast of v / 2^e (exact power-of-two scaling)."""
    R, C = shape
    x = synthetic.bf16_bits(synthetic.normal_with_entry_outliers(R, C, seed=R + C))
    out = oracle.mx_quantize(x, ROW | COL)
    xv = f32(x).astype(np.float64)
    for orient, codes, scales in ((0, out["codes_row"], out["scales_row"]),
                                  (1, out["codes_col"], out["scales_col"])):
        v = (xv if orient == 0 else xv.T).reshape(-1, 32)
        amax = np.abs(v).max(1)
        e = np.floor(np.log2(amax)) - 2
        assert np.array_equal(scales.reshape(-1), (e + 127).astype(np.uint8))
        y = np.clip(v / 2.0 ** e[:, None], -6, 6).astype(np.float32)
        want = y.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
        assert np.array_equal(nibbles(codes).reshape(-1, 32), want)


def test_columns_are_rows_of_the_transpose():
    x = synthetic.bf16_bits(synthetic.weight(64, 96, seed=2))
    a = oracle.mx_quantize(x, COL | RHT, seed=5)
    b = oracle.mx_quantize(np.ascontiguousarray(x.T), ROW | RHT, seed=5)
    assert np.array_equal(a["codes_col"], b["codes_row"])
    assert np.array_equal(a["scales_col"], b["scales_row"])


def test_round_trip_on_representable_blocks():
    """Blocks of E2M1 values times 2^e holding one +-4 or +-6 quantize back to
    the same codes and scale, and dequantize to the same values."""
    rng = np.random.default_rng(3)
    R, C = 32, 256
    codes = rng.integers(0, 16, (R, C)).astype(np.uint8)
    e = rng.integers(-20, 20, (R, C // 32))
    for r in range(R):
        for b in range(C // 32):
            codes[r, 32 * b + rng.integers(32)] = rng.choice([6, 7, 14, 15])
    vals = e2m1_lib_value(codes) * np.repeat(2.0 ** e, 32, 1)
    x = synthetic.bf16_bits(torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16))
    out = oracle.mx_quantize(x, ROW)
    got = nibbles(out["codes_row"])
    # the sign of zero survives: compare magnitudes and the sign of non-zeros
    assert np.array_equal(got & 7, codes & 7)
    nz = (codes & 7) != 0
    assert np.array_equal((got >> 3)[nz], (codes >> 3)[nz])
    assert np.array_equal(out["scales_row"], (e + 127).astype(np.uint8))
    y = oracle.mx_dequantize(out["codes_row"], out["scales_row"], R, C)
    assert np.array_equal(y, vals.astype(np.float32))


def test_rotation_is_the_16_wide_hadamard_per_half_block():
    """With small integer inputs the rotated values are exact in bf16, so MX
    with the rotation equals MX without it applied to the tensor rotated in
    float64 with scipy's Hadamard matrix (each 16-half of a block, signs D)."""
    rng = np.random.default_rng(4)
    R, C, seed = 16, 128, 9
    xi = rng.integers(-3, 4, (R, C)).astype(np.float64)
    x = synthetic.bf16_bits(torch.from_numpy(xi.astype(np.float32)).to(torch.bfloat16))
    signs = oracle.sign_bits(seed)
    d = np.array([-1.0 if (signs >> i) & 1 else 1.0 for i in range(16)])
    rot = (0.25 * (xi.reshape(-1, 16) * d) @ H16.T).reshape(R, C)
    xr = synthetic.bf16_bits(torch.from_numpy(rot.astype(np.float32)).to(torch.bfloat16))
    assert np.array_equal(f32(xr).astype(np.float64), rot)
    a = oracle.mx_quantize(x, ROW | RHT, seed=seed)
    b = oracle.mx_quantize(xr, ROW)
    assert np.array_equal(a["codes_row"], b["codes_row"])
    assert np.array_equal(a["scales_row"], b["scales_row"])
    # and the inverse rotation in dequantization undoes it up to the rounding
    y = oracle.mx_dequantize(a["codes_row"], a["scales_row"], R, C, INV, seed)
    yr = oracle.mx_dequantize(b["codes_row"], b["scales_row"], R, C)
    back = ((yr.reshape(-1, 16).astype(np.float64) @ H16.T) * 0.25 * d).reshape(R, C)
    assert np.allclose(y, back, rtol=0, atol=1e-6)


def test_dequantize_matches_library_decode():
    x = synthetic.bf16_bits(synthetic.normal_with_channel_outliers(64, 256, seed=6))
    out = oracle.mx_quantize(x, ROW)
    y = oracle.mx_dequantize(out["codes_row"], out["scales_row"], 64, 256)
    want = e2m1_lib_value(nibbles(out["codes_row"])) * np.repeat(e8m0_lib_value(out["scales_row"]), 32, 1)
    assert np.array_equal(y, want.astype(np.float32))


def test_saturation_clips_block_maxima_in_6_to_8():
    """Block maxima in [6, 8) 2^e (the range the power-of-two scale cannot
    reach) store 6 2^e: the known MXFP4 clipping that the NVFP4 write-up §五
    counts against the format."""
    v = np.zeros((1, 32), np.float32)
    v[0, 0], v[0, 1] = 7.5, -0.3
    x = synthetic.bf16_bits(torch.from_numpy(v).to(torch.bfloat16))
    out = oracle.mx_quantize(x, ROW)
    assert out["scales_row"][0, 0] == 127
    y = oracle.mx_dequantize(out["codes_row"], out["scales_row"], 1, 32)
    assert y[0, 0] == 6.0 and y[0, 1] == -0.5


def test_errors():
    x = np.zeros((32, 32), np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.mx_quantize(np.zeros((32, 48), np.uint16), ROW)
    with pytest.raises(oracle.OracleError):
        oracle.mx_quantize(np.zeros((48, 32), np.uint16), COL)
    with pytest.raises(oracle.OracleError):
        oracle.mx_quantize(x, 0)
    x[3, 4] = 0x7F80   # +Inf
    with pytest.raises(oracle.OracleError):
        oracle.mx_quantize(x, ROW)
    z = oracle.mx_quantize(np.zeros((32, 32), np.uint16), ROW | COL)
    assert (z["scales_row"] == 0).all() and (z["codes_row"] == 0).all()


def test_mx_gemm_matches_numpy_on_library_decoded_operands():
    """The FP64 MXFP4 GEMM equals numpy's float64 matmul of the operands
    decoded with ml_dtypes (E2M1 x UE8M0), on all and on selected outputs."""
    rng = np.random.default_rng(12)
    M, N, K = 48, 40, 256
    A = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    B = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sA = rng.integers(100, 150, (M, K // 32), dtype=np.uint8)
    sB = rng.integers(100, 150, (N, K // 32), dtype=np.uint8)
    da = e2m1_lib_value(nibbles(A)).astype(np.float64) * np.repeat(e8m0_lib_value(sA), 32, 1)
    db = e2m1_lib_value(nibbles(B)).astype(np.float64) * np.repeat(e8m0_lib_value(sB), 32, 1)
    want = da @ db.T
    got = oracle.mx_gemm_f64(A, sA, B, sB, M, N, K)
    assert np.allclose(got, want, rtol=1e-12, atol=0)
    rows, cols = np.array([3, 47, 0]), np.array([39, 5])
    sub = oracle.mx_gemm_f64(A, sA, B, sB, M, N, K, rows=rows, cols=cols)
    assert np.array_equal(sub, got[np.ix_(rows, cols)])
