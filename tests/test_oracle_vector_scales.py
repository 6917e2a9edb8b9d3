"""Pins of the oracle's finer tensor scales (one Eq. 1 tensor scale per row of
the quantized operand; the NVFP4 pretraining write-up §九 names per-row or
per-block global scales as the remedy for a single global amax).

Each pin checks the oracle against something other than itself: numpy's
IEEE float32 division for the closed form, scipy's Hadamard matrix for the
rotated maxima, the consequence that each vector's largest block gets the
E4M3 maximum 448, the per-tensor path (already pinned) applied to a
one-vector tensor, and numpy's float64 matmul for the GEMM reference.
"""
import numpy as np
import pytest
import scipy.linalg

import oracle
from nvfp4_block_quantization_amax_b200 import synthetic
from test_oracle_pins import e2m1_lib_value, e4m3_lib_value, unpack

ROW, COL, RHT, VS, HEADROOM = oracle.ROWWISE, oracle.COLWISE, oracle.RHT, oracle.VECTOR_SCALES, oracle.HEADROOM
H16 = scipy.linalg.hadamard(16).astype(np.float64)


def f32(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32)


@pytest.fixture(scope="module")
def x():
    # rows with very different ranges: channel outliers plus a few scaled rows
    t = synthetic.normal_with_channel_outliers(48, 128, seed=61).float()
    t[5] *= 1e-3
    t[17] *= 37.0
    t[30] = 0.0
    return synthetic.bf16_bits(synthetic.to_bf16(t.numpy()))


@pytest.mark.parametrize("headroom", [False, True])
def test_vector_alpha_is_eq1_per_vector(x, headroom):
    flags = ROW | COL | VS | (HEADROOM if headroom else 0)
    o = oracle.quantize(x, oracle.RTN, flags)
    den = np.float32(1792 if headroom else 2688)
    xf = np.abs(f32(x))
    assert np.array_equal(o["alpha_row"], (xf.max(1).astype(np.float32) / den).astype(np.float32))
    assert np.array_equal(o["alpha_col"], (xf.max(0).astype(np.float32) / den).astype(np.float32))
    assert o["amax_row"] == float(xf.max()) and o["amax_col"] == float(xf.max())
    assert o["alpha_row"][30] == 0.0 and not o["codes_row"][30].any()


def test_vector_alpha_of_rotated_vectors_matches_scipy_hadamard():
    # small-integer inputs: the rotated values are exact in float32
    rng = np.random.default_rng(62)
    t = (4 * rng.integers(-60, 60, (32, 64))).astype(np.float32)
    bits = synthetic.bf16_bits(synthetic.to_bf16(t))
    seed = 9
    s = oracle.sign_bits(seed)
    d = np.array([-1.0 if (s >> i) & 1 else 1.0 for i in range(16)])
    rows = 0.25 * (t.reshape(32, 4, 16).astype(np.float64) * d) @ H16.T
    cols = 0.25 * (t.T.reshape(64, 2, 16).astype(np.float64) * d) @ H16.T
    o = oracle.quantize(bits, oracle.MS_EDEN, ROW | COL | VS, seed=seed)
    want_r = (np.abs(rows).max((1, 2)).astype(np.float32) / np.float32(2688)).astype(np.float32)
    want_c = (np.abs(cols).max((1, 2)).astype(np.float32) / np.float32(2688)).astype(np.float32)
    assert np.array_equal(o["alpha_row"], want_r)
    assert np.array_equal(o["alpha_col"], want_c)
    assert np.array_equal(oracle.amax_vectors(bits, 0, True, seed), np.abs(rows).max((1, 2)).astype(np.float32))


def test_each_vectors_largest_block_gets_448(x):
    o = oracle.quantize(x, oracle.RTN, ROW | COL | VS)
    xf = np.abs(f32(x))
    for side, t in (("row", xf), ("col", xf.T)):
        sc = o[f"scales_{side}"]
        for i in range(t.shape[0]):
            if t[i].max() == 0:
                continue
            blk = int(np.argmax(t[i])) // 16
            assert sc[i, blk] == 0x7E, (side, i)


@pytest.mark.parametrize("mode", [oracle.RTN, oracle.FOUR_SIX])
@pytest.mark.parametrize("rot", [0, RHT])
def test_vector_equals_quantizing_that_vector_alone(x, mode, rot):
    # row i with its own scale == the one-row tensor x[i] quantized with Eq. 1;
    # column j == row j of the transpose (no random streams in these modes)
    o = oracle.quantize(x, mode, ROW | COL | VS | rot, seed=4)
    for i in (0, 5, 17, 30, 47):
        one = oracle.quantize(np.ascontiguousarray(x[i:i + 1]), mode, ROW | rot, seed=4)
        assert np.array_equal(o["codes_row"][i], one["codes_row"][0]), i
        assert np.array_equal(o["scales_row"][i], one["scales_row"][0]), i
        assert o["alpha_row"][i] == one["alpha_row"]
    xt = np.ascontiguousarray(x.T)
    for j in (0, 3, 64, 127):
        one = oracle.quantize(np.ascontiguousarray(xt[j:j + 1]), mode, ROW | rot, seed=4)
        assert np.array_equal(o["codes_col"][j], one["codes_row"][0]), j
        assert np.array_equal(o["scales_col"][j], one["scales_row"][0]), j
        assert o["alpha_col"][j] == one["alpha_row"]


@pytest.mark.parametrize("mode", [oracle.RHT_SR, oracle.MS_EDEN, oracle.RHT_SR_HW])
def test_random_modes_use_the_tensor_wide_streams(x, mode):
    # the random draws are keyed by the block's index in the whole tensor, as
    # without vector scales: vector i equals the per-tensor 1D path on that
    # vector given its own alpha
    o = oracle.quantize(x, mode, ROW | COL | VS, seed=11, stream_id=3)
    for orient, side in ((0, "row"), (1, "col")):
        for i in (1, 17, 40):
            a = float(o[f"alpha_{side}"][i])
            c, s = oracle.quantize_1d_range(x, orient, mode, 0, 11, 3, a, i, i + 1)
            assert np.array_equal(o[f"codes_{side}"][i], c[0]) and np.array_equal(o[f"scales_{side}"][i], s[0])


def test_vector_scales_reject_2d_and_provided_alpha(x):
    with pytest.raises(oracle.OracleError):
        oracle.quantize_vector_scales(x, oracle.RTN, ROW | oracle.BLOCK2D | VS)
    with pytest.raises(ValueError):
        oracle.quantize(x, oracle.RTN, ROW | VS, alpha=1.0)


def test_gemm_f64_vector_scales_matches_numpy():
    rng = np.random.default_rng(63)
    M, N, K = 40, 24, 64
    A = rng.integers(0, 256, (M, K // 2)).astype(np.uint8)
    B = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    sA = rng.integers(0, 0x7F, (M, K // 16)).astype(np.uint8)
    sB = rng.integers(0, 0x7F, (N, K // 16)).astype(np.uint8)
    aA = rng.uniform(0.01, 3, M).astype(np.float32)
    aB = rng.uniform(0.01, 3, N).astype(np.float32)
    dA = e2m1_lib_value(unpack(A)).astype(np.float64) * np.repeat(e4m3_lib_value(sA), 16, 1)
    dB = e2m1_lib_value(unpack(B)).astype(np.float64) * np.repeat(e4m3_lib_value(sB), 16, 1)
    want = (dA @ dB.T) * np.outer(aA.astype(np.float64), aB.astype(np.float64))
    got = oracle.gemm_f64(A, sA, aA, B, sB, aB, M, N, K)
    assert np.allclose(got, want, rtol=1e-12, atol=0)
    rows, cols = np.array([39, 2]), np.array([0, 23, 7])
    assert np.allclose(oracle.gemm_f64(A, sA, aA, B, sB, aB, M, N, K, rows, cols), want[np.ix_(rows, cols)],
                       rtol=1e-12, atol=0)
