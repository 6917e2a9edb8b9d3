"""Pins of the CPU oracle against what the pages and the mathematics fix.

Every check here compares the oracle with something other than itself: values
printed on the pages (tests/golden), independent library encoders and
decoders (ml_dtypes, torch float8), an independent Philox (PyTorch's ATen
engine), scipy's Hadamard matrix, numpy's float64 matmul, closed forms and
statistical invariants.  No GPU is needed.
"""
import json
import os
import shutil
import subprocess

import ml_dtypes
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from nvfp4_block_quantization_amax_b200 import synthetic

HERE = os.path.dirname(os.path.abspath(__file__))
GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


# --------------------------------------------------------------------------
# helpers built on library types only
# --------------------------------------------------------------------------
def e4m3_lib_value(b):
    return np.asarray(b, np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float32)


def e4m3_lib_rne(v):
    """ml_dtypes RNE cast; the format saturates at 448 in our spec."""
    v = np.minimum(np.asarray(v, np.float32), np.float32(448))
    return v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)


def e2m1_lib_value(codes):
    """4-bit codes (one per byte) decoded by ml_dtypes' float4_e2m1fn."""
    return np.asarray(codes, np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float32)


def e2m1_lib_rne_code(y):
    """ml_dtypes float4_e2m1fn cast -> 4-bit code (one per byte)."""
    return np.asarray(y, np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF


def unpack(codes):
    return oracle.unpack_codes(codes)


# --------------------------------------------------------------------------
# Philox4x32-10 against PyTorch's independent engine
# --------------------------------------------------------------------------
@pytest.fixture(scope="module")
def aten_philox(tmp_path_factory):
    gxx = shutil.which("g++")
    inc = os.path.join(os.path.dirname(torch.__file__), "include")
    if gxx is None or not os.path.exists(os.path.join(inc, "ATen/core/PhiloxRNGEngine.h")):
        pytest.skip("g++ or the ATen Philox header is not available")
    exe = str(tmp_path_factory.mktemp("philox") / "aten_philox")
    subprocess.run([gxx, "-std=c++17", "-O1", "-I", inc,
                    os.path.join(HERE, "helpers", "aten_philox_ref.cpp"), "-o", exe], check=True)

    def run(rows):
        inp = "\n".join(" ".join(str(int(v)) for v in r) for r in rows) + "\n"
        out = subprocess.run([exe], input=inp, capture_output=True, text=True, check=True).stdout
        return np.array([[int(t) for t in line.split()] for line in out.strip().splitlines()],
                        np.uint64).astype(np.uint32)
    return run


def test_philox_matches_aten_engine(aten_philox):
    rng = np.random.default_rng(123)
    rows = [[0] * 6, [0xFFFFFFFF] * 6, [1, 0, 0, 0, 0, 0], [0, 0, 0, 3, 7, 0]]
    rows += rng.integers(0, 2**32, size=(300, 6), dtype=np.uint64).tolist()
    ref = aten_philox(rows)
    for r, want in zip(rows, ref):
        got = oracle.philox(r[:4], r[4:])
        assert np.array_equal(got, want), (r, got, want)


def test_sign_vector_is_first_word_of_tag3(aten_philox):
    seeds = [0, 1, 42, 2**40 + 5, 2**64 - 1]
    rows = [[0, 0, 0, 3, s & 0xFFFFFFFF, s >> 32] for s in seeds]
    ref = aten_philox(rows)
    for s, w in zip(seeds, ref):
        assert oracle.sign_bits(s) == int(w[0]) & 0xFFFF


# --------------------------------------------------------------------------
# E4M3 scale encoder
# --------------------------------------------------------------------------
def test_e4m3_decode_matches_ml_dtypes():
    for b in range(0x7F):
        assert oracle.e4m3_value(b) == float(e4m3_lib_value(b))


def _e4m3_probe_points():
    vals = e4m3_lib_value(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)
    pts = [0.0, 1e-30, 2.0**-12, 2.0**-10, 448.0, 449.0, 464.0, 500.0, 1e30]
    rng = np.random.default_rng(7)
    for lo, hi in zip(vals[:-1], vals[1:]):
        mid = (lo + hi) / 2
        pts += [lo, mid, np.nextafter(np.float32(mid), np.float32(0)),
                np.nextafter(np.float32(mid), np.float32(1e9))]
        pts += list(rng.uniform(lo, hi, 8))
    return np.array(pts, np.float32)


def test_e4m3_rne_matches_library_casts():
    pts = _e4m3_probe_points()
    got = np.array([oracle.e4m3_rne(v) for v in pts], np.uint8)
    want = e4m3_lib_rne(pts)
    assert np.array_equal(got, want)
    # torch's own float8 cast agrees inside the finite range
    inr = pts[pts < 448]
    t = torch.from_numpy(inr).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(np.array([oracle.e4m3_rne(v) for v in inr], np.uint8), t)
    # the page's worked example: 40/6 = 6.667 -> 6.5, not 7
    assert oracle.e4m3_value(oracle.e4m3_rne(np.float32(40) / np.float32(6))) == 6.5


def test_e4m3_ceil_is_smallest_value_not_below():
    pts = _e4m3_probe_points()
    for v in pts:
        b = oracle.e4m3_ceil(v)
        if v >= 448:
            assert b == 0x7E
            continue
        assert oracle.e4m3_value(b) >= v
        if b > 0:
            assert oracle.e4m3_value(b - 1) < v


def test_e4m3_sr_threshold_and_expectation():
    rng = np.random.default_rng(3)
    for v in rng.uniform(2.0**-12, 440, 200).astype(np.float32):
        lo_b = oracle.e4m3_ceil(v)
        if oracle.e4m3_value(lo_b) == v:
            continue
        lo_b -= 1
        lo, hi = oracle.e4m3_value(lo_b), oracle.e4m3_value(lo_b + 1)
        t = (float(v) - lo) / (hi - lo) * 2**24  # exact in float64
        k = int(np.ceil(t))  # number of u24 values that round up
        assert oracle.e4m3_sr(v, k - 1) == lo_b + 1
        assert oracle.e4m3_sr(v, min(k, 2**24 - 1)) == (lo_b if k < 2**24 else lo_b + 1)
        # expectation over all u24: lo + k/2^24 (hi - lo), within one 2^-24 step of v
        mean = lo + k / 2**24 * (hi - lo)
        assert abs(mean - float(v)) <= (hi - lo) * 2.0**-24


# --------------------------------------------------------------------------
# E2M1 value encoder: Eq. 3 of the Four Over Six page, and library casts
# --------------------------------------------------------------------------
def eq3_page(y):
    """Eq. 3 as printed (Four Over Six, §2.1), with round-half-even integers,
    saturated at 6 outside the printed range."""
    y = np.asarray(y, np.float64)
    a = np.abs(y)
    q = np.where(a < 2, 0.5 * np.rint(2 * y), np.where(a < 4, np.rint(y), 2 * np.rint(y / 2)))
    return np.clip(q, -6, 6)


def test_e2m1_rne_all_bf16_in_range_eq3_and_ml_dtypes():
    bits = np.arange(65536, dtype=np.uint32)
    vals = (bits << 16).view(np.float32)
    vals = vals[np.isfinite(vals) & (np.abs(vals) <= 8)]
    got = np.array([oracle.e2m1_rne(v) for v in vals], np.uint8)
    mag = GRID[got & 7] * np.where(got & 8, -1, 1)
    assert np.array_equal(mag, eq3_page(vals) * 1.0)
    assert np.array_equal(np.abs(mag), np.abs(e2m1_lib_value(e2m1_lib_rne_code(vals))))
    # sign bit follows the sign of y, including values that round to zero
    assert np.array_equal(got >> 3, (vals.view(np.uint32) >> 31).astype(np.uint8))


def test_e2m1_rne_random_fp32():
    rng = np.random.default_rng(11)
    vals = rng.uniform(-7, 7, 20000).astype(np.float32)
    got = np.array([oracle.e2m1_rne(v) for v in vals], np.uint8)
    mag = GRID[got & 7] * np.where(got & 8, -1, 1)
    assert np.array_equal(mag, eq3_page(vals))
    assert np.array_equal(got & 7, e2m1_lib_rne_code(np.abs(vals)))


def test_e2m1_decode_matches_ml_dtypes():
    for c in range(16):
        assert oracle.e2m1_value(c) == float(e2m1_lib_value(np.uint8(c)))


def test_e2m1_sr_threshold():
    rng = np.random.default_rng(5)
    for y in rng.uniform(-5.99, 5.99, 400).astype(np.float32):
        a = abs(float(y))
        lo = GRID[GRID <= a].max()
        if lo == a:
            assert oracle.e2m1_value(oracle.e2m1_sr(y, 0)) == float(y)
            continue
        hi = GRID[GRID > a].min()
        k = int(np.ceil((a - lo) / (hi - lo) * 65536))
        up = oracle.e2m1_value(oracle.e2m1_sr(y, k - 1))
        dn = oracle.e2m1_value(oracle.e2m1_sr(y, min(k, 65535)))
        assert abs(up) == hi
        assert abs(dn) == (lo if k < 65536 else hi)
        assert np.sign(up) == np.sign(y)


def test_e2m1_sr_hw_threshold_and_expectation():
    """Hardware stochastic rounding ([NV] §四): over all 2^16 fields the number
    that round up is floor(f 2^16), f the exact fraction of |y| between its grid
    neighbours, so the expectation is within gap / 2^16 of y; the smallest
    field that rounds up is 2^16 - floor(f 2^16); magnitudes >= 6 give 6."""
    from fractions import Fraction
    rng = np.random.default_rng(6)
    ys = np.concatenate([rng.uniform(-5.99, 5.99, 150), GRID[:-1] + 0.25 * np.diff(GRID)]).astype(np.float32)
    for y in ys:
        a = Fraction(abs(float(y)))
        lo = Fraction(float(GRID[GRID <= a].max()))
        codes = {oracle.e2m1_sr_hw(y, r) for r in (0, 65535)}
        if lo == a:
            assert codes == {oracle.e2m1_sr(y, 0)}
            continue
        hi = Fraction(float(GRID[GRID > a].min()))
        ups = int((a - lo) / (hi - lo) * 65536)          # floor
        first_up = 65536 - ups
        if first_up <= 65535:
            assert abs(oracle.e2m1_value(oracle.e2m1_sr_hw(y, first_up))) == float(hi)
        assert abs(oracle.e2m1_value(oracle.e2m1_sr_hw(y, first_up - 1))) == float(lo)
        assert np.sign(oracle.e2m1_value(oracle.e2m1_sr_hw(y, 65535))) == np.sign(y)
        mean = lo + (hi - lo) * Fraction(ups, 65536)
        assert 0 <= a - mean < (hi - lo) / 65536
    for y in (6.0, 7.5, -300.0):
        assert abs(oracle.e2m1_value(oracle.e2m1_sr_hw(y, 65535))) == 6.0
    assert oracle.e2m1_sr_hw(-0.0, 65535) == 8 and oracle.e2m1_sr_hw(0.0, 65535) == 0


def test_sr_hw_fields_uniform_and_paired():
    """Each element's 16-bit field must be uniform when the draw word is: for
    every position the map from the word's two bytes it reads to the field is
    a bijection, positions 0/1 read bytes 0 and 2, positions 2/3 bytes 1 and 3."""
    w = np.arange(65536, dtype=np.uint64)
    even = ((w >> 8) << 16) | (w & 0xFF)               # bytes 0 and 2
    odd = even << 8                                    # bytes 1 and 3
    for j, src in ((0, even), (1, even), (2, odd), (3, odd)):
        f = [oracle.sr_hw_field(int(v), j) for v in src]
        assert len(set(f)) == 65536, j
        mask = 0xFF00FF00 if j < 2 else 0x00FF00FF     # the other two bytes are ignored
        for i in range(0, 65536, 257):
            assert oracle.sr_hw_field(int(src[i]) | mask, j) == f[i]


# --------------------------------------------------------------------------
# 16-wide random Hadamard transform
# --------------------------------------------------------------------------
H16 = scipy.linalg.hadamard(16).astype(np.int64)


def test_hadamard_orthogonal_integers():
    assert np.array_equal(H16 @ H16.T, 16 * np.eye(16, dtype=np.int64))


def test_rht_exact_on_integers():
    rng = np.random.default_rng(2)
    for _ in range(200):
        signs = int(rng.integers(0, 1 << 16))
        d = np.array([-1 if (signs >> i) & 1 else 1 for i in range(16)], np.int64)
        x = 4 * rng.integers(-1000, 1000, 16)
        want = (H16 @ (d * x)) // 4  # exact: every entry of H d x is a multiple of 4
        got = oracle.rht16(x.astype(np.float32), signs)
        assert np.array_equal(got.astype(np.int64), want)
        back = oracle.irht16(got, signs)
        assert np.array_equal(back.astype(np.int64), x)


def test_rht_float_close_to_f64_and_norm_preserving():
    rng = np.random.default_rng(4)
    for _ in range(200):
        signs = int(rng.integers(0, 1 << 16))
        d = np.array([-1.0 if (signs >> i) & 1 else 1.0 for i in range(16)])
        x = rng.standard_normal(16).astype(np.float32) * np.float32(rng.uniform(0.01, 100))
        want = 0.25 * (H16 @ (d * x.astype(np.float64)))
        got = oracle.rht16(x, signs)
        bound = 4 * 2.0**-24 * np.abs(x).sum() * 4
        assert np.max(np.abs(got - want)) <= bound
        assert abs(np.linalg.norm(got) - np.linalg.norm(x)) <= 1e-5 * np.linalg.norm(x)
        back = oracle.irht16(got, signs)
        assert np.max(np.abs(back - x)) <= 8 * 2.0**-24 * np.abs(x).sum()


# --------------------------------------------------------------------------
# Eq. 1 (tensor scale) and the block-scale consequences
# --------------------------------------------------------------------------
@pytest.fixture(scope="module")
def pr1():
    d = synthetic.pr1()
    return {k: synthetic.bf16_bits(v) for k, v in d.items()}


def f32(x_bits):
    return (x_bits.astype(np.uint32) << 16).view(np.float32)


def test_alpha_is_eq1(pr1):
    x = pr1["x"]
    out = oracle.quantize(x, oracle.RTN, oracle.ROWWISE)
    amax = np.abs(f32(x)).max()
    assert out["amax_row"] == amax
    assert out["alpha_row"] == float(np.float32(amax) / np.float32(6 * 448))
    # the block holding the tensor max gets the largest E4M3 scale, 448
    r, c = np.unravel_index(np.argmax(np.abs(f32(x))), x.shape)
    assert out["scales_row"][r, c // 16] == 0x7E


def test_worked_example_table1():
    g = json.load(open(os.path.join(HERE, "golden", "four_over_six_table1.json")))
    v = np.zeros(16, np.float32)
    v[:4] = g["block"]
    alpha = g["alpha"]
    c6, s6 = oracle.quantize_block16(v, alpha, oracle.RTN)
    assert oracle.e4m3_value(s6) == g["M6"]["scale"]
    y30 = 30 / oracle.e4m3_value(s6)
    assert round(y30, 2) == g["M6"]["scaled_30"]
    assert oracle.e2m1_value(c6[2]) == g["M6"]["rounded_30"]
    deq = np.array([oracle.e2m1_value(c) for c in c6]) * oracle.e4m3_value(s6)
    # the page prints 13.4% = (4.62 - 4) / 4.62 from its rounded value; the
    # exact relative error of 30 is 4/30 = 13.3%
    rel = abs(deq[2] - 30) / 30
    assert 0.133 <= rel <= 0.135
    assert abs(g["M6"]["relative_error_percent"] / 100 - (y30 - 4) / y30) < 0.001
    # Four Over Six keeps the M = 4 encoding: scale 10, 30 -> 3 exactly
    c46, s46 = oracle.quantize_block16(v, alpha, oracle.FOUR_SIX)
    assert oracle.e4m3_value(s46) == g["M4"]["scale"]
    assert oracle.e2m1_value(c46[2]) == g["M4"]["rounded_30"]
    deq46 = np.array([oracle.e2m1_value(c) for c in c46]) * oracle.e4m3_value(s46)
    assert np.array_equal(deq46[:4], np.array(g["block"], np.float64))
    # byte encodings agree with the library types
    assert s6 == int(e4m3_lib_rne(6.5)) and s46 == int(e4m3_lib_rne(10.0))


def _lib_rtn_rows(x_bits, alpha, M=6.0):
    """RTN row quantization restated with numpy float32 steps and the
    ml_dtypes encoders (Eq. 2, Eq. 3 of Four Over Six)."""
    x = f32(x_bits)
    R, C = x.shape
    blocks = x.reshape(R, C // 16, 16)
    amax_b = np.abs(blocks).max(axis=2)
    den = np.float32(alpha) * np.float32(M)
    draw = (amax_b / den).astype(np.float32)
    sb = e4m3_lib_rne(draw)
    s = (np.float32(alpha) * e4m3_lib_value(sb)).astype(np.float32)
    with np.errstate(divide="ignore"):
        rinv = (np.float32(1) / s).astype(np.float32)
    y = (blocks * rinv[..., None]).astype(np.float32)
    codes = e2m1_lib_rne_code(np.abs(y)) | ((y.view(np.uint32) >> 31).astype(np.uint8) << 3)
    codes = np.where(np.isinf(rinv)[..., None], codes & 8, codes)
    return codes.reshape(R, C), sb


def test_rtn_rows_match_library_encoders(pr1):
    x = pr1["x"]
    out = oracle.quantize(x, oracle.RTN, oracle.ROWWISE)
    codes, sb = _lib_rtn_rows(x, out["alpha_row"])
    assert np.array_equal(out["scales_row"], sb)
    assert np.array_equal(unpack(out["codes_row"]), codes)


def test_colwise_is_rowwise_of_transpose(pr1):
    x = pr1["x"]
    out = oracle.quantize(x, oracle.RTN, oracle.COLWISE)
    codes, sb = _lib_rtn_rows(np.ascontiguousarray(x.T), out["alpha_col"])
    assert np.array_equal(out["scales_col"], sb)
    assert np.array_equal(unpack(out["codes_col"]), codes)


@pytest.mark.parametrize("mode", [oracle.RTN, oracle.FOUR_SIX, oracle.RHT_SR, oracle.MS_EDEN, oracle.RHT_SR_HW])
def test_grid_membership_and_scale_range(pr1, mode):
    out = oracle.quantize(pr1["x"], mode, oracle.ROWWISE | oracle.COLWISE, seed=9)
    for k in ("codes_row", "codes_col"):
        vals = np.array([oracle.e2m1_value(c) for c in range(16)])[unpack(out[k])]
        assert np.isin(np.abs(vals), GRID).all()
    for k in ("scales_row", "scales_col"):
        s = out[k]
        assert (s <= 0x7E).all()  # sign bit clear, never NaN, at most 448
        assert np.isfinite(e4m3_lib_value(s)).all()


def _representable_tensor(rng, R, C, two_d=False):
    codes = rng.integers(0, 16, (R, C)).astype(np.uint8)
    if two_d:
        sb = rng.integers(0x20, 0x60, (R // 16, C // 16)).astype(np.uint8)
        scale = np.repeat(np.repeat(e4m3_lib_value(sb), 16, 0), 16, 1)
        for br in range(R // 16):
            for bc in range(C // 16):
                codes[16 * br + rng.integers(16), 16 * bc + rng.integers(16)] = 7 | (8 * rng.integers(2))
    else:
        sb = rng.integers(0x20, 0x60, (R, C // 16)).astype(np.uint8)
        scale = np.repeat(e4m3_lib_value(sb), 16, 1)
        for r in range(R):
            for b in range(C // 16):
                codes[r, 16 * b + rng.integers(16)] = 7 | (8 * rng.integers(2))  # one +-6 per block
    vals = e2m1_lib_value(codes) * scale
    return synthetic.bf16_bits(torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16)), vals


@pytest.mark.parametrize("mode", [oracle.RTN, oracle.FOUR_SIX])
@pytest.mark.parametrize("two_d", [False, True])
def test_round_trip_identity_on_representable_inputs(mode, two_d):
    rng = np.random.default_rng(17 + mode + 2 * two_d)
    R, C = 64, 128
    x, vals = _representable_tensor(rng, R, C, two_d)
    assert np.array_equal(f32(x), vals)  # the values are exact in bf16
    f2d = oracle.BLOCK2D if two_d else 0
    out = oracle.quantize(x, mode, oracle.ROWWISE | oracle.COLWISE * two_d | f2d, alpha=1.0)
    dq = oracle.dequantize(out["codes_row"], out["scales_row"], 1.0, R, C, f2d)
    assert np.array_equal(dq, vals)
    if two_d:
        dqc = oracle.dequantize(out["codes_col"], out["scales_col"], 1.0, C, R, f2d)
        assert np.array_equal(dqc.T, vals)
    else:
        # column blocks: the transpose of a row-representable tensor
        xt = np.ascontiguousarray(x.T)
        out = oracle.quantize(xt, mode, oracle.COLWISE, alpha=1.0)
        dqc = oracle.dequantize(out["codes_col"], out["scales_col"], 1.0, R, C)
        assert np.array_equal(dqc, vals)


def test_block_max_stored_near_8bit(pr1):
    x = pr1["x"]
    out = oracle.quantize(x, oracle.RTN, oracle.ROWWISE)
    dq = oracle.dequantize(out["codes_row"], out["scales_row"], out["alpha_row"], *x.shape)
    xf = f32(x).reshape(x.shape[0], -1, 16)
    dqb = dq.reshape(xf.shape)
    idx = np.argmax(np.abs(xf), axis=2)
    xm = np.take_along_axis(xf, idx[..., None], 2)[..., 0]
    dm = np.take_along_axis(dqb, idx[..., None], 2)[..., 0]
    normal = out["scales_row"] >= 0x08
    rel = np.abs(dm - xm) / np.abs(xm)
    assert (rel[normal] <= 2.0**-4 + 1e-6).all()


def test_dead_zone_and_three_quarters():
    # M = 6: values between 2/3 and 1 of the block max land on 4 or 6
    rng = np.random.default_rng(8)
    for _ in range(200):
        v = np.zeros(16, np.float32)
        v[0] = 6.0
        v[1:] = rng.uniform(4.0001, 5.9999, 15).astype(np.float32)
        c, s = oracle.quantize_block16(v, 1.0, oracle.RTN)
        assert oracle.e4m3_value(s) == 1.0
        assert set(np.abs([oracle.e2m1_value(q) for q in c[1:]])) <= {4.0, 6.0}
    # M = 4: 75% of the block max is the representable value 3
    v = np.zeros(16, np.float32)
    v[:2] = [40.0, 30.0]
    c, s = oracle.quantize_block16(v, 1.0, oracle.FOUR_SIX)
    assert oracle.e4m3_value(s) == 10.0 and oracle.e2m1_value(c[1]) == 3.0


def test_four_six_keeps_the_lower_error_candidate(pr1):
    x = f32(pr1["x"]).reshape(-1, 16)
    sweep = f32(synthetic.bf16_bits(synthetic.sweep(256, seed=3))).reshape(-1, 16)
    alpha = float(np.float32(np.abs(x).max()) / np.float32(2688))
    alpha2 = float(np.float32(np.abs(sweep).max()) / np.float32(2688))
    n4 = 0
    for blocks, a in ((x[:3000], alpha), (sweep[:3000], alpha2)):
        for v in blocks:
            c6, s6 = oracle.quantize_block16(v, a, oracle.RTN)
            c46, s46 = oracle.quantize_block16(v, a, oracle.FOUR_SIX)
            e6 = oracle.block_sq_error(v, a, c6, s6)
            e46 = oracle.block_sq_error(v, a, c46, s46)
            assert e46 <= e6
            # independent M = 4 candidate from library encoders, fp64 error
            amax_b = np.float32(np.abs(v).max())
            s4 = int(e4m3_lib_rne(amax_b / (np.float32(a) * np.float32(4))))
            sc4 = np.float32(a) * e4m3_lib_value(s4)
            y4 = v * (np.float32(1) / sc4) if sc4 > 0 else np.zeros(16, np.float32)
            q4 = e2m1_lib_value(e2m1_lib_rne_code(np.abs(y4))) * np.sign(v)
            err4 = float(np.sum((v.astype(np.float64) - q4 * np.float64(sc4)) ** 2))
            q6 = np.array([oracle.e2m1_value(t) for t in c6], np.float64)
            err6 = float(np.sum((v - q6 * np.float64(a * oracle.e4m3_value(s6))) ** 2))
            if s46 != s6 or not np.array_equal(c46, c6):
                n4 += 1
                assert s46 == s4
                assert err4 <= err6 * (1 + 1e-5) + 1e-30
            else:
                assert err6 <= err4 * (1 + 1e-5) + 1e-30
    assert n4 > 0  # the M = 4 candidate does win on some blocks


def test_four_six_exact_tie_keeps_six():
    """A block both candidates represent exactly (errors both 0): with
    alpha = 1 and maximum 6, M = 6 gives Delta = 1 and M = 4 gives Delta = 1.5,
    each mapping 6 onto the grid.  The tie keeps M = 6 (the selection rule is
    strict: M = 4 only when its error is lower)."""
    v = np.zeros(16, np.float32)
    v[0], v[5] = 6.0, -3.0          # 6 and 3 on the M = 6 grid (Delta 1); 4 and 2 on M = 4's (Delta 1.5)
    c6, s6 = oracle.quantize_block16(v, 1.0, oracle.RTN)
    c46, s46 = oracle.quantize_block16(v, 1.0, oracle.FOUR_SIX)
    assert oracle.e4m3_value(s6) == 1.0 and oracle.block_sq_error(v, 1.0, c6, s6) == 0.0
    assert s46 == s6 and np.array_equal(c46, c6)
    s4 = int(e4m3_lib_rne(1.5))
    q4 = np.zeros(16, np.uint8)
    q4[0], q4[5] = 6, 8 | 4          # 4 and -2 under Delta 1.5
    assert oracle.block_sq_error(v, 1.0, q4, s4) == 0.0   # the M = 4 candidate is exact too


def test_2d_blocks_consistent_across_orientations(pr1):
    w = pr1["w"]
    R, C = w.shape
    for mode in (oracle.RTN, oracle.FOUR_SIX):
        out = oracle.quantize(w, mode, oracle.ROWWISE | oracle.COLWISE | oracle.BLOCK2D)
        assert np.array_equal(out["scales_col"], out["scales_row"].T)
        a = out["alpha_row"]
        dr = oracle.dequantize(out["codes_row"], out["scales_row"], a, R, C, oracle.BLOCK2D)
        dc = oracle.dequantize(out["codes_col"], out["scales_col"], a, C, R, oracle.BLOCK2D)
        assert np.array_equal(dr, dc.T)
        # the scale of each tile follows Eq. 2 from the tile's max (RTN)
        if mode == oracle.RTN:
            wt = np.abs(f32(w)).reshape(R // 16, 16, C // 16, 16).max(axis=(1, 3))
            draw = (wt / (np.float32(a) * np.float32(6))).astype(np.float32)
            assert np.array_equal(out["scales_row"], e4m3_lib_rne(draw))


def test_dequant_matches_library_decode(pr1):
    x = pr1["x"]
    out = oracle.quantize(x, oracle.FOUR_SIX, oracle.ROWWISE)
    R, C = x.shape
    dq = oracle.dequantize(out["codes_row"], out["scales_row"], out["alpha_row"], R, C)
    s = (np.float32(out["alpha_row"]) * e4m3_lib_value(out["scales_row"])).astype(np.float32)
    want = (e2m1_lib_value(unpack(out["codes_row"])) * np.repeat(s, 16, 1)).astype(np.float32)
    assert np.array_equal(dq, want)


def test_gemm_f64_matches_numpy_matmul():
    rng = np.random.default_rng(21)
    M, N, K = 48, 40, 96
    A = rng.integers(0, 256, (M, K // 2)).astype(np.uint8)
    B = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    sA = rng.integers(0, 0x7F, (M, K // 16)).astype(np.uint8)
    sB = rng.integers(0, 0x7F, (N, K // 16)).astype(np.uint8)
    aA, aB = 0.37, 1.9
    dA = e2m1_lib_value(unpack(A)).astype(np.float64) * np.repeat(e4m3_lib_value(sA), 16, 1)
    dB = e2m1_lib_value(unpack(B)).astype(np.float64) * np.repeat(e4m3_lib_value(sB), 16, 1)
    want = (dA @ dB.T) * np.float64(np.float32(aA)) * np.float64(np.float32(aB))
    got = oracle.gemm_f64(A, sA, aA, B, sB, aB, M, N, K)
    assert np.allclose(got, want, rtol=1e-12, atol=0)
    rows, cols = np.array([3, 0, 47]), np.array([39, 5])
    sub = oracle.gemm_f64(A, sA, aA, B, sB, aB, M, N, K, rows, cols)
    assert np.allclose(sub, want[np.ix_(rows, cols)], rtol=1e-12, atol=0)


def test_inverse_rht_dequant_recovers_input(pr1):
    x = pr1["x"][:64]
    R, C = x.shape
    out = oracle.quantize(x, oracle.RTN, oracle.ROWWISE | oracle.RHT, seed=5)
    dq = oracle.dequantize(out["codes_row"], out["scales_row"], out["alpha_row"], R, C,
                           oracle.INVERSE_RHT, seed=5)
    xf = f32(x)
    # error of 4-bit quantization: a fraction of the block scale, far from 0
    assert np.linalg.norm(dq - xf) / np.linalg.norm(xf) < 0.2
    # rotated RTN codes equal RTN codes of the explicitly rotated tensor
    signs = oracle.sign_bits(5)
    rot = np.stack([oracle.rht16(b, signs) for b in xf.reshape(-1, 16)]).reshape(R, C)
    codes, sb = _lib_rtn_rows_from_f32(rot, out["alpha_row"])
    assert np.array_equal(out["scales_row"], sb)
    assert np.array_equal(unpack(out["codes_row"]), codes)


def _lib_rtn_rows_from_f32(x, alpha):
    R, C = x.shape
    blocks = x.reshape(R, C // 16, 16)
    amax_b = np.abs(blocks).max(axis=2)
    draw = (amax_b / (np.float32(alpha) * np.float32(6))).astype(np.float32)
    sb = e4m3_lib_rne(draw)
    s = (np.float32(alpha) * e4m3_lib_value(sb)).astype(np.float32)
    rinv = (np.float32(1) / s).astype(np.float32)
    y = (blocks * rinv[..., None]).astype(np.float32)
    codes = e2m1_lib_rne_code(np.abs(y)) | ((y.view(np.uint32) >> 31).astype(np.uint8) << 3)
    return codes.reshape(R, C), sb


def test_rotated_amax_is_max_of_rotated_blocks(pr1):
    x = pr1["x"]
    xf = f32(x)
    signs = oracle.sign_bits(77)
    rot_r = np.stack([oracle.rht16(b, signs) for b in xf.reshape(-1, 16)])
    assert oracle.amax(x, 0, True, 77) == np.abs(rot_r).max()
    rot_c = np.stack([oracle.rht16(b, signs) for b in np.ascontiguousarray(xf.T).reshape(-1, 16)])
    assert oracle.amax(x, 1, True, 77) == np.abs(rot_c).max()


# --------------------------------------------------------------------------
# Randomised modes: unbiasedness (10^4 seeds) and the MS-EDEN error claim
# --------------------------------------------------------------------------
@pytest.fixture(scope="module")
def seeds_runs():
    """10^4 seeds of both randomised modes on one fixed 16x256 tensor.  The
    rotation is undone in float64 with scipy's Hadamard matrix."""
    R, C = 16, 256
    x = synthetic.bf16_bits(synthetic.normal_with_entry_outliers(R, C, seed=31))
    xf = f32(x).astype(np.float64)
    xb = xf.reshape(-1, 16)
    n = 10000
    res = {}
    for mode in (oracle.RHT_SR, oracle.MS_EDEN):
        acc = np.zeros((R, C))
        acc2 = np.zeros((R, C))
        ratios = np.zeros((n, R * C // 16))
        for seed in range(n):
            out = oracle.quantize(x, mode, oracle.ROWWISE, seed=seed)
            dq_rot = oracle.dequantize(out["codes_row"], out["scales_row"], out["alpha_row"],
                                       R, C, 0, seed).reshape(-1, 16).astype(np.float64)
            signs = oracle.sign_bits(seed)
            d = np.array([-1.0 if (signs >> i) & 1 else 1.0 for i in range(16)])
            r = 0.25 * (xb * d) @ H16.T            # rotated blocks (rows)
            ratios[seed] = (r * dq_rot).sum(1) / (r ** 2).sum(1)
            back = (0.25 * dq_rot @ H16.T * d).reshape(R, C)
            acc += back
            acc2 += back ** 2
        mean = acc / n
        var = acc2 / n - mean ** 2
        res[mode] = dict(mean=mean, var=var, ratios=ratios,
                         mse=float(np.mean(var + (mean - xf) ** 2)))
    return xf, n, res


@pytest.mark.slow
def test_rht_sr_unbiased_over_seeds(seeds_runs):
    xf, n, res = seeds_runs
    r = res[oracle.RHT_SR]
    se = np.sqrt(np.maximum(r["var"], 1e-30) / n)
    z = (r["mean"] - xf) / se
    assert np.max(np.abs(z)) < 5.0
    assert np.linalg.norm(r["mean"] - xf) / np.linalg.norm(xf) < 3 * np.sqrt(np.mean(r["var"]) / n) \
        * np.sqrt(xf.size) / np.linalg.norm(xf) + 1e-12


@pytest.mark.slow
def test_rht_sr_hw_unbiased_over_seeds():
    """The hardware-rounded mode is unbiased too: over 4000 seeds the mean of
    the de-rotated dequantized tensor matches the input within 5 standard
    errors (the rounding keeps a downward bias below gap / 2^16 per element,
    far under the standard error here)."""
    R, C, n = 16, 64, 4000
    x = synthetic.bf16_bits(synthetic.normal_with_entry_outliers(R, C, seed=32))
    xf = f32(x).astype(np.float64)
    acc = np.zeros((R, C))
    acc2 = np.zeros((R, C))
    for seed in range(n):
        out = oracle.quantize(x, oracle.RHT_SR_HW, oracle.ROWWISE, seed=seed)
        back = oracle.dequantize(out["codes_row"], out["scales_row"], out["alpha_row"], R, C,
                                 oracle.INVERSE_RHT, seed).astype(np.float64)
        acc += back
        acc2 += back ** 2
    mean = acc / n
    se = np.sqrt(np.maximum(acc2 / n - mean ** 2, 1e-30) / n)
    assert np.max(np.abs((mean - xf) / se)) < 5.0


@pytest.mark.slow
def test_ms_eden_unbiased_inner_product(seeds_runs):
    xf, n, res = seeds_runs
    ratios = res[oracle.MS_EDEN]["ratios"]
    m = ratios.mean(0)
    se = ratios.std(0) / np.sqrt(n)
    assert np.max(np.abs((m - 1) / np.maximum(se, 1e-12))) < 5.0


@pytest.mark.slow
def test_ms_eden_error_at_least_twice_lower_than_sr(seeds_runs):
    """Quartet II page, §一: MS-EDEN has more than 2x lower quantization error
    than element-wise stochastic rounding."""
    xf, n, res = seeds_runs
    print("MSE ratio SR / MS-EDEN:", res[oracle.RHT_SR]["mse"] / res[oracle.MS_EDEN]["mse"])
    assert res[oracle.MS_EDEN]["mse"] <= 0.5 * res[oracle.RHT_SR]["mse"]


# --------------------------------------------------------------------------
# errors and degenerate cases
# --------------------------------------------------------------------------
def test_nonfinite_input_is_reported():
    x = np.zeros((16, 32), np.uint16)
    x[3, 7] = 0x7FC0  # NaN
    with pytest.raises(oracle.OracleError) as e:
        oracle.quantize(x, oracle.RTN, oracle.ROWWISE)
    assert e.value.status == oracle.ERR_NONFINITE
    x[3, 7] = 0xFF80  # -Inf
    with pytest.raises(oracle.OracleError):
        oracle.quantize(x, oracle.FOUR_SIX, oracle.COLWISE)


def test_shape_and_argument_errors():
    x = np.zeros((16, 40), np.uint16)
    with pytest.raises(oracle.OracleError) as e:
        oracle.quantize(x, oracle.RTN, oracle.ROWWISE)  # C % 16 != 0
    assert e.value.status == oracle.ERR_SHAPE
    with pytest.raises(oracle.OracleError) as e:
        oracle.quantize(np.zeros((16, 32), np.uint16), oracle.RHT_SR,
                        oracle.ROWWISE | oracle.BLOCK2D)
    assert e.value.status == oracle.ERR_ARG
    with pytest.raises(oracle.OracleError):
        oracle.quantize(np.zeros((16, 32), np.uint16), oracle.RTN, oracle.ROWWISE,
                        alpha=float("nan"))


def test_all_zero_tensor_gives_zero_scale_and_signed_zero_codes():
    x = np.zeros((16, 32), np.uint16)
    x[0, 1] = 0x8000  # -0.0
    for mode in range(5):
        out = oracle.quantize(x, mode, oracle.ROWWISE, seed=1)
        assert out["alpha_row"] == 0.0
        assert (out["scales_row"] == 0).all()
        c = unpack(out["codes_row"])
        assert ((c & 7) == 0).all()


def test_ranges_reproduce_full_tensor(pr1):
    x = pr1["x"]
    for mode in range(5):
        full = oracle.quantize(x, mode, oracle.ROWWISE | oracle.COLWISE, seed=3, stream_id=2)
        cr, sr = oracle.quantize_1d_range(x, 0, mode, 0, 3, 2, full["alpha_row"], 40, 77)
        assert np.array_equal(cr, full["codes_row"][40:77])
        assert np.array_equal(sr, full["scales_row"][40:77])
        cc, sc = oracle.quantize_1d_range(x, 1, mode, 0, 3, 2, full["alpha_col"], 100, 333)
        assert np.array_equal(cc, full["codes_col"][100:333])
        assert np.array_equal(sc, full["scales_col"][100:333])


def test_stream_ids_and_seeds_change_the_noise(pr1):
    x = pr1["x"]
    a = oracle.quantize(x, oracle.RHT_SR, oracle.ROWWISE, seed=3, stream_id=0)
    b = oracle.quantize(x, oracle.RHT_SR, oracle.ROWWISE, seed=3, stream_id=1)
    c = oracle.quantize(x, oracle.RHT_SR, oracle.ROWWISE, seed=3, stream_id=0)
    assert not np.array_equal(a["codes_row"], b["codes_row"])
    assert np.array_equal(a["codes_row"], c["codes_row"])


def test_headroom_alpha_keeps_the_four_candidate_in_range():
    """Four Over Six (§2.1 Eq. 1-2, §1 Table 1) with the plain tensor scale
    amax / (6 * 448): a block whose maximum exceeds 2/3 of the tensor amax gets
    an M = 4 raw scale above 448, which E4M3 clips.  With the headroom scale
    amax / (4 * 448) no M = 4 raw scale passes 448 (beyond the rounding of
    alpha).  Either way every stored scale is one of the block's two
    candidates, computed here in float32 from the block maxima."""
    from nvfp4_block_quantization_amax_b200 import synthetic
    x = synthetic.normal_with_channel_outliers(64, 256, seed=11)
    bits = synthetic.bf16_bits(x)
    vals = (bits.astype(np.uint32) << 16).view(np.float32)
    amax_b = np.abs(vals.reshape(-1, 16)).max(axis=1).astype(np.float32)
    for flags, expect_clip in ((oracle.ROWWISE, True), (oracle.ROWWISE | oracle.HEADROOM, False)):
        out = oracle.quantize(bits, 1, flags)
        a = np.float32(out["alpha_row"])
        amax = np.float32(out["amax_row"])
        assert a == (amax / np.float32(1792 if flags & oracle.HEADROOM else 2688))
        raw4 = amax_b / np.float32(a * np.float32(4))
        raw6 = amax_b / np.float32(a * np.float32(6))
        s4 = np.array([oracle.e4m3_rne(float(r)) for r in raw4])
        s6 = np.array([oracle.e4m3_rne(float(r)) for r in raw6])
        chosen = out["scales_row"].reshape(-1)
        assert np.all((chosen == s4) | (chosen == s6))
        assert bool(np.any(raw4 > 448 * (1 + 2 ** -20))) == expect_clip
        if not expect_clip:
            assert np.any(chosen == s4)  # the M = 4 candidate still wins somewhere
