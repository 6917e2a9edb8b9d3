"""GPU parity of nvfp4_quantize / nvfp4_dequantize against the CPU oracle.

Codes, scales and the tensor scale must match bit for bit in every mode, on
the same seeded inputs; the library is called through its C ABI (ctypes).
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_quantization_amax_b200 import synthetic

pytestmark = pytest.mark.gpu

ROW, COL, B2D, RHT, GEMM = 0x1, 0x2, 0x4, 0x40, 0x20
HEADROOM = 0x200
MODES = {"rtn": 0, "four_six": 1, "rht_sr": 2, "ms_eden": 3, "rht_sr_hw": 4}


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_block_quantization_amax_b200 import api as _api
    return _api


def gemm_to_plain(flat, rows, kb):
    """Undo the tcgen05 scale layout: -> [rows, kb]."""
    m = np.arange(rows)[:, None]
    j = np.arange(kb)[None, :]
    off = ((m >> 7) * (kb >> 2) + (j >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (j & 3)
    return np.asarray(flat)[off]


def run_both(api, x_t, mode, flags, seed=0, stream_id=0, alpha=None):
    """Quantize on the GPU and in the oracle; return (gpu dict, oracle dict)."""
    x_dev = x_t.cuda()
    a_dev = None if alpha is None else torch.tensor([alpha], dtype=torch.float32, device="cuda")
    q = api.nvfp4_quantize(x_dev, mode, flags, seed=seed, stream_id=stream_id, alpha=a_dev)
    torch.cuda.synchronize()
    bits = synthetic.bf16_bits(x_t)
    o = oracle.quantize(bits, mode, flags & (ROW | COL | B2D | RHT | HEADROOM), seed=seed, stream_id=stream_id,
                        alpha=alpha)
    g = {}
    R, C = x_t.shape
    if flags & ROW:
        g["codes_row"] = q.codes_row.cpu().numpy()
        s = q.scales_row.cpu().numpy()
        if flags & GEMM:
            s = gemm_to_plain(s, R, C // 16)
            if flags & B2D:
                s = s[::16]  # one row of each 16-row group carries the 2D scale
        g["scales_row"] = s
        g["alpha_row"] = float(q.alpha_row.item())
    if flags & COL:
        g["codes_col"] = q.codes_col.cpu().numpy()
        s = q.scales_col.cpu().numpy()
        if flags & GEMM:
            s = gemm_to_plain(s, C, R // 16)
            if flags & B2D:
                s = s[::16]
        g["scales_col"] = s
        g["alpha_col"] = float(q.alpha_col.item())
    g["amax"] = q.amax.cpu().numpy()
    return g, o, q


def assert_same(g, o, flags):
    for side in ("row", "col"):
        if not flags & (ROW if side == "row" else COL):
            continue
        assert g[f"alpha_{side}"] == o[f"alpha_{side}"], side
        sg, so = g[f"scales_{side}"], o[f"scales_{side}"]
        assert sg.shape == so.shape
        bad = np.argwhere(sg != so)
        assert bad.size == 0, f"{side} scales differ at {bad[:5].tolist()} ({sg[tuple(bad[0])]} vs {so[tuple(bad[0])]})"
        cg, co = g[f"codes_{side}"], o[f"codes_{side}"]
        bad = np.argwhere(cg != co)
        assert bad.size == 0, f"{side} codes differ at {bad[:5].tolist()} ({cg[tuple(bad[0])]:#x} vs {co[tuple(bad[0])]:#x})"


@pytest.fixture(scope="module")
def pr1():
    return synthetic.pr1()


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("orient", ["row", "col", "dual"])
def test_pr1_all_modes(api, pr1, mode, orient):
    flags = {"row": ROW, "col": COL, "dual": ROW | COL}[orient]
    g, o, _ = run_both(api, pr1["x"], MODES[mode], flags, seed=1234, stream_id=3)
    assert_same(g, o, flags)


@pytest.mark.parametrize("mode", ["rtn", "four_six"])
@pytest.mark.parametrize("orient", ["row", "col", "dual"])
def test_pr1_rotated_rtn_and_four_six(api, pr1, mode, orient):
    flags = {"row": ROW, "col": COL, "dual": ROW | COL}[orient] | RHT
    g, o, _ = run_both(api, pr1["x"], MODES[mode], flags, seed=77)
    assert_same(g, o, flags)


@pytest.mark.parametrize("mode", ["rtn", "four_six"])
@pytest.mark.parametrize("orient", ["row", "col", "dual"])
def test_2d_weight_blocks(api, pr1, mode, orient):
    flags = {"row": ROW, "col": COL, "dual": ROW | COL}[orient] | B2D
    g, o, _ = run_both(api, pr1["w"], MODES[mode], flags)
    assert_same(g, o, flags)


@pytest.mark.parametrize("shape", [(48, 144), (16, 16), (80, 272), (37, 48), (1, 16)])
@pytest.mark.parametrize("mode", list(MODES))
def test_ragged_tiles(api, shape, mode):
    R, C = shape
    x = synthetic.normal_with_entry_outliers(R, C, seed=R * 1000 + C)
    flags = ROW | COL if R % 16 == 0 else ROW
    g, o, _ = run_both(api, x, MODES[mode], flags, seed=5)
    assert_same(g, o, flags)


@pytest.mark.parametrize("mode", list(MODES))
def test_gemm_scale_layout(api, mode):
    x = synthetic.normal_with_channel_outliers(256, 384, seed=8)
    flags = ROW | COL | GEMM
    g, o, _ = run_both(api, x, MODES[mode], flags, seed=9)
    assert_same(g, o, flags)


@pytest.mark.parametrize("mode", ["rtn", "four_six"])
def test_gemm_scale_layout_2d(api, pr1, mode):
    flags = ROW | COL | GEMM | B2D
    g, o, q = run_both(api, pr1["w"], MODES[mode], flags)
    assert_same(g, o, flags)
    # every row of a 16-row group carries its tile's scale
    R, C = pr1["w"].shape
    full = gemm_to_plain(q.scales_row.cpu().numpy(), R, C // 16)
    assert np.array_equal(full, np.repeat(o["scales_row"], 16, 0))


def test_alpha_provided_exercises_every_bf16_value(api):
    # blocks [6, v1..v15] with alpha = 1: Delta = 1, so y = v for every bf16
    # v in [-6, 6] -- the value encoder sees all of them, ties included.
    bits = np.arange(65536, dtype=np.uint32)
    vals = (bits << 16).view(np.float32)
    vals = vals[np.isfinite(vals) & (np.abs(vals) <= 6)]
    n = -(-len(vals) // 15)
    pad = np.zeros(n * 15, np.float32)
    pad[:len(vals)] = vals
    blocks = np.concatenate([np.full((n, 1), 6.0, np.float32), pad.reshape(n, 15)], axis=1)
    R = -(-n // 64)
    arr = np.zeros((R * 64, 16), np.float32)
    arr[:n] = blocks
    x = synthetic.to_bf16(arr.reshape(R * 16, 64))
    for mode in ("rtn", "four_six"):
        g, o, _ = run_both(api, x, MODES[mode], ROW, alpha=1.0)
        assert_same(g, o, ROW)


def test_zero_tensor_and_negative_zero(api):
    x = torch.zeros((32, 64), dtype=torch.bfloat16)
    x[3, 5] = -0.0
    for mode in MODES.values():
        g, o, _ = run_both(api, x, mode, ROW | COL, seed=2)
        assert_same(g, o, ROW | COL)


def test_tiny_values_subnormal_scales(api):
    rng = np.random.default_rng(3)
    a = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-30, 0, (64, 1)))).astype(np.float32)
    x = synthetic.to_bf16(a)
    for mode in MODES.values():
        g, o, _ = run_both(api, x, mode, ROW | COL, seed=4)
        assert_same(g, o, ROW | COL)


def test_nonfinite_sets_status(api):
    x = torch.randn(64, 128, dtype=torch.bfloat16, device="cuda")
    x[7, 9] = float("nan")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.nvfp4_quantize(x, 0, ROW, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -4
    x[7, 9] = float("inf")
    status.zero_()
    api.nvfp4_quantize(x, 2, COL, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -4
    status.zero_()
    api.nvfp4_quantize(x, 1, ROW, alpha=torch.ones(1, device="cuda"), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -4


def test_host_errors_return_before_launch(api):
    from nvfp4_block_quantization_amax_b200 import _lib as L
    x = torch.randn(64, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(api.NVFP4Error) as e:
        api.nvfp4_quantize(x[:, :120], 0, ROW)
    assert e.value.status == L.NVFP4_ERR_SHAPE
    with pytest.raises(api.NVFP4Error) as e:
        api.nvfp4_quantize(x, 2, ROW | B2D)
    assert e.value.status == L.NVFP4_ERR_ARG
    with pytest.raises(api.NVFP4Error) as e:
        api.nvfp4_quantize(x[:, 8:], 0, ROW)
    assert e.value.status in (L.NVFP4_ERR_ALIGN, L.NVFP4_ERR_SHAPE)
    assert api.nvfp4_quantize(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"), 0, ROW) is not None


def test_strided_input(api, pr1):
    big = torch.zeros((256, 1024 + 64), dtype=torch.bfloat16)
    big[:, :1024] = pr1["x"]
    view = big.cuda()[:, :1024]
    q = api.nvfp4_quantize(view, 1, ROW | COL, seed=3)
    torch.cuda.synchronize()
    o = oracle.quantize(synthetic.bf16_bits(pr1["x"]), 1, ROW | COL, seed=3)
    assert np.array_equal(q.codes_row.cpu().numpy(), o["codes_row"])
    assert np.array_equal(q.codes_col.cpu().numpy(), o["codes_col"])


# ------------------------------------------------------------------ dequant
@pytest.mark.parametrize("mode", list(MODES))
def test_dequantize_matches_oracle(api, pr1, mode):
    x = pr1["x"]
    R, C = x.shape
    m = MODES[mode]
    q = api.nvfp4_quantize(x.cuda(), m, ROW, seed=11)
    inv = 0x80 if m >= 2 else 0
    y = api.nvfp4_dequantize(q.codes_row, q.scales_row, q.alpha_row, R, C, inv, seed=11)
    yb = api.nvfp4_dequantize(q.codes_row, q.scales_row, q.alpha_row, R, C, inv | 0x100, seed=11)
    torch.cuda.synchronize()
    want = oracle.dequantize(q.codes_row.cpu().numpy(), q.scales_row.cpu().numpy(),
                             float(q.alpha_row.item()), R, C, inv, seed=11)
    assert np.array_equal(y.cpu().numpy(), want)
    assert torch.equal(yb.cpu(), torch.from_numpy(want).to(torch.bfloat16))


def test_dequantize_2d_and_gemm_layout(api, pr1):
    w = pr1["w"]
    R, C = w.shape
    q = api.nvfp4_quantize(w.cuda(), 1, ROW | B2D)
    y = api.nvfp4_dequantize(q.codes_row, q.scales_row, q.alpha_row, R, C, B2D)
    qg = api.nvfp4_quantize(w.cuda(), 1, ROW | B2D | GEMM)
    yg = api.nvfp4_dequantize(qg.codes_row, qg.scales_row, qg.alpha_row, R, C, GEMM)
    torch.cuda.synchronize()
    want = oracle.dequantize(q.codes_row.cpu().numpy(), q.scales_row.cpu().numpy(),
                             float(q.alpha_row.item()), R, C, B2D)
    assert np.array_equal(y.cpu().numpy(), want)
    assert np.array_equal(yg.cpu().numpy(), want)


# ------------------------------------------------- full sizes, sampled rows
def _sampled_rows_check(api, x_t, mode, flags, seed, stream_id, nsample=24):
    R, C = x_t.shape
    q = api.nvfp4_quantize(x_t.cuda(), mode, flags, seed=seed, stream_id=stream_id)
    torch.cuda.synchronize()
    bits = synthetic.bf16_bits(x_t)
    rng = np.random.default_rng(seed)
    rot = mode >= 2 or bool(flags & RHT)
    for side, orient in (("row", 0), ("col", 1)):
        if not flags & (ROW if side == "row" else COL):
            continue
        amax = oracle.amax(bits, orient, rot, seed)
        alpha = oracle.alpha_from_amax(amax)
        assert float(getattr(q, f"alpha_{side}").item()) == alpha
        n = R if orient == 0 else C
        picks = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, nsample)]))
        codes = getattr(q, f"codes_{side}")
        scales = getattr(q, f"scales_{side}")
        for v in picks:
            c_o, s_o = oracle.quantize_1d_range(bits, orient, mode, flags & RHT, seed, stream_id,
                                                alpha, int(v), int(v) + 1)
            assert np.array_equal(codes[v].cpu().numpy(), c_o[0]), (side, v)
            assert np.array_equal(scales[v].cpu().numpy(), s_o[0]), (side, v)


@pytest.fixture(scope="module")
def layer8b():
    return synthetic.fwd_bwd_8b()


def test_full_size_activation_four_six(api, layer8b):
    _sampled_rows_check(api, layer8b["x"], 1, ROW, seed=0, stream_id=0)


@pytest.mark.parametrize("mode", [2, 3])
def test_full_size_gradient_dual(api, layer8b, mode):
    _sampled_rows_check(api, layer8b["dy"], mode, ROW | COL, seed=1000 + mode, stream_id=1)


def test_full_size_weight_2d(api, layer8b):
    w = layer8b["w"]
    R, C = w.shape
    q = api.nvfp4_quantize(w.cuda(), 1, ROW | COL | B2D, seed=0)
    torch.cuda.synchronize()
    bits = synthetic.bf16_bits(w)
    alpha = oracle.alpha_from_amax(oracle.amax(bits))
    assert float(q.alpha_row.item()) == alpha
    for br in (0, 17, R // 16 - 1):
        cr, sr, cc, sc = oracle.quantize_2d_range(bits, 1, alpha, br, br + 1)
        assert np.array_equal(q.codes_row[16 * br:16 * br + 16].cpu().numpy(), cr)
        assert np.array_equal(q.scales_row[br].cpu().numpy(), sr[0])
        assert np.array_equal(q.codes_col[:, 8 * br:8 * br + 8].cpu().numpy(), cc)
        assert np.array_equal(q.scales_col[:, br].cpu().numpy(), sc[:, 0])


def test_full_size_rotated_rtn_requantization(api, layer8b):
    # the partner operands of the rotated backward GEMMs: W along its output
    # features, X along tokens (columns), RTN with the gradient's sign vector
    _sampled_rows_check(api, layer8b["w"], 0, COL | RHT, seed=1002, stream_id=2, nsample=8)
    _sampled_rows_check(api, layer8b["x"], 0, COL | RHT, seed=1002, stream_id=3, nsample=8)


# ---------------------------------------------------------------------------
# Single pass (NVFP4_SINGLE_PASS): amax, a grid barrier and the quantization
# in one cooperative launch.  Same results as the two-pass path, bit for bit,
# so the same oracle comparisons apply.
# ---------------------------------------------------------------------------
SP = 0x8


def assert_amax(g, o, flags):
    if flags & ROW:
        assert float(g["amax"][0]) == o["amax_row"]
    if flags & COL:
        assert float(g["amax"][1]) == o["amax_col"]


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("orient", ["row", "col", "dual"])
def test_single_pass_all_modes(api, pr1, mode, orient):
    flags = {"row": ROW, "col": COL, "dual": ROW | COL}[orient] | SP
    g, o, _ = run_both(api, pr1["x"], MODES[mode], flags, seed=1234, stream_id=3)
    assert_same(g, o, flags)
    assert_amax(g, o, flags)


@pytest.mark.parametrize("mode", ["rtn", "four_six"])
@pytest.mark.parametrize("extra", [RHT, B2D, B2D | GEMM])
def test_single_pass_rotated_and_2d(api, pr1, mode, extra):
    flags = ROW | COL | SP | extra
    x = pr1["w"] if extra & B2D else pr1["x"]
    g, o, _ = run_both(api, x, MODES[mode], flags, seed=77)
    assert_same(g, o, flags)


@pytest.mark.parametrize("shape", [(48, 144), (37, 48), (1, 16), (80, 272), (1040, 1552)])
@pytest.mark.parametrize("mode", list(MODES))
def test_single_pass_ragged_and_many_tiles(api, shape, mode):
    R, C = shape
    x = synthetic.normal_with_entry_outliers(R, C, seed=R * 1000 + C + 1)
    flags = (ROW | COL if R % 16 == 0 else ROW) | SP
    g, o, _ = run_both(api, x, MODES[mode], flags, seed=6, stream_id=2)
    assert_same(g, o, flags)
    assert_amax(g, o, flags)


def test_single_pass_equals_two_pass_full_size(api, layer8b):
    # the dY dual MS-EDEN call of the step, GEMM scale layout, both ways
    dy = layer8b["dy"].cuda()
    flags = ROW | COL | GEMM
    a = api.nvfp4_quantize(dy, 3, flags, seed=11, stream_id=1)
    b = api.nvfp4_quantize(dy, 3, flags | SP, seed=11, stream_id=1)
    torch.cuda.synchronize()
    for name in ("codes_row", "scales_row", "alpha_row", "codes_col", "scales_col", "alpha_col", "amax"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    # and sampled rows of it against the oracle
    _sampled_rows_check(api, layer8b["dy"], 3, ROW | COL | SP, seed=12, stream_id=1, nsample=4)


def test_single_pass_nonfinite_sets_status(api):
    x = torch.randn(64, 128, dtype=torch.bfloat16, device="cuda")
    x[5, 3] = float("nan")
    for mode, flags in ((0, ROW), (3, ROW | COL), (1, ROW | B2D)):
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        api.nvfp4_quantize(x, mode, flags | SP, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == -4, (mode, flags)


@pytest.mark.parametrize("mode,flags", [(3, ROW | COL), (1, ROW), (1, ROW | B2D), (0, COL | RHT)])
def test_single_pass_barrier_timeout_sets_status(api, pr1, monkeypatch, mode, flags):
    # A barrier limit of 0 ns makes the wait run out for every CTA that is not
    # the last to arrive (the grid always has more than one CTA): the call
    # returns, the status word says NVFP4_ERR_TIMEOUT, and the next call with
    # the default limit is bit-exact with the oracle again.
    from nvfp4_block_quantization_amax_b200 import _lib as L
    x = pr1["w"] if flags & B2D else pr1["x"]
    xd = x.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    monkeypatch.setenv("NVFP4_BARRIER_TIMEOUT_NS", "0")
    api.nvfp4_quantize(xd, mode, flags | SP, seed=9, stream_id=1, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == L.NVFP4_ERR_TIMEOUT
    monkeypatch.delenv("NVFP4_BARRIER_TIMEOUT_NS")
    status.zero_()
    g, o, _ = run_both(api, x, mode, flags | SP, seed=9, stream_id=1)
    assert_same(g, o, flags)
    api.nvfp4_quantize(xd, mode, flags | SP, seed=9, stream_id=1, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_single_pass_workspace_is_scratch(api, pr1):
    # the barrier counter is cleared by the call itself: a workspace full of
    # garbage, reused call after call, gives the same result
    x = pr1["x"].cuda()
    R, C = x.shape
    ws = torch.full((api.workspace_for(R, C, ROW | COL | SP, x.device).numel(),), 0x7B,
                    dtype=torch.uint8, device="cuda")
    ref = api.nvfp4_quantize(x, 3, ROW | COL, seed=3)
    for _ in range(3):
        q = api.nvfp4_quantize(x, 3, ROW | COL | SP, seed=3, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(q.codes_row, ref.codes_row) and torch.equal(q.codes_col, ref.codes_col)
        assert torch.equal(q.scales_row, ref.scales_row) and torch.equal(q.scales_col, ref.scales_col)


def test_four_six_near_tie_blocks(api):
    # Two blocks of the 4096 x 1024 sweep tensor whose M = 4 and M = 6 squared
    # errors lie two ulps apart (0.119696319 vs 0.119696334 for the first):
    # the selector must see exactly the oracle's rounded products q * s.
    blocks = [[0.337890625, -1.2109375, 0.5078125, -1.8515625, -0.056640625, -1.5390625, -0.328125, 0.462890625,
               -1.828125, 0.294921875, -0.9453125, 0.6796875, -0.45703125, 0.400390625, 1.1015625, 0.447265625],
              [-1.578125, 0.05615234375, -1.03125, 1.046875, -2.203125, 0.26171875, 0.90625, -0.10595703125,
               -1.265625, 0.65234375, -0.5234375, -0.1689453125, 0.69921875, -0.478515625, 0.93359375, -0.99609375]]
    alpha = float(np.float32(0.0714285746216774))
    a = np.zeros((64, 128), np.float32)
    a[0, :16], a[33, 32:48] = blocks[0], blocks[1]   # rows 0 / 33: both lanes of a row pair
    a[17, 16:32] = blocks[1]
    x = synthetic.to_bf16(a)
    for flags in (ROW, ROW | COL, COL):
        g, o, _ = run_both(api, x if flags != COL else synthetic.to_bf16(a.T.copy()), 1, flags, alpha=alpha)
        assert_same(g, o, flags)


# ---------------------------------------------------------------------------
# Headroom tensor scale (NVFP4_HEADROOM): alpha = amax / (4 * 448).
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("orient", ["row", "col", "dual"])
def test_headroom_all_modes(api, pr1, mode, orient):
    flags = {"row": ROW, "col": COL, "dual": ROW | COL}[orient] | HEADROOM
    g, o, _ = run_both(api, pr1["x"], MODES[mode], flags, seed=99, stream_id=2)
    assert_same(g, o, flags)


@pytest.mark.parametrize("extra", [B2D, B2D | SP, SP, SP | RHT])
def test_headroom_four_six_2d_and_single_pass(api, pr1, extra):
    flags = ROW | COL | HEADROOM | extra
    x = pr1["w"] if extra & B2D else pr1["x"]
    g, o, _ = run_both(api, x, MODES["four_six"], flags, seed=8)
    assert_same(g, o, flags)


@pytest.mark.parametrize("mode", ["rtn", "four_six", "ms_eden"])
@pytest.mark.parametrize("eps", [2.0 ** -22, -(2.0 ** -23), 0.0])
def test_scale_rounding_near_e4m3_midpoints(api, mode, eps):
    # alpha = 0.5 (1 + eps) makes the M = 6 divisor 3 (1 + eps): block maxima
    # 3 m, m an E4M3 rounding midpoint, give quotients within a few ulps of m
    # (eps = 0: exactly m, a tie).  The scale must still round as the oracle's
    # correctly rounded quotient does.
    alpha = float(np.float32(0.5) * np.float32(1.0 + eps))
    mids = [1.0625, 1.1875, 1.3125, 1.4375, 1.5625, 1.6875, 1.8125, 1.9375, 0.53125, 2.125, 4.25, 9.5,
            19.0, 38.0, 0.28125, 0.140625]
    rng = np.random.default_rng(17)
    a = (rng.standard_normal((64, 256)) * 0.1).astype(np.float32)
    blocks = a.reshape(64, 16, 16)
    for r in range(64):
        for b in range(16):
            m = mids[(r + b) % len(mids)]
            blocks[r, b, (r * 7 + b) % 16] = np.float32(3.0 * m) * (1 if (r + b) % 3 else -1)
            blocks[r, b] = np.clip(blocks[r, b], -abs(3.0 * m), abs(3.0 * m))
    x = synthetic.to_bf16(blocks.reshape(64, 256))
    for flags in (ROW, ROW | COL):
        g, o, _ = run_both(api, x, MODES[mode], flags, seed=13, alpha=alpha)
        assert_same(g, o, flags)
