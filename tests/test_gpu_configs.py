"""GPU parity on the two remaining named workloads, against the CPU oracle.

* Quantizer sweep: bf16 4096 x N, N(0,1) with 0.1% channel outliers x50.
  Small N are compared in full in every mode, two-pass and single-pass;
  a large N on sampled rows and columns.
* 12B-hybrid-shaped linear step: tokens 16384, hidden 5120, FFN 20480.  The
  up-projection's fprop / dgrad / wgrad and the down-projection's fprop, on
  sampled output entries at full K (FP64 oracle product), with the operands
  the step uses (4/6 1D activations, 4/6 2D weights, MS-EDEN or RHT+SR
  gradients, rotated RTN partner operands).
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_quantization_amax_b200 import synthetic

pytestmark = pytest.mark.gpu

ROW, COL, B2D, SP, RHT, GEMM = 0x1, 0x2, 0x4, 0x8, 0x40, 0x20
FP32 = 1
FROB_TOL = 1e-5
MODES = {"rtn": 0, "four_six": 1, "rht_sr": 2, "ms_eden": 3, "rht_sr_hw": 4}


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_block_quantization_amax_b200 import api as _api
    return _api


def frob(D, ref):
    return float(np.linalg.norm(D.astype(np.float64) - ref) / np.linalg.norm(ref))


# ------------------------------------------------------------------ sweep
@pytest.mark.parametrize("n", [256, 1024])
@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("single", [False, True])
def test_sweep_small_full(api, n, mode, single):
    x = synthetic.sweep(n, seed=n)
    flags = ROW | COL | (SP if single else 0)
    q = api.nvfp4_quantize(x.cuda(), MODES[mode], flags, seed=21, stream_id=4)
    torch.cuda.synchronize()
    o = oracle.quantize(synthetic.bf16_bits(x), MODES[mode], ROW | COL, seed=21, stream_id=4)
    for side in ("row", "col"):
        assert float(getattr(q, f"alpha_{side}").item()) == o[f"alpha_{side}"], side
        assert np.array_equal(getattr(q, f"scales_{side}").cpu().numpy(), o[f"scales_{side}"]), side
        assert np.array_equal(getattr(q, f"codes_{side}").cpu().numpy(), o[f"codes_{side}"]), side


@pytest.mark.parametrize("mode,flags", [(1, ROW), (3, ROW | COL), (0, COL | RHT)])
def test_sweep_4096_full(api, mode, flags):
    x = synthetic.sweep(4096, seed=4096)
    q = api.nvfp4_quantize(x.cuda(), mode, flags | SP, seed=22, stream_id=5)
    torch.cuda.synchronize()
    o = oracle.quantize(synthetic.bf16_bits(x), mode, flags, seed=22, stream_id=5)
    for side, bit in (("row", ROW), ("col", COL)):
        if flags & bit:
            assert np.array_equal(getattr(q, f"codes_{side}").cpu().numpy(), o[f"codes_{side}"]), side
            assert np.array_equal(getattr(q, f"scales_{side}").cpu().numpy(), o[f"scales_{side}"]), side


def test_sweep_16384_sampled(api):
    n = 16384
    x = synthetic.sweep(n, seed=n)
    bits = synthetic.bf16_bits(x)
    rng = np.random.default_rng(7)
    for mode, flags in ((3, ROW | COL), (1, ROW)):
        for sp in (0, SP):
            q = api.nvfp4_quantize(x.cuda(), mode, flags | sp, seed=23, stream_id=6)
            torch.cuda.synchronize()
            for side, orient, bit in (("row", 0, ROW), ("col", 1, COL)):
                if not flags & bit:
                    continue
                rot = mode >= 2
                alpha = oracle.alpha_from_amax(oracle.amax(bits, orient, rot, 23))
                assert float(getattr(q, f"alpha_{side}").item()) == alpha
                lim = x.shape[orient]
                for v in np.unique(np.concatenate([[0, lim - 1], rng.integers(0, lim, 6)])):
                    c, s = oracle.quantize_1d_range(bits, orient, mode, 0, 23, 6, alpha, int(v), int(v) + 1)
                    assert np.array_equal(getattr(q, f"codes_{side}")[v].cpu().numpy(), c[0]), (mode, side, v)
                    assert np.array_equal(getattr(q, f"scales_{side}")[v].cpu().numpy(), s[0]), (mode, side, v)


# ------------------------------------------------------------- 12B step
@pytest.fixture(scope="module")
def step12b():
    return synthetic.step_12b(seed=5)


def _row_operand(bits, orient, mode, rot_flag, seed, sid, idx):
    rot = mode >= 2 or bool(rot_flag)
    alpha = oracle.alpha_from_amax(oracle.amax(bits, orient, rot, seed))
    codes, scales = [], []
    for v in idx:
        c, s = oracle.quantize_1d_range(bits, orient, mode, rot_flag, seed, sid, alpha, int(v), int(v) + 1)
        codes.append(c[0])
        scales.append(s[0])
    return np.stack(codes), np.stack(scales), alpha


def _weight_2d_rows(bits, rows):
    alpha = oracle.alpha_from_amax(oracle.amax(bits))
    codes, scales = [], []
    for n in rows:
        cr, sr, _, _ = oracle.quantize_2d_range(bits, 1, alpha, int(n) // 16, int(n) // 16 + 1)
        codes.append(cr[int(n) % 16])
        scales.append(sr[0])
    return np.stack(codes), np.stack(scales), alpha


def _check(D, rows, cols, A, B, K, what):
    ref = oracle.gemm_f64(A[0], A[1], A[2], B[0], B[1], B[2], len(rows), len(cols), K)
    got = D.cpu().numpy()[np.ix_(rows, cols)]
    e = frob(got, ref)
    print(f"{what}: frob {e:.2e}")
    assert e <= FROB_TOL, what


def test_12b_up_projection_fprop(api, step12b):
    x, w = step12b["x"], step12b["w"]                  # [16384, 5120], [20480, 5120]
    qx = api.nvfp4_quantize(x.cuda(), 1, ROW | GEMM)
    qw = api.nvfp4_quantize(w.cuda(), 1, ROW | B2D | GEMM)
    D = api.nvfp4_gemm(qx.codes_row, qx.scales_row, qx.alpha_row, qw.codes_row, qw.scales_row, qw.alpha_row,
                       out_dtype=FP32)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(x.shape[0], 32, replace=False))
    cols = np.sort(rng.choice(w.shape[0], 32, replace=False))
    A = _row_operand(synthetic.bf16_bits(x), 0, 1, 0, 0, 0, rows)
    B = _weight_2d_rows(synthetic.bf16_bits(w), cols)
    _check(D, rows, cols, A, B, x.shape[1], "12B fprop")


@pytest.mark.parametrize("mode", [2, 3])
def test_12b_up_projection_dgrad_wgrad(api, step12b, mode):
    x, w, dy = step12b["x"], step12b["w"], step12b["dy"]   # dy [16384, 20480]
    seed = 3000 + mode
    qdy = api.nvfp4_quantize(dy.cuda(), mode, ROW | COL | GEMM, seed=seed, stream_id=0)
    qwt = api.nvfp4_quantize(w.cuda(), 0, COL | RHT | GEMM, seed=seed, stream_id=1)
    dX = api.nvfp4_gemm(qdy.codes_row, qdy.scales_row, qdy.alpha_row, qwt.codes_col, qwt.scales_col,
                        qwt.alpha_col, out_dtype=FP32)           # [16384, 5120], K = 20480
    qxt = api.nvfp4_quantize(x.cuda(), 0, COL | RHT | GEMM, seed=seed, stream_id=2)
    dW = api.nvfp4_gemm(qdy.codes_col, qdy.scales_col, qdy.alpha_col, qxt.codes_col, qxt.scales_col,
                        qxt.alpha_col, out_dtype=FP32)           # [20480, 5120], K = 16384
    torch.cuda.synchronize()
    rng = np.random.default_rng(10 + mode)
    dyb, wb, xb = synthetic.bf16_bits(dy), synthetic.bf16_bits(w), synthetic.bf16_bits(x)
    rows = np.sort(rng.choice(dy.shape[0], 24, replace=False))
    cols = np.sort(rng.choice(w.shape[1], 24, replace=False))
    A = _row_operand(dyb, 0, mode, 0, seed, 0, rows)
    B = _row_operand(wb, 1, 0, RHT, seed, 1, cols)
    _check(dX, rows, cols, A, B, dy.shape[1], f"12B dgrad mode {mode}")
    rows = np.sort(rng.choice(dy.shape[1], 24, replace=False))
    cols = np.sort(rng.choice(x.shape[1], 24, replace=False))
    A = _row_operand(dyb, 1, mode, 0, seed, 0, rows)
    B = _row_operand(xb, 1, 0, RHT, seed, 2, cols)
    _check(dW, rows, cols, A, B, dy.shape[0], f"12B wgrad mode {mode}")


def test_12b_down_projection_fprop(api):
    # FFN 20480 -> hidden 5120: activations [16384, 20480], weight [5120, 20480]
    layer = synthetic.layer(16384, 20480, 5120, seed=9)
    x, w = layer["x"], layer["w"]
    qx = api.nvfp4_quantize(x.cuda(), 1, ROW | GEMM)
    qw = api.nvfp4_quantize(w.cuda(), 1, ROW | B2D | GEMM)
    D = api.nvfp4_gemm(qx.codes_row, qx.scales_row, qx.alpha_row, qw.codes_row, qw.scales_row, qw.alpha_row,
                       out_dtype=FP32)
    torch.cuda.synchronize()
    rng = np.random.default_rng(2)
    rows = np.sort(rng.choice(x.shape[0], 24, replace=False))
    cols = np.sort(rng.choice(w.shape[0], 24, replace=False))
    A = _row_operand(synthetic.bf16_bits(x), 0, 1, 0, 0, 0, rows)
    B = _weight_2d_rows(synthetic.bf16_bits(w), cols)
    _check(D, rows, cols, A, B, x.shape[1], "12B down fprop")
