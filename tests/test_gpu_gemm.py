"""GPU parity of nvfp4_gemm against the FP64 oracle product.

D = alphaA alphaB (qA DeltaA)(qB DeltaB)^T.  fp32 output: relative Frobenius
error <= 1e-5 against the FP64 product of the same operands; bf16 output:
within one bf16 ulp of the FP64 product rounded to bf16.  The maximum
elementwise relative error (entries with |D_ref| >= 1e-3 RMS) is reported.
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_quantization_amax_b200 import synthetic

pytestmark = pytest.mark.gpu

ROW, COL, B2D, RHT, GEMM = 0x1, 0x2, 0x4, 0x40, 0x20
FP32, BF16 = 1, 0
FROB_TOL = 1e-5


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_block_quantization_amax_b200 import api as _api
    return _api


def plain_to_gemm(plain):
    """[rows, kb] row-major scales -> the tcgen05 layout (flat)."""
    rows, kb = plain.shape
    m = np.arange(rows)[:, None]
    j = np.arange(kb)[None, :]
    off = ((m >> 7) * (kb >> 2) + (j >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (j & 3)
    out = np.zeros(rows * kb, np.uint8)
    out[off.ravel()] = plain.ravel()
    return out


def rand_operand(rng, rows, K, lo=0x28, hi=0x48):
    codes = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    scales = rng.integers(lo, hi, (rows, K // 16), dtype=np.uint8)
    return codes, scales


def frob(D, ref):
    return float(np.linalg.norm(D.astype(np.float64) - ref) / np.linalg.norm(ref))


def max_rel(D, ref):
    rms = np.sqrt(np.mean(ref ** 2))
    mask = np.abs(ref) >= 1e-3 * rms
    return float(np.max(np.abs(D.astype(np.float64) - ref)[mask] / np.abs(ref[mask])))


def bf16_within_one_ulp(Dbf, ref):
    r = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)
    d = Dbf.float().numpy().astype(np.float64)
    mag = np.maximum(np.abs(r), np.finfo(np.float32).tiny)
    ulp = 2.0 ** (np.floor(np.log2(mag)) - 7)
    return bool(np.all(np.abs(d - r) <= ulp * 1.0000001))


def run_gemm(api, A, sA, aA, B, sB, aB, out_dtype):
    dev = "cuda"
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    D = api.nvfp4_gemm(t(A), t(plain_to_gemm(sA)), torch.tensor([aA], dtype=torch.float32, device=dev),
                       t(B), t(plain_to_gemm(sB)), torch.tensor([aB], dtype=torch.float32, device=dev),
                       out_dtype=out_dtype)
    torch.cuda.synchronize()
    return D.cpu()


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (128, 256, 256), (256, 384, 384), (384, 512, 1024),
                                   (256, 256, 4096), (128, 128, 2048 + 128), (512, 512, 384),
                                   (768, 1024, 2048), (2048, 1536, 256)])
def test_random_operands(api, M, N, K):
    rng = np.random.default_rng(M * 7 + N * 13 + K)
    A, sA = rand_operand(rng, M, K)
    B, sB = rand_operand(rng, N, K)
    aA, aB = 0.75, 1.3125
    ref = oracle.gemm_f64(A, sA, aA, B, sB, aB, M, N, K)
    D = run_gemm(api, A, sA, aA, B, sB, aB, FP32).numpy()
    e = frob(D, ref)
    print(f"M={M} N={N} K={K}: frob {e:.2e} max_rel {max_rel(D, ref):.2e}")
    assert e <= FROB_TOL
    Db = run_gemm(api, A, sA, aA, B, sB, aB, BF16)
    assert bf16_within_one_ulp(Db, ref)


def test_scale_and_value_extremes(api):
    # every E4M3 scale byte and every FP4 code appear; values of both signs
    rng = np.random.default_rng(99)
    M, N, K = 128, 128, 2048
    A, sA = rand_operand(rng, M, K, 0x00, 0x7F)
    B, sB = rand_operand(rng, N, K, 0x00, 0x7F)
    ref = oracle.gemm_f64(A, sA, 1.0, B, sB, 1.0, M, N, K)
    D = run_gemm(api, A, sA, 1.0, B, sB, 1.0, FP32).numpy()
    assert frob(D, ref) <= FROB_TOL


def test_single_scale_position(api):
    # one non-zero scale at a time pins where each (row, K-block) scale is read
    M, N, K = 256, 128, 512
    rng = np.random.default_rng(5)
    A, _ = rand_operand(rng, M, K)
    B, sB = rand_operand(rng, N, K)
    for (m, j) in [(0, 0), (37, 3), (128 + 95, 17), (255, 31), (64, 4)]:
        sA = np.zeros((M, K // 16), np.uint8)
        sA[m, j] = 0x38  # 1.0
        ref = oracle.gemm_f64(A, sA, 1.0, B, sB, 1.0, M, N, K)
        D = run_gemm(api, A, sA, 1.0, B, sB, 1.0, FP32).numpy()
        assert np.count_nonzero(ref) > 0
        assert frob(D, ref) <= FROB_TOL, (m, j)


def test_pr1_quantized_operands(api):
    d = synthetic.pr1()
    x, w = d["x"], d["w"]
    R, C = x.shape
    qa = api.nvfp4_quantize(x.cuda(), 1, ROW | GEMM)
    qw = api.nvfp4_quantize(w.cuda(), 0, ROW | B2D | GEMM)
    for out_dtype in (FP32, BF16):
        D = api.nvfp4_gemm(qa.codes_row, qa.scales_row, qa.alpha_row, qw.codes_row, qw.scales_row,
                           qw.alpha_row, out_dtype=out_dtype)
        torch.cuda.synchronize()
        oa = oracle.quantize(synthetic.bf16_bits(x), 1, ROW)
        ow = oracle.quantize(synthetic.bf16_bits(w), 0, ROW | B2D)
        ref = oracle.gemm_f64(oa["codes_row"], oa["scales_row"], oa["alpha_row"], ow["codes_row"],
                              np.repeat(ow["scales_row"], 16, 0), ow["alpha_row"], R, w.shape[0], C)
        if out_dtype == FP32:
            e = frob(D.cpu().numpy(), ref)
            print(f"PR1 GEMM frob {e:.2e} max_rel {max_rel(D.cpu().numpy(), ref):.2e}")
            assert e <= FROB_TOL
        else:
            assert bf16_within_one_ulp(D.cpu(), ref)


def test_timeout_status_word_stays_zero(api):
    rng = np.random.default_rng(1)
    M = N = K = 256
    A, sA = rand_operand(rng, M, K)
    B, sB = rand_operand(rng, N, K)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    ws = torch.zeros(1, dtype=torch.int32, device="cuda")
    from nvfp4_block_quantization_amax_b200 import _lib as L
    D = torch.empty((M, N), dtype=torch.float32, device="cuda")
    one = torch.ones(1, device="cuda")
    st = L.nvfp4_gemm(t(A).data_ptr(), t(plain_to_gemm(sA)).data_ptr(), one.data_ptr(), t(B).data_ptr(),
                      t(plain_to_gemm(sB)).data_ptr(), one.data_ptr(), M, N, K, D.data_ptr(), FP32, N,
                      ws.data_ptr(), 4, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == 0 and int(ws.item()) == 0


# ------------------------------------------- full 8B-shaped GEMMs, sampled
@pytest.fixture(scope="module")
def layer8b():
    return synthetic.fwd_bwd_8b()


def _sampled_ref(bits_a, flags_a, mode_a, bits_b, flags_b, mode_b, rows, cols, seed=0, sid_a=0, sid_b=1,
                 orient_a=0, orient_b=0):
    """Oracle operands for sampled output rows / columns (1D blocks), FP64
    product.  orient 1 quantizes columns of the source (the transposed use)."""
    def operand(bits, flags, mode, orient, idx, sid):
        rot = mode >= 2 or bool(flags & RHT)
        alpha = oracle.alpha_from_amax(oracle.amax(bits, orient, rot, seed))
        codes, scales = [], []
        for v in idx:
            c, s = oracle.quantize_1d_range(bits, orient, mode, flags & RHT, seed, sid, alpha, int(v), int(v) + 1)
            codes.append(c[0])
            scales.append(s[0])
        return np.stack(codes), np.stack(scales), alpha
    A, sA, aA = operand(bits_a, flags_a, mode_a, orient_a, rows, sid_a)
    B, sB, aB = operand(bits_b, flags_b, mode_b, orient_b, cols, sid_b)
    K = 2 * A.shape[1]
    return oracle.gemm_f64(A, sA, aA, B, sB, aB, len(rows), len(cols), K)


def test_fprop_8b_sampled(api, layer8b):
    x, w = layer8b["x"], layer8b["w"]
    qa = api.nvfp4_quantize(x.cuda(), 1, ROW | GEMM)
    qw = api.nvfp4_quantize(w.cuda(), 1, ROW | B2D | GEMM)
    D = api.nvfp4_gemm(qa.codes_row, qa.scales_row, qa.alpha_row, qw.codes_row, qw.scales_row, qw.alpha_row,
                       out_dtype=FP32)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(x.shape[0], 64, replace=False))
    wb = synthetic.bf16_bits(w)
    # W uses 2D blocks: quantize the 16-row groups that hold the sampled rows
    cols = np.sort(rng.choice(w.shape[0], 64, replace=False))
    alpha_w = oracle.alpha_from_amax(oracle.amax(wb))
    Bc, Bs = [], []
    for n in cols:
        cr, sr, _, _ = oracle.quantize_2d_range(wb, 1, alpha_w, int(n) // 16, int(n) // 16 + 1)
        Bc.append(cr[int(n) % 16])
        Bs.append(sr[0])
    xb = synthetic.bf16_bits(x)
    alpha_x = oracle.alpha_from_amax(oracle.amax(xb))
    Ac, As = [], []
    for m in rows:
        c, s = oracle.quantize_1d_range(xb, 0, 1, 0, 0, 0, alpha_x, int(m), int(m) + 1)
        Ac.append(c[0])
        As.append(s[0])
    K = x.shape[1]
    ref = oracle.gemm_f64(np.stack(Ac), np.stack(As), alpha_x, np.stack(Bc), np.stack(Bs), alpha_w,
                          len(rows), len(cols), K)
    got = D.cpu().numpy()[np.ix_(rows, cols)]
    e = frob(got, ref)
    print(f"fprop 8B sampled frob {e:.2e} max_rel {max_rel(got, ref):.2e}")
    assert e <= FROB_TOL


@pytest.mark.parametrize("mode", [2, 3])
def test_dgrad_wgrad_8b_sampled(api, layer8b, mode):
    x, w, dy = layer8b["x"], layer8b["w"], layer8b["dy"]
    seed = 1000 + mode
    # dgrad: dX[t, h] = sum_o dY[t, o] W[o, h]; both rotated along o (same seed)
    qdy = api.nvfp4_quantize(dy.cuda(), mode, ROW | COL | GEMM, seed=seed, stream_id=0)
    qwt = api.nvfp4_quantize(w.cuda(), 0, COL | RHT | GEMM, seed=seed, stream_id=1)
    dX = api.nvfp4_gemm(qdy.codes_row, qdy.scales_row, qdy.alpha_row, qwt.codes_col, qwt.scales_col,
                        qwt.alpha_col, out_dtype=FP32)
    # wgrad: dW[o, h] = sum_t dY[t, o] X[t, h]; both rotated along t
    qxt = api.nvfp4_quantize(x.cuda(), 0, COL | RHT | GEMM, seed=seed, stream_id=2)
    dW = api.nvfp4_gemm(qdy.codes_col, qdy.scales_col, qdy.alpha_col, qxt.codes_col, qxt.scales_col,
                        qxt.alpha_col, out_dtype=FP32)
    torch.cuda.synchronize()
    rng = np.random.default_rng(mode)
    dyb, wb, xb = synthetic.bf16_bits(dy), synthetic.bf16_bits(w), synthetic.bf16_bits(x)
    rows = np.sort(rng.choice(dy.shape[0], 32, replace=False))
    cols = np.sort(rng.choice(w.shape[1], 32, replace=False))
    ref = _sampled_ref(dyb, 0, mode, wb, RHT, 0, rows, cols, seed=seed, sid_a=0, sid_b=1, orient_a=0, orient_b=1)
    got = dX.cpu().numpy()[np.ix_(rows, cols)]
    e = frob(got, ref)
    print(f"dgrad mode {mode} frob {e:.2e}")
    assert e <= FROB_TOL
    rows = np.sort(rng.choice(dy.shape[1], 32, replace=False))
    cols = np.sort(rng.choice(x.shape[1], 32, replace=False))
    ref = _sampled_ref(dyb, 0, mode, xb, RHT, 0, rows, cols, seed=seed, sid_a=0, sid_b=2, orient_a=1, orient_b=1)
    got = dW.cpu().numpy()[np.ix_(rows, cols)]
    e = frob(got, ref)
    print(f"wgrad mode {mode} frob {e:.2e}")
    assert e <= FROB_TOL


# ----------------------------------------- epilogue quantization (fused)
def _fused_operands(api, M, N, K, seed):
    a = synthetic.normal_with_channel_outliers(M, K, seed=seed)
    w = synthetic.weight(N, K, seed=seed + 1)
    qa = api.nvfp4_quantize(a.cuda(), 1, ROW | GEMM)
    qw = api.nvfp4_quantize(w.cuda(), 1, ROW | B2D | GEMM)
    return qa, qw


@pytest.mark.parametrize("M,N,K", [(512, 512, 384), (768, 1024, 2048)])
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("layout", [0, GEMM])
def test_gemm_quantize_epilogue_matches_quantize_of_output(api, M, N, K, mode, layout):
    qa, qw = _fused_operands(api, M, N, K, seed=M + N + K)
    ops = (qa.codes_row, qa.scales_row, qa.alpha_row, qw.codes_row, qw.scales_row, qw.alpha_row)
    D_ref = api.nvfp4_gemm(*ops)
    torch.cuda.synchronize()
    # the output's tensor scale, as a caller would take it from the previous step
    alpha_out = torch.tensor([float(D_ref.float().abs().max()) / 2688.0], dtype=torch.float32, device="cuda")
    D, codes, scales, amax = api.nvfp4_gemm_quantize(*ops, mode, alpha_out, flags=layout)
    torch.cuda.synchronize()
    assert torch.equal(D, D_ref)
    assert float(amax.item()) == float(D_ref.float().abs().max())
    bits = synthetic.bf16_bits(D.cpu())
    o = oracle.quantize(bits, mode, ROW, alpha=float(alpha_out.item()))
    assert np.array_equal(codes.cpu().numpy(), o["codes_row"])
    s = scales.cpu().numpy().reshape(-1)
    if layout:
        m = np.arange(M)[:, None]
        j = np.arange(N // 16)[None, :]
        kb = N // 16
        off = ((m >> 7) * (kb >> 2) + (j >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (j & 3)
        s = s[off]
    else:
        s = s.reshape(M, N // 16)
    assert np.array_equal(s, o["scales_row"])
    # without writing D: the same codes, scales and amax
    D2, codes2, scales2, amax2 = api.nvfp4_gemm_quantize(*ops, mode, alpha_out, flags=layout, write_d=False)
    torch.cuda.synchronize()
    assert D2 is None
    assert torch.equal(codes2, codes) and torch.equal(scales2, scales) and torch.equal(amax2, amax)


def test_gemm_quantize_epilogue_8b_sampled(api, layer8b):
    x, w = layer8b["x"], layer8b["w"]
    qa = api.nvfp4_quantize(x.cuda(), 1, ROW | GEMM)
    qw = api.nvfp4_quantize(w.cuda(), 1, ROW | B2D | GEMM)
    ops = (qa.codes_row, qa.scales_row, qa.alpha_row, qw.codes_row, qw.scales_row, qw.alpha_row)
    alpha_out = torch.tensor([0.37 / 2688.0], dtype=torch.float32, device="cuda")
    D, codes, scales, amax = api.nvfp4_gemm_quantize(*ops, 1, alpha_out, flags=0)
    torch.cuda.synchronize()
    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([[0, D.shape[0] - 1], rng.integers(0, D.shape[0], 12)]))
    bits = synthetic.bf16_bits(D[torch.as_tensor(rows, device="cuda")].cpu())
    a = float(alpha_out.item())
    for i, r in enumerate(rows):
        c, s = oracle.quantize_1d_range(bits[i:i + 1], 0, 1, 0, 0, 0, a, 0, 1)
        assert np.array_equal(codes[r].cpu().numpy(), c[0]), r
        assert np.array_equal(scales[r].cpu().numpy(), s[0]), r
    assert float(amax.item()) == float(D.float().abs().max())
