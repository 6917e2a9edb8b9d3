"""GPU parity of the MXFP4 path (mxfp4_quantize / mxfp4_dequantize through
the C ABI) against the CPU oracle: codes and UE8M0 scale bytes bit-exact,
dequantized values exact (fp32) or equal after the same bf16 rounding."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_quantization_amax_b200 import synthetic

pytestmark = pytest.mark.gpu

ROW, COL, RHT, INV, BF16 = 0x1, 0x2, 0x40, 0x80, 0x100


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_block_quantization_amax_b200 import api as _api
    return _api


def run_both(api, x, flags, seed=0):
    q = api.mxfp4_quantize(x.cuda(), flags, seed=seed)
    torch.cuda.synchronize()
    o = oracle.mx_quantize(synthetic.bf16_bits(x), flags, seed=seed)
    for side, bit in (("row", ROW), ("col", COL)):
        if flags & bit:
            assert np.array_equal(getattr(q, f"scales_{side}").cpu().numpy(), o[f"scales_{side}"]), side
            assert np.array_equal(getattr(q, f"codes_{side}").cpu().numpy(), o[f"codes_{side}"]), side
    return q, o


@pytest.mark.parametrize("orient", [ROW, COL, ROW | COL])
@pytest.mark.parametrize("rot", [0, RHT])
def test_pr1_shapes(api, orient, rot):
    x = synthetic.pr1()["x"]
    run_both(api, x, orient | rot, seed=17)


@pytest.mark.parametrize("shape", [(32, 32), (96, 160), (64, 128), (1056, 1568), (224, 4128)])
@pytest.mark.parametrize("rot", [0, RHT])
def test_ragged_and_many_tiles(api, shape, rot):
    x = synthetic.normal_with_entry_outliers(*shape, seed=shape[0] + shape[1])
    run_both(api, x, ROW | COL | rot, seed=3)


@pytest.mark.parametrize("shape", [(37, 64), (1, 32), (5, 96)])
def test_rows_only_any_row_count(api, shape):
    run_both(api, synthetic.weight(*shape, seed=1), ROW)


def test_every_bf16_value_through_the_encoder(api):
    # blocks [6, v1..v31]: the block maximum is 6, so e = 0 and y = v for every
    # bf16 v in [-6, 6], ties included
    bits = np.arange(65536, dtype=np.uint32)
    vals = (bits << 16).view(np.float32)
    vals = vals[np.isfinite(vals) & (np.abs(vals) <= 6)]
    n = -(-len(vals) // 31)
    pad = np.zeros(n * 31, np.float32)
    pad[:len(vals)] = vals
    blocks = np.concatenate([np.full((n, 1), 6.0, np.float32), pad.reshape(n, 31)], axis=1)
    R = -(-n // 4)
    arr = np.zeros((R * 4, 32), np.float32)
    arr[:n] = blocks
    run_both(api, synthetic.to_bf16(arr.reshape(R, 128)), ROW)


def test_extreme_exponents_and_zeros(api):
    rng = np.random.default_rng(8)
    a = rng.standard_normal((64, 256)).astype(np.float64)
    a *= np.exp2(rng.integers(-133, 126, (64, 1)).astype(np.float64))   # subnormal to near-max bf16 rows
    a[5] = 0.0
    a[6, :32] = -0.0
    a[7, 3] = 3.0e38
    x = synthetic.to_bf16(np.clip(a, -3.0e38, 3.0e38).astype(np.float32))
    run_both(api, x, ROW | COL)
    run_both(api, x, ROW | COL | RHT, seed=2)


def test_nonfinite_sets_status(api):
    for v in (float("inf"), float("nan")):
        x = torch.zeros((64, 128), dtype=torch.bfloat16)
        x[40, 77] = v
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        api.mxfp4_quantize(x.cuda(), ROW | COL, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == -4


@pytest.mark.parametrize("flags", [0, BF16, INV, INV | BF16])
def test_dequantize_matches_oracle(api, flags):
    x = synthetic.normal_with_channel_outliers(256, 1024, seed=4)
    rot = RHT if flags & INV else 0
    q = api.mxfp4_quantize(x.cuda(), ROW | rot, seed=11)
    y = api.mxfp4_dequantize(q.codes_row, q.scales_row, 256, 1024, flags, seed=11)
    torch.cuda.synchronize()
    want = oracle.mx_dequantize(q.codes_row.cpu().numpy(), q.scales_row.cpu().numpy(), 256, 1024,
                                flags & INV, seed=11)
    if flags & BF16:
        assert torch.equal(y.cpu(), torch.from_numpy(want).to(torch.bfloat16))
    else:
        assert np.array_equal(y.cpu().numpy(), want)


def test_full_size_activation_dual_rotated(api):
    """X [8192, 4096] rows + columns with the fixed rotation: the first 1024
    rows (32-row column blocks never cross them) compared in full."""
    x = synthetic.fwd_bwd_8b(seed=0)["x"]
    q = api.mxfp4_quantize(x.cuda(), ROW | COL | RHT, seed=0)
    torch.cuda.synchronize()
    o = oracle.mx_quantize(synthetic.bf16_bits(x[:1024]), ROW | COL | RHT, seed=0)
    assert np.array_equal(q.codes_row[:1024].cpu().numpy(), o["codes_row"])
    assert np.array_equal(q.scales_row[:1024].cpu().numpy(), o["scales_row"])
    assert np.array_equal(q.codes_col[:, :512].cpu().numpy(), o["codes_col"])
    assert np.array_equal(q.scales_col[:, :32].cpu().numpy(), o["scales_col"])


# ------------------------------------------------------------------ GEMM
GEMM_LAYOUT, FP32 = 0x20, 1


def plain_to_gemm(plain):
    """[rows, kb] row-major scales -> the tcgen05 block-scale layout (flat)."""
    rows, kb = plain.shape
    m = np.arange(rows)[:, None]
    j = np.arange(kb)[None, :]
    off = ((m >> 7) * (kb >> 2) + (j >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (j & 3)
    out = np.zeros(rows * kb, np.uint8)
    out[off.ravel()] = plain.ravel()
    return out


def frob(D, ref):
    return float(np.linalg.norm(D.astype(np.float64) - ref) / np.linalg.norm(ref))


def bf16_within_bound(Dbf, ref, S, K):
    """bf16 output against the FP64 product: the kernel rounds an FP32
    accumulator to bf16, so |d - ref| <= E + ulp_bf16(|ref| + E), where
    E = K 2^-24 S bounds the FP32 summation error (S = sum |a_k b_k|).  With
    power-of-two scales spanning 2^+-9 on both operands, cancellation makes E
    exceed half a bf16 ulp of small outputs, so a plain one-ulp check of
    RN_bf16(ref) does not hold for a correct kernel."""
    d = Dbf.float().numpy().astype(np.float64)
    E = K * 2.0 ** -24 * S
    mag = np.maximum(np.abs(ref) + E, np.finfo(np.float32).tiny)
    ulp = 2.0 ** (np.floor(np.log2(mag)) - 7)
    return bool(np.all(np.abs(d - ref) <= (ulp + E) * 1.0000001))


def test_quantizer_writes_the_gemm_scale_layout(api):
    x = synthetic.normal_with_channel_outliers(256, 512, seed=21)
    g = api.mxfp4_quantize(x.cuda(), ROW | COL | GEMM_LAYOUT, seed=4)
    p = api.mxfp4_quantize(x.cuda(), ROW | COL, seed=4)
    torch.cuda.synchronize()
    assert torch.equal(g.codes_row, p.codes_row) and torch.equal(g.codes_col, p.codes_col)
    assert np.array_equal(g.scales_row.cpu().numpy(), plain_to_gemm(p.scales_row.cpu().numpy()))
    assert np.array_equal(g.scales_col.cpu().numpy(), plain_to_gemm(p.scales_col.cpu().numpy()))


@pytest.mark.parametrize("M,N,K", [(256, 256, 128), (512, 768, 384), (1024, 512, 2048)])
def test_mx_gemm_random_operands(api, M, N, K):
    rng = np.random.default_rng(M + N + K)
    A = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    B = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sA = rng.integers(118, 136, (M, K // 32), dtype=np.uint8)
    sB = rng.integers(118, 136, (N, K // 32), dtype=np.uint8)
    ref = oracle.mx_gemm_f64(A, sA, B, sB, M, N, K)
    S = oracle.mx_gemm_f64(A & 0x77, sA, B & 0x77, sB, M, N, K)   # sum of |products|: signs cleared
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    args = (dev(A), dev(plain_to_gemm(sA)), dev(B), dev(plain_to_gemm(sB)))
    D32 = api.mxfp4_gemm(*args, out_dtype=FP32)
    Dbf = api.mxfp4_gemm(*args)
    torch.cuda.synchronize()
    e = frob(D32.cpu().numpy(), ref)
    print(f"MX GEMM {M}x{N}x{K}: frob {e:.2e}")
    assert e <= 1e-5
    assert bf16_within_bound(Dbf.cpu(), ref, S, K)


def test_mx_gemm_of_quantized_operands(api):
    """X-like and W-like bf16 operands through mxfp4_quantize (GEMM layout)
    and the GEMM, against the FP64 product of the oracle's own quantization."""
    M, N, K = 512, 512, 1024
    x = synthetic.normal_with_channel_outliers(M, K, seed=31)
    w = synthetic.weight(N, K, seed=32)
    qx = api.mxfp4_quantize(x.cuda(), ROW | GEMM_LAYOUT | RHT, seed=5)
    qw = api.mxfp4_quantize(w.cuda(), ROW | GEMM_LAYOUT | RHT, seed=5)
    D = api.mxfp4_gemm(qx.codes_row, qx.scales_row, qw.codes_row, qw.scales_row, out_dtype=FP32)
    torch.cuda.synchronize()
    ox = oracle.mx_quantize(synthetic.bf16_bits(x), ROW | RHT, seed=5)
    ow = oracle.mx_quantize(synthetic.bf16_bits(w), ROW | RHT, seed=5)
    ref = oracle.mx_gemm_f64(ox["codes_row"], ox["scales_row"], ow["codes_row"], ow["scales_row"], M, N, K)
    assert frob(D.cpu().numpy(), ref) <= 1e-5
    # the shared rotation cancels in the product: close to the bf16 product
    xf = x.float().numpy().astype(np.float64)
    wf = w.float().numpy().astype(np.float64)
    # loose sanity bound (the oracle gives 0.175 for these inputs; a rotation
    # that failed to cancel would give about 1.4)
    print("MX GEMM vs unquantized product: frob", frob(D.cpu().numpy(), xf @ wf.T))
    assert frob(D.cpu().numpy(), xf @ wf.T) < 0.5
