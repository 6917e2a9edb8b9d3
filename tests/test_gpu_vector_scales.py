"""GPU parity of NVFP4_VECTOR_SCALES (one Eq. 1 tensor scale per row of the
quantized operand; the NVFP4 pretraining write-up §九 names finer-than-tensor
global scales as the remedy for one global amax) and of
nvfp4_gemm_vector_scales, against the CPU oracle.

Codes, scales, the alpha vectors and the per-orientation maxima must match
bit for bit in every mode and orientation; the GEMM against the FP64 oracle
product with per-row / per-column tensor scales (fp32 output: relative
Frobenius error <= 1e-5; bf16 output: within one bf16 ulp).
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_quantization_amax_b200 import synthetic

pytestmark = pytest.mark.gpu

ROW, COL, B2D, SP, PROV, GEMM, RHT, HEADROOM, VS = 0x1, 0x2, 0x4, 0x8, 0x10, 0x20, 0x40, 0x200, 0x400
MODES = {"rtn": 0, "four_six": 1, "rht_sr": 2, "ms_eden": 3, "rht_sr_hw": 4}
FP32, BF16 = 1, 0


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_block_quantization_amax_b200 import api as _api
    return _api


def gemm_to_plain(flat, rows, kb):
    m = np.arange(rows)[:, None]
    j = np.arange(kb)[None, :]
    off = ((m >> 7) * (kb >> 2) + (j >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (j & 3)
    return np.asarray(flat)[off]


def tensor_with_row_ranges(R, C, seed):
    """Rows (and columns) of very different ranges, so per-vector scales
    differ from the tensor scale."""
    t = synthetic.normal_with_channel_outliers(R, C, seed=seed).float()
    g = torch.Generator().manual_seed(seed)
    t *= torch.exp2(torch.randint(-6, 7, (R, 1), generator=g).float())
    t[R // 3] = 0.0
    return synthetic.to_bf16(t.numpy())


def check_against_oracle(api, x, mode, flags, seed=3, sid=1):
    R, C = x.shape
    q = api.nvfp4_quantize(x.cuda(), mode, flags | VS, seed=seed, stream_id=sid)
    torch.cuda.synchronize()
    o = oracle.quantize(synthetic.bf16_bits(x), mode, (flags & (ROW | COL | RHT | HEADROOM)) | oracle.VECTOR_SCALES,
                        seed=seed, stream_id=sid)
    for side, bit, n, length in (("row", ROW, R, C), ("col", COL, C, R)):
        if not flags & bit:
            continue
        assert np.array_equal(getattr(q, f"alpha_{side}").cpu().numpy()[:n], o[f"alpha_{side}"]), side
        assert np.array_equal(getattr(q, f"codes_{side}").cpu().numpy(), o[f"codes_{side}"]), side
        s = getattr(q, f"scales_{side}").cpu().numpy()
        if flags & GEMM:
            s = gemm_to_plain(s, n, length // 16)
        assert np.array_equal(s, o[f"scales_{side}"]), side
    amax = q.amax.cpu().numpy()
    if flags & ROW:
        assert float(amax[0]) == o["amax_row"]
    if flags & COL:
        assert float(amax[1]) == o["amax_col"]
    return q, o


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("orient", ["row", "col", "dual"])
def test_vector_scales_all_modes(api, mode, orient):
    x = tensor_with_row_ranges(256, 1024, seed=71)
    check_against_oracle(api, x, MODES[mode], {"row": ROW, "col": COL, "dual": ROW | COL}[orient])


@pytest.mark.parametrize("extra", [RHT, HEADROOM, GEMM, RHT | GEMM | HEADROOM])
@pytest.mark.parametrize("mode", ["rtn", "four_six"])
def test_vector_scales_rotation_headroom_layout(api, mode, extra):
    x = tensor_with_row_ranges(256, 512, seed=72)
    check_against_oracle(api, x, MODES[mode], ROW | COL | extra)


@pytest.mark.parametrize("shape", [(48, 144), (37, 48), (1, 16), (80, 272), (1040, 1552)])
@pytest.mark.parametrize("mode", ["four_six", "ms_eden"])
def test_vector_scales_ragged_and_many_tiles(api, shape, mode):
    R, C = shape
    x = tensor_with_row_ranges(R, C, seed=R + C)
    check_against_oracle(api, x, MODES[mode], ROW | COL if R % 16 == 0 else ROW)


def test_vector_scales_reject_incompatible_flags(api):
    from nvfp4_block_quantization_amax_b200 import _lib as L
    x = tensor_with_row_ranges(64, 128, seed=73).cuda()
    for bad in (ROW | B2D, ROW | SP):
        with pytest.raises(api.NVFP4Error) as e:
            api.nvfp4_quantize(x, 0, bad | VS)
        assert e.value.status == L.NVFP4_ERR_ARG
    with pytest.raises(api.NVFP4Error) as e:
        api.nvfp4_quantize(x, 0, ROW | VS, alpha=torch.ones(1, device="cuda"))
    assert e.value.status == L.NVFP4_ERR_ARG


def test_vector_scales_nonfinite_sets_status(api):
    x = torch.randn(64, 128, dtype=torch.bfloat16, device="cuda")
    x[7, 9] = float("inf")
    for mode, flags in ((0, ROW), (3, ROW | COL), (1, COL)):
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        api.nvfp4_quantize(x, mode, flags | VS, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == -4, (mode, flags)


def _frob(D, ref):
    return float(np.linalg.norm(D.astype(np.float64) - ref) / np.linalg.norm(ref))


def _bf16_within_one_ulp(Dbf, ref):
    r = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)
    d = Dbf.float().numpy().astype(np.float64)
    mag = np.maximum(np.abs(r), np.finfo(np.float32).tiny)
    ulp = 2.0 ** (np.floor(np.log2(mag)) - 7)
    return bool(np.all(np.abs(d - r) <= ulp * 1.0000001))


@pytest.mark.parametrize("M,N,K", [(256, 256, 512), (512, 768, 1024), (1024, 512, 2048)])
def test_gemm_vector_scales_four_six_operands(api, M, N, K):
    a = tensor_with_row_ranges(M, K, seed=M + K)
    w = tensor_with_row_ranges(N, K, seed=N + K + 1)
    qa = api.nvfp4_quantize(a.cuda(), 1, ROW | GEMM | VS)
    qw = api.nvfp4_quantize(w.cuda(), 1, ROW | GEMM | VS)
    oa = oracle.quantize(synthetic.bf16_bits(a), 1, ROW | oracle.VECTOR_SCALES)
    ow = oracle.quantize(synthetic.bf16_bits(w), 1, ROW | oracle.VECTOR_SCALES)
    ref = oracle.gemm_f64(oa["codes_row"], oa["scales_row"], oa["alpha_row"], ow["codes_row"], ow["scales_row"],
                          ow["alpha_row"], M, N, K)
    for dt in (FP32, BF16):
        D = api.nvfp4_gemm_vector_scales(qa.codes_row, qa.scales_row, qa.alpha_row, qw.codes_row, qw.scales_row,
                                         qw.alpha_row, out_dtype=dt)
        torch.cuda.synchronize()
        if dt == FP32:
            e = _frob(D.cpu().numpy(), ref)
            print(f"vector-scale GEMM {M}x{N}x{K}: frob {e:.2e}")
            assert e <= 1e-5
        else:
            assert _bf16_within_one_ulp(D.cpu(), ref)


def test_gemm_vector_scales_rotated_backward_operands(api):
    # dgrad-shaped: dY rows (MS-EDEN) x W rotated along its output features
    # (columns), both with per-vector scales; the rotations cancel
    T, H, O = 512, 256, 1024
    layer = synthetic.layer(T, H, O, seed=74)
    dy, w = layer["dy"], layer["w"]
    seed = 75
    qd = api.nvfp4_quantize(dy.cuda(), 3, ROW | GEMM | VS, seed=seed, stream_id=0)
    qwt = api.nvfp4_quantize(w.cuda(), 0, COL | RHT | GEMM | VS, seed=seed, stream_id=1)
    D = api.nvfp4_gemm_vector_scales(qd.codes_row, qd.scales_row, qd.alpha_row, qwt.codes_col, qwt.scales_col,
                                     qwt.alpha_col, out_dtype=FP32)
    torch.cuda.synchronize()
    od = oracle.quantize(synthetic.bf16_bits(dy), 3, ROW | oracle.VECTOR_SCALES, seed=seed, stream_id=0)
    ow = oracle.quantize(synthetic.bf16_bits(w), 0, COL | RHT | oracle.VECTOR_SCALES, seed=seed, stream_id=1)
    ref = oracle.gemm_f64(od["codes_row"], od["scales_row"], od["alpha_row"], ow["codes_col"], ow["scales_col"],
                          ow["alpha_col"], T, H, O)
    e = _frob(D.cpu().numpy(), ref)
    print(f"vector-scale dgrad frob {e:.2e}")
    assert e <= 1e-5
