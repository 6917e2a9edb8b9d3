"""nvfp4_quantize_noalloc against nvfp4_quantize.

The no-allocation entry point serves callers that may not allocate device
memory while they run (a plugin inside a runtime that owns all device memory,
a program whose memory plan is fixed at start-up).  Its scratch is a fixed
array inside the library instead of a caller workspace.  Two calls in a row,
through the C ABI, must give the same bytes as the workspace entry point on
the same inputs.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from nvfp4_block_quantization_amax_b200 import synthetic

pytestmark = pytest.mark.gpu


def _outputs(api, R, C, flags):
    return api.alloc_outputs(R, C, flags, torch.device("cuda"))


def _call_noalloc(L, api, x, mode, flags, seed, stream_id):
    R, C = x.shape
    q = _outputs(api, R, C, flags)
    p = lambda t: None if t is None else t.data_ptr()
    qt = L.nvfp4_qtensor_t(p(q.codes_row), p(q.scales_row), p(q.alpha_row), p(q.codes_col),
                           p(q.scales_col), p(q.alpha_col), p(q.amax), None)
    st = L.nvfp4_quantize_noalloc(x.data_ptr(), R, C, x.stride(0), mode, flags, seed, stream_id, None, qt,
                                  torch.cuda.current_stream().cuda_stream)
    assert st == L.NVFP4_OK, L.nvfp4_status_string(st)
    return q


def _same(a, b):
    for k in ("codes_row", "scales_row", "alpha_row", "codes_col", "scales_col", "alpha_col"):
        ta, tb = getattr(a, k), getattr(b, k)
        if ta is None and tb is None:
            continue
        assert torch.equal(ta.cpu(), tb.cpu()), k


def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_block_quantization_amax_b200 import _lib as L
    from nvfp4_block_quantization_amax_b200 import api
    ROW, COL, GEMM = L.NVFP4_ROWWISE, L.NVFP4_COLWISE, L.NVFP4_GEMM_SCALE_LAYOUT
    g = synthetic.laplace_with_spikes(512, 1024, seed=41).cuda()
    x = synthetic.normal_with_channel_outliers(256, 2048, seed=42).cuda()
    cases = [(g, L.NVFP4_MS_EDEN, ROW | COL | GEMM, 5, 1), (x, L.NVFP4_FOUR_SIX, ROW, 0, 0)]
    for t, mode, flags, seed, sid in cases:  # two calls in a row, different work
        got = _call_noalloc(L, api, t, mode, flags, seed, sid)
        want = api.nvfp4_quantize(t, mode, flags, seed=seed, stream_id=sid)
        torch.cuda.synchronize()
        _same(got, want)
        assert float(got.alpha_row.item()) > 0.0


def _oracle_same(q, x_cpu, mode, flags, seed, stream_id, alpha=None):
    """Compare the plain-layout outputs of one call with the oracle, byte for
    byte (codes, scales, alpha)."""
    import oracle
    o = oracle.quantize(synthetic.bf16_bits(x_cpu), mode, flags & 0x47, seed=seed, stream_id=stream_id,
                        alpha=alpha)
    for side, bit in (("row", 0x1), ("col", 0x2)):
        if not flags & bit:
            continue
        assert float(getattr(q, f"alpha_{side}").item()) == o[f"alpha_{side}"], side
        assert np.array_equal(getattr(q, f"codes_{side}").cpu().numpy(), o[f"codes_{side}"]), side
        assert np.array_equal(getattr(q, f"scales_{side}").cpu().numpy(), o[f"scales_{side}"]), side


def test_noalloc_paths_against_the_oracle():
    # The paths that use the fixed array in their own way: the two-pass amax
    # partials (rotated rows + columns), the single pass (partials plus the
    # barrier counter, cooperative launch), a provided alpha (no scratch at
    # all), and a rows + columns call right after a rows-only call (the
    # column partials left by earlier calls must never be read).
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_block_quantization_amax_b200 import _lib as L
    from nvfp4_block_quantization_amax_b200 import api
    ROW, COL, SP = L.NVFP4_ROWWISE, L.NVFP4_COLWISE, L.NVFP4_SINGLE_PASS
    g = synthetic.laplace_with_spikes(256, 512, seed=43)
    x = synthetic.normal_with_channel_outliers(192, 1024, seed=44)
    gd, xd = g.cuda(), x.cuda()
    cases = [(gd, g, L.NVFP4_MS_EDEN, ROW | COL, 5, 1),
             (xd, x, L.NVFP4_FOUR_SIX, ROW | SP, 0, 0),
             (gd, g, L.NVFP4_RHT_SR, ROW | COL | SP, 6, 2),
             (xd, x, L.NVFP4_RHT_SR, ROW, 8, 0),
             (gd, g, L.NVFP4_MS_EDEN, ROW | COL, 9, 3)]
    for t, t_cpu, mode, flags, seed, sid in cases:
        q = _call_noalloc(L, api, t, mode, flags, seed, sid)
        torch.cuda.synchronize()
        _oracle_same(q, t_cpu, mode, flags, seed, sid)
    # provided alpha: no scratch, the array untouched
    R, C = x.shape
    alpha = torch.tensor([0.0123], dtype=torch.float32, device="cuda")
    q = _outputs(api, R, C, ROW)
    p = lambda t: None if t is None else t.data_ptr()
    qt = L.nvfp4_qtensor_t(p(q.codes_row), p(q.scales_row), p(q.alpha_row), None, None, None, p(q.amax), None)
    st = L.nvfp4_quantize_noalloc(xd.data_ptr(), R, C, C, L.NVFP4_RTN, ROW | L.NVFP4_ALPHA_PROVIDED, 0, 0,
                                  alpha.data_ptr(), qt, torch.cuda.current_stream().cuda_stream)
    assert st == L.NVFP4_OK
    torch.cuda.synchronize()
    _oracle_same(q, x, L.NVFP4_RTN, ROW, 0, 0, alpha=float(alpha.item()))
