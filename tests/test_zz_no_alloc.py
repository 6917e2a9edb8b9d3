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
