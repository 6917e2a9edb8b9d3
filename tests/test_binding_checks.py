"""Host-side checks of the Python binding (CPU): buffers a caller hands in
are validated before the library writes through their raw pointers.  The
buffers the binding allocates itself, with the flags of every call the bench
step makes, pass the same checks."""
import pytest
import torch

from nvfp4_block_quantization_amax_b200 import api

ROW, COL, B2D, GEMM, RHT = (api.NVFP4_ROWWISE, api.NVFP4_COLWISE, api.NVFP4_BLOCK2D,
                            api.NVFP4_GEMM_SCALE_LAYOUT, api.NVFP4_RHT)
CPU = torch.device("cpu")


@pytest.mark.parametrize("R,C,flags", [(8192, 4096, ROW | GEMM), (14336, 4096, ROW | B2D | GEMM),
                                       (8192, 14336, ROW | COL | GEMM), (14336, 4096, COL | RHT | GEMM),
                                       (256, 1024, ROW | COL), (256, 1024, ROW | COL | B2D)])
def test_own_allocations_pass(R, C, flags):
    api.check_outputs(api.alloc_outputs(R, C, flags, CPU), R, C, flags, CPU)


@pytest.mark.parametrize("R,C,flags", [(8192, 14336, ROW | COL | RHT), (512, 1024, ROW | GEMM), (64, 128, COL)])
def test_own_mx_allocations_pass(R, C, flags):
    api.mx_check_outputs(api.mx_alloc_outputs(R, C, flags, CPU), R, C, flags, CPU)


def test_short_wrong_type_or_strided_buffers_are_rejected():
    R, C = 256, 1024
    q = api.alloc_outputs(R, C, ROW | B2D, CPU)       # 2D scales are smaller than the GEMM layout's
    with pytest.raises(ValueError, match="scales_row"):
        api.check_outputs(q, R, C, ROW | B2D | GEMM, CPU)
    q = api.alloc_outputs(R, C, ROW, CPU)
    with pytest.raises(ValueError, match="codes_col"):
        api.check_outputs(q, R, C, ROW | COL, CPU)
    q.alpha_row = torch.empty(1, dtype=torch.float64)
    with pytest.raises(TypeError, match="alpha_row"):
        api.check_outputs(q, R, C, ROW, CPU)
    q = api.alloc_outputs(R, C, ROW, CPU)
    q.codes_row = torch.empty((R, C), dtype=torch.uint8)[:, ::2]
    with pytest.raises(ValueError, match="contiguous"):
        api.check_outputs(q, R, C, ROW, CPU)
    m = api.mx_alloc_outputs(R, C, ROW, CPU)
    m.scales_row = m.scales_row[:-1]
    with pytest.raises(ValueError, match="scales_row"):
        api.mx_check_outputs(m, R, C, ROW, CPU)


def test_gemm_output_matrix_checks():
    api._need_matrix(torch.empty((256, 512), dtype=torch.bfloat16), 256, 512, torch.bfloat16, "out")
    api._need_matrix(torch.empty((256, 1024), dtype=torch.bfloat16)[:, :512], 256, 512, torch.bfloat16, "out")
    with pytest.raises(ValueError):
        api._need_matrix(torch.empty((128, 512), dtype=torch.bfloat16), 256, 512, torch.bfloat16, "out")
    with pytest.raises(ValueError):
        api._need_matrix(torch.empty((512, 256), dtype=torch.bfloat16).t(), 256, 512, torch.bfloat16, "out")
    with pytest.raises(TypeError):
        api._need_matrix(torch.empty((256, 512), dtype=torch.float32), 256, 512, torch.bfloat16, "out")
