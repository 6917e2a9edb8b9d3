"""torch-facing wrappers of the C ABI: allocate outputs with torch (device
memory and the current stream are the only things torch supplies) and call
libnvfp4.so.  Every step of the computation runs in the library's kernels.
"""
import math
from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib as L
from ._lib import (NVFP4_ALPHA_PROVIDED, NVFP4_AMAX_PROVIDED, NVFP4_BLOCK2D, NVFP4_COLWISE, NVFP4_FOUR_SIX,  # noqa: F401
                   NVFP4_GEMM_SCALE_LAYOUT, NVFP4_INVERSE_RHT, NVFP4_MS_EDEN, NVFP4_OUT_BF16,
                   NVFP4_OUT_DTYPE_BF16, NVFP4_OUT_DTYPE_FP32, NVFP4_RHT, NVFP4_RHT_SR, NVFP4_RHT_SR_HW,
                   NVFP4_ROWWISE, NVFP4_RTN, NVFP4_SINGLE_PASS, NVFP4_VECTOR_SCALES)


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {L.nvfp4_status_string(status)} (status {status})")
        self.status = status


def _check(status: int, what: str):
    if status != L.NVFP4_OK:
        raise NVFP4Error(status, what)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _need(t: Optional[torch.Tensor], numel: int, dtype, what: str, device=None):
    """Raise unless t can hold `numel` contiguous elements of `dtype` (on
    `device`): the library writes through raw pointers and cannot check."""
    if t is None:
        raise ValueError(f"{what}: buffer missing")
    if t.dtype != dtype:
        raise TypeError(f"{what}: dtype {t.dtype}, expected {dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{what}: on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{what}: must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{what}: {t.numel()} elements, {numel} needed")


def _need_matrix(t: torch.Tensor, rows: int, cols: int, dtype, what: str, device=None):
    """A row-major matrix view of at least rows x cols (row stride >= cols)."""
    if t.dtype != dtype:
        raise TypeError(f"{what}: dtype {t.dtype}, expected {dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{what}: on {t.device}, expected {device}")
    if t.dim() != 2 or t.shape[0] < rows or t.shape[1] < cols or t.stride(1) != 1:
        raise ValueError(f"{what}: shape {tuple(t.shape)} / strides {t.stride()}, need a row-major "
                         f"[>= {rows}, >= {cols}] matrix")


def check_outputs(q: "QTensor", R: int, C: int, flags: int, device=None):
    """Raise unless q's buffers can take the outputs of nvfp4_quantize on an
    [R, C] tensor with these flags."""
    vec = bool(flags & NVFP4_VECTOR_SCALES)
    if flags & NVFP4_ROWWISE:
        _need(q.codes_row, R * (C // 2), torch.uint8, "codes_row", device)
        _need(q.scales_row, math.prod(scale_shape(R, C, flags)), torch.uint8, "scales_row", device)
        _need(q.alpha_row, R if vec else 1, torch.float32, "alpha_row", device)
    if flags & NVFP4_COLWISE:
        _need(q.codes_col, C * (R // 2), torch.uint8, "codes_col", device)
        _need(q.scales_col, math.prod(scale_shape(C, R, flags)), torch.uint8, "scales_col", device)
        _need(q.alpha_col, C if vec else 1, torch.float32, "alpha_col", device)
    if q.amax is not None:
        _need(q.amax, 2, torch.float32, "amax", device)


@dataclass
class QTensor:
    """NVFP4 outputs of one quantize call (device tensors)."""
    codes_row: Optional[torch.Tensor] = None
    scales_row: Optional[torch.Tensor] = None
    alpha_row: Optional[torch.Tensor] = None
    codes_col: Optional[torch.Tensor] = None
    scales_col: Optional[torch.Tensor] = None
    alpha_col: Optional[torch.Tensor] = None
    amax: Optional[torch.Tensor] = None


def scale_shape(rows: int, cols: int, flags: int):
    """Shape of the scale tensor of an operand [rows, cols] (cols = the
    blocked axis)."""
    if flags & NVFP4_GEMM_SCALE_LAYOUT:
        return (rows * (cols // 16),)
    if flags & NVFP4_BLOCK2D:
        return (rows // 16, cols // 16)
    return (rows, cols // 16)


def alloc_outputs(R: int, C: int, flags: int, device) -> QTensor:
    q = QTensor()
    u8 = dict(dtype=torch.uint8, device=device)
    vec = bool(flags & NVFP4_VECTOR_SCALES)   # one tensor scale per row / column
    if flags & NVFP4_ROWWISE:
        q.codes_row = torch.empty((R, C // 2), **u8)
        q.scales_row = torch.empty(scale_shape(R, C, flags), **u8)
        q.alpha_row = torch.empty(max(R, 1) if vec else 1, dtype=torch.float32, device=device)
    if flags & NVFP4_COLWISE:
        q.codes_col = torch.empty((C, R // 2), **u8)
        q.scales_col = torch.empty(scale_shape(C, R, flags), **u8)
        q.alpha_col = torch.empty(max(C, 1) if vec else 1, dtype=torch.float32, device=device)
    q.amax = torch.zeros(2, dtype=torch.float32, device=device)
    return q


def workspace_for(R: int, C: int, flags: int, device) -> Optional[torch.Tensor]:
    n = L.nvfp4_workspace_size(R, C, flags)
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def nvfp4_amax(x: torch.Tensor, flags: int = 0, seed: int = 0, out: Optional[torch.Tensor] = None,
               status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The amax values of Eq. 1 from one read of x with the C ABI's
    nvfp4_amax: [plain, rotated rows, rotated columns] as a float32 CUDA
    tensor of 3 (rotated entries with NVFP4_RHT and the orientation flag)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise TypeError("x must be a 2D bfloat16 CUDA tensor")
    if x.numel() and x.stride(1) != 1:
        raise ValueError("x must have unit column stride")
    R, C = x.shape
    ld = x.stride(0) if x.numel() else C
    if out is not None:
        _need(out, 3, torch.float32, "out", x.device)
    if status is not None:
        _need(status, 1, torch.int32, "status", x.device)
    a = out if out is not None else torch.empty(3, dtype=torch.float32, device=x.device)
    st = L.nvfp4_amax(_p(x), R, C, ld, flags, seed, _p(a), _p(status), _stream())
    _check(st, "nvfp4_amax")
    return a


def nvfp4_quantize(x: torch.Tensor, mode: int, flags: int, seed: int = 0, stream_id: int = 0,
                   alpha: Optional[torch.Tensor] = None, out: Optional[QTensor] = None,
                   workspace: Optional[torch.Tensor] = None,
                   status: Optional[torch.Tensor] = None, amax: Optional[torch.Tensor] = None) -> QTensor:
    """Quantize a 2D bf16 CUDA tensor (unit column stride) with the C ABI's
    nvfp4_quantize; allocates outputs and workspace when not given.  alpha
    (a device float) replaces Eq. 1 (NVFP4_ALPHA_PROVIDED); amax (the three
    device floats nvfp4_amax writes) replaces the amax pass
    (NVFP4_AMAX_PROVIDED)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise TypeError("x must be a 2D bfloat16 CUDA tensor")
    if x.numel() and x.stride(1) != 1:
        raise ValueError("x must have unit column stride")
    R, C = x.shape
    ld = x.stride(0) if x.numel() else C
    if alpha is not None and amax is not None:
        raise ValueError("give alpha or amax, not both")
    if alpha is not None:
        flags |= NVFP4_ALPHA_PROVIDED
    if amax is not None:
        if amax.dtype != torch.float32 or not amax.is_cuda or amax.device != x.device or amax.numel() < 3 \
                or not amax.is_contiguous():
            raise ValueError("amax must be a contiguous float32 tensor on x's device")
        flags |= NVFP4_AMAX_PROVIDED
        alpha = amax
    if out is not None:
        check_outputs(out, R, C, flags, x.device)
    if status is not None:
        _need(status, 1, torch.int32, "status", x.device)
    q = out if out is not None else alloc_outputs(R, C, flags, x.device)
    ws = workspace if workspace is not None else workspace_for(R, C, flags, x.device)
    qt = L.nvfp4_qtensor_t(_p(q.codes_row), _p(q.scales_row), _p(q.alpha_row), _p(q.codes_col),
                           _p(q.scales_col), _p(q.alpha_col), _p(q.amax), _p(status))
    st = L.nvfp4_quantize(_p(x), R, C, ld, mode, flags, seed, stream_id, _p(alpha), qt, _p(ws),
                          0 if ws is None else ws.numel(), _stream())
    _check(st, "nvfp4_quantize")
    return q


def nvfp4_dequantize(codes: torch.Tensor, scales: torch.Tensor, alpha: torch.Tensor, R: int, C: int,
                     flags: int = 0, seed: int = 0, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Decode [R, C/2] codes to fp32 (or bf16 with NVFP4_OUT_BF16)."""
    dtype = torch.bfloat16 if flags & NVFP4_OUT_BF16 else torch.float32
    if out is not None:
        _need(out, R * C, dtype, "out", codes.device)
    y = out if out is not None else torch.empty((R, C), dtype=dtype, device=codes.device)
    st = L.nvfp4_dequantize(_p(codes), _p(scales), _p(alpha), R, C, flags, seed, _p(y), _stream())
    _check(st, "nvfp4_dequantize")
    return y


def nvfp4_gemm(A: torch.Tensor, sA: torch.Tensor, alphaA: torch.Tensor, B: torch.Tensor,
               sB: torch.Tensor, alphaB: torch.Tensor, out_dtype: int = NVFP4_OUT_DTYPE_BF16,
               out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """D[M, N] = alphaA alphaB (A dequantized) (B dequantized)^T; A codes
    [M, K/2], B codes [N, K/2], scales in the GEMM layout."""
    M, K2 = A.shape
    N = B.shape[0]
    K = 2 * K2
    dt = torch.bfloat16 if out_dtype == NVFP4_OUT_DTYPE_BF16 else torch.float32
    if out is not None:
        _need_matrix(out, M, N, dt, "out", A.device)
    D = out if out is not None else torch.empty((M, N), dtype=dt, device=A.device)
    st = L.nvfp4_gemm(_p(A), _p(sA), _p(alphaA), _p(B), _p(sB), _p(alphaB), M, N, K, _p(D), out_dtype,
                      D.stride(0), None, 0, _stream())
    _check(st, "nvfp4_gemm")
    return D


def nvfp4_gemm_vector_scales(A: torch.Tensor, sA: torch.Tensor, alphaA: torch.Tensor, B: torch.Tensor,
                             sB: torch.Tensor, alphaB: torch.Tensor, out_dtype: int = NVFP4_OUT_DTYPE_BF16,
                             out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """nvfp4_gemm for operands quantized with NVFP4_VECTOR_SCALES: alphaA
    holds one tensor scale per row of A ([M]), alphaB one per row of B ([N])."""
    M, K2 = A.shape
    N = B.shape[0]
    K = 2 * K2
    _need(alphaA, M, torch.float32, "alphaA", A.device)
    _need(alphaB, N, torch.float32, "alphaB", A.device)
    dt = torch.bfloat16 if out_dtype == NVFP4_OUT_DTYPE_BF16 else torch.float32
    if out is not None:
        _need_matrix(out, M, N, dt, "out", A.device)
    D = out if out is not None else torch.empty((M, N), dtype=dt, device=A.device)
    st = L.nvfp4_gemm_vector_scales(_p(A), _p(sA), _p(alphaA), _p(B), _p(sB), _p(alphaB), M, N, K, _p(D),
                                    out_dtype, D.stride(0), None, 0, _stream())
    _check(st, "nvfp4_gemm_vector_scales")
    return D


def nvfp4_gemm_quantize(A: torch.Tensor, sA: torch.Tensor, alphaA: torch.Tensor, B: torch.Tensor,
                        sB: torch.Tensor, alphaB: torch.Tensor, mode: int, alpha_out: torch.Tensor,
                        flags: int = NVFP4_GEMM_SCALE_LAYOUT, write_d: bool = True,
                        out: Optional[torch.Tensor] = None):
    """nvfp4_gemm with the bf16 output also quantized rowwise in the epilogue
    (RTN or FOUR_SIX, tensor scale alpha_out).  Returns (D or None, codes
    [M, N/2], scales, amax [1])."""
    M, K2 = A.shape
    N = B.shape[0]
    K = 2 * K2
    dev = A.device
    D = None
    if write_d:
        if out is not None:
            _need_matrix(out, M, N, torch.bfloat16, "out", dev)
        D = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    codes = torch.empty((M, N // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((M, N // 16), dtype=torch.uint8, device=dev)
    amax = torch.empty(1, dtype=torch.float32, device=dev)
    st = L.nvfp4_gemm_quantize(_p(A), _p(sA), _p(alphaA), _p(B), _p(sB), _p(alphaB), M, N, K,
                               _p(D) if D is not None else None, D.stride(0) if D is not None else N,
                               mode, flags, _p(alpha_out), _p(codes), _p(scales), _p(amax), None, 0, _stream())
    _check(st, "nvfp4_gemm_quantize")
    return D, codes, scales, amax


@dataclass
class MXTensor:
    """MXFP4 outputs of one quantize call (device tensors): codes [rows, len/2],
    UE8M0 scale bytes [rows, len/32] per requested orientation."""
    codes_row: Optional[torch.Tensor] = None
    scales_row: Optional[torch.Tensor] = None
    codes_col: Optional[torch.Tensor] = None
    scales_col: Optional[torch.Tensor] = None


def mx_alloc_outputs(R: int, C: int, flags: int, device) -> MXTensor:
    """Output buffers of mxfp4_quantize on an [R, C] tensor: codes [rows,
    len/2] and UE8M0 scales [rows, len/32] (flat in the GEMM layout)."""
    q = MXTensor()
    u8 = dict(dtype=torch.uint8, device=device)
    gemm = bool(flags & NVFP4_GEMM_SCALE_LAYOUT)
    if flags & NVFP4_ROWWISE:
        q.codes_row = torch.empty((R, C // 2), **u8)
        q.scales_row = torch.empty((R * (C // 32),) if gemm else (R, C // 32), **u8)
    if flags & NVFP4_COLWISE:
        q.codes_col = torch.empty((C, R // 2), **u8)
        q.scales_col = torch.empty((C * (R // 32),) if gemm else (C, R // 32), **u8)
    return q


def mx_check_outputs(q: MXTensor, R: int, C: int, flags: int, device=None):
    """Raise unless q's buffers can take the outputs of mxfp4_quantize."""
    if flags & NVFP4_ROWWISE:
        _need(q.codes_row, R * (C // 2), torch.uint8, "codes_row", device)
        _need(q.scales_row, R * (C // 32), torch.uint8, "scales_row", device)
    if flags & NVFP4_COLWISE:
        _need(q.codes_col, C * (R // 2), torch.uint8, "codes_col", device)
        _need(q.scales_col, C * (R // 32), torch.uint8, "scales_col", device)


def mxfp4_quantize(x: torch.Tensor, flags: int, seed: int = 0, status: Optional[torch.Tensor] = None,
                   out: Optional[MXTensor] = None) -> MXTensor:
    """Quantize a 2D bf16 CUDA tensor (unit column stride) to MXFP4 with the C
    ABI's mxfp4_quantize (flags: NVFP4_ROWWISE / NVFP4_COLWISE, NVFP4_RHT)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise TypeError("x must be a 2D bfloat16 CUDA tensor")
    if x.numel() and x.stride(1) != 1:
        raise ValueError("x must have unit column stride")
    R, C = x.shape
    ld = x.stride(0) if x.numel() else C
    if out is not None:
        mx_check_outputs(out, R, C, flags, x.device)
    if status is not None:
        _need(status, 1, torch.int32, "status", x.device)
    q = out if out is not None else mx_alloc_outputs(R, C, flags, x.device)
    st = L.mxfp4_quantize(_p(x), R, C, ld, flags, seed, _p(q.codes_row), _p(q.scales_row), _p(q.codes_col),
                          _p(q.scales_col), _p(status), _stream())
    _check(st, "mxfp4_quantize")
    return q


def mxfp4_dequantize(codes: torch.Tensor, scales: torch.Tensor, R: int, C: int, flags: int = 0, seed: int = 0,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Decode MXFP4 codes [R, C/2] and scales [R, C/32] to fp32 (or bf16 with
    NVFP4_OUT_BF16)."""
    dtype = torch.bfloat16 if flags & NVFP4_OUT_BF16 else torch.float32
    if out is not None:
        _need(out, R * C, dtype, "out", codes.device)
    y = out if out is not None else torch.empty((R, C), dtype=dtype, device=codes.device)
    st = L.mxfp4_dequantize(_p(codes), _p(scales), R, C, flags, seed, _p(y), _stream())
    _check(st, "mxfp4_dequantize")
    return y


def mxfp4_gemm(A: torch.Tensor, sA: torch.Tensor, B: torch.Tensor, sB: torch.Tensor,
               out_dtype: int = NVFP4_OUT_DTYPE_BF16, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """D[M, N] = (A dequantized) (B dequantized)^T for MXFP4 operands: codes
    [M, K/2] and [N, K/2], UE8M0 scales in the GEMM layout."""
    M, K2 = A.shape
    N = B.shape[0]
    K = 2 * K2
    dt = torch.bfloat16 if out_dtype == NVFP4_OUT_DTYPE_BF16 else torch.float32
    if out is not None:
        _need_matrix(out, M, N, dt, "out", A.device)
    D = out if out is not None else torch.empty((M, N), dtype=dt, device=A.device)
    st = L.mxfp4_gemm(_p(A), _p(sA), _p(B), _p(sB), M, N, K, _p(D), out_dtype, D.stride(0), None, 0, _stream())
    _check(st, "mxfp4_gemm")
    return D
