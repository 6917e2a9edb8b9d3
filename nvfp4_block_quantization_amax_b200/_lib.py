"""ctypes binding of libnvfp4.so (include/nvfp4.h), names as in the header.

Argument marshalling only.  The shared library must exist next to this file
(built by ``build.py``); loading fails loudly otherwise -- there is no CPU
fallback.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libnvfp4.so")

NVFP4_OK, NVFP4_ERR_ARG, NVFP4_ERR_SHAPE, NVFP4_ERR_ALIGN = 0, -1, -2, -3
NVFP4_ERR_NONFINITE, NVFP4_ERR_LAUNCH, NVFP4_ERR_TIMEOUT, NVFP4_ERR_CUDA = -4, -5, -6, -7
NVFP4_ERR_WORKSPACE = -8

NVFP4_RTN, NVFP4_FOUR_SIX, NVFP4_RHT_SR, NVFP4_MS_EDEN, NVFP4_RHT_SR_HW = 0, 1, 2, 3, 4

NVFP4_ROWWISE = 0x1
NVFP4_COLWISE = 0x2
NVFP4_BLOCK2D = 0x4
NVFP4_SINGLE_PASS = 0x8
NVFP4_HEADROOM = 0x200
NVFP4_VECTOR_SCALES = 0x400
NVFP4_ALPHA_PROVIDED = 0x10
NVFP4_AMAX_PROVIDED = 0x800
NVFP4_GEMM_SCALE_LAYOUT = 0x20
NVFP4_RHT = 0x40
NVFP4_INVERSE_RHT = 0x80
NVFP4_OUT_BF16 = 0x100

NVFP4_OUT_DTYPE_BF16 = 0
NVFP4_OUT_DTYPE_FP32 = 1

EXPORTED = ("nvfp4_workspace_size", "nvfp4_quantize", "nvfp4_quantize_noalloc", "nvfp4_amax", "nvfp4_dequantize",
            "nvfp4_gemm", "nvfp4_gemm_vector_scales", "nvfp4_gemm_quantize", "mxfp4_quantize", "mxfp4_dequantize", "mxfp4_gemm", "nvfp4_launch_count",
            "nvfp4_status_string", "nvfp4_version")


class nvfp4_qtensor_t(ctypes.Structure):
    _fields_ = [("codes_row", ctypes.c_void_p), ("scales_row", ctypes.c_void_p),
                ("alpha_row", ctypes.c_void_p), ("codes_col", ctypes.c_void_p),
                ("scales_col", ctypes.c_void_p), ("alpha_col", ctypes.c_void_p),
                ("amax_out", ctypes.c_void_p), ("status", ctypes.c_void_p)]


_lib = None


def load(path=LIB_PATH):
    """Load libnvfp4.so and declare every exported function."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with nvfp4_block_quantization_amax_b200/build.py "
                           "(the library has no CPU fallback)")
    L = ctypes.CDLL(path)
    vp, i64, u32, u64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_size_t
    L.nvfp4_workspace_size.argtypes = [i64, i64, u32]
    L.nvfp4_workspace_size.restype = sz
    L.nvfp4_quantize.argtypes = [vp, i64, i64, i64, ctypes.c_int, u32, u64, u32, vp,
                                 ctypes.POINTER(nvfp4_qtensor_t), vp, sz, vp]
    L.nvfp4_quantize.restype = ctypes.c_int
    L.nvfp4_quantize_noalloc.argtypes = [vp, i64, i64, i64, ctypes.c_int, u32, u64, u32, vp,
                                         ctypes.POINTER(nvfp4_qtensor_t), vp]
    L.nvfp4_quantize_noalloc.restype = ctypes.c_int
    L.nvfp4_amax.argtypes = [vp, i64, i64, i64, u32, u64, vp, vp, vp]
    L.nvfp4_amax.restype = ctypes.c_int
    L.nvfp4_dequantize.argtypes = [vp, vp, vp, i64, i64, u32, u64, vp, vp]
    L.nvfp4_dequantize.restype = ctypes.c_int
    L.nvfp4_gemm.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, ctypes.c_int, i64, vp, sz, vp]
    L.nvfp4_gemm.restype = ctypes.c_int
    L.nvfp4_gemm_vector_scales.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, ctypes.c_int, i64, vp, sz, vp]
    L.nvfp4_gemm_vector_scales.restype = ctypes.c_int
    L.nvfp4_gemm_quantize.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, i64, ctypes.c_int, u32, vp,
                                      vp, vp, vp, vp, sz, vp]
    L.nvfp4_gemm_quantize.restype = ctypes.c_int
    L.mxfp4_quantize.argtypes = [vp, i64, i64, i64, u32, u64, vp, vp, vp, vp, vp, vp]
    L.mxfp4_quantize.restype = ctypes.c_int
    L.mxfp4_dequantize.argtypes = [vp, vp, i64, i64, u32, u64, vp, vp]
    L.mxfp4_gemm.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, ctypes.c_int, i64, vp, sz, vp]
    L.mxfp4_gemm.restype = ctypes.c_int
    L.mxfp4_dequantize.restype = ctypes.c_int
    L.nvfp4_status_string.argtypes = [ctypes.c_int]
    L.nvfp4_status_string.restype = ctypes.c_char_p
    L.nvfp4_version.argtypes = []
    L.nvfp4_version.restype = ctypes.c_int
    L.nvfp4_launch_count.argtypes = []
    L.nvfp4_launch_count.restype = ctypes.c_uint64
    _lib = L
    return L


def nvfp4_workspace_size(R, C, flags):
    return int(load().nvfp4_workspace_size(R, C, flags))


def nvfp4_quantize(x, R, C, ld, mode, flags, seed, stream_id, alpha_in, out, workspace,
                   workspace_bytes, stream):
    return int(load().nvfp4_quantize(x, R, C, ld, mode, flags, seed, stream_id, alpha_in,
                                     ctypes.byref(out), workspace, workspace_bytes, stream))


def nvfp4_quantize_noalloc(x, R, C, ld, mode, flags, seed, stream_id, alpha_in, out, stream):
    """nvfp4_quantize without a workspace, for callers that may not allocate
    device memory while they run; its scratch is a fixed array inside the
    library shared by every call on a device (order such calls on one
    stream)."""
    return int(load().nvfp4_quantize_noalloc(x, R, C, ld, mode, flags, seed, stream_id, alpha_in,
                                             ctypes.byref(out), stream))


def nvfp4_amax(x, R, C, ld, flags, seed, amax_out, status, stream):
    return int(load().nvfp4_amax(x, R, C, ld, flags, seed, amax_out, status, stream))


def nvfp4_dequantize(codes, scales, alpha, R, C, flags, seed, y, stream):
    return int(load().nvfp4_dequantize(codes, scales, alpha, R, C, flags, seed, y, stream))


def nvfp4_gemm(A, sA, alphaA, B, sB, alphaB, M, N, K, D, out_dtype, ldd, workspace,
               workspace_bytes, stream):
    return int(load().nvfp4_gemm(A, sA, alphaA, B, sB, alphaB, M, N, K, D, out_dtype, ldd,
                                 workspace, workspace_bytes, stream))


def nvfp4_gemm_vector_scales(A, sA, alphaA, B, sB, alphaB, M, N, K, D, out_dtype, ldd, workspace,
                             workspace_bytes, stream):
    return int(load().nvfp4_gemm_vector_scales(A, sA, alphaA, B, sB, alphaB, M, N, K, D, out_dtype, ldd,
                                               workspace, workspace_bytes, stream))


def nvfp4_gemm_quantize(A, sA, alphaA, B, sB, alphaB, M, N, K, D, ldd, mode, flags, alpha_out, codes, scales,
                        amax_out, workspace, workspace_bytes, stream):
    return int(load().nvfp4_gemm_quantize(A, sA, alphaA, B, sB, alphaB, M, N, K, D, ldd, mode, flags, alpha_out,
                                          codes, scales, amax_out, workspace, workspace_bytes, stream))


def mxfp4_quantize(x, R, C, ld, flags, seed, codes_row, scales_row, codes_col, scales_col, status, stream):
    return int(load().mxfp4_quantize(x, R, C, ld, flags, seed, codes_row, scales_row, codes_col, scales_col,
                                     status, stream))


def mxfp4_gemm(A, sA, B, sB, M, N, K, D, out_dtype, ldd, workspace, workspace_bytes, stream):
    return int(load().mxfp4_gemm(A, sA, B, sB, M, N, K, D, out_dtype, ldd, workspace, workspace_bytes, stream))


def mxfp4_dequantize(codes, scales, R, C, flags, seed, y, stream):
    return int(load().mxfp4_dequantize(codes, scales, R, C, flags, seed, y, stream))


def nvfp4_status_string(status):
    return load().nvfp4_status_string(status).decode()


def nvfp4_launch_count():
    return int(load().nvfp4_launch_count())


def nvfp4_version():
    return int(load().nvfp4_version())
