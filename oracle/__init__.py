"""CPU oracle for NVFP4 block quantization -- TEST INFRASTRUCTURE ONLY.

A plain, slow restatement of the method (see ``nvfp4_oracle.c`` for the
step-by-step definitions and their sources) that the CUDA library is checked
against.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import this package.  It shares no code with the CUDA
library and never calls it.

Arrays: bf16 tensors are passed as ``numpy.uint16`` bit patterns, row-major
with a row stride ``ld`` (elements).  Outputs are numpy arrays in the plain
row-major layouts described in ``nvfp4_oracle.c``.
"""
import contextlib
import ctypes
import os

import numpy as np

from . import build as _build

ROWWISE, COLWISE, BLOCK2D, ALPHA_PROVIDED, RHT, INVERSE_RHT = 0x1, 0x2, 0x4, 0x10, 0x40, 0x80
HEADROOM = 0x200
VECTOR_SCALES = 0x400
RTN, FOUR_SIX, RHT_SR, MS_EDEN, RHT_SR_HW = 0, 1, 2, 3, 4
OK, ERR_ARG, ERR_SHAPE, ERR_NONFINITE = 0, -1, -2, -4

_lib = None

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_u32p = ctypes.POINTER(ctypes.c_uint32)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64


def lib():
    global _lib
    if _lib is None:
        _lib = _configure(ctypes.CDLL(_build.build()))
    return _lib


@contextlib.contextmanager
def use_library(path):
    """Run the oracle's functions against another build of its source (the
    mutation tests' planted mistakes) inside the block."""
    global _lib
    saved = lib()
    _lib = _configure(ctypes.CDLL(path))
    try:
        yield
    finally:
        _lib = saved


def _configure(L):
    L.oracle_philox4x32_10.argtypes = [_u32p, _u32p, _u32p]
    L.oracle_philox4x32_10.restype = None
    L.oracle_sign_bits.argtypes = [ctypes.c_uint64]
    L.oracle_sign_bits.restype = ctypes.c_uint32
    L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
    L.oracle_e4m3_value.restype = ctypes.c_float
    for n in ("oracle_e4m3_rne", "oracle_e4m3_ceil", "oracle_e2m1_rne"):
        getattr(L, n).argtypes = [ctypes.c_float]
        getattr(L, n).restype = ctypes.c_uint8
    L.oracle_sr_hw_field.argtypes = [ctypes.c_uint32, ctypes.c_int]
    L.oracle_sr_hw_field.restype = ctypes.c_uint32
    for n in ("oracle_e4m3_sr", "oracle_e2m1_sr", "oracle_e2m1_sr_hw"):
        getattr(L, n).argtypes = [ctypes.c_float, ctypes.c_uint32]
        getattr(L, n).restype = ctypes.c_uint8
    L.oracle_e2m1_value.argtypes = [ctypes.c_uint8]
    L.oracle_e2m1_value.restype = ctypes.c_float
    L.oracle_rht16.argtypes = [_f32p, ctypes.c_uint32, _f32p]
    L.oracle_irht16.argtypes = [_f32p, ctypes.c_uint32, _f32p]
    L.oracle_alpha_from_amax.argtypes = [ctypes.c_float]
    L.oracle_alpha_from_amax.restype = ctypes.c_float
    L.oracle_alpha_headroom.argtypes = [ctypes.c_float]
    L.oracle_alpha_headroom.restype = ctypes.c_float
    L.oracle_amax.argtypes = [_u16p, _i64, _i64, _i64, ctypes.c_int, ctypes.c_int,
                              ctypes.c_uint64, _f32p]
    L.oracle_amax.restype = ctypes.c_int
    L.oracle_quantize_1d.argtypes = [_u16p, _i64, _i64, _i64, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_uint32, ctypes.c_uint64, ctypes.c_uint32,
                                     ctypes.c_float, _i64, _i64, _u8p, _u8p]
    L.oracle_quantize_1d.restype = ctypes.c_int
    L.oracle_quantize_2d.argtypes = [_u16p, _i64, _i64, _i64, ctypes.c_int, ctypes.c_float,
                                     _i64, _i64, _u8p, _u8p, _u8p, _u8p]
    L.oracle_quantize_2d.restype = ctypes.c_int
    L.oracle_quantize.argtypes = [_u16p, _i64, _i64, _i64, ctypes.c_int, ctypes.c_uint32,
                                  ctypes.c_uint64, ctypes.c_uint32, _f32p,
                                  _u8p, _u8p, _f32p, _u8p, _u8p, _f32p, _f32p, _f32p]
    L.oracle_quantize.restype = ctypes.c_int
    L.oracle_dequantize.argtypes = [_u8p, _u8p, ctypes.c_float, _i64, _i64, ctypes.c_uint32,
                                    ctypes.c_uint64, _f32p]
    L.oracle_dequantize.restype = ctypes.c_int
    L.oracle_gemm_f64.argtypes = [_u8p, _u8p, ctypes.c_float, _u8p, _u8p, ctypes.c_float,
                                  _i64, _i64, _i64, _i64p, _i64, _i64p, _i64, _f64p]
    L.oracle_gemm_f64.restype = None
    L.oracle_amax_vectors.argtypes = [_u16p, _i64, _i64, _i64, ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                                      _f32p]
    L.oracle_amax_vectors.restype = ctypes.c_int
    L.oracle_quantize_vector_scales.argtypes = [_u16p, _i64, _i64, _i64, ctypes.c_int, ctypes.c_uint32,
                                                ctypes.c_uint64, ctypes.c_uint32, _u8p, _u8p, _f32p,
                                                _u8p, _u8p, _f32p, _f32p, _f32p]
    L.oracle_quantize_vector_scales.restype = ctypes.c_int
    L.oracle_gemm_f64_vector_scales.argtypes = [_u8p, _u8p, _f32p, _u8p, _u8p, _f32p, _i64, _i64, _i64,
                                                _i64p, _i64, _i64p, _i64, _f64p]
    L.oracle_gemm_f64_vector_scales.restype = None
    L.oracle_quantize_block16.argtypes = [_f32p, ctypes.c_float, ctypes.c_int, ctypes.c_uint64,
                                          ctypes.c_uint32, ctypes.c_uint64, _u8p, _u8p]
    L.oracle_quantize_block16.restype = ctypes.c_int
    L.oracle_block_sq_error.argtypes = [_f32p, ctypes.c_float, _u8p, ctypes.c_uint8]
    L.oracle_block_sq_error.restype = ctypes.c_float
    L.oracle_mx_exponent.argtypes = [ctypes.c_float]
    L.oracle_mx_exponent.restype = ctypes.c_int
    L.oracle_e8m0_value.argtypes = [ctypes.c_uint8]
    L.oracle_e8m0_value.restype = ctypes.c_float
    L.oracle_mx_quantize.argtypes = [_u16p, _i64, _i64, _i64, ctypes.c_uint32, ctypes.c_uint64,
                                     _u8p, _u8p, _u8p, _u8p]
    L.oracle_mx_quantize.restype = ctypes.c_int
    L.oracle_mx_dequantize.argtypes = [_u8p, _u8p, _i64, _i64, ctypes.c_uint32, ctypes.c_uint64, _f32p]
    L.oracle_mx_dequantize.restype = ctypes.c_int
    L.oracle_mx_gemm_f64.argtypes = [_u8p, _u8p, _u8p, _u8p, _i64, _i64, _i64, _i64p, _i64, _i64p, _i64, _f64p]
    L.oracle_mx_gemm_f64.restype = None
    return L


def _p(a, t):
    return a.ctypes.data_as(t) if a is not None else None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


class OracleError(RuntimeError):
    def __init__(self, status):
        super().__init__(f"oracle returned status {status}")
        self.status = status


def _check(st):
    if st != OK:
        raise OracleError(st)


# ---- generator and number formats -----------------------------------------
def philox(ctr, key):
    c = _c(ctr, np.uint32)
    k = _c(key, np.uint32)
    o = np.zeros(4, np.uint32)
    lib().oracle_philox4x32_10(_p(c, _u32p), _p(k, _u32p), _p(o, _u32p))
    return o


def sign_bits(seed):
    return int(lib().oracle_sign_bits(seed))


def e4m3_value(b):
    return float(lib().oracle_e4m3_value(int(b)))


def e4m3_rne(v):
    return int(lib().oracle_e4m3_rne(float(v)))


def e4m3_ceil(v):
    return int(lib().oracle_e4m3_ceil(float(v)))


def e4m3_sr(v, u24):
    return int(lib().oracle_e4m3_sr(float(v), int(u24)))


def e2m1_value(c):
    return float(lib().oracle_e2m1_value(int(c)))


def e2m1_rne(y):
    return int(lib().oracle_e2m1_rne(float(y)))


def e2m1_sr(y, u16):
    return int(lib().oracle_e2m1_sr(float(y), int(u16)))


def e2m1_sr_hw(y, r16):
    """E2M1 code of y stochastically rounded the way the sm_100a convert with
    caller random bits does it, for its 16-bit field r16."""
    return int(lib().oracle_e2m1_sr_hw(float(y), int(r16)))


def sr_hw_field(w, j):
    """16-bit field of the 32-bit word w used for element j of a group of four."""
    return int(lib().oracle_sr_hw_field(int(w) & 0xFFFFFFFF, int(j)))


def rht16(x, signs):
    a = _c(x, np.float32)
    r = np.zeros(16, np.float32)
    lib().oracle_rht16(_p(a, _f32p), signs, _p(r, _f32p))
    return r


def irht16(r, signs):
    a = _c(r, np.float32)
    x = np.zeros(16, np.float32)
    lib().oracle_irht16(_p(a, _f32p), signs, _p(x, _f32p))
    return x


def alpha_from_amax(amax):
    return float(lib().oracle_alpha_from_amax(float(amax)))


def alpha_headroom(amax):
    return float(lib().oracle_alpha_headroom(float(amax)))


# ---- tensor level ----------------------------------------------------------
def _bf16_bits(x):
    x = np.asarray(x)
    if x.dtype != np.uint16:
        raise TypeError("bf16 tensors are passed as uint16 bit patterns")
    if x.ndim != 2:
        raise ValueError("expected a 2D array")
    return np.ascontiguousarray(x)


def amax(x, orient=0, rot=False, seed=0, C=None):
    x = _bf16_bits(x)
    R, ld = x.shape
    C = ld if C is None else C
    out = np.zeros(1, np.float32)
    _check(lib().oracle_amax(_p(x, _u16p), R, C, ld, orient, int(rot), seed, _p(out, _f32p)))
    return float(out[0])


def amax_vectors(x, orient=0, rot=False, seed=0, C=None):
    """amax of every row (orient 0) or column (orient 1), over rotated
    16-blocks when rot is set."""
    x = _bf16_bits(x)
    R, ld = x.shape
    C = ld if C is None else C
    out = np.zeros(C if orient else R, np.float32)
    _check(lib().oracle_amax_vectors(_p(x, _u16p), R, C, ld, orient, int(rot), seed, _p(out, _f32p)))
    return out


def quantize_vector_scales(x, mode, flags, seed=0, stream_id=0, C=None):
    """1D quantization with one tensor scale per row (row orientation) or per
    column (column orientation).  alpha_row [R] / alpha_col [C] are arrays;
    amax_row / amax_col the largest vector amax."""
    x = _bf16_bits(x)
    R, ld = x.shape
    C = ld if C is None else C
    out = {}
    cr = sr = cc = sc = ar = ac = None
    if flags & ROWWISE:
        cr = np.zeros((R, C // 2), np.uint8)
        sr = np.zeros((R, C // 16), np.uint8)
        ar = np.zeros(max(R, 1), np.float32)
    if flags & COLWISE:
        cc = np.zeros((C, R // 2), np.uint8)
        sc = np.zeros((C, R // 16), np.uint8)
        ac = np.zeros(max(C, 1), np.float32)
    mr = np.zeros(1, np.float32)
    mc = np.zeros(1, np.float32)
    _check(lib().oracle_quantize_vector_scales(_p(x, _u16p), R, C, ld, mode, flags & ~VECTOR_SCALES, seed,
                                               stream_id, _p(cr, _u8p), _p(sr, _u8p), _p(ar, _f32p),
                                               _p(cc, _u8p), _p(sc, _u8p), _p(ac, _f32p), _p(mr, _f32p),
                                               _p(mc, _f32p)))
    if flags & ROWWISE:
        out.update(codes_row=cr, scales_row=sr, alpha_row=ar[:R], amax_row=float(mr[0]))
    if flags & COLWISE:
        out.update(codes_col=cc, scales_col=sc, alpha_col=ac[:C], amax_col=float(mc[0]))
    return out


def quantize(x, mode, flags, seed=0, stream_id=0, alpha=None, C=None):
    """Quantize a [R, ld] uint16 (bf16) array whose first C columns are the
    tensor.  Returns a dict with the requested outputs.  With VECTOR_SCALES
    (one tensor scale per row / column) see quantize_vector_scales."""
    if flags & VECTOR_SCALES:
        if alpha is not None:
            raise ValueError("VECTOR_SCALES computes its own tensor scales")
        return quantize_vector_scales(x, mode, flags, seed=seed, stream_id=stream_id, C=C)
    x = _bf16_bits(x)
    R, ld = x.shape
    C = ld if C is None else C
    two_d = bool(flags & BLOCK2D)
    out = {}
    a_in = None
    if alpha is not None:
        a_in = np.array([alpha], np.float32)
    cr = sr = cc = sc = None
    if flags & ROWWISE:
        cr = np.zeros((R, C // 2), np.uint8)
        sr = np.zeros((R // 16, C // 16) if two_d else (R, C // 16), np.uint8)
    if flags & COLWISE:
        cc = np.zeros((C, R // 2), np.uint8)
        sc = np.zeros((C // 16, R // 16) if two_d else (C, R // 16), np.uint8)
    ar = np.zeros(1, np.float32)
    ac = np.zeros(1, np.float32)
    mr = np.zeros(1, np.float32)
    mc = np.zeros(1, np.float32)
    st = lib().oracle_quantize(_p(x, _u16p), R, C, ld, mode, flags, seed, stream_id,
                               _p(a_in, _f32p), _p(cr, _u8p), _p(sr, _u8p), _p(ar, _f32p),
                               _p(cc, _u8p), _p(sc, _u8p), _p(ac, _f32p),
                               _p(mr, _f32p), _p(mc, _f32p))
    _check(st)
    if flags & ROWWISE:
        out.update(codes_row=cr, scales_row=sr, alpha_row=float(ar[0]), amax_row=float(mr[0]))
    if flags & COLWISE:
        out.update(codes_col=cc, scales_col=sc, alpha_col=float(ac[0]), amax_col=float(mc[0]))
    return out


def quantize_1d_range(x, orient, mode, flags, seed, stream_id, alpha, v0, v1, C=None):
    """1D quantization of rows (orient 0) or columns (orient 1) v0..v1-1."""
    x = _bf16_bits(x)
    R, ld = x.shape
    C = ld if C is None else C
    length = R if orient else C
    codes = np.zeros((v1 - v0, length // 2), np.uint8)
    scales = np.zeros((v1 - v0, length // 16), np.uint8)
    _check(lib().oracle_quantize_1d(_p(x, _u16p), R, C, ld, orient, mode, flags, seed,
                                    stream_id, alpha, v0, v1, _p(codes, _u8p), _p(scales, _u8p)))
    return codes, scales


def quantize_2d_range(x, mode, alpha, br0, br1, C=None):
    x = _bf16_bits(x)
    R, ld = x.shape
    C = ld if C is None else C
    nb = br1 - br0
    cr = np.zeros((16 * nb, C // 2), np.uint8)
    sr = np.zeros((nb, C // 16), np.uint8)
    cc = np.zeros((C, 8 * nb), np.uint8)
    sc = np.zeros((C // 16, nb), np.uint8)
    _check(lib().oracle_quantize_2d(_p(x, _u16p), R, C, ld, mode, alpha, br0, br1,
                                    _p(cr, _u8p), _p(sr, _u8p), _p(cc, _u8p), _p(sc, _u8p)))
    return cr, sr, cc, sc


def dequantize(codes, scales, alpha, R, C, flags=0, seed=0):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    y = np.zeros((R, C), np.float32)
    _check(lib().oracle_dequantize(_p(codes, _u8p), _p(scales, _u8p), alpha, R, C, flags,
                                   seed, _p(y, _f32p)))
    return y


def gemm_f64(A, sA, alphaA, B, sB, alphaB, M, N, K, rows=None, cols=None):
    """FP64 reference D = alphaA alphaB (qA DeltaA)(qB DeltaB)^T on the given
    rows / columns (None = all).  alphaA / alphaB may be per-row arrays ([M],
    [N]: one tensor scale per operand row)."""
    if np.ndim(alphaA) or np.ndim(alphaB):
        aA = np.broadcast_to(np.asarray(alphaA, np.float32), (M,)).copy()
        aB = np.broadcast_to(np.asarray(alphaB, np.float32), (N,)).copy()
        A = _c(A, np.uint8)
        B = _c(B, np.uint8)
        sA = _c(sA, np.uint8)
        sB = _c(sB, np.uint8)
        r = None if rows is None else _c(rows, np.int64)
        c = None if cols is None else _c(cols, np.int64)
        nr = M if r is None else len(r)
        nc = N if c is None else len(c)
        D = np.zeros((nr, nc), np.float64)
        lib().oracle_gemm_f64_vector_scales(_p(A, _u8p), _p(sA, _u8p), _p(aA, _f32p), _p(B, _u8p), _p(sB, _u8p),
                                            _p(aB, _f32p), M, N, K, _p(r, _i64p), nr, _p(c, _i64p), nc,
                                            _p(D, _f64p))
        return D
    A = _c(A, np.uint8)
    B = _c(B, np.uint8)
    sA = _c(sA, np.uint8)
    sB = _c(sB, np.uint8)
    r = None if rows is None else _c(rows, np.int64)
    c = None if cols is None else _c(cols, np.int64)
    nr = M if r is None else len(r)
    nc = N if c is None else len(c)
    D = np.zeros((nr, nc), np.float64)
    lib().oracle_gemm_f64(_p(A, _u8p), _p(sA, _u8p), alphaA, _p(B, _u8p), _p(sB, _u8p), alphaB,
                          M, N, K, _p(r, _i64p), nr, _p(c, _i64p), nc, _p(D, _f64p))
    return D


def quantize_block16(v, alpha, mode, seed=0, c2=0, blk=0):
    a = _c(v, np.float32)
    codes = np.zeros(16, np.uint8)
    scale = np.zeros(1, np.uint8)
    _check(lib().oracle_quantize_block16(_p(a, _f32p), alpha, mode, seed, c2, blk,
                                         _p(codes, _u8p), _p(scale, _u8p)))
    return codes, int(scale[0])


def block_sq_error(v, alpha, codes, scale):
    a = _c(v, np.float32)
    c = _c(codes, np.uint8)
    return float(lib().oracle_block_sq_error(_p(a, _f32p), alpha, _p(c, _u8p), int(scale)))


def unpack_codes(codes):
    """[n, L/2] packed bytes -> [n, L] 4-bit codes (element 2j = low nibble)."""
    codes = np.asarray(codes, np.uint8)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = codes & 0xF
    out[..., 1::2] = codes >> 4
    return out


# --------------------------------------------------------------------- MXFP4
def mx_exponent(amax):
    """Shared exponent of a 32-block with maximum magnitude amax."""
    return int(lib().oracle_mx_exponent(float(amax)))


def e8m0_value(b):
    return float(lib().oracle_e8m0_value(int(b)))


def mx_quantize(x, flags, seed=0, C=None):
    """MXFP4 quantization of a [R, ld] uint16 (bf16) array in the requested
    orientations (ROWWISE / COLWISE, optional RHT)."""
    x = _bf16_bits(x)
    R, ld = x.shape
    C = ld if C is None else C
    cr = sr = cc = sc = None
    if flags & ROWWISE:
        cr = np.zeros((R, C // 2), np.uint8)
        sr = np.zeros((R, C // 32), np.uint8)
    if flags & COLWISE:
        cc = np.zeros((C, R // 2), np.uint8)
        sc = np.zeros((C, R // 32), np.uint8)
    _check(lib().oracle_mx_quantize(_p(x, _u16p), R, C, ld, flags, seed, _p(cr, _u8p), _p(sr, _u8p),
                                    _p(cc, _u8p), _p(sc, _u8p)))
    out = {}
    if flags & ROWWISE:
        out.update(codes_row=cr, scales_row=sr)
    if flags & COLWISE:
        out.update(codes_col=cc, scales_col=sc)
    return out


def mx_dequantize(codes, scales, R, C, flags=0, seed=0):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    y = np.zeros((R, C), np.float32)
    _check(lib().oracle_mx_dequantize(_p(codes, _u8p), _p(scales, _u8p), R, C, flags, seed, _p(y, _f32p)))
    return y


def mx_gemm_f64(A, sA, B, sB, M, N, K, rows=None, cols=None):
    """FP64 reference D = (qA 2^eA)(qB 2^eB)^T for MXFP4 operands (row-major
    UE8M0 scales) on the given rows / columns (None = all)."""
    A = _c(A, np.uint8)
    B = _c(B, np.uint8)
    sA = _c(sA, np.uint8)
    sB = _c(sB, np.uint8)
    r = None if rows is None else _c(rows, np.int64)
    c = None if cols is None else _c(cols, np.int64)
    nr = M if r is None else len(r)
    nc = N if c is None else len(c)
    D = np.zeros((nr, nc), np.float64)
    lib().oracle_mx_gemm_f64(_p(A, _u8p), _p(sA, _u8p), _p(B, _u8p), _p(sB, _u8p), M, N, K,
                             _p(r, _i64p), nr, _p(c, _i64p), nc, _p(D, _f64p))
    return D
