"""The C-ABI library loads without a GPU and exports every entry point that
include/nvfp4.h declares; host-side argument checks run without a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"NVFP4_API\s+[\w\s\*]+?\b((?:nv|mx)fp4_\w+)\s*\(", text)


@pytest.fixture(scope="module")
def lib():
    from nvfp4_block_quantization_amax_b200 import build, _lib
    build.build()
    return _lib.load()


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert {"nvfp4_quantize", "nvfp4_dequantize", "nvfp4_gemm", "nvfp4_workspace_size",
            "nvfp4_status_string", "nvfp4_version", "mxfp4_quantize", "mxfp4_dequantize"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_binding_names_match_header():
    from nvfp4_block_quantization_amax_b200 import _lib
    for name in declared_functions():
        assert hasattr(_lib, name), name
    assert set(_lib.EXPORTED) == set(declared_functions())


def test_status_strings_and_version(lib):
    from nvfp4_block_quantization_amax_b200 import _lib
    assert _lib.nvfp4_status_string(0) == "ok"
    assert "NaN" in _lib.nvfp4_status_string(-4)
    assert _lib.nvfp4_version() >= 10000


def test_host_argument_checks_need_no_gpu(lib):
    from nvfp4_block_quantization_amax_b200 import _lib as L
    out = L.nvfp4_qtensor_t()
    fake = 0x10000  # never dereferenced: every call below fails its checks first
    # bad mode, bad flags, no orientation
    assert L.nvfp4_quantize(fake, 16, 16, 16, 7, L.NVFP4_ROWWISE, 0, 0, None, out, None, 0, None) == L.NVFP4_ERR_ARG
    assert L.nvfp4_quantize(fake, 16, 16, 16, 0, 0x8000, 0, 0, None, out, None, 0, None) == L.NVFP4_ERR_ARG
    assert L.nvfp4_quantize(fake, 16, 16, 16, 0, 0, 0, 0, None, out, None, 0, None) == L.NVFP4_ERR_ARG
    # missing outputs
    assert L.nvfp4_quantize(fake, 16, 16, 16, 0, L.NVFP4_ROWWISE, 0, 0, None, out, None, 0, None) == L.NVFP4_ERR_ARG
    out = L.nvfp4_qtensor_t(fake, fake, fake, fake, fake, fake, None, None)
    # C not a multiple of 16; R not a multiple of 16 for columns
    assert L.nvfp4_quantize(fake, 16, 24, 24, 0, L.NVFP4_ROWWISE, 0, 0, None, out, None, 0, None) == L.NVFP4_ERR_SHAPE
    assert L.nvfp4_quantize(fake, 20, 32, 32, 0, L.NVFP4_COLWISE, 0, 0, None, out, None, 0, None) == L.NVFP4_ERR_SHAPE
    # 2D blocks only for RTN / FOUR_SIX
    assert L.nvfp4_quantize(fake, 16, 16, 16, 2, L.NVFP4_ROWWISE | L.NVFP4_BLOCK2D, 0, 0, None, out, None, 0,
                            None) == L.NVFP4_ERR_ARG
    # misaligned input, then missing workspace
    assert L.nvfp4_quantize(fake + 2, 16, 16, 16, 0, L.NVFP4_ROWWISE, 0, 0, None, out, None, 0, None) == L.NVFP4_ERR_ALIGN
    assert L.nvfp4_quantize(fake, 16, 16, 16, 0, L.NVFP4_ROWWISE, 0, 0, None, out, None, 0, None) == L.NVFP4_ERR_WORKSPACE
    assert L.nvfp4_workspace_size(16, 16, L.NVFP4_ROWWISE) > 0
    assert L.nvfp4_workspace_size(16, 16, L.NVFP4_ROWWISE | L.NVFP4_ALPHA_PROVIDED) == 0
    # single pass: the partials plus a 16-byte slot for the grid barrier's counter
    two = L.nvfp4_workspace_size(16, 16, L.NVFP4_ROWWISE)
    assert L.nvfp4_workspace_size(16, 16, L.NVFP4_ROWWISE | L.NVFP4_SINGLE_PASS) == two + 16
    assert L.nvfp4_workspace_size(16, 16, L.NVFP4_ROWWISE | L.NVFP4_SINGLE_PASS | L.NVFP4_ALPHA_PROVIDED) == 0
    # single pass is checked like the two-pass call (here: its workspace is missing)
    assert L.nvfp4_quantize(fake, 16, 16, 16, 0, L.NVFP4_ROWWISE | L.NVFP4_SINGLE_PASS, 0, 0, None, out, None, 0,
                            None) == L.NVFP4_ERR_WORKSPACE
    # empty tensors are a no-op
    assert L.nvfp4_quantize(None, 0, 16, 16, 0, L.NVFP4_ROWWISE, 0, 0, None, out, None, 0, None) == L.NVFP4_OK
    # amax pass: flags, output, shapes, alignment; AMAX_PROVIDED needs the amax
    # input, excludes ALPHA_PROVIDED / SINGLE_PASS / VECTOR_SCALES, needs no workspace
    assert L.nvfp4_amax(fake, 16, 16, 16, L.NVFP4_BLOCK2D, 0, fake, None, None) == L.NVFP4_ERR_ARG
    assert L.nvfp4_amax(fake, 16, 16, 16, 0, 0, None, None, None) == L.NVFP4_ERR_ARG
    assert L.nvfp4_amax(fake, 16, 24, 24, 0, 0, fake, None, None) == L.NVFP4_ERR_SHAPE
    assert L.nvfp4_amax(fake, 24, 16, 16, L.NVFP4_COLWISE | L.NVFP4_RHT, 0, fake, None, None) == L.NVFP4_ERR_SHAPE
    assert L.nvfp4_amax(fake + 8, 16, 16, 16, 0, 0, fake, None, None) == L.NVFP4_ERR_ALIGN
    assert L.nvfp4_amax(fake, 16, 16, 16, 0, 0, fake + 2, None, None) == L.NVFP4_ERR_ALIGN
    assert L.nvfp4_workspace_size(16, 16, L.NVFP4_ROWWISE | L.NVFP4_AMAX_PROVIDED) == 0
    amax = L.NVFP4_AMAX_PROVIDED
    assert L.nvfp4_quantize(fake, 16, 16, 16, 0, L.NVFP4_ROWWISE | amax, 0, 0, None, out, None, 0,
                            None) == L.NVFP4_ERR_ARG
    for other in (L.NVFP4_ALPHA_PROVIDED, L.NVFP4_SINGLE_PASS, L.NVFP4_VECTOR_SCALES):
        assert L.nvfp4_quantize(fake, 16, 16, 16, 0, L.NVFP4_ROWWISE | amax | other, 0, 0, fake, out, None, 0,
                                None) == L.NVFP4_ERR_ARG
    assert L.nvfp4_quantize(fake, 16, 16, 16, 0, L.NVFP4_ROWWISE | amax, 0, 0, fake + 2, out, None, 0,
                            None) == L.NVFP4_ERR_ALIGN
    # dequantize / gemm checks
    assert L.nvfp4_dequantize(fake, fake, fake, 16, 24, 0, 0, fake, None) == L.NVFP4_ERR_SHAPE
    assert L.nvfp4_dequantize(fake, fake, fake, 16, 16, 0x8000, 0, fake, None) == L.NVFP4_ERR_ARG
    assert L.nvfp4_gemm(fake, fake, fake, fake, fake, fake, 100, 128, 128, fake, 0, 128, None, 0, None) == L.NVFP4_ERR_SHAPE
    assert L.nvfp4_gemm(fake, fake, fake, fake, fake, fake, 128, 128, 128, fake, 5, 128, None, 0, None) == L.NVFP4_ERR_ARG
    assert L.nvfp4_gemm(None, fake, fake, fake, fake, fake, 128, 128, 128, fake, 0, 128, None, 0, None) == L.NVFP4_ERR_ARG
    # gemm with epilogue quantization: RTN / FOUR_SIX only, CTA-pair shapes only
    assert L.nvfp4_gemm_quantize(fake, fake, fake, fake, fake, fake, 256, 256, 128, None, 256, 3, 0, fake, fake,
                                 fake, None, None, 0, None) == L.NVFP4_ERR_ARG
    assert L.nvfp4_gemm_quantize(fake, fake, fake, fake, fake, fake, 256, 384, 128, None, 384, 1, 0, fake, fake,
                                 fake, None, None, 0, None) == L.NVFP4_ERR_SHAPE
    assert L.nvfp4_gemm_quantize(fake, fake, fake, fake, fake, fake, 256, 256, 128, None, 256, 1, 0x1, fake, fake,
                                 fake, None, None, 0, None) == L.NVFP4_ERR_ARG
    assert L.nvfp4_gemm_quantize(fake, fake, fake, fake, fake, fake, 256, 256, 128, None, 256, 1, 0, None, fake,
                                 fake, None, None, 0, None) == L.NVFP4_ERR_ARG


def test_mxfp4_host_checks_need_no_gpu(lib):
    from nvfp4_block_quantization_amax_b200 import _lib as L
    fake = 0x10000  # never dereferenced: every call below fails its checks first
    ROW, COL = L.NVFP4_ROWWISE, L.NVFP4_COLWISE
    q = lambda x, R, C, ld, flags, cr=fake, sr=fake, cc=fake, sc=fake: L.mxfp4_quantize(
        x, R, C, ld, flags, 0, cr, sr, cc, sc, None, None)
    assert q(fake, 32, 32, 32, 0) == L.NVFP4_ERR_ARG                      # no orientation
    assert q(fake, 32, 32, 32, ROW | L.NVFP4_BLOCK2D) == L.NVFP4_ERR_ARG  # NVFP4-only flag
    assert q(fake, 32, 48, 48, ROW) == L.NVFP4_ERR_SHAPE                  # rows need C % 32
    assert q(fake, 48, 32, 32, COL) == L.NVFP4_ERR_SHAPE                  # columns need R % 32
    assert q(fake, 32, 32, 16, ROW) == L.NVFP4_ERR_SHAPE                  # ld < C
    assert q(fake, 32, 32, 32, ROW, cr=None) == L.NVFP4_ERR_ARG
    assert q(fake, 32, 32, 32, COL, sc=None) == L.NVFP4_ERR_ARG
    assert q(fake + 2, 32, 32, 32, ROW) == L.NVFP4_ERR_ALIGN
    assert q(fake, 32, 32, 36, ROW) == L.NVFP4_ERR_ALIGN                  # ld % 8
    assert q(fake, 32, 32, 32, ROW, cr=fake + 8) == L.NVFP4_ERR_ALIGN
    assert q(None, 0, 32, 32, ROW) == L.NVFP4_OK                          # empty: no-op
    assert q(fake, 64, 128, 128, ROW | L.NVFP4_GEMM_SCALE_LAYOUT) == L.NVFP4_ERR_SHAPE   # layout: R % 128
    g = L.mxfp4_gemm
    assert g(fake, fake, fake, fake, 128, 256, 128, fake, 0, 256, None, 0, None) == L.NVFP4_ERR_SHAPE   # M % 256
    assert g(fake, fake, fake, fake, 256, 256, 64, fake, 0, 256, None, 0, None) == L.NVFP4_ERR_SHAPE    # K % 128
    assert g(fake, fake, fake, fake, 256, 256, 128, fake, 7, 256, None, 0, None) == L.NVFP4_ERR_ARG
    assert g(None, fake, fake, fake, 256, 256, 128, fake, 0, 256, None, 0, None) == L.NVFP4_ERR_ARG
    assert g(fake + 8, fake, fake, fake, 256, 256, 128, fake, 0, 256, None, 0, None) == L.NVFP4_ERR_ALIGN
    d = L.mxfp4_dequantize
    assert d(fake, fake, 16, 48, 0, 0, fake, None) == L.NVFP4_ERR_SHAPE
    assert d(fake, fake, 16, 32, L.NVFP4_BLOCK2D, 0, fake, None) == L.NVFP4_ERR_ARG
    assert d(None, fake, 16, 32, 0, 0, fake, None) == L.NVFP4_ERR_ARG
    assert d(fake + 4, fake, 16, 32, 0, 0, fake, None) == L.NVFP4_ERR_ALIGN
    assert d(None, None, 0, 32, 0, 0, None, None) == L.NVFP4_OK


def test_header_is_plain_c_and_the_library_links_from_c(lib, tmp_path):
    """A C11 program (-Wall -Wextra -pedantic -Werror) includes the header,
    links libnvfp4.so and runs the host-side checks of every entry point."""
    import shutil
    import subprocess
    from nvfp4_block_quantization_amax_b200 import build
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    so = build.build()
    exe = str(tmp_path / "abi_from_c")
    subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "helpers", "abi_from_c.c"), so, "-Wl,-rpath," + os.path.dirname(so),
                    "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout
