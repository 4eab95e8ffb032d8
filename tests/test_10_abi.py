"""The C ABI library loads and exports every entry point include/mx.h declares;
host-side argument checks reject bad calls before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

from fp8_quantization_block_b200 import build as mxbuild
from fp8_quantization_block_b200 import mx

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    mxbuild.build()
    return mx.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "mx.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(mx_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(mx.EXPORTED)


def test_header_constants_match_the_binding():
    """Every enumerator (and the scratch-size macro) that include/mx.h
    declares has the same value in the Python binding."""
    src = open(os.path.join(ROOT, "include", "mx.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    consts = {}
    for body in re.findall(r"typedef\s+enum\s*\{(.*?)\}", src, flags=re.S):
        for name, value in re.findall(r"\b(MX_[A-Z0-9_]+)\s*=\s*(\d+)", body):
            consts[name] = int(value)
    assert len(consts) >= 20
    for name, value in consts.items():
        assert getattr(mx, name) == value, name
    assert mx.MX_NOALLOC_SCRATCH_BYTES == 4 << 20 and "((size_t)4 << 20)" in src


def test_sizes_match_layout(L):
    assert mx.mx_codes_bytes(mx.MX_MXFP8_E4M3, 3, 64) == 192
    assert mx.mx_codes_bytes(mx.MX_NVFP4, 3, 64) == 96
    assert mx.mx_scales_bytes(mx.MX_MXFP4, 3, 64) == 128 * 4
    assert mx.mx_scales_bytes(mx.MX_NVFP4, 129, 80) == 256 * 8
    assert mx.mx_block_size(mx.MX_NVFP4) == 16 and mx.mx_block_size(mx.MX_MXFP4) == 32
    assert mx.mx_codes_bytes(mx.MX_MXFP6_E3M2, 3, 64) == 144 and mx.mx_block_size(mx.MX_MXFP6_E3M2) == 32
    assert mx.mx_scales_bytes(mx.MX_MXFP4_MBS, 3, 256) == 128 * 16 + 16 and mx.mx_block_size(mx.MX_MXFP4_MBS) == 16
    assert mx.mx_codes_bytes(7, 4, 4) == 0 and mx.mx_block_size(-1) == 0


def test_sizes_agree_with_oracle(L):
    import oracle
    for fmt in range(6):
        for (r, c) in [(1, 128), (127, 128), (129, 4096), (4608, 3072)]:
            assert mx.mx_codes_bytes(fmt, r, c) == oracle.codes_bytes(fmt, r, c)
            assert mx.mx_scales_bytes(fmt, r, c) == oracle.scales_bytes(fmt, r, c)


def test_status_strings_and_version(L):
    assert mx.mx_status_string(mx.MX_ERR_TIMEOUT) == "MX_ERR_TIMEOUT"
    assert mx.mx_version() >= 100
    assert mx.mx_debug_set(99, 0) == mx.MX_ERR_INVALID_ARG
    # the grid cap is host state only: set and restored without a GPU
    assert mx.mx_debug_set(mx.MX_DEBUG_MAX_GEMM_CTAS, 2) == mx.MX_OK
    assert mx.mx_debug_set(mx.MX_DEBUG_MAX_GEMM_CTAS, 0) == mx.MX_OK


def _t(fmt, rows, cols, codes=0x1000, scales=0x2000, g=0x3000):
    return mx.MxTensorC(fmt, 0, rows, cols, codes, scales, g)


def test_host_checks_reject_bad_arguments(L):
    # these all fail before any CUDA call
    dst = _t(0, 4, 64)
    assert mx.mx_quantize(9, 0x1000, 4, 64, 64, dst, None, None) == mx.MX_ERR_INVALID_ARG
    assert mx.mx_quantize(0, 0x1000, 4, 64, 64, _t(1, 4, 64), None, None) == mx.MX_ERR_INVALID_ARG   # fmt mismatch
    assert mx.mx_quantize(0, 0x1000, 4, 48, 48, _t(0, 4, 48), None, None) == mx.MX_ERR_UNSUPPORTED_SHAPE
    assert mx.mx_quantize(0, 0x1008, 4, 64, 64, dst, None, None) == mx.MX_ERR_MISALIGNED
    assert mx.mx_quantize(0, 0x1000, 4, 64, 60, dst, None, None) == mx.MX_ERR_MISALIGNED      # ld < K
    assert mx.mx_quantize(0, None, 4, 64, 64, dst, None, None) == mx.MX_ERR_INVALID_ARG
    assert mx.mx_quantize(3, 0x1000, 4, 64, 64, _t(3, 4, 64, g=None), None, None) == mx.MX_ERR_INVALID_ARG
    assert mx.mx_quantize(0, None, 0, 64, 64, _t(0, 0, 64), None, None) == mx.MX_OK            # empty: no-op
    A, B = _t(0, 8, 256), _t(0, 8, 256)
    assert mx.mx_gemm(A, _t(3, 8, 256), 0x4000, 8, None) == mx.MX_ERR_INVALID_ARG               # NVFP4 x MXFP8
    assert mx.mx_gemm(_t(3, 8, 256), _t(4, 8, 256), 0x4000, 8, None) == mx.MX_ERR_INVALID_ARG
    # MX formats mix on kind::mxf8f6f4, whose FP6 / FP4 operands need 32-byte aligned codes
    assert mx.mx_gemm(_t(4, 8, 256, codes=0x1010), B, 0x4000, 8, None) == mx.MX_ERR_MISALIGNED
    assert mx.mx_gemm(A, _t(2, 8, 256, codes=0x1010), 0x4000, 8, None) == mx.MX_ERR_MISALIGNED
    assert mx.mx_gemm(_t(4, 8, 64), _t(4, 8, 64), 0x4000, 8, None) == mx.MX_ERR_UNSUPPORTED_SHAPE
    assert mx.mx_quantize(4, 0x1000, 4, 48, 48, _t(4, 4, 48), None, None) == mx.MX_ERR_UNSUPPORTED_SHAPE
    # MXFP4 with macro-block scaling: K a multiple of 128; not a GEMM or rotation format
    assert mx.mx_quantize(5, 0x1000, 4, 64, 64, _t(5, 4, 64), None, None) == mx.MX_ERR_UNSUPPORTED_SHAPE
    assert mx.mx_gemm(_t(5, 8, 256), _t(2, 8, 256), 0x4000, 8, None) == mx.MX_ERR_INVALID_ARG   # MBS x MXFP4
    assert mx.mx_quantize_rht(5, 0x1000, 4, 256, 256, _t(5, 4, 256), None, None) == mx.MX_ERR_INVALID_ARG
    assert mx.mx_dequantize(_t(5, 4, 64), 0x4000, 64, None) == mx.MX_ERR_UNSUPPORTED_SHAPE
    assert mx.mx_gemm(A, _t(0, 8, 128), 0x4000, 8, None) == mx.MX_ERR_INVALID_ARG               # K mismatch
    assert mx.mx_gemm(_t(0, 8, 96), _t(0, 8, 96), 0x4000, 8, None) == mx.MX_ERR_UNSUPPORTED_SHAPE
    assert mx.mx_gemm(A, B, 0x4004, 8, None) == mx.MX_ERR_MISALIGNED
    assert mx.mx_gemm(A, B, 0x4000, 4, None) == mx.MX_ERR_INVALID_ARG                           # ldc < N
    assert mx.mx_gemm(_t(0, 0, 256), B, None, 8, None) == mx.MX_OK                              # empty: no-op
    assert mx.mx_gemm(_t(0, 8, 256, codes=0x1001), B, 0x4000, 8, None) == mx.MX_ERR_MISALIGNED
    assert mx.mx_dequantize(_t(3, 4, 64, g=None), 0x4000, 64, None) == mx.MX_ERR_INVALID_ARG
    assert mx.mx_dequantize(_t(0, 4, 64), 0x4000, 60, None) == mx.MX_ERR_MISALIGNED


def test_host_checks_oas_and_qsnr(L):
    # fail before any CUDA call
    assert mx.mx_quantize_oas(0x1000, 4, 64, 64, _t(0, 4, 64), None) == mx.MX_ERR_INVALID_ARG      # not MXFP4
    assert mx.mx_quantize_oas(0x1000, 4, 48, 48, _t(2, 4, 48), None) == mx.MX_ERR_UNSUPPORTED_SHAPE
    assert mx.mx_quantize_oas(0x1000, 4, 64, 64, _t(2, 4, 32), None) == mx.MX_ERR_INVALID_ARG      # shape mismatch
    assert mx.mx_quantize_oas(0x1008, 4, 64, 64, _t(2, 4, 64), None) == mx.MX_ERR_MISALIGNED
    assert mx.mx_quantize_oas(None, 0, 64, 64, _t(2, 0, 64), None) == mx.MX_OK                    # empty: no-op
    assert mx.mx_qsnr(_t(2, 4, 64), 0x1000, 64, None, None) == mx.MX_ERR_INVALID_ARG               # no sums
    assert mx.mx_qsnr(_t(2, 4, 64), 0x1000, 64, 0x5004, None) == mx.MX_ERR_MISALIGNED
    assert mx.mx_qsnr(_t(9, 4, 64), 0x1000, 64, 0x5000, None) == mx.MX_ERR_INVALID_ARG
