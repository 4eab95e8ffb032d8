"""CPU oracle for microscaling quantization and the block-scaled GEMM.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``fp8_quantization_block_b200``) never imports it
and shares no code with it.

The arithmetic lives in ``mx_oracle.c`` (plain C, fp64, one element at a
time); this module only builds it with gcc and marshals numpy arrays.  The
independent exact-arithmetic checker used to pin the C code is ``exact.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mx_oracle.c")
_LIB = os.path.join(_HERE, "libmxoracle.so")

MXFP8_E4M3, MXFP8_E5M2, MXFP4, NVFP4, MXFP6_E3M2, MXFP4_MBS = 0, 1, 2, 3, 4, 5
FORMAT_NAMES = {MXFP8_E4M3: "mxfp8_e4m3", MXFP8_E5M2: "mxfp8_e5m2", MXFP4: "mxfp4", NVFP4: "nvfp4",
                MXFP6_E3M2: "mxfp6_e3m2", MXFP4_MBS: "mxfp4_mbs"}

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile mx_oracle.c into libmxoracle.so (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", _LIB, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            d, u8, u16, i64, f32, i32 = (ctypes.c_double, ctypes.c_uint8, ctypes.c_uint16,
                                         ctypes.c_int64, ctypes.c_float, ctypes.c_int)
            P = ctypes.c_void_p
            sig = {
                "orc_bf16_to_double": (d, [u16]),
                "orc_double_to_bf16_rne": (u16, [d]),
                "orc_e2m1_decode": (d, [u8]),
                "orc_e4m3_decode": (d, [u8]),
                "orc_e5m2_decode": (d, [u8]),
                "orc_e3m2_decode": (d, [u8]),
                "orc_e8m0_decode": (d, [u8]),
                "orc_e2m1_encode": (u8, [d]),
                "orc_e4m3_encode": (u8, [d]),
                "orc_e5m2_encode": (u8, [d]),
                "orc_e3m2_encode": (u8, [d]),
                "orc_block_size": (i32, [i32]),
                "orc_max_element": (d, [i32]),
                "orc_codes_bytes": (ctypes.c_size_t, [i32, i64, i64]),
                "orc_scales_bytes": (ctypes.c_size_t, [i32, i64, i64]),
                "orc_sf_offset": (ctypes.c_size_t, [i64, i64, i64]),
                "orc_mbs_macro_offset": (ctypes.c_size_t, [i64, i64, i64, i64]),
                "orc_mbs_static_mantissa": (i32, [d]),
                "orc_mbs_block_exponent": (i32, [d, i32]),
                "orc_mx_scale_byte": (i32, [d, d]),
                "orc_nvfp4_global_scale": (f32, [d]),
                "orc_nvfp4_block_scale": (u8, [d, f32]),
                "orc_amax_bf16": (d, [P, i64, i64, i64]),
                "orc_quantize": (i32, [i32, P, i64, i64, i64, P, P, P, i32]),
                "orc_quantize_oas": (i32, [P, i64, i64, i64, P, P]),
                "orc_quantize_mbs_dynamic": (i32, [P, i64, i64, i64, P, P]),
                "orc_mbs_macro_sse": (d, [P, i32]),
                "orc_mbs_dynamic_mantissa": (i32, [P]),
                "orc_quantize_f32": (i32, [i32, P, i64, i64, i64, P, P, P, i32]),
                "orc_rht32_f32": (i32, [P, i64, i64, i64, P]),
                "orc_qsnr_db": (d, [P, i64, i64, i64, P, P]),
                "orc_dequantize_f64": (i32, [i32, P, P, f32, i64, i64, P]),
                "orc_dequantize_bf16": (i32, [i32, P, P, f32, i64, i64, P, i64]),
                "orc_gemm_f64": (i32, [P, P, P, i64, i64, i64, P, P]),
                "orc_gelu": (d, [d]),
                "orc_gelu_array": (None, [P, P, i64]),
                "orc_set_threads": (None, [i32]),
                "orc_get_threads": (i32, []),
            }
            for name, (res, args) in sig.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def lib():
    return _load()


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> None:
    _load().orc_set_threads(int(n))


def get_threads() -> int:
    return int(_load().orc_get_threads())


# --- scalar codecs ---------------------------------------------------------
def bf16_to_double(b: int) -> float:
    return _load().orc_bf16_to_double(int(b))


def double_to_bf16(v: float) -> int:
    return int(_load().orc_double_to_bf16_rne(float(v)))


def decode(fmt_name: str, code: int) -> float:
    return getattr(_load(), f"orc_{fmt_name}_decode")(int(code))


def encode(fmt_name: str, v: float) -> int:
    return int(getattr(_load(), f"orc_{fmt_name}_encode")(float(v)))


def block_size(fmt: int) -> int:
    return int(_load().orc_block_size(fmt))


def max_element(fmt: int) -> float:
    return float(_load().orc_max_element(fmt))


def codes_bytes(fmt: int, rows: int, cols: int) -> int:
    return int(_load().orc_codes_bytes(fmt, rows, cols))


def scales_bytes(fmt: int, rows: int, cols: int) -> int:
    return int(_load().orc_scales_bytes(fmt, rows, cols))


def sf_offset(r: int, c: int, sf_cols: int) -> int:
    return int(_load().orc_sf_offset(r, c, sf_cols))


def mx_scale_byte(amax: float, maxelem: float) -> int:
    return int(_load().orc_mx_scale_byte(float(amax), float(maxelem)))


def mbs_macro_offset(rows: int, cols: int, r: int, mb: int) -> int:
    return int(_load().orc_mbs_macro_offset(rows, cols, r, mb))


def mbs_static_mantissa(alpha: float) -> int:
    return int(_load().orc_mbs_static_mantissa(float(alpha)))


def mbs_block_exponent(amax_b: float, m: int) -> int:
    return int(_load().orc_mbs_block_exponent(float(amax_b), int(m)))


def mbs_macro_bytes(scales: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """The [rows, cols/128] macro mantissas stored after an MXFP4-MBS scale buffer's tiles."""
    off = mbs_macro_offset(rows, cols, 0, 0)
    return np.asarray(scales[off:off + rows * (cols // 128)]).reshape(rows, cols // 128)


def nvfp4_global_scale(amax_t: float) -> float:
    return float(_load().orc_nvfp4_global_scale(float(amax_t)))


def nvfp4_block_scale(amax_b: float, g: float) -> int:
    return int(_load().orc_nvfp4_block_scale(float(amax_b), float(g)))


# --- tensor operations -------------------------------------------------------
def amax_bf16(src_bits: np.ndarray) -> float:
    src = np.ascontiguousarray(src_bits, dtype=np.uint16)
    M, K = src.shape
    return float(_load().orc_amax_bf16(_ptr(src), M, K, K))


def quantize(fmt: int, src_bits: np.ndarray, gscale: float | None = None):
    """bf16 bits [M, K] -> (codes uint8, scales uint8 (swizzled, padded), g float32)."""
    src = np.ascontiguousarray(src_bits, dtype=np.uint16)
    M, K = src.shape
    codes = np.zeros(codes_bytes(fmt, M, K), dtype=np.uint8)
    scales = np.zeros(scales_bytes(fmt, M, K), dtype=np.uint8)
    g = np.array([1.0 if gscale is None else gscale], dtype=np.float32)
    rc = _load().orc_quantize(fmt, _ptr(src), M, K, K, _ptr(codes), _ptr(scales), _ptr(g),
                              0 if gscale is None else 1)
    if rc != 0:
        raise ValueError(f"oracle quantize failed with code {rc}")
    return codes, scales, float(g[0])


def quantize_oas(src_bits: np.ndarray):
    """MXFP4 with overflow-aware scaling (block max mapped into (3.5, 7]) ->
    (codes, scales), in MXFP4 storage."""
    src = np.ascontiguousarray(src_bits, dtype=np.uint16)
    M, K = src.shape
    codes = np.zeros(codes_bytes(2, M, K), dtype=np.uint8)
    scales = np.zeros(scales_bytes(2, M, K), dtype=np.uint8)
    rc = _load().orc_quantize_oas(_ptr(src), M, K, K, _ptr(codes), _ptr(scales))
    if rc != 0:
        raise ValueError(f"oracle quantize_oas failed with code {rc}")
    return codes, scales


def quantize_mbs_dynamic(src_bits: np.ndarray):
    """MXFP4 with dynamic macro-block scaling (reading R21: per 128 elements the
    macro mantissa of the smallest squared error) -> (codes, scales), in
    MXFP4-MBS storage (macro bytes after the scale tiles)."""
    src = np.ascontiguousarray(src_bits, dtype=np.uint16)
    M, K = src.shape
    codes = np.zeros(codes_bytes(MXFP4_MBS, M, K), dtype=np.uint8)
    scales = np.zeros(scales_bytes(MXFP4_MBS, M, K), dtype=np.uint8)
    rc = _load().orc_quantize_mbs_dynamic(_ptr(src), M, K, K, _ptr(codes), _ptr(scales))
    if rc != 0:
        raise ValueError(f"oracle quantize_mbs_dynamic failed with code {rc}")
    return codes, scales


def mbs_macro_sse(block_values: np.ndarray, m: int) -> float:
    """fp64 squared error of one 128-value macro block quantized with macro
    mantissa m (reading R21's sum, in element order)."""
    v = np.ascontiguousarray(block_values, dtype=np.float64)
    assert v.shape == (128,)
    return float(_load().orc_mbs_macro_sse(_ptr(v), int(m)))


def mbs_dynamic_mantissa(block_values: np.ndarray) -> int:
    v = np.ascontiguousarray(block_values, dtype=np.float64)
    assert v.shape == (128,)
    return int(_load().orc_mbs_dynamic_mantissa(_ptr(v)))


def rht32(src_bits: np.ndarray) -> np.ndarray:
    """32-point Walsh-Hadamard rotation of every block along K, fp32 [M, K]
    (butterflies of half-width 1, 2, 4, 8, 16 in fp32, then x RN_fp32(1/sqrt(32)))."""
    src = np.ascontiguousarray(src_bits, dtype=np.uint16)
    M, K = src.shape
    out = np.empty((M, K), dtype=np.float32)
    rc = _load().orc_rht32_f32(_ptr(src), M, K, K, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle rht32 failed with code {rc}")
    return out


def quantize_f32(fmt: int, src: np.ndarray, gscale: float | None = None):
    """fp32 [M, K] -> (codes, scales, g), the same rules as quantize()."""
    x = np.ascontiguousarray(src, dtype=np.float32)
    M, K = x.shape
    codes = np.zeros(codes_bytes(fmt, M, K), dtype=np.uint8)
    scales = np.zeros(scales_bytes(fmt, M, K), dtype=np.uint8)
    g = np.array([1.0 if gscale is None else gscale], dtype=np.float32)
    rc = _load().orc_quantize_f32(fmt, _ptr(x), M, K, K, _ptr(codes), _ptr(scales), _ptr(g),
                                  0 if gscale is None else 1)
    if rc != 0:
        raise ValueError(f"oracle quantize_f32 failed with code {rc}")
    return codes, scales, float(g[0])


def quantize_rht(fmt: int, src_bits: np.ndarray, gscale: float | None = None):
    """Rotate every 32-element block (rht32), then quantize the fp32 result."""
    return quantize_f32(fmt, rht32(src_bits), gscale)


def qsnr_db(src_bits: np.ndarray, xhat: np.ndarray):
    """(QSNR in dB, sum x^2, sum (x - xhat)^2) of bf16 bits [M, K] against fp64 xhat [M, K]."""
    src = np.ascontiguousarray(src_bits, dtype=np.uint16)
    xh = np.ascontiguousarray(xhat, dtype=np.float64)
    M, K = src.shape
    assert xh.shape == (M, K)
    sums = np.zeros(2, dtype=np.float64)
    db = float(_load().orc_qsnr_db(_ptr(src), M, K, K, _ptr(xh), _ptr(sums)))
    return db, float(sums[0]), float(sums[1])


def dequantize_f64(fmt: int, codes: np.ndarray, scales: np.ndarray, gscale: float, M: int, K: int):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    out = np.empty((M, K), dtype=np.float64)
    rc = _load().orc_dequantize_f64(fmt, _ptr(codes), _ptr(scales), float(gscale), M, K, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle dequantize failed with code {rc}")
    return out


def dequantize_bf16(fmt: int, codes: np.ndarray, scales: np.ndarray, gscale: float, M: int, K: int):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    out = np.empty((M, K), dtype=np.uint16)
    rc = _load().orc_dequantize_bf16(fmt, _ptr(codes), _ptr(scales), float(gscale), M, K, _ptr(out), K)
    if rc != 0:
        raise ValueError(f"oracle dequantize failed with code {rc}")
    return out


def gemm_f64(A: np.ndarray, B: np.ndarray, rows=None):
    """C = A[rows] @ B^T and |A[rows]| @ |B|^T in fp64 (plain triple loop in C)."""
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2
    if rows is None:
        nrows, rptr, keep = M, None, None
    else:
        keep = np.ascontiguousarray(rows, dtype=np.int64)
        nrows, rptr = keep.shape[0], _ptr(keep)
    C = np.empty((nrows, N), dtype=np.float64)
    Cabs = np.empty((nrows, N), dtype=np.float64)
    _load().orc_gemm_f64(_ptr(A), _ptr(B), rptr, nrows, N, K, _ptr(C), _ptr(Cabs))
    return C, Cabs


def gelu(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    _load().orc_gelu_array(_ptr(x), _ptr(y), x.size)
    return y


def gemm_tolerance_ok(C: np.ndarray, Cref: np.ndarray, Cabs: np.ndarray):
    """Elementwise |C - Cref| <= 2^-8 |Cref| + 1e-4 (|A_dq| |B_dq|^T)_ij.

    Returns (ok, worst_ratio) where ratio = err / bound (ok <=> ratio <= 1)."""
    C = np.asarray(C, dtype=np.float64)
    bound = 2.0 ** -8 * np.abs(Cref) + 1e-4 * Cabs
    err = np.abs(C - Cref)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / bound, np.where(err > 0, np.inf, 0.0))
    return bool(np.all(err <= bound)), float(np.max(ratio)) if ratio.size else 0.0
