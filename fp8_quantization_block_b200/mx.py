"""Thin Python binding of libmx.so (the C ABI in include/mx.h).

Argument marshalling only: every step of quantize / dequantize / GEMM runs in
the library's CUDA kernels.  torch is used for device memory and streams.  If
the library is missing this module raises; there is no fallback path.

The raw entry points keep the C names (``mx_quantize``, ``mx_gemm``, ...) and
take integer device pointers and an ``MxTensorC`` struct; the helpers below
(``quantize``, ``dequantize``, ``gemm``, ``gemm_fused_act``) wrap them for
torch tensors.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmx.so")

MX_MXFP8_E4M3, MX_MXFP8_E5M2, MX_MXFP4, MX_NVFP4, MX_MXFP6_E3M2, MX_MXFP4_MBS = 0, 1, 2, 3, 4, 5
FORMATS = {"mxfp8_e4m3": 0, "mxfp8_e5m2": 1, "mxfp4": 2, "nvfp4": 3, "mxfp6_e3m2": 4, "mxfp4_mbs": 5}
MX_OK, MX_ERR_INVALID_ARG, MX_ERR_UNSUPPORTED_SHAPE, MX_ERR_MISALIGNED = 0, 1, 2, 3
MX_ERR_CUDA, MX_ERR_TIMEOUT, MX_ERR_DEVICE = 4, 5, 6
MX_EPI_NONE, MX_EPI_GELU = 0, 1
MX_DEBUG_WAIT_LIMIT_NS, MX_DEBUG_SKIP_PRODUCER, MX_DEBUG_PAIR_GEMM, MX_DEBUG_OVERLAP_LAUNCH = 1, 2, 3, 4
MX_DEBUG_MAX_GEMM_CTAS = 5
MX_DEBUG_FUSED_MODE = 6
MX_FUSED_PIPELINED, MX_FUSED_IN_KERNEL, MX_FUSED_TWO_KERNELS = 0, 1, 2
MX_DEBUG_K_SPLIT = 7
MX_K_SPLIT_AUTO, MX_K_SPLIT_NEVER, MX_K_SPLIT_ALWAYS = 0, 1, 2
KUNIT_WHOLE, KUNIT_PARTIAL, KUNIT_FINISH = 0, 1, 2

EXPORTED = [
    "mx_codes_bytes", "mx_scales_bytes", "mx_block_size", "mx_quantize", "mx_dequantize", "mx_gemm",
    "mx_gemm_fused_act", "mx_fused_workspace_bytes", "mx_check_device_error", "mx_status_string",
    "mx_version", "mx_debug_set", "mx_gemm_fused_act_noalloc", "mx_quantize_oas", "mx_qsnr",
    "mx_quantize_rht", "mx_quantize_mbs_dynamic", "mx_fused_split_workspace_bytes", "mx_debug_split_units",
]
MX_NOALLOC_SCRATCH_BYTES = 4 << 20


class MxError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class MxTensorC(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("reserved", ctypes.c_int32), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("gscale", ctypes.c_void_p)]


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"libmx.so not built ({LIB_PATH}); run python -m fp8_quantization_block_b200.build")
            L = ctypes.CDLL(LIB_PATH)
            P, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
            T = ctypes.POINTER(MxTensorC)
            sigs = {
                "mx_codes_bytes": (sz, [i32, i64, i64]),
                "mx_scales_bytes": (sz, [i32, i64, i64]),
                "mx_block_size": (i32, [i32]),
                "mx_quantize": (i32, [i32, P, i64, i64, i64, T, P, P]),
                "mx_dequantize": (i32, [T, P, i64, P]),
                "mx_quantize_oas": (i32, [P, i64, i64, i64, T, P]),
                "mx_quantize_mbs_dynamic": (i32, [P, i64, i64, i64, T, P]),
                "mx_quantize_rht": (i32, [i32, P, i64, i64, i64, T, P, P]),
                "mx_qsnr": (i32, [T, P, i64, P, P]),
                "mx_gemm": (i32, [T, T, P, i64, P]),
                "mx_gemm_fused_act": (i32, [i32, P, i64, i64, i64, T, P, i64, i32, P, P, P, P, sz, P]),
                "mx_fused_workspace_bytes": (sz, [i32, i64, i64]),
                "mx_fused_split_workspace_bytes": (sz, [i32, i64, i64]),
                "mx_debug_split_units": (i32, [i64, i32, i32, i32, i32, P, i32, P]),
                "mx_gemm_fused_act_noalloc": (i32, [i32, P, i64, i64, i64, T, P, i64, i32, P, P, P, P]),
                "mx_check_device_error": (i32, [P, ctypes.POINTER(ctypes.c_uint32)]),
                "mx_status_string": (ctypes.c_char_p, [i32]),
                "mx_version": (i32, []),
                "mx_debug_set": (i32, [i32, ctypes.c_uint64]),
            }
            for name, (res, args) in sigs.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


# ----------------------------------------------------------------- raw C names
def mx_codes_bytes(fmt: int, rows: int, cols: int) -> int:
    return int(lib().mx_codes_bytes(fmt, rows, cols))


def mx_scales_bytes(fmt: int, rows: int, cols: int) -> int:
    return int(lib().mx_scales_bytes(fmt, rows, cols))


def mx_block_size(fmt: int) -> int:
    return int(lib().mx_block_size(fmt))


def mx_quantize(fmt, src_ptr, M, K, ld, dst: MxTensorC, gscale_in_ptr, stream) -> int:
    return int(lib().mx_quantize(fmt, src_ptr, M, K, ld, ctypes.byref(dst), gscale_in_ptr, stream))


def mx_quantize_oas(src_ptr, M, K, ld, dst: MxTensorC, stream) -> int:
    return int(lib().mx_quantize_oas(src_ptr, M, K, ld, ctypes.byref(dst), stream))


def mx_quantize_mbs_dynamic(src_ptr, M, K, ld, dst: MxTensorC, stream) -> int:
    return int(lib().mx_quantize_mbs_dynamic(src_ptr, M, K, ld, ctypes.byref(dst), stream))


def mx_quantize_rht(fmt, src_ptr, M, K, ld, dst: MxTensorC, gscale_in_ptr, stream) -> int:
    return int(lib().mx_quantize_rht(fmt, src_ptr, M, K, ld, ctypes.byref(dst), gscale_in_ptr, stream))


def mx_qsnr(q: MxTensorC, src_ptr, ld, sums_ptr, stream) -> int:
    return int(lib().mx_qsnr(ctypes.byref(q), src_ptr, ld, sums_ptr, stream))


def mx_dequantize(src: MxTensorC, dst_ptr, ld, stream) -> int:
    return int(lib().mx_dequantize(ctypes.byref(src), dst_ptr, ld, stream))


def mx_gemm(A: MxTensorC, B: MxTensorC, C_ptr, ldc, stream) -> int:
    return int(lib().mx_gemm(ctypes.byref(A), ctypes.byref(B), C_ptr, ldc, stream))


def mx_gemm_fused_act(fmt, X_ptr, M, K, ldx, W: MxTensorC, C_ptr, ldc, epilogue, amax_out_ptr, x_gscale_ptr,
                      x_amax_ptr, ws_ptr, ws_bytes, stream) -> int:
    return int(lib().mx_gemm_fused_act(fmt, X_ptr, M, K, ldx, ctypes.byref(W), C_ptr, ldc, epilogue, amax_out_ptr,
                                       x_gscale_ptr, x_amax_ptr, ws_ptr, ws_bytes, stream))


def mx_gemm_fused_act_noalloc(fmt, X_ptr, M, K, ldx, W: MxTensorC, C_ptr, ldc, epilogue, amax_out_ptr, x_gscale_ptr,
                              x_amax_ptr, stream) -> int:
    """The fused call with the library's own fixed scratch (no workspace; allocates nothing)."""
    return int(lib().mx_gemm_fused_act_noalloc(fmt, X_ptr, M, K, ldx, ctypes.byref(W), C_ptr, ldc, epilogue,
                                               amax_out_ptr, x_gscale_ptr, x_amax_ptr, stream))


def mx_fused_workspace_bytes(fmt: int, M: int, K: int) -> int:
    return int(lib().mx_fused_workspace_bytes(fmt, M, K))


def mx_fused_split_workspace_bytes(fmt: int, M: int, K: int) -> int:
    return int(lib().mx_fused_split_workspace_bytes(fmt, M, K))


def split_units(tiles: int, workers: int, kt: int, mode: int, worker: int):
    """The GEMM work schedule of one worker (host only): (grid workers, [(tile,
    kb, ke, kind, first), ...])."""
    n_workers = ctypes.c_int(0)
    n = int(lib().mx_debug_split_units(tiles, workers, kt, mode, worker, None, 0, ctypes.byref(n_workers)))
    if n < 0:
        raise MxError(MX_ERR_INVALID_ARG, "mx_debug_split_units")
    buf = (ctypes.c_int32 * (5 * max(n, 1)))()
    lib().mx_debug_split_units(tiles, workers, kt, mode, worker, buf, n, None)
    return n_workers.value, [tuple(buf[5 * u:5 * u + 5]) for u in range(n)]


def mx_check_device_error(stream=None):
    info = (ctypes.c_uint32 * 4)()
    s = int(lib().mx_check_device_error(stream, info))
    return s, list(info)


def mx_status_string(s: int) -> str:
    return lib().mx_status_string(int(s)).decode()


def mx_version() -> int:
    return int(lib().mx_version())


def mx_debug_set(key: int, value: int) -> int:
    return int(lib().mx_debug_set(key, value))


status_string = mx_status_string


def check(status: int, what: str = "libmx") -> None:
    if status != MX_OK:
        raise MxError(status, what)


# ----------------------------------------------------------------- torch helpers
def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


@dataclass
class MxTensor:
    """A quantized matrix whose buffers are torch CUDA tensors."""
    fmt: int
    rows: int
    cols: int
    codes: torch.Tensor          # uint8, mx_codes_bytes
    scales: torch.Tensor         # uint8, mx_scales_bytes (tensor-core tiled layout)
    gscale: torch.Tensor | None  # float32 [1] for NVFP4

    def c(self) -> MxTensorC:
        return MxTensorC(self.fmt, 0, self.rows, self.cols, _ptr(self.codes), _ptr(self.scales), _ptr(self.gscale))

    @property
    def nbytes(self) -> int:
        return self.codes.numel() + self.scales.numel() + (4 if self.gscale is not None else 0)


def empty(fmt: int, rows: int, cols: int, device="cuda") -> MxTensor:
    codes = torch.empty(max(mx_codes_bytes(fmt, rows, cols), 1), dtype=torch.uint8, device=device)
    scales = torch.empty(max(mx_scales_bytes(fmt, rows, cols), 1), dtype=torch.uint8, device=device)
    g = torch.empty(1, dtype=torch.float32, device=device) if fmt == MX_NVFP4 else None
    return MxTensor(fmt, rows, cols, codes, scales, g)


def quantize(x: torch.Tensor, fmt: int, gscale: torch.Tensor | None = None, out: MxTensor | None = None,
             stream=None) -> MxTensor:
    """bf16 [M, K] CUDA tensor (row pitch x.stride(0)) -> MxTensor."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    M, K = x.shape
    out = out if out is not None else empty(fmt, M, K, x.device)
    check(mx_quantize(fmt, x.data_ptr(), M, K, x.stride(0), out.c(), _ptr(gscale), _stream(stream)), "mx_quantize")
    return out


def quantize_oas(x: torch.Tensor, out: MxTensor | None = None, stream=None) -> MxTensor:
    """bf16 [M, K] CUDA tensor -> MXFP4 MxTensor with overflow-aware block scales."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    M, K = x.shape
    out = out if out is not None else empty(MX_MXFP4, M, K, x.device)
    check(mx_quantize_oas(x.data_ptr(), M, K, x.stride(0), out.c(), _stream(stream)), "mx_quantize_oas")
    return out


def quantize_mbs_dynamic(x: torch.Tensor, out: MxTensor | None = None, stream=None) -> MxTensor:
    """bf16 [M, K] CUDA tensor -> MXFP4-MBS MxTensor whose macro factors minimise the squared error."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    M, K = x.shape
    out = out if out is not None else empty(MX_MXFP4_MBS, M, K, x.device)
    check(mx_quantize_mbs_dynamic(x.data_ptr(), M, K, x.stride(0), out.c(), _stream(stream)),
          "mx_quantize_mbs_dynamic")
    return out


def quantize_rht(x: torch.Tensor, fmt: int, gscale: torch.Tensor | None = None, out: MxTensor | None = None,
                 stream=None) -> MxTensor:
    """bf16 [M, K] CUDA tensor -> MxTensor of its 32-element Walsh-Hadamard rotation."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    M, K = x.shape
    out = out if out is not None else empty(fmt, M, K, x.device)
    check(mx_quantize_rht(fmt, x.data_ptr(), M, K, x.stride(0), out.c(), _ptr(gscale), _stream(stream)),
          "mx_quantize_rht")
    return out


def qsnr_sums(t: MxTensor, x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """float64 CUDA tensor [sum x^2, sum (x - dequant(t))^2]; QSNR dB = 10 log10(s[0] / s[1])."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    out = out if out is not None else torch.empty(2, dtype=torch.float64, device=x.device)
    check(mx_qsnr(t.c(), x.data_ptr(), x.stride(0), out.data_ptr(), _stream(stream)), "mx_qsnr")
    return out


def dequantize(t: MxTensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    out = out if out is not None else torch.empty((t.rows, t.cols), dtype=torch.bfloat16, device=t.codes.device)
    check(mx_dequantize(t.c(), out.data_ptr(), out.stride(0), _stream(stream)), "mx_dequantize")
    return out


def gemm(A: MxTensor, B: MxTensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    out = out if out is not None else torch.empty((A.rows, B.rows), dtype=torch.bfloat16, device=A.codes.device)
    check(mx_gemm(A.c(), B.c(), out.data_ptr(), out.stride(0), _stream(stream)), "mx_gemm")
    return out


def gemm_fused_act(x: torch.Tensor, W: MxTensor, out: torch.Tensor | None = None, epilogue: int = MX_EPI_NONE,
                   amax_out: torch.Tensor | None = None, x_gscale: torch.Tensor | None = None,
                   x_amax: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                   stream=None, x_fmt: int | None = None) -> torch.Tensor:
    """x_fmt: the format X is quantized to (default W's; any MX format pairs with an MX W)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    M, K = x.shape
    fmt = W.fmt if x_fmt is None else x_fmt
    out = out if out is not None else torch.empty((M, W.rows), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = fused_workspace(fmt, M, K, x.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    check(mx_gemm_fused_act(fmt, x.data_ptr(), M, K, x.stride(0), W.c(), out.data_ptr(), out.stride(0), epilogue,
                            _ptr(amax_out), _ptr(x_gscale), _ptr(x_amax), _ptr(workspace), ws_bytes,
                            _stream(stream)), "mx_gemm_fused_act")
    return out


def fused_workspace(fmt: int, M: int, K: int, device="cuda", split: bool = True) -> torch.Tensor:
    """A workspace for gemm_fused_act (torch's allocator hands out 256-B aligned
    blocks); split: with room for the K split of the last wave."""
    n = mx_fused_split_workspace_bytes(fmt, M, K) if split else mx_fused_workspace_bytes(fmt, M, K)
    return torch.empty(n, dtype=torch.uint8, device=device)


def check_device_error(stream=None) -> None:
    s, info = mx_check_device_error(None if stream is None else stream.cuda_stream)
    if s != MX_OK:
        raise MxError(s, f"device error {info}")
