"""mx_gemm_fused_act_noalloc: the fused quantize + GEMM for callers that cannot
allocate device memory (for example code inside an inference engine's plugin
callback, where the engine owns all memory, or a runtime under a fixed memory
budget).  It uses a fixed scratch array inside the library instead of a caller
workspace.

Checked through the C ABI against the workspace-taking mx_gemm_fused_act on the
same inputs, on two calls in a row (the second call reuses the scratch the
first one left behind), and against the fp64 oracle's tolerance.  This file is
collected last; one test also makes the call first thing in a fresh process
(where the first call looks up the scratch array's device address)."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from fp8_quantization_block_b200 import build as mxbuild
from fp8_quantization_block_b200 import mx, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def library():
    mxbuild.build()
    mx.lib()


def _scratch_sized() -> torch.Tensor:
    """A workspace of exactly the scratch array's size: the workspace entry then
    makes the same choices (the K split needs room) as the no-allocation one."""
    return torch.empty(mx.MX_NOALLOC_SCRATCH_BYTES, dtype=torch.uint8, device="cuda")


def _noalloc(x: torch.Tensor, W: mx.MxTensor, **kw) -> torch.Tensor:
    M, K = x.shape
    out = torch.empty((M, W.rows), dtype=torch.bfloat16, device=x.device)
    ptr = lambda t: None if t is None else t.data_ptr()
    s = mx.mx_gemm_fused_act_noalloc(W.fmt, x.data_ptr(), M, K, x.stride(0), W.c(), out.data_ptr(), out.stride(0),
                                     kw.get("epilogue", 0), ptr(kw.get("amax_out")), ptr(kw.get("x_gscale")),
                                     ptr(kw.get("x_amax")), torch.cuda.current_stream().cuda_stream)
    mx.check(s, "mx_gemm_fused_act_noalloc")
    return out


@pytest.mark.parametrize("fmt", [0, 2, 3])
def test_noalloc_matches_workspace_entry_two_calls(fmt):
    N, K = 640, 1024
    W_bits = synth.gaussian_weights(900 + fmt, N, K)
    W = mx.quantize(synth.bits_to_tensor(W_bits).cuda(), fmt)
    for call, (M, seed) in enumerate([(256, 901), (96, 902)]):
        X_bits = synth.student_t(seed + fmt, M, K)
        X = synth.bits_to_tensor(X_bits).cuda()
        got = _noalloc(X, W)
        want = mx.gemm_fused_act(X, W, workspace=_scratch_sized())
        torch.cuda.synchronize()
        mx.check_device_error()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), f"call {call}"
        # and within the GEMM tolerance of the fp64 oracle
        cx, sx, gx = oracle.quantize(fmt, X_bits)
        cw, sw, gw = oracle.quantize(fmt, W_bits)
        Cref, Cabs = oracle.gemm_f64(oracle.dequantize_f64(fmt, cx, sx, gx, M, K),
                                     oracle.dequantize_f64(fmt, cw, sw, gw, N, K))
        ok, worst = oracle.gemm_tolerance_ok(got.float().cpu().double().numpy(), Cref, Cabs)
        assert ok, (call, worst)


def test_noalloc_epilogue_and_amax_chain():
    M, D, F = 128, 512, 768
    X = synth.bits_to_tensor(synth.student_t(910, M, D)).cuda()
    W1 = mx.quantize(synth.bits_to_tensor(synth.gaussian_weights(911, F, D)).cuda(), 3)
    W2 = mx.quantize(synth.bits_to_tensor(synth.gaussian_weights(912, D, F)).cuda(), 3)
    a1, a2 = torch.empty(1, device="cuda"), torch.empty(1, device="cuda")
    H1 = _noalloc(X, W1, epilogue=mx.MX_EPI_GELU, amax_out=a1)
    Y1 = _noalloc(H1, W2, x_amax=a1)
    H2 = mx.gemm_fused_act(X, W1, epilogue=mx.MX_EPI_GELU, amax_out=a2, workspace=_scratch_sized())
    Y2 = mx.gemm_fused_act(H2, W2, x_amax=a2, workspace=_scratch_sized())
    torch.cuda.synchronize()
    mx.check_device_error()
    assert torch.equal(H1.view(torch.int16), H2.view(torch.int16))
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    assert float(a1.cpu()[0]) == float(a2.cpu()[0])


def _largest_accepted_rows(fmt: int, K: int) -> int:
    """The largest M whose fused workspace fits the scratch array (the size is
    non-decreasing in M, so M + 1 is the smallest rejected shape)."""
    lo, hi = 0, mx.MX_NOALLOC_SCRATCH_BYTES    # fits at lo, not at hi
    assert mx.mx_fused_workspace_bytes(fmt, hi, K) > mx.MX_NOALLOC_SCRATCH_BYTES
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if mx.mx_fused_workspace_bytes(fmt, mid, K) <= mx.MX_NOALLOC_SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid
    return lo


@pytest.mark.parametrize("fmt", [0, 2, 3])
def test_noalloc_largest_shape_runs_and_the_next_is_rejected(fmt):
    K, N = 4096, 256
    M = _largest_accepted_rows(fmt, K)
    assert M > 128
    W = mx.quantize(synth.bits_to_tensor(synth.gaussian_weights(914 + fmt, N, K)).cuda(), fmt)
    # one row more: rejected on the host before any launch (the pointers are never used)
    s = mx.mx_gemm_fused_act_noalloc(fmt, 0x1000, M + 1, K, K, W.c(), 0x2000, N, 0, None, None, None, None)
    assert s == mx.MX_ERR_UNSUPPORTED_SHAPE
    # sizes whose byte count would overflow are rejected too
    for big_m, big_k in ((1 << 40, K), (256, 1 << 40), ((1 << 62) // 4096, 4096)):
        s = mx.mx_gemm_fused_act_noalloc(fmt, 0x1000, big_m, big_k, big_k, W.c(), 0x2000, N, 0, None, None, None,
                                         None)
        assert s in (mx.MX_ERR_UNSUPPORTED_SHAPE, mx.MX_ERR_INVALID_ARG)
    # the largest accepted shape fills the array to its end: bit for bit the workspace entry
    X = synth.bits_to_tensor(synth.sweep_tensor(913 + fmt, M, K)).cuda()
    got = _noalloc(X, W)
    want = mx.gemm_fused_act(X, W, workspace=_scratch_sized())
    torch.cuda.synchronize()
    mx.check_device_error()
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))


_FRESH = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
from fp8_quantization_block_b200 import mx, synth
fmt, M, N, K = 0, 200, 384, 512
W = mx.quantize(synth.bits_to_tensor(synth.gaussian_weights(920, N, K)).cuda(), fmt)
X = synth.bits_to_tensor(synth.student_t(921, M, K)).cuda()
outs = []
for _ in range(2):
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    s = mx.mx_gemm_fused_act_noalloc(fmt, X.data_ptr(), M, K, K, W.c(), out.data_ptr(), N, 0, None, None, None,
                                     torch.cuda.current_stream().cuda_stream)
    mx.check(s, "mx_gemm_fused_act_noalloc")
    outs.append(out)
want = mx.gemm_fused_act(X, W, workspace=torch.empty(mx.MX_NOALLOC_SCRATCH_BYTES, dtype=torch.uint8, device="cuda"))
torch.cuda.synchronize()
mx.check_device_error()
for o in outs:
    assert torch.equal(o.view(torch.int16), want.view(torch.int16))
print("fresh-process noalloc ok")
"""


def test_noalloc_first_call_in_a_fresh_process():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _FRESH, root], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "fresh-process noalloc ok" in r.stdout
