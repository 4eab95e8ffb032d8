"""mx_gemm_fused_act_noalloc: the fused quantize + GEMM for callers that cannot
allocate device memory (for example while a stream is being captured, inside an
inference engine's plugin callback, or under a fixed memory budget).  It uses a
fixed scratch array inside the library instead of a caller workspace.

Checked through the C ABI against the workspace-taking mx_gemm_fused_act on the
same inputs, on two calls in a row (the second call reuses the scratch the
first one left behind), and against the fp64 oracle's tolerance.  This file is
collected last and also runs on its own in a fresh process."""
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
        want = mx.gemm_fused_act(X, W)
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
    H2 = mx.gemm_fused_act(X, W1, epilogue=mx.MX_EPI_GELU, amax_out=a2)
    Y2 = mx.gemm_fused_act(H2, W2, x_amax=a2)
    torch.cuda.synchronize()
    mx.check_device_error()
    assert torch.equal(H1.view(torch.int16), H2.view(torch.int16))
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    assert float(a1.cpu()[0]) == float(a2.cpu()[0])


def test_noalloc_rejects_shapes_beyond_its_scratch():
    fmt, K = 0, 4096
    M = mx.MX_NOALLOC_SCRATCH_BYTES // K + 128       # codes alone exceed the scratch
    assert mx.mx_fused_workspace_bytes(fmt, M, K) > mx.MX_NOALLOC_SCRATCH_BYTES
    W = mx.quantize(torch.zeros((64, K), dtype=torch.bfloat16, device="cuda"), fmt)
    s = mx.mx_gemm_fused_act_noalloc(fmt, 0x1000, M, K, K, W.c(), 0x2000, 64, 0, None, None, None, None)
    assert s == mx.MX_ERR_UNSUPPORTED_SHAPE
    # the largest accepted shape runs
    M_ok = 256
    assert mx.mx_fused_workspace_bytes(fmt, M_ok, K) <= mx.MX_NOALLOC_SCRATCH_BYTES
    X = synth.bits_to_tensor(synth.sweep_tensor(913, M_ok, K)).cuda()
    got = _noalloc(X, W)
    want = mx.gemm_fused_act(X, W)
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
