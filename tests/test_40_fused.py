"""Fused activation-quantize + GEMM: bitwise equal to mx_quantize + mx_gemm,
GELU / |C| max epilogue against the fp64 oracle, and the NVFP4 MLP chain
(GEMM1 -> GELU -> amax -> GEMM2) without a host sync."""
import numpy as np
import pytest
import torch

import oracle
from fp8_quantization_block_b200 import mx, synth
from gpu_helpers import gemm_check, host, to_dev

pytestmark = pytest.mark.gpu
FMTS = [0, 1, 2, 3]
# GELU is Lipschitz with constant max |GELU'(x)| = Phi(sqrt 2) + sqrt 2 phi(sqrt 2)
# = 1.128904 (at x = sqrt 2; the minimum, -0.128904, is at x = -sqrt 2), so an
# error e in the pre-activation moves GELU by at most 1.129 e: the GEMM bound
# times this factor, plus the bf16 rounding of H (2^-8 relative), bounds H.
GELU_LIPSCHITZ = 1.13


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,N,K", [(64, 64, 256), (200, 300, 384), (512, 768, 1024), (16, 384, 512)])
def test_fused_equals_unfused(fmt, M, N, K):
    X_bits = synth.sweep_tensor(300 + M, M, K)
    W_bits = synth.gaussian_weights(400 + N, N, K)
    X, Wt = to_dev(X_bits), to_dev(W_bits)
    W = mx.quantize(Wt, fmt)
    # without room for the K split, whose partial sums change the fp32 order
    C_f = mx.gemm_fused_act(X, W, workspace=mx.fused_workspace(fmt, M, K, split=False))
    C_u = mx.gemm(mx.quantize(X, fmt), W)
    torch.cuda.synchronize()
    mx.check_device_error()
    assert torch.equal(C_f.view(torch.int16), C_u.view(torch.int16))


def test_nvfp4_gscale_sources_agree():
    M, N, K = 256, 512, 768
    X = to_dev(synth.student_t(50, M, K))
    W = mx.quantize(to_dev(synth.gaussian_weights(51, N, K)), 3)
    C_pre = mx.gemm_fused_act(X, W)                                       # amax pre-pass
    amax = X.abs().max().float().reshape(1)
    C_amax = mx.gemm_fused_act(X, W, x_amax=amax)                         # g from amax
    g = mx.quantize(X, 3).gscale
    C_g = mx.gemm_fused_act(X, W, x_gscale=g)                             # g given
    torch.cuda.synchronize()
    assert torch.equal(C_pre.view(torch.int16), C_amax.view(torch.int16))
    assert torch.equal(C_pre.view(torch.int16), C_g.view(torch.int16))
    assert float(g.cpu()[0]) == oracle.nvfp4_global_scale(float(amax.cpu()[0]))


@pytest.mark.parametrize("fmt", [0, 3])
@pytest.mark.parametrize("M", [192, 20])
def test_gelu_and_amax_epilogue(fmt, M):
    N, K = 320, 512
    X_bits = synth.student_t(60, M, K)
    W_bits = synth.gaussian_weights(61, N, K)
    X = to_dev(X_bits)
    W = mx.quantize(to_dev(W_bits), fmt)
    amax = torch.full((1,), 123.0, device="cuda")
    H = mx.gemm_fused_act(X, W, epilogue=mx.MX_EPI_GELU, amax_out=amax)
    torch.cuda.synchronize()
    mx.check_device_error()
    # oracle: quantize X and W on the host, fp64 GEMM, fp64 GELU
    cx, sx, gx = oracle.quantize(fmt, X_bits)
    cw, sw, gw = host(W)
    Xd = oracle.dequantize_f64(fmt, cx, sx, gx, M, K)
    Wd = oracle.dequantize_f64(fmt, cw, sw, gw, N, K)
    Cref, Cabs = oracle.gemm_f64(Xd, Wd)
    Href = oracle.gelu(Cref)
    Hg = H.float().cpu().double().numpy()
    bound = GELU_LIPSCHITZ * (2.0 ** -8 * np.abs(Cref) + 1e-4 * Cabs) + 2.0 ** -8 * np.abs(Href) + 1e-30
    assert np.all(np.abs(Hg - Href) <= bound), float(np.max(np.abs(Hg - Href) / bound))
    assert float(amax.cpu()[0]) == float(H.abs().max().float().cpu())     # zeroed, then max |H|


@pytest.mark.parametrize("fmt", [0, 2, 3])
@pytest.mark.parametrize("M,N,K", [(300, 1000, 256), (300, 1000, 2048), (100, 1000, 256), (100, 1000, 2048),
                                   (20, 1000, 2048), (300, 100, 512)])
def test_several_tiles_per_cta(fmt, M, N, K):
    """A grid of one CTA (or one CTA pair) walks every tile, so consecutive
    tiles alternate between the two accumulators whose TMEM columns overlap.
    With GELU those shared columns are drained by the epilogue and the scale
    warps together, before (K > 4 stages) or after (K within the scale slots)
    the scale warps' last wait.  Shapes: the CTA-pair kernel (M = 300: a ragged
    second row block whose upper CTA has no rows), the single-CTA 128 x 256 and
    32-row variants, 128-wide N tiles; N = 1000 ends in a partial chunk.  The
    result must equal the one-tile-per-CTA launch bitwise, and GELU the fp64
    oracle within the GEMM bound."""
    X_bits = synth.student_t(90 + M, M, K)
    W_bits = synth.gaussian_weights(91 + N, N, K)
    X = to_dev(X_bits)
    W = mx.quantize(to_dev(W_bits), fmt)
    qX = mx.quantize(X, fmt)
    a_ref = torch.empty(1, device="cuda")
    H_ref = mx.gemm_fused_act(X, W, epilogue=mx.MX_EPI_GELU, amax_out=a_ref)
    C_ref = mx.gemm(qX, W)
    a = torch.empty(1, device="cuda")
    try:
        assert mx.mx_debug_set(mx.MX_DEBUG_MAX_GEMM_CTAS, 1) == mx.MX_OK
        H = mx.gemm_fused_act(X, W, epilogue=mx.MX_EPI_GELU, amax_out=a)
        C = mx.gemm(qX, W)
        torch.cuda.synchronize()
        mx.check_device_error()
    finally:
        mx.mx_debug_set(mx.MX_DEBUG_MAX_GEMM_CTAS, 0)
    assert torch.equal(C.view(torch.int16), C_ref.view(torch.int16))
    assert torch.equal(H.view(torch.int16), H_ref.view(torch.int16))
    assert float(a.cpu()[0]) == float(a_ref.cpu()[0]) == float(H.abs().max().float().cpu())
    cx, sx, gx = oracle.quantize(fmt, X_bits)
    cw, sw, gw = host(W)
    Cref, Cabs = oracle.gemm_f64(oracle.dequantize_f64(fmt, cx, sx, gx, M, K),
                                 oracle.dequantize_f64(fmt, cw, sw, gw, N, K))
    Href = oracle.gelu(Cref)
    Hg = H.float().cpu().double().numpy()
    bound = GELU_LIPSCHITZ * (2.0 ** -8 * np.abs(Cref) + 1e-4 * Cabs) + 2.0 ** -8 * np.abs(Href) + 1e-30
    assert np.all(np.abs(Hg - Href) <= bound), float(np.max(np.abs(Hg - Href) / bound))


def test_nvfp4_mlp_chain_without_host_sync():
    M, D, F = 256, 512, 1024
    X = to_dev(synth.student_t(70, M, D))
    W1 = mx.quantize(to_dev(synth.gaussian_weights(71, F, D)), 3)
    W2 = mx.quantize(to_dev(synth.gaussian_weights(72, D, F)), 3)
    aH = torch.empty(1, device="cuda")
    H = mx.gemm_fused_act(X, W1, epilogue=mx.MX_EPI_GELU, amax_out=aH)
    Y = mx.gemm_fused_act(H, W2, x_amax=aH, workspace=mx.fused_workspace(3, M, F, split=False))
    torch.cuda.synchronize()
    mx.check_device_error()
    # the same chain unfused: quantize H (g from its own amax) then GEMM
    qH = mx.quantize(H, 3)
    Y_u = mx.gemm(qH, W2)
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Y_u.view(torch.int16))
    # and against the oracle on H as produced by the GPU
    H_bits = bits16(H)
    ch, sh, gh = oracle.quantize(3, H_bits)
    assert np.array_equal(qH.codes.cpu().numpy(), ch) and np.array_equal(qH.scales.cpu().numpy(), sh)
    cw, sw, gw = host(W2)
    Hd = oracle.dequantize_f64(3, ch, sh, gh, M, F)
    W2d = oracle.dequantize_f64(3, cw, sw, gw, D, F)
    ok, worst = gemm_check(Y, Hd, W2d)
    assert ok, worst


def test_workspace_checks():
    X = torch.zeros((64, 256), dtype=torch.bfloat16, device="cuda")
    W = mx.quantize(torch.zeros((64, 256), dtype=torch.bfloat16, device="cuda"), 0)
    C = torch.empty((64, 64), dtype=torch.bfloat16, device="cuda")
    need = mx.mx_fused_workspace_bytes(0, 64, 256)
    ws = torch.empty(need + 512, dtype=torch.uint8, device="cuda")
    s = mx.mx_gemm_fused_act(0, X.data_ptr(), 64, 256, 256, W.c(), C.data_ptr(), 64, 0, None, None, None,
                             ws.data_ptr(), need - 1, None)
    assert s == mx.MX_ERR_INVALID_ARG
    s = mx.mx_gemm_fused_act(0, X.data_ptr(), 64, 256, 256, W.c(), C.data_ptr(), 64, 0, None, None, None,
                             ws.data_ptr() + 16, need, None)
    assert s == mx.MX_ERR_MISALIGNED
    s = mx.mx_gemm_fused_act(3, X.data_ptr(), 64, 256, 256, W.c(), C.data_ptr(), 64, 0, None, None, None,
                             ws.data_ptr(), need, None)
    assert s == mx.MX_ERR_INVALID_ARG                                      # NVFP4 X with an MXFP8 W
    torch.cuda.synchronize()


def test_nvfp4_mlp_pair_full_size_sampled_rows():
    """The NVFP4 MLP pair at its full size (X [4608 x 3072] Student-t, W1
    [12288 x 3072], W2 [3072 x 12288]): H = GELU(X W1^T) by the fused call
    with |H| max, then Y = H W2^T with H quantized in the call from that max,
    as one chain without a host sync.  Y equals the unfused chain bitwise; on
    sampled rows, X's and H's codes equal the oracle's and H and Y are within
    the tolerance of the fp64 oracle."""
    M, D, F = 4608, 3072, 12288
    X_bits = synth.student_t(3, M, D)
    W1 = mx.quantize(to_dev(synth.gaussian_weights(4, F, D)), 3)
    W2 = mx.quantize(to_dev(synth.gaussian_weights(5, D, F)), 3)
    X = to_dev(X_bits)
    aH = torch.empty(1, device="cuda")
    H = mx.gemm_fused_act(X, W1, epilogue=mx.MX_EPI_GELU, amax_out=aH)
    Y = mx.gemm_fused_act(H, W2, x_amax=aH, workspace=mx.fused_workspace(3, M, F, split=False))
    qX = mx.quantize(X, 3)
    qH = mx.quantize(H, 3)
    Y_u = mx.gemm(qH, W2)
    torch.cuda.synchronize()
    mx.check_device_error()
    assert torch.equal(Y.view(torch.int16), Y_u.view(torch.int16))
    assert float(aH.cpu()[0]) == float(H.abs().max().float().cpu())
    rows = np.sort(np.random.default_rng(11).choice(M, 24, replace=False))
    sel = torch.from_numpy(rows).cuda()

    def rows_quantized(q, row_bits, amax):
        """The oracle's codes of the sampled rows with the tensor's g, checked
        against the GPU's, and their fp64 values."""
        g = oracle.nvfp4_global_scale(amax)
        assert np.float32(float(q.gscale.cpu()[0])) == np.float32(g)
        c, s, _ = oracle.quantize(3, row_bits, gscale=g)
        K = row_bits.shape[1]
        gpu_codes = q.codes.view(-1, K // 2)[sel].cpu().numpy().reshape(-1)
        assert np.array_equal(gpu_codes, c)
        return oracle.dequantize_f64(3, c, s, g, len(rows), K)

    Xd = rows_quantized(qX, X_bits[rows], float(X.abs().max().float().cpu()))
    cw1, sw1, gw1 = host(W1)
    W1d = oracle.dequantize_f64(3, cw1, sw1, gw1, F, D)
    C1, C1abs = oracle.gemm_f64(Xd, W1d)
    del W1d
    Href = oracle.gelu(C1)
    Hg = H[sel].float().cpu().double().numpy()
    bound = GELU_LIPSCHITZ * (2.0 ** -8 * np.abs(C1) + 1e-4 * C1abs) + 2.0 ** -8 * np.abs(Href) + 1e-30
    assert np.all(np.abs(Hg - Href) <= bound), float(np.max(np.abs(Hg - Href) / bound))
    Hd = rows_quantized(qH, bits16(H[sel]), float(aH.cpu()[0]))
    cw2, sw2, gw2 = host(W2)
    W2d = oracle.dequantize_f64(3, cw2, sw2, gw2, D, F)
    Yref, Yabs = oracle.gemm_f64(Hd, W2d)
    ok, worst = oracle.gemm_tolerance_ok(Y[sel].float().cpu().double().numpy(), Yref, Yabs)
    assert ok, worst
