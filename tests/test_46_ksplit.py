"""The fused call with the last wave of tiles split along K (partial sums in the
workspace, added by the worker that finishes each tile): within the GEMM
tolerance of the fp64 oracle on both GEMM kernels, every format pairing,
ragged shapes and grids small enough that every tile is split; the same bits
from call to call and in every fused mode; |C| max equal to the output's; and
at the full DiT and skinny shapes, on sampled rows and weight bands."""
import numpy as np
import pytest
import torch

import oracle
from fp8_quantization_block_b200 import mx, synth
from gpu_helpers import gemm_check, host, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture
def debug_keys():
    set_keys = []

    def set_key(key, value):
        assert mx.mx_debug_set(key, value) == mx.MX_OK
        set_keys.append(key)

    yield set_key
    defaults = {mx.MX_DEBUG_K_SPLIT: mx.MX_K_SPLIT_AUTO, mx.MX_DEBUG_MAX_GEMM_CTAS: 0,
                mx.MX_DEBUG_FUSED_MODE: mx.MX_FUSED_PIPELINED}
    for k in set_keys:
        mx.mx_debug_set(k, defaults[k])


def plan(fmt, M, N, K, cap, epilogue=0):
    """(tiles, workers, stages) of the launch the library makes for this shape."""
    kbytes = K // (2 if fmt in (2, 3) else 1)
    kt = (kbytes + 127) // 128
    sms = 148
    if M > 128 and N > 128:
        bn = 128 if epilogue else 256
        tiles = -(-M // 256) * -(-N // bn)
        workers = (cap + 1) // 2 if 0 < cap < sms else sms // 2
    else:
        bn = 128 if N <= 128 else 256
        tiles = -(-M // 128) * -(-N // bn)
        workers = cap if 0 < cap < sms else sms
    return tiles, workers, kt


def x_dequantized(X_bits, fmt):
    M, K = X_bits.shape
    c, s, g = oracle.quantize(fmt, X_bits)
    return oracle.dequantize_f64(fmt, c, s, g, M, K)


# (X format, W format, M, N, K, grid cap): every case leaves a ragged last wave
# that the split covers (checked against the host plan below)
CASES = [
    (0, 0, 100, 1000, 1024, 6),      # single-CTA kernel, 4 tiles on 6 CTAs: all split, 1 partial sum each
    (0, 0, 100, 1000, 2048, 7),      # 2 partial sums per tile
    (3, 3, 16, 2048, 8192, 19),      # decode-shape kernel (32-row A), NVFP4, up to 3 partial sums
    (2, 2, 1, 1300, 2048, 8),        # one row, ragged N
    (1, 1, 128, 640, 1536, 6),       # E5M2, 12 stages per tile
    (0, 0, 384, 128, 4096, 8),       # N <= 128 tiles, M > 128 (128-row slots), 3 partial sums
    (0, 0, 600, 700, 2048, 10),      # CTA pairs, ragged M and N: 5 whole tiles, then 4 split over 5 pairs
    (3, 3, 512, 512, 8192, 22),      # CTA pairs, NVFP4, 3 partial sums
    (0, 2, 300, 520, 2048, 20),      # CTA pairs, MXFP8 x MXFP4 (run-time operand types), 2 partial sums
    (4, 4, 260, 1024, 2048, 6),      # CTA pairs, MXFP6
]


@pytest.mark.parametrize("xf,wf,M,N,K,cap", CASES)
def test_split_within_tolerance_and_deterministic(debug_keys, xf, wf, M, N, K, cap):
    tiles, workers, kt = plan(wf if xf == wf else 0, M, N, K, cap)
    n, units = mx.split_units(tiles, workers, kt, mx.MX_K_SPLIT_ALWAYS, 0)
    assert any(u[3] != mx.KUNIT_WHOLE for c in range(n) for u in mx.split_units(tiles, workers, kt, 2, c)[1])
    debug_keys(mx.MX_DEBUG_MAX_GEMM_CTAS, cap)
    debug_keys(mx.MX_DEBUG_K_SPLIT, mx.MX_K_SPLIT_ALWAYS)
    X_bits = synth.student_t(4600 + M, M, K)
    W_bits = synth.gaussian_weights(4700 + N, N, K)
    X = to_dev(X_bits)
    W = mx.quantize(to_dev(W_bits), wf)
    ws = mx.fused_workspace(xf, M, K)
    amax = torch.empty(1, device="cuda")
    C1 = mx.gemm_fused_act(X, W, workspace=ws, x_fmt=xf, amax_out=amax)
    C2 = mx.gemm_fused_act(X, W, workspace=ws, x_fmt=xf)
    C0 = mx.gemm_fused_act(X, W, workspace=mx.fused_workspace(xf, M, K, split=False), x_fmt=xf)
    torch.cuda.synchronize()
    mx.check_device_error()
    assert torch.equal(C1.view(torch.int16), C2.view(torch.int16))          # the same bits every call
    assert float(amax.cpu()[0]) == float(C1.abs().max().float().cpu())
    cw, sw, gw = host(W)
    Wd = oracle.dequantize_f64(wf, cw, sw, gw, N, K)
    Xd = x_dequantized(X_bits, xf)
    for C in (C1, C0):
        ok, worst = gemm_check(C, Xd, Wd)
        assert ok, worst


@pytest.mark.parametrize("xf,M,N,K,cap", [(0, 600, 700, 2048, 10), (3, 512, 512, 8192, 22), (2, 100, 1000, 1024, 6)])
def test_split_same_bits_in_every_fused_mode(debug_keys, xf, M, N, K, cap):
    debug_keys(mx.MX_DEBUG_MAX_GEMM_CTAS, cap)
    debug_keys(mx.MX_DEBUG_K_SPLIT, mx.MX_K_SPLIT_ALWAYS)
    X = to_dev(synth.dit_activations(4800, M, K))
    W = mx.quantize(to_dev(synth.gaussian_weights(4801, N, K)), xf)
    ws = mx.fused_workspace(xf, M, K)
    out = {}
    for mode in (mx.MX_FUSED_PIPELINED, mx.MX_FUSED_IN_KERNEL, mx.MX_FUSED_TWO_KERNELS):
        debug_keys(mx.MX_DEBUG_FUSED_MODE, mode)
        ws.fill_(0xA5)                                                     # a dirty workspace
        out[mode] = mx.gemm_fused_act(X, W, workspace=ws)
    torch.cuda.synchronize()
    mx.check_device_error()
    ref = out[mx.MX_FUSED_PIPELINED]
    for mode, c in out.items():
        assert torch.equal(c.view(torch.int16), ref.view(torch.int16)), mode


def test_gelu_is_never_split(debug_keys):
    """The split is planned only for the plain epilogue; GELU calls run whole
    tiles and equal the same call without room for the split."""
    debug_keys(mx.MX_DEBUG_MAX_GEMM_CTAS, 10)
    debug_keys(mx.MX_DEBUG_K_SPLIT, mx.MX_K_SPLIT_ALWAYS)
    M, N, K = 512, 512, 2048
    X = to_dev(synth.student_t(4900, M, K))
    W = mx.quantize(to_dev(synth.gaussian_weights(4901, N, K)), 0)
    H1 = mx.gemm_fused_act(X, W, epilogue=mx.MX_EPI_GELU, workspace=mx.fused_workspace(0, M, K))
    H0 = mx.gemm_fused_act(X, W, epilogue=mx.MX_EPI_GELU, workspace=mx.fused_workspace(0, M, K, split=False))
    torch.cuda.synchronize()
    mx.check_device_error()
    assert torch.equal(H1.view(torch.int16), H0.view(torch.int16))


def test_dit_shape_full_size_sampled_rows(debug_keys):
    """The DiT MXFP8 GEMM at full size through the fused call with the split
    of its last wave forced (192 pair tiles on 74 pairs: the last 44 split
    along K; the default leaves GEMMs of several waves whole) on rows from
    every band, the split bands included; the same bits on a second call."""
    debug_keys(mx.MX_DEBUG_K_SPLIT, mx.MX_K_SPLIT_ALWAYS)
    M, N, K = 4096, 3072, 3072
    tiles, workers, kt = plan(0, M, N, K, 0)
    assert mx.split_units(tiles, workers, kt, mx.MX_K_SPLIT_ALWAYS, 0)[1][-1][3] != mx.KUNIT_WHOLE
    X_bits = synth.dit_activations(1, M, K)
    W_bits = synth.gaussian_weights(2, N, K)
    X = to_dev(X_bits)
    W = mx.quantize(to_dev(W_bits), 0)
    ws = mx.fused_workspace(0, M, K)
    C1 = mx.gemm_fused_act(X, W, workspace=ws)
    C2 = mx.gemm_fused_act(X, W, workspace=ws)
    torch.cuda.synchronize()
    mx.check_device_error()
    assert torch.equal(C1.view(torch.int16), C2.view(torch.int16))
    rows = np.sort(np.concatenate([np.random.default_rng(21).choice(3072, 8, replace=False),
                                   np.random.default_rng(22).choice(np.arange(3072, 4096), 16, replace=False),
                                   [3072, 3327, 3328, 4095]]))
    cw, sw, gw = host(W)
    ok, worst = gemm_check(C1, x_dequantized(X_bits, 0), oracle.dequantize_f64(0, cw, sw, gw, N, K), rows=rows)
    assert ok, worst


def _band_rows(q: mx.MxTensor, fmt: int, bands, K: int):
    """Codes and scales of whole 128-row bands of a quantized weight."""
    codes, scales, g = host(q)
    codes = codes.reshape(q.rows, -1)
    tiles_k = -(-K // (16 if fmt == 3 else 32) // 4)
    sc = scales.reshape(-1, tiles_k * 512)
    c = np.concatenate([codes[b * 128:(b + 1) * 128] for b in bands])
    s = np.concatenate([sc[b] for b in bands])
    return c.reshape(-1), s.reshape(-1), g


@pytest.mark.parametrize("fmt,M,N,K,mode", [
    (3, 16, 8192, 28672, mx.MX_K_SPLIT_AUTO),     # a down projection at decode: 32 tiles on 148 CTAs
    (2, 1, 8192, 28672, mx.MX_K_SPLIT_AUTO),
    (3, 128, 8192, 28672, mx.MX_K_SPLIT_AUTO),
    (3, 16, 28672, 8192, mx.MX_K_SPLIT_ALWAYS),   # 112 tiles on 148 CTAs, split when forced
])
def test_skinny_full_size_weight_bands(debug_keys, fmt, M, N, K, mode):
    """Weight-streaming GEMMs at full size with their tiles split along K over
    all 148 SMs: every row of C on four 128-row bands of W, the first and last
    among them."""
    debug_keys(mx.MX_DEBUG_K_SPLIT, mode)
    tiles, workers, kt = plan(fmt, M, N, K, 0)
    n, units = mx.split_units(tiles, workers, kt, mode, 0)
    assert any(u[3] != mx.KUNIT_WHOLE for u in units)
    X_bits = synth.student_t(5000 + M, M, K)
    X = to_dev(X_bits)
    W = mx.quantize(to_dev(synth.gaussian_weights(5001, N, K)), fmt)
    C = mx.gemm_fused_act(X, W)
    torch.cuda.synchronize()
    mx.check_device_error()
    nb = N // 128
    bands = [0, nb // 3, 2 * nb // 3, nb - 1]
    c, s, g = _band_rows(W, fmt, bands, K)
    Wd = oracle.dequantize_f64(fmt, c, s, g, 128 * len(bands), K)
    cols = np.concatenate([np.arange(b * 128, (b + 1) * 128) for b in bands])
    Cref, Cabs = oracle.gemm_f64(x_dequantized(X_bits, fmt), Wd)
    ok, worst = oracle.gemm_tolerance_ok(C.float().cpu().double().numpy()[:, cols], Cref, Cabs)
    assert ok, worst
