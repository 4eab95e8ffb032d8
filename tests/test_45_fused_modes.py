"""The fused call's activation quantize, band by band: X is quantized into the
workspace 128 rows at a time, each band counted as written, and the GEMM's TMA
producers load A from a band once its count is complete.  Two producers of the
bands: the quantize kernel, with the GEMM kernel launched to overlap it
(MX_FUSED_PIPELINED, the default), or the GEMM kernel's own epilogue warps,
which claim 32-row x 128-column items from a work counter before their first
tile (MX_FUSED_IN_KERNEL).

Every mode must give, bit for bit, the result of the quantize kernel followed
by the GEMM in plain stream order (MX_FUSED_TWO_KERNELS) and of mx_gemm on
mx_quantize's output, for every format pairing the fused call takes, ragged
shapes, both GEMM kernels, GELU and |C| max, grids capped so that one CTA (or
one pair) runs every output tile (and, in-kernel, quantizes every item), and
workspaces that start dirty or are reused.  The quantized X in the workspace
must equal mx_quantize's codes and scales; the full-size DiT shape is checked
against the oracle on sampled rows."""
import numpy as np
import pytest
import torch

import oracle
from fp8_quantization_block_b200 import mx, synth
from gpu_helpers import gemm_check, host, to_dev

pytestmark = pytest.mark.gpu


def i16(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.int16)


class debug:
    """Set libmx debug keys for a block, restoring their defaults after it."""
    DEFAULTS = {mx.MX_DEBUG_FUSED_MODE: mx.MX_FUSED_PIPELINED, mx.MX_DEBUG_MAX_GEMM_CTAS: 0, mx.MX_DEBUG_PAIR_GEMM: 1}

    def __init__(self, **kv):
        self.kv = {getattr(mx, "MX_DEBUG_" + k.upper()): v for k, v in kv.items()}

    def __enter__(self):
        for k, v in self.kv.items():
            assert mx.mx_debug_set(k, v) == mx.MX_OK

    def __exit__(self, *a):
        for k in self.kv:
            mx.mx_debug_set(k, self.DEFAULTS[k])


MODES = (mx.MX_FUSED_PIPELINED, mx.MX_FUSED_IN_KERNEL)


def run_modes(X, W, x_fmt=None, **kw):
    """The fused call in each mode, same arguments: {mode: C}."""
    out = {}
    for mode in MODES + (mx.MX_FUSED_TWO_KERNELS,):
        with debug(fused_mode=mode):
            out[mode] = mx.gemm_fused_act(X, W, x_fmt=x_fmt, **kw)
    torch.cuda.synchronize()
    mx.check_device_error()
    return out


def assert_all_equal(outs, ref):
    for mode, c in outs.items():
        assert torch.equal(i16(c), i16(ref)), f"mode {mode}"


SHAPES = [(64, 64, 256), (200, 300, 384), (333, 520, 1024), (512, 768, 1024), (16, 384, 512), (1, 640, 2048),
          (130, 128, 640), (257, 2000, 256)]


@pytest.mark.parametrize("fmt", [0, 1, 2, 3])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_fused_modes_equal_two_kernels_and_unfused(fmt, M, N, K):
    X = to_dev(synth.sweep_tensor(500 + M, M, K))
    W = mx.quantize(to_dev(synth.gaussian_weights(600 + N, N, K)), fmt)
    outs = run_modes(X, W)
    ref = mx.gemm(mx.quantize(X, fmt), W)
    torch.cuda.synchronize()
    assert_all_equal(outs, ref)


@pytest.mark.parametrize("x_fmt,w_fmt", [(4, 4), (0, 2), (2, 0), (1, 0), (0, 4), (4, 2)])
@pytest.mark.parametrize("M,N,K", [(200, 300, 384), (16, 384, 512), (333, 520, 1024)])
def test_fused_modes_mixed_and_mxfp6(x_fmt, w_fmt, M, N, K):
    """X quantized to any MX format inside the run-time-typed kind::mxf8f6f4 kernel."""
    X = to_dev(synth.student_t(510 + M, M, K))
    W = mx.quantize(to_dev(synth.gaussian_weights(610 + N, N, K)), w_fmt)
    outs = run_modes(X, W, x_fmt=x_fmt)
    ref = mx.gemm(mx.quantize(X, x_fmt), W)
    torch.cuda.synchronize()
    assert_all_equal(outs, ref)


@pytest.mark.parametrize("fmt", [0, 2, 3])
@pytest.mark.parametrize("ctas", [1, 3, 8])
@pytest.mark.parametrize("M,N,K", [(300, 1000, 256), (300, 1000, 2048), (100, 1000, 1024), (20, 1000, 2048)])
def test_fused_modes_with_few_ctas(fmt, ctas, M, N, K):
    """A grid of one CTA (or pair) runs every output tile (in-kernel: and
    quantizes every item of X itself before its first tile); a few CTAs share
    them.  GELU and |C| max included."""
    X = to_dev(synth.student_t(520 + M, M, K))
    W = mx.quantize(to_dev(synth.gaussian_weights(620 + N, N, K)), fmt)
    a_ref = torch.empty(1, device="cuda")
    with debug(fused_mode=mx.MX_FUSED_TWO_KERNELS):
        H_ref = mx.gemm_fused_act(X, W, epilogue=mx.MX_EPI_GELU, amax_out=a_ref)
    for mode in MODES:
        a = torch.empty(1, device="cuda")
        with debug(max_gemm_ctas=ctas, fused_mode=mode):
            H = mx.gemm_fused_act(X, W, epilogue=mx.MX_EPI_GELU, amax_out=a)
        torch.cuda.synchronize()
        mx.check_device_error()
        assert torch.equal(i16(H), i16(H_ref)), mode
        assert float(a.cpu()[0]) == float(a_ref.cpu()[0]) == float(H.abs().max().float().cpu())


@pytest.mark.parametrize("fmt", [0, 3])
def test_fused_modes_single_cta_tiles(fmt):
    """The single-CTA kernel for M > 128 (CTA pairs switched off): band-major
    tiles of 128 rows."""
    M, N, K = 400, 700, 768
    X = to_dev(synth.student_t(530, M, K))
    W = mx.quantize(to_dev(synth.gaussian_weights(630, N, K)), fmt)
    ref = mx.gemm(mx.quantize(X, fmt), W)
    with debug(pair_gemm=0):
        outs = run_modes(X, W)
    assert_all_equal(outs, ref)


def test_fused_modes_nvfp4_gscale_sources():
    M, N, K = 300, 512, 768
    X = to_dev(synth.student_t(540, M, K))
    W = mx.quantize(to_dev(synth.gaussian_weights(640, N, K)), 3)
    amax = X.abs().max().float().reshape(1)
    g = mx.quantize(X, 3).gscale
    ref = mx.gemm(mx.quantize(X, 3), W)
    for kw in ({}, {"x_amax": amax}, {"x_gscale": g}):
        outs = run_modes(X, W, **kw)
        for mode, c in outs.items():
            assert torch.equal(i16(c), i16(ref)), (mode, kw)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("fmt", [0, 3])
def test_workspace_dirty_and_reused(fmt, mode):
    """The call clears its counters itself: a workspace full of 0xFF gives the
    same result, and one workspace serves calls of different shapes in a row
    (on one stream, so they do not overlap)."""
    K, N = 1024, 512
    W = mx.quantize(to_dev(synth.gaussian_weights(650, N, K)), fmt)
    ws = mx.fused_workspace(fmt, 600, K)
    ws.fill_(0xFF)
    outs, refs = [], []
    for i, M in enumerate((600, 130, 300, 600, 1)):
        X = to_dev(synth.sweep_tensor(660 + i, M, K))
        with debug(fused_mode=mode):
            outs.append(mx.gemm_fused_act(X, W, workspace=ws))
        refs.append(mx.gemm(mx.quantize(X, fmt), W))
    torch.cuda.synchronize()
    mx.check_device_error()
    for o, r in zip(outs, refs):
        assert torch.equal(i16(o), i16(r))


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("fmt", [0, 1, 2, 3, 4])
def test_workspace_holds_mx_quantize_output(fmt, mode):
    """X's codes and scales, as the GEMM kernel wrote them into the workspace,
    equal mx_quantize's (the workspace layout is the header, then the codes,
    then the scales, each on a 256-byte boundary; the header holds 64 bytes,
    a counter per 128-row band and the 148 partial-sum slot counters)."""
    M, N, K = 333, 384, 1024
    X = to_dev(synth.sweep_tensor(670, M, K))
    W = mx.quantize(to_dev(synth.gaussian_weights(671, N, K)), 4 if fmt == 4 else fmt)
    ws = mx.fused_workspace(fmt, M, K)
    with debug(fused_mode=mode):
        mx.gemm_fused_act(X, W, workspace=ws, x_fmt=fmt)
    q = mx.quantize(X, fmt)
    torch.cuda.synchronize()
    header = ((64 + 4 * ((M + 127) // 128) + 4 * 148) + 255) // 256 * 256
    nc, ns = mx.mx_codes_bytes(fmt, M, K), mx.mx_scales_bytes(fmt, M, K)
    codes = ws[header:header + nc]
    so = header + (nc + 255) // 256 * 256
    scales = ws[so:so + ns]
    assert torch.equal(codes, q.codes[:nc])
    assert torch.equal(scales, q.scales[:ns])
    # every band counter reached its count: in-kernel, four 32-row items per
    # 128 x 128 tile, and the work counter ran past the last item; pipelined,
    # one quantize-kernel CTA per tile
    words = ws[:header].view(torch.int32).cpu().numpy()
    bands, items_k = (M + 127) // 128, (K + 127) // 128
    if mode == mx.MX_FUSED_IN_KERNEL:
        assert np.all(words[16:16 + bands] == 4 * items_k)
        assert words[2] >= bands * items_k * 4
    else:
        assert np.all(words[16:16 + bands] == items_k)


def test_dit_full_size_fused_modes():
    """The DiT MXFP8 Linear at its full size, 4096 x 3072 x 3072: every fused
    mode equals mx_quantize + mx_gemm bit for bit, and sampled rows are within
    the oracle's tolerance."""
    M, N, K = 4096, 3072, 3072
    X_bits = synth.dit_activations(1, M, K)
    W_bits = synth.gaussian_weights(2, N, K)
    X = to_dev(X_bits)
    W = mx.quantize(to_dev(W_bits), 0)
    outs = run_modes(X, W)
    one = outs[mx.MX_FUSED_PIPELINED]
    ref = mx.gemm(mx.quantize(X, 0), W)
    torch.cuda.synchronize()
    mx.check_device_error()
    assert_all_equal(outs, ref)
    rows = np.sort(np.random.default_rng(12).choice(M, 32, replace=False))
    cx, sx, gx = oracle.quantize(0, np.ascontiguousarray(X_bits[rows]))
    cw, sw, gw = host(W)
    ok, worst = gemm_check(one[torch.from_numpy(rows).cuda()],
                           oracle.dequantize_f64(0, cx, sx, gx, len(rows), K),
                           oracle.dequantize_f64(0, cw, sw, gw, N, K))
    assert ok, worst
