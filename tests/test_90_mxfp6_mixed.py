"""GPU parity for MXFP6 E3M2 (quantize / dequantize / QSNR bit for bit or to
fp64 rounding against the oracle) and for GEMMs on MXFP6 and on mixed MX
operands (kind::mxf8f6f4 with each operand's element type chosen at run
time), through the C ABI.

Page "Microscaling MXFP4/NVFP4 on Blackwell for reasoning LLMs", format table
(MXFP6 = E3M2 elements, E8M0 scale per 32 elements, 6.25 bits/element) and
section "Arquitetura Blackwell SM100" (the tensor core applies the block scales
during FP32 accumulation).
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_quantization_block_b200 import mx, synth
from gpu_helpers import assert_quant_equal, first_mismatch, gemm_check, host, quantize_dev, to_dev

pytestmark = pytest.mark.gpu
MXFP6 = 4


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    mx.check_device_error()


def test_mxfp6_tiny_edge_and_tie_rows():
    A, B = synth.tiny_pair()
    for bits in (A, B, np.vstack([synth.edge_rows(256), synth.tie_rows(256, MXFP6)])):
        assert_quant_equal(quantize_dev(bits, MXFP6), bits, MXFP6)


@pytest.mark.parametrize("M,K", [(1, 32), (200, 96), (129, 4096), (300, 160), (5, 2080), (1000, 3072)])
def test_mxfp6_ragged_shapes(M, K):
    bits = synth.sweep_tensor(90 + M, M, K)
    assert_quant_equal(quantize_dev(bits, MXFP6), bits, MXFP6)


def test_mxfp6_row_pitch_larger_than_k():
    bits = synth.sweep_tensor(91, 70, 640)
    padded = torch.zeros((70, 704), dtype=torch.bfloat16, device="cuda")
    padded[:, :640] = to_dev(bits)
    q = mx.quantize(padded[:, :640], MXFP6)
    torch.cuda.synchronize()
    assert_quant_equal(q, bits, MXFP6)


def test_mxfp6_dequantize_matches_oracle():
    bits = synth.student_t(92, 133, 1024)
    q = quantize_dev(bits, MXFP6)
    c, s, _ = host(q)
    d = mx.dequantize(q)
    torch.cuda.synchronize()
    got = d.view(torch.int16).cpu().numpy().view(np.uint16).ravel()
    want = oracle.dequantize_bf16(MXFP6, c, s, 1.0, 133, 1024).ravel()
    assert first_mismatch(got, want) is None, first_mismatch(got, want)


def test_mxfp6_rotation_matches_oracle():
    bits = synth.dit_activations(93, 129, 1024)
    q = mx.quantize_rht(to_dev(bits), MXFP6)
    torch.cuda.synchronize()
    c, s, _ = oracle.quantize_rht(MXFP6, bits)
    gc, gs, _ = host(q)
    assert first_mismatch(gc, c) is None and first_mismatch(gs, s) is None


def test_mxfp6_qsnr_sums_and_ordering():
    bits = synth.dit_activations(94, 256, 3072)
    q = quantize_dev(bits, MXFP6)
    c, s, _ = oracle.quantize(MXFP6, bits)
    db, sx, se = oracle.qsnr_db(bits, oracle.dequantize_f64(MXFP6, c, s, 1.0, 256, 3072))
    got = mx.qsnr_sums(q, to_dev(bits)).cpu().numpy()
    assert got[0] == pytest.approx(sx, rel=1e-12) and got[1] == pytest.approx(se, rel=1e-10)
    # 6 bits sit between MXFP4 and MXFP8
    q4, q8 = quantize_dev(bits, 2), quantize_dev(bits, 0)
    s4 = mx.qsnr_sums(q4, to_dev(bits)).cpu().numpy()
    s8 = mx.qsnr_sums(q8, to_dev(bits)).cpu().numpy()
    assert s8[1] < got[1] < s4[1]


GEMM_SHAPES = [(256, 384, 1024), (100, 96, 512), (128, 300, 256), (300, 520, 384), (24, 288, 640)]


def _dq(bits, fmt):
    c, s, g = oracle.quantize(fmt, bits)
    return oracle.dequantize_f64(fmt, c, s, g, *bits.shape)


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_mxfp6(M, N, K):
    xa = synth.dit_activations(95, M, K)
    wb = synth.gaussian_weights(96, N, K)
    C = mx.gemm(quantize_dev(xa, MXFP6), quantize_dev(wb, MXFP6))
    torch.cuda.synchronize()
    mx.check_device_error()
    ok, worst = gemm_check(C, _dq(xa, MXFP6), _dq(wb, MXFP6))
    assert ok, worst


MIXED = [(0, 2), (0, 4), (4, 2), (2, 0), (4, 0), (1, 0), (1, 4), (2, 4)]


@pytest.mark.parametrize("fa,fb", MIXED)
@pytest.mark.parametrize("M,N,K", [(256, 384, 1024), (100, 96, 512), (300, 520, 384), (9, 272, 512)])
def test_gemm_mixed_operands(fa, fb, M, N, K):
    xa = synth.dit_activations(97, M, K)
    wb = synth.gaussian_weights(98, N, K)
    C = mx.gemm(quantize_dev(xa, fa), quantize_dev(wb, fb))
    torch.cuda.synchronize()
    mx.check_device_error()
    ok, worst = gemm_check(C, _dq(xa, fa), _dq(wb, fb))
    assert ok, worst


def test_gemm_mixed_one_hot_probe():
    # A = e_i scaled, B = one code in one block: C picks exactly one product, so a
    # wrong nibble / 6-bit order, a swapped operand type or a misread scale shows
    # up as a wrong value at a wrong place
    M, N, K = 128, 128, 256
    rng = np.random.default_rng(99)
    for fa, fb in ((0, 4), (4, 2), (2, 4)):
        for _ in range(4):
            i, j, k = int(rng.integers(M)), int(rng.integers(N)), int(rng.integers(K))
            a = np.zeros((M, K), np.float32)
            b = np.zeros((N, K), np.float32)
            a[i, k] = 1.5 * 2.0 ** int(rng.integers(-3, 4))
            b[j, k] = -3.0 * 2.0 ** int(rng.integers(-3, 4))
            ab, bb = synth.to_bf16_bits(a), synth.to_bf16_bits(b)
            C = mx.gemm(quantize_dev(ab, fa), quantize_dev(bb, fb)).float().cpu().numpy()
            want = np.zeros((M, N))
            want[i, j] = float(a[i, k]) * float(b[j, k])
            assert np.array_equal(C, want), (fa, fb, i, j, k)


@pytest.mark.parametrize("xf,wf", [(0, 2), (0, 4), (4, 4), (4, 2)])
def test_fused_act_with_mixed_weights(xf, wf):
    M, N, K = 300, 384, 1024
    xa = synth.dit_activations(100, M, K)
    wb = synth.gaussian_weights(101, N, K)
    W = quantize_dev(wb, wf)
    C = mx.gemm_fused_act(to_dev(xa), W, x_fmt=xf)
    torch.cuda.synchronize()
    mx.check_device_error()
    ok, worst = gemm_check(C, _dq(xa, xf), _dq(wb, wf))
    assert ok, worst


@pytest.mark.parametrize("xf,wf", [(0, 2), (4, 4), (1, 0)])
@pytest.mark.parametrize("M,N,K", [(300, 1000, 256), (100, 1000, 2048)])
def test_several_tiles_per_cta_mixed(xf, wf, M, N, K):
    """The runtime-typed kernel (mixed operands, MXFP6) with a grid of one CTA
    (or one CTA pair), so that every CTA walks several tiles through both
    accumulators: plain and GELU results equal the one-tile-per-CTA launch
    bitwise, and GELU the fp64 oracle within the GEMM bound."""
    xa = synth.dit_activations(102, M, K)
    wb = synth.gaussian_weights(103, N, K)
    X = to_dev(xa)
    W = quantize_dev(wb, wf)
    qX = quantize_dev(xa, xf)
    H_ref = mx.gemm_fused_act(X, W, x_fmt=xf, epilogue=mx.MX_EPI_GELU)
    C_ref = mx.gemm(qX, W)
    try:
        assert mx.mx_debug_set(mx.MX_DEBUG_MAX_GEMM_CTAS, 1) == mx.MX_OK
        H = mx.gemm_fused_act(X, W, x_fmt=xf, epilogue=mx.MX_EPI_GELU)
        C = mx.gemm(qX, W)
        torch.cuda.synchronize()
        mx.check_device_error()
    finally:
        mx.mx_debug_set(mx.MX_DEBUG_MAX_GEMM_CTAS, 0)
    assert torch.equal(C.view(torch.int16), C_ref.view(torch.int16))
    assert torch.equal(H.view(torch.int16), H_ref.view(torch.int16))
    Cref, Cabs = oracle.gemm_f64(_dq(xa, xf), _dq(wb, wf))
    Href = oracle.gelu(Cref)
    Hg = H.float().cpu().double().numpy()
    bound = 1.13 * (2.0 ** -8 * np.abs(Cref) + 1e-4 * Cabs) + 2.0 ** -8 * np.abs(Href) + 1e-30
    assert np.all(np.abs(Hg - Href) <= bound), float(np.max(np.abs(Hg - Href) / bound))
