"""GPU parity for the Walsh-Hadamard rotation fused with quantization: codes,
scales and the NVFP4 global scale bit for bit against the oracle (which
rotates in fp32 with the same butterfly order and then quantizes), a GEMM on
rotated operands against the unrotated product, and the error reduction the
page claims for outlier channels."""
import numpy as np
import pytest
import torch

import oracle
from fp8_quantization_block_b200 import mx, synth
from gpu_helpers import first_mismatch, gemm_check, host, to_dev

pytestmark = pytest.mark.gpu
FMTS = [0, 1, 2, 3]


def rht_dev(bits, fmt, gscale=None):
    g = None if gscale is None else torch.tensor([gscale], dtype=torch.float32, device="cuda")
    q = mx.quantize_rht(to_dev(bits), fmt, gscale=g)
    torch.cuda.synchronize()
    mx.check_device_error()
    return q


def assert_rht_equal(q, bits, fmt, gscale=None):
    c, s, g = oracle.quantize_rht(fmt, bits, gscale=gscale)
    gc, gs, gg = host(q)
    assert first_mismatch(gc, c) is None, f"codes differ: {first_mismatch(gc, c)}"
    assert first_mismatch(gs, s) is None, f"scales differ: {first_mismatch(gs, s)}"
    if fmt == 3:
        assert np.float32(gg) == np.float32(g), (gg, g)


def edge_rows_in_range(K):
    """The codec edge rows without the one at the bf16 maximum (the sum of 32
    such values overflows fp32, which the rotation leaves outside its
    contract), plus a row of +-1e37 whose block sums stay finite."""
    rows = synth.edge_rows(K)
    big = synth.bits_to_tensor(rows).float().abs().amax(dim=1).numpy()
    keep = rows[big < 1e38]
    near = synth.to_bf16_bits(np.where(np.arange(K) % 5 == 0, -1e37, 1e37).astype(np.float32)[None, :])
    # all equal: the first rotated value is 32 c x ~ 5.6e37, near the largest a
    # finite block reaches (MXFP4 scale byte 250)
    flat = synth.to_bf16_bits(np.full((1, K), 1e37, dtype=np.float32))
    return np.vstack([keep, near, flat])


@pytest.mark.parametrize("fmt", FMTS)
def test_rht_tiny_edge_and_tie_rows(fmt):
    A, B = synth.tiny_pair()
    for bits in (A, B, np.vstack([edge_rows_in_range(256), synth.tie_rows(256, fmt)])):
        assert_rht_equal(rht_dev(bits, fmt), bits, fmt)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,K", [(1, 32), (200, 96), (129, 4096), (300, 160), (5, 2080)])
def test_rht_ragged_shapes(fmt, M, K):
    bits = synth.dit_activations(50 + M, M, K, n_outlier=min(8, K // 32))
    assert_rht_equal(rht_dev(bits, fmt), bits, fmt)


@pytest.mark.parametrize("g", [0.01, 1.0])
def test_rht_nvfp4_given_gscale(g):
    bits = synth.student_t(51, 96, 512)
    g32 = float(np.float32(g))
    assert_rht_equal(rht_dev(bits, 3, gscale=g32), bits, 3, gscale=g32)


@pytest.mark.parametrize("scale_exp", [-122, 100])
def test_rht_nvfp4_extreme_global_scales(scale_exp):
    # the rotated tensor near the bottom of the range (g subnormal) or near the top
    x = synth.bits_to_tensor(synth.student_t(56, 64, 512)).float().numpy() * np.float32(2.0 ** scale_exp)
    bits = synth.to_bf16_bits(x)
    assert_rht_equal(rht_dev(bits, 3), bits, 3)


def test_rht_row_pitch_larger_than_k():
    bits = synth.sweep_tensor(52, 70, 640)
    padded = torch.zeros((70, 704), dtype=torch.bfloat16, device="cuda")
    padded[:, :640] = to_dev(bits)
    q = mx.quantize_rht(padded[:, :640], 2)
    torch.cuda.synchronize()
    assert_rht_equal(q, bits, 2)


@pytest.mark.parametrize("fmt", [0, 2, 3])
def test_gemm_on_rotated_operands_approximates_the_plain_product(fmt):
    # (H x)(H w)^T = 32 x w^T, and c^2 * 32 = 1 up to fp32 rounding of c
    M, N, K = 256, 384, 1024
    xa = synth.dit_activations(53, M, K)
    wb = synth.gaussian_weights(54, N, K)
    qa, qb = rht_dev(xa, fmt), rht_dev(wb, fmt)
    Ct = mx.gemm(qa, qb)
    torch.cuda.synchronize()
    mx.check_device_error()
    C = Ct.float().cpu().double().numpy()
    ref = synth.bits_to_tensor(xa).double().numpy() @ synth.bits_to_tensor(wb).double().numpy().T
    rel = np.linalg.norm(C - ref) / np.linalg.norm(ref)
    assert rel < {0: 0.05, 2: 0.25, 3: 0.2}[fmt], rel
    # and the rotated GEMM is the oracle's rotated product within the GEMM tolerance
    ca, sa, ga = oracle.quantize_rht(fmt, xa)
    cb, sb, gb = oracle.quantize_rht(fmt, wb)
    Ad, Bd = oracle.dequantize_f64(fmt, ca, sa, ga, M, K), oracle.dequantize_f64(fmt, cb, sb, gb, N, K)
    ok, worst = gemm_check(Ct, Ad, Bd)
    assert ok, worst


def test_rotation_lowers_mxfp4_error_with_outlier_channels():
    bits = synth.dit_activations(55, 1024, 3072)
    x = to_dev(bits)
    plain = mx.qsnr_sums(mx.quantize(x, 2), x).cpu().numpy()
    rot = mx.quantize_rht(x, 2)
    torch.cuda.synchronize()
    # error of the rotated tensor, measured against the oracle's fp32 rotation
    y = oracle.rht32(bits).astype(np.float64)
    c, s, _ = host(rot)
    err = np.sum((y - oracle.dequantize_f64(2, c, s, 1.0, *bits.shape)) ** 2)
    assert err < 0.7 * plain[1], (err, plain[1])
