"""GPU parity for MXFP4 with overflow-aware scaling (codes and scales bit for
bit against the oracle, and the GEMM on OAS operands) and for the QSNR sums
(against the oracle's fp64 sums), through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from fp8_quantization_block_b200 import mx, synth
from gpu_helpers import first_mismatch, gemm_check, host, to_dev

pytestmark = pytest.mark.gpu
MXFP4 = 2


def oas_dev(bits: np.ndarray) -> mx.MxTensor:
    q = mx.quantize_oas(to_dev(bits))
    torch.cuda.synchronize()
    mx.check_device_error()
    return q


def assert_oas_equal(q: mx.MxTensor, bits: np.ndarray):
    c, s = oracle.quantize_oas(bits)
    gc, gs, _ = host(q)
    assert first_mismatch(gc, c) is None, f"codes differ: {first_mismatch(gc, c)}"
    assert first_mismatch(gs, s) is None, f"scales differ: {first_mismatch(gs, s)}"
    return c, s


def test_oas_tiny_edge_and_tie_rows():
    A, B = synth.tiny_pair()
    for bits in (A, B, np.vstack([synth.edge_rows(256), synth.tie_rows(256, MXFP4)])):
        assert_oas_equal(oas_dev(bits), bits)


@pytest.mark.parametrize("M,K", [(1, 32), (200, 96), (129, 4096), (300, 160), (5, 2080), (1000, 3072)])
def test_oas_ragged_shapes(M, K):
    bits = synth.sweep_tensor(70 + M, M, K)
    assert_oas_equal(oas_dev(bits), bits)


def test_oas_differs_from_ocp_only_in_the_saturating_band():
    bits = synth.dit_activations(71, 256, 3072)
    q_oas, q_ocp = oas_dev(bits), mx.quantize(to_dev(bits), MXFP4)
    torch.cuda.synchronize()
    so, sc = q_oas.scales.cpu().numpy().astype(int), q_ocp.scales.cpu().numpy().astype(int)
    d = so - sc
    assert set(np.unique(d)) <= {-1, 0}
    assert (d == -1).sum() > 0          # the band (3, 3.5] is hit by some blocks


def test_gemm_on_oas_operands():
    M, N, K = 300, 384, 1024
    xa = synth.dit_activations(72, M, K)
    wb = synth.gaussian_weights(73, N, K)
    qa, qb = oas_dev(xa), oas_dev(wb)
    C = mx.gemm(qa, qb)
    torch.cuda.synchronize()
    mx.check_device_error()
    ca, sa = oracle.quantize_oas(xa)
    cb, sb = oracle.quantize_oas(wb)
    ok, worst = gemm_check(C, oracle.dequantize_f64(MXFP4, ca, sa, 1.0, M, K),
                           oracle.dequantize_f64(MXFP4, cb, sb, 1.0, N, K))
    assert ok, worst


def _qsnr_dev(q: mx.MxTensor, bits: np.ndarray):
    s = mx.qsnr_sums(q, to_dev(bits))
    torch.cuda.synchronize()
    mx.check_device_error()
    return s.cpu().numpy()


@pytest.mark.parametrize("fmt", [0, 1, 2, 3, "oas"])
@pytest.mark.parametrize("gen,M,K", [("student_t", 257, 1024), ("dit", 128, 3072), ("sweep", 33, 4096)])
def test_qsnr_sums_match_oracle(fmt, gen, M, K):
    bits = {"student_t": synth.student_t, "dit": synth.dit_activations, "sweep": synth.sweep_tensor}[gen](74, M, K)
    if fmt == "oas":
        q = oas_dev(bits)
        c, s = oracle.quantize_oas(bits)
        xh = oracle.dequantize_f64(MXFP4, c, s, 1.0, M, K)
    else:
        q = mx.quantize(to_dev(bits), fmt)
        c, s, g = oracle.quantize(fmt, bits)
        xh = oracle.dequantize_f64(fmt, c, s, g, M, K)
    db, sx, se = oracle.qsnr_db(bits, xh)
    got = _qsnr_dev(q, bits)
    assert got[0] == pytest.approx(sx, rel=1e-12)
    assert got[1] == pytest.approx(se, rel=1e-10)
    assert 10 * np.log10(got[0] / got[1]) == pytest.approx(db, abs=1e-8)


def test_qsnr_of_an_exactly_representable_tensor_has_zero_error():
    # codes 0..7 scaled by a power of two in every MXFP4 block: quantization is exact
    rng = np.random.default_rng(75)
    vals = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float32)
    x = vals[rng.integers(0, 8, size=(64, 256))] * np.float32(2.0 ** -3)
    x[:, ::32] = 6.0 * 2.0 ** -3                      # each block reaches the format maximum
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    got = _qsnr_dev(mx.quantize(to_dev(bits), MXFP4), bits)
    assert got[1] == 0.0 and got[0] > 0.0
