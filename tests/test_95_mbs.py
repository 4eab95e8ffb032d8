"""GPU parity for MXFP4 with static macro-block scaling (codes, base-block
scales and macro mantissas bit for bit against the oracle; dequantize and
QSNR), through the C ABI.

Page "Unveiling the Potential of Quantization with MXFP4: Strategies for
Quantization Error Reduction", section B (Macro Block Scaling).
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_quantization_block_b200 import mx, synth
from gpu_helpers import assert_quant_equal, first_mismatch, host, quantize_dev, to_dev

pytestmark = pytest.mark.gpu
MBS = 5


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    mx.check_device_error()


def test_mbs_tiny_edge_and_tie_rows():
    A, B = synth.tiny_pair()
    for bits in (A, B, np.vstack([synth.edge_rows(256), synth.tie_rows(256, 2), synth.tie_rows(256, 3)])):
        assert_quant_equal(quantize_dev(bits, MBS), bits, MBS)


@pytest.mark.parametrize("gen", ["sweep", "dit", "student_t"])
@pytest.mark.parametrize("M,K", [(1, 128), (200, 256), (129, 4096), (300, 384), (5, 2048)])
def test_mbs_shapes(gen, M, K):
    bits = {"sweep": synth.sweep_tensor, "dit": synth.dit_activations, "student_t": synth.student_t}[gen](95 + M, M, K)
    c, s, _ = assert_quant_equal(quantize_dev(bits, MBS), bits, MBS)
    assert oracle.mbs_macro_bytes(s, M, K).any() or gen == "sweep"


def test_mbs_row_pitch_larger_than_k():
    bits = synth.sweep_tensor(96, 70, 640)
    padded = torch.zeros((70, 704), dtype=torch.bfloat16, device="cuda")
    padded[:, :640] = to_dev(bits)
    q = mx.quantize(padded[:, :640], MBS)
    torch.cuda.synchronize()
    assert_quant_equal(q, bits, MBS)


def test_mbs_outliers_and_tiny_blocks():
    # outliers of every size in one macro block, subnormal-only blocks, zero blocks
    rng = np.random.default_rng(97)
    x = rng.normal(0, 1, (64, 512)).astype(np.float32)
    x[:, 5::128] = (10.0 ** rng.uniform(-2, 3, (64, 4))).astype(np.float32)
    x[::7, 128:256] = 0.0
    x[3::9, 256:384] = (rng.normal(0, 1, (len(range(3, 64, 9)), 128)) * 2.0 ** -130).astype(np.float32)
    bits = synth.to_bf16_bits(x)
    assert_quant_equal(quantize_dev(bits, MBS), bits, MBS)


def test_mbs_dequantize_matches_oracle():
    bits = synth.dit_activations(98, 133, 1024)
    q = quantize_dev(bits, MBS)
    c, s, _ = host(q)
    d = mx.dequantize(q)
    torch.cuda.synchronize()
    got = d.view(torch.int16).cpu().numpy().view(np.uint16).ravel()
    want = oracle.dequantize_bf16(MBS, c, s, 1.0, 133, 1024).ravel()
    assert first_mismatch(got, want) is None, first_mismatch(got, want)


def test_mbs_qsnr_sums_and_gap_to_nvfp4():
    bits = synth.student_t(99, 256, 3072)
    q = quantize_dev(bits, MBS)
    c, s, _ = oracle.quantize(MBS, bits)
    db, sx, se = oracle.qsnr_db(bits, oracle.dequantize_f64(MBS, c, s, 1.0, 256, 3072))
    got = mx.qsnr_sums(q, to_dev(bits)).cpu().numpy()
    assert got[0] == pytest.approx(sx, rel=1e-12) and got[1] == pytest.approx(se, rel=1e-10)
    s4 = mx.qsnr_sums(quantize_dev(bits, 2), to_dev(bits)).cpu().numpy()
    assert got[1] < s4[1] / 1.5                     # well above plain MXFP4


def test_gemm_rejects_mbs_with_another_format():
    """MXFP4-MBS multiplies only with MXFP4-MBS (tests/test_96_mbs_gemm.py)."""
    bits = synth.gaussian_weights(100, 128, 256)
    q = quantize_dev(bits, MBS)
    for other in (0, 2, 3):
        o = quantize_dev(bits, other)
        C = torch.empty((128, 128), dtype=torch.bfloat16, device="cuda")
        assert mx.mx_gemm(q.c(), o.c(), C.data_ptr(), 128, None) == mx.MX_ERR_INVALID_ARG
        assert mx.mx_gemm(o.c(), q.c(), C.data_ptr(), 128, None) == mx.MX_ERR_INVALID_ARG
