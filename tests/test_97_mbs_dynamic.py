"""GPU parity of MXFP4 with dynamic macro-block scaling (the macro mantissa of
each 128 elements chosen by exhaustive error search): codes, base-block
exponents and macro bytes bit for bit against the oracle, through the C ABI;
the result feeds dequantize, QSNR and the MBS GEMM unchanged.

Page "Unveiling the Potential of Quantization with MXFP4", section 2.B."""
import numpy as np
import pytest
import torch

import oracle
from fp8_quantization_block_b200 import mx, synth
from gpu_helpers import first_mismatch, gemm_check, host, to_dev

pytestmark = pytest.mark.gpu
MBS = 5


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    mx.check_device_error()


def assert_dynamic_equal(bits):
    M, K = bits.shape
    q = mx.quantize_mbs_dynamic(to_dev(bits))
    torch.cuda.synchronize()
    c, s, _ = host(q)
    oc, os_ = oracle.quantize_mbs_dynamic(bits)
    assert first_mismatch(c, oc) is None, first_mismatch(c, oc)
    assert first_mismatch(s, os_) is None, first_mismatch(s, os_)
    return q


def test_dynamic_tiny_edge_and_tie_rows():
    A, B = synth.tiny_pair()
    for bits in (A, B, np.vstack([synth.edge_rows(256), synth.tie_rows(256, 2), synth.tie_rows(256, 3)])):
        assert_dynamic_equal(bits)


@pytest.mark.parametrize("gen", ["sweep", "dit", "student_t"])
@pytest.mark.parametrize("M,K", [(1, 128), (130, 256), (37, 1024), (300, 384)])
def test_dynamic_shapes(gen, M, K):
    bits = {"sweep": synth.sweep_tensor, "dit": synth.dit_activations, "student_t": synth.student_t}[gen](970 + M, M, K)
    assert_dynamic_equal(bits)


def test_dynamic_wide_range_blocks():
    rng = np.random.default_rng(975)
    x = rng.normal(0, 1, (48, 512)).astype(np.float32)
    x[:, 5::128] = (10.0 ** rng.uniform(-2, 3, (48, 4))).astype(np.float32)
    x[::7, 128:256] = 0.0
    x[3::9, 256:384] = (rng.normal(0, 1, (len(range(3, 48, 9)), 128)) * 2.0 ** -130).astype(np.float32)
    assert_dynamic_equal(synth.to_bf16_bits(x))


def test_dynamic_not_below_static_qsnr_and_gemm():
    M, N, K = 256, 384, 1024
    X_bits = synth.student_t(976, M, K)
    W_bits = synth.gaussian_weights(977, N, K)
    X = to_dev(X_bits)
    qd = mx.quantize_mbs_dynamic(X)
    qs = mx.quantize(X, MBS)
    sd = mx.qsnr_sums(qd, X).cpu().numpy()
    ss = mx.qsnr_sums(qs, X).cpu().numpy()
    assert sd[1] <= ss[1]                 # no more squared error than the static choice
    qw = mx.quantize_mbs_dynamic(to_dev(W_bits))
    C = mx.gemm(qd, qw)
    torch.cuda.synchronize()
    ca, sa, _ = host(qd)
    cb, sb, _ = host(qw)
    ok, worst = gemm_check(C, oracle.dequantize_f64(MBS, ca, sa, 1.0, M, K), oracle.dequantize_f64(MBS, cb, sb, 1.0, N, K))
    assert ok, worst


def test_dynamic_argument_checks():
    q = mx.empty(MBS, 4, 256)
    assert mx.mx_quantize_mbs_dynamic(0x1000, 4, 200, 256, mx.empty(MBS, 4, 200).c(), None) == mx.MX_ERR_UNSUPPORTED_SHAPE
    assert mx.mx_quantize_mbs_dynamic(0x1000, 4, 256, 256, mx.empty(2, 4, 256).c(), None) == mx.MX_ERR_INVALID_ARG
    assert mx.mx_quantize_mbs_dynamic(0x1008, 4, 256, 256, q.c(), None) == mx.MX_ERR_MISALIGNED
