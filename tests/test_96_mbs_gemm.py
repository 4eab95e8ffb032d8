"""GPU parity of the MXFP4-MBS GEMM (macro-block scaling, page "Unveiling the
Potential of Quantization with MXFP4", section 2.B): C = A_dq B_dq^T with both
operands MXFP4-MBS, within the GEMM tolerance of the fp64 oracle on the
oracle's own dequantized operands, through the C ABI.

The kernel runs each 128-element macro block as two block32 MMA passes (one
per 16-element base block of every 32-element group, the other half cleared)
and applies the macro factors (1 + mA/256)(1 + mB/256) to the partial sum on
the CUDA cores.  Shapes cover a ragged last stage (K an odd multiple of 128),
ragged M and N, a single row, and inputs whose two base blocks per group have
very different exponents (so a wrong pass or scale assignment shows)."""
import numpy as np
import pytest
import torch

import oracle
from fp8_quantization_block_b200 import mx, synth
from gpu_helpers import gemm_check, host, to_dev

pytestmark = pytest.mark.gpu
MBS = 5


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    mx.check_device_error()


def check_mbs_gemm(A_bits, B_bits, rows=None):
    M, K = A_bits.shape
    N = B_bits.shape[0]
    qa, qb = mx.quantize(to_dev(A_bits), MBS), mx.quantize(to_dev(B_bits), MBS)
    C = mx.gemm(qa, qb)
    torch.cuda.synchronize()
    ca, sa, _ = host(qa)
    cb, sb, _ = host(qb)
    # the GPU's operands are the oracle's, bit for bit
    oa, osa, _ = oracle.quantize(MBS, A_bits)
    assert np.array_equal(ca, oa) and np.array_equal(sa, osa)
    Ad = oracle.dequantize_f64(MBS, ca, sa, 1.0, M, K)
    Bd = oracle.dequantize_f64(MBS, cb, sb, 1.0, N, K)
    ok, worst = gemm_check(C, Ad, Bd, rows=rows)
    assert ok, worst
    return C


@pytest.mark.parametrize("M,N,K", [(64, 64, 256), (200, 300, 384), (333, 520, 1024), (1, 640, 2048),
                                   (130, 128, 640), (257, 129, 128), (128, 256, 3072)])
def test_mbs_gemm_against_oracle(M, N, K):
    check_mbs_gemm(synth.student_t(960 + M, M, K), synth.gaussian_weights(961 + N, N, K))


def test_mbs_gemm_alternating_block_exponents():
    """Every 32-element group's two base blocks differ by ~2^12 in magnitude,
    on both operands, with outliers that push the macro factors around."""
    rng = np.random.default_rng(962)
    M, N, K = 192, 256, 768
    def gen(rows, seed):
        x = np.random.default_rng(seed).normal(0, 1, (rows, K))
        scale = np.where((np.arange(K) // 16) % 2 == 0, 2.0 ** 6, 2.0 ** -6)
        x = x * scale
        x[:, 7::128] *= 30.0
        return synth.to_bf16_bits(x.astype(np.float32))
    check_mbs_gemm(gen(M, 963), gen(N, 964))


def test_mbs_gemm_dit_shape_sampled_rows():
    """The DiT-like Linear shape, 4096 x 3072 x 3072, with both operands MBS."""
    M, N, K = 4096, 3072, 3072
    rows = np.sort(np.random.default_rng(965).choice(M, 24, replace=False))
    check_mbs_gemm(synth.dit_activations(1, M, K), synth.gaussian_weights(2, N, K), rows=rows)


def test_mbs_fused_call_equals_quantize_then_gemm():
    M, N, K = 300, 520, 1024
    X = to_dev(synth.student_t(966, M, K))
    W = mx.quantize(to_dev(synth.gaussian_weights(967, N, K)), MBS)
    C_f = mx.gemm_fused_act(X, W)
    C_u = mx.gemm(mx.quantize(X, MBS), W)
    torch.cuda.synchronize()
    assert torch.equal(C_f.view(torch.int16), C_u.view(torch.int16))
    # GELU / |C| max are not offered for MBS operands
    C = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = mx.fused_workspace(MBS, M, K)
    s = mx.mx_gemm_fused_act(MBS, X.data_ptr(), M, K, K, W.c(), C.data_ptr(), N, mx.MX_EPI_GELU, None, None, None,
                             ws.data_ptr(), ws.numel(), None)
    assert s == mx.MX_ERR_INVALID_ARG


def test_mbs_gemm_repeatable_and_strided_c():
    M, N, K = 200, 300, 512
    qa = mx.quantize(to_dev(synth.student_t(968, M, K)), MBS)
    qb = mx.quantize(to_dev(synth.gaussian_weights(969, N, K)), MBS)
    C1 = mx.gemm(qa, qb)
    big = torch.zeros((M, N + 37), dtype=torch.bfloat16, device="cuda")
    s = mx.mx_gemm(qa.c(), qb.c(), big.data_ptr(), N + 37, None)
    assert s == mx.MX_OK
    torch.cuda.synchronize()
    assert torch.equal(C1.view(torch.int16), big[:, :N].contiguous().view(torch.int16))
    assert not big[:, N:].any()
