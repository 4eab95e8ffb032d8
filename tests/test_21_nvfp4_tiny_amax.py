"""NVFP4 without a given g on tensors of at most 16384 elements: every CTA of
the quantize kernel takes amax(|X|) itself instead of running the pre-pass.
Codes, scales and g must equal the oracle's bit for bit on both sides of that
size, wherever the tensor's largest magnitude lies (another CTA's tile, the
last segment, a row past the first, a padded row pitch), and the fused call
must give the same C as with amax(|X|) supplied."""
import numpy as np
import pytest
import torch

from fp8_quantization_block_b200 import mx, synth
from gpu_helpers import assert_quant_equal, quantize_dev, to_dev

pytestmark = pytest.mark.gpu
TINY = 16384


def with_peak(bits: np.ndarray, r: int, c: int, value: float) -> np.ndarray:
    out = bits.copy()
    out[r, c] = synth.to_bf16_bits(np.array([[value]], dtype=np.float32))[0, 0]
    return out


@pytest.mark.parametrize("M,K", [(1, 16384), (128, 128), (2, 8192), (1, 16), (3, 4096),
                                 (129, 128), (1, 16400), (2, 8208)])
@pytest.mark.parametrize("where", ["first", "last", "far_tile", "row_past_first"])
def test_quantize_without_g_matches_oracle(M, K, where):
    bits = synth.student_t(60 + M, M, K)
    r, c = {"first": (0, 0), "last": (M - 1, K - 1), "far_tile": (0, K - 1 - K // 3),
            "row_past_first": (M // 2, K // 2)}[where]
    bits = with_peak(bits, r, c, -37.5)
    assert_quant_equal(quantize_dev(bits, 3), bits, 3)


@pytest.mark.parametrize("M,K", [(1, 8192), (64, 256), (130, 96)])
def test_quantize_without_g_row_pitch(M, K):
    bits = with_peak(synth.student_t(70 + M, M, K), M - 1, 5, 91.0)
    padded = torch.zeros((M, K + 40), dtype=torch.bfloat16, device="cuda")
    padded[:, :K] = to_dev(bits)
    padded[:, K:] = 1.0e4   # past the row: must not count towards amax
    q = mx.quantize(padded[:, :K], 3)
    torch.cuda.synchronize()
    mx.check_device_error()
    assert_quant_equal(q, bits, 3)


def test_quantize_without_g_all_zero():
    bits = np.zeros((4, 1024), dtype=np.uint16)
    _, _, g = assert_quant_equal(quantize_dev(bits, 3), bits, 3)
    assert g == 1.0


@pytest.mark.parametrize("M,K", [(1, 8192), (2, 8192), (16, 1024), (128, 128), (1, 16384)])
def test_fused_call_tiny_x_equals_amax_route(M, K):
    N = 512
    X = to_dev(with_peak(synth.student_t(80 + M, M, K), M - 1, K - 1, 12.25))
    W = mx.quantize(to_dev(synth.gaussian_weights(81, N, K)), 3)
    C_tiny = mx.gemm_fused_act(X, W)
    C_amax = mx.gemm_fused_act(X, W, x_amax=X.abs().max().float().reshape(1))
    C_unfused = mx.gemm(mx.quantize(X, 3), W)
    torch.cuda.synchronize()
    mx.check_device_error()
    assert M * K <= TINY
    assert torch.equal(C_tiny.view(torch.int16), C_amax.view(torch.int16))
    assert torch.equal(C_tiny.view(torch.int16), C_unfused.view(torch.int16))
