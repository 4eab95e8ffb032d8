"""The GELU epilogue on its own: A has one nonzero per row, x_i (an MXFP8
value, so the quantization is exact), and B's rows are all e_0, so every
C[i][j] is x_i exactly and the epilogue's output is GELU(x_i) rounded to bf16.
It must be within one bf16 ulp of the correctly rounded exact-erf GELU (fp64),
for x over [-16, 16] with 4 significant bits (8..15 times powers of two),
positive and negative, through the CTA-pair kernel with 256 x 128 tiles and
through the single-CTA kernel."""
import numpy as np
import pytest
import torch

import oracle
from fp8_quantization_block_b200 import mx, synth

pytestmark = pytest.mark.gpu


def _values():
    vals = []
    for k in range(-14, 1):
        for m in range(8, 16):
            v = m * 2.0 ** k
            if v <= 16.0:
                vals += [v, -v]
    vals += [0.0, -0.0]
    return np.array(vals, dtype=np.float32)


def _bf16_of_f64(v: np.ndarray) -> np.ndarray:
    """RNE of fp64 values to bf16 bit patterns (through the oracle's rounding)."""
    return np.array([oracle.double_to_bf16(float(x)) for x in v], dtype=np.uint16)


@pytest.mark.parametrize("M,N", [(512, 256), (64, 256)])
def test_gelu_epilogue_within_one_bf16_ulp(M, N):
    x = _values()
    rows = np.resize(x, M)
    K = 128
    A = np.zeros((M, K), dtype=np.float32)
    A[:, 0] = rows
    B = np.zeros((N, K), dtype=np.float32)
    B[:, 0] = 1.0
    qa = mx.quantize(synth.bits_to_tensor(synth.to_bf16_bits(A)).cuda(), 0)
    qb = mx.quantize(synth.bits_to_tensor(synth.to_bf16_bits(B)).cuda(), 0)
    X = synth.bits_to_tensor(synth.to_bf16_bits(A)).cuda()
    H = mx.gemm_fused_act(X, qb, epilogue=mx.MX_EPI_GELU)
    C = mx.gemm(qa, qb)
    torch.cuda.synchronize()
    mx.check_device_error()
    # the GEMM is exact here: C[i][j] = x_i
    c = C.float().cpu().numpy()
    assert np.array_equal(c, np.repeat(rows[:, None], N, axis=1))
    got = H.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    want = _bf16_of_f64(oracle.gelu(rows.astype(np.float64)))
    # distance in bf16 steps, sign-aware (the ordered integer of the bit pattern)
    def ordered(b):
        b = b.astype(np.int64)
        return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    d = np.abs(ordered(got) - ordered(want)[:, None])
    assert d.max() <= 1, (d.max(), rows[np.argmax(d.max(axis=1))])
    # and exact for most values
    assert np.count_nonzero(d) <= d.size // 50
