"""Oracle pins for the 32-point Walsh-Hadamard rotation and for quantizing
fp32 values (the rotated tensor).

Page "Microscaling MXFP4/NVFP4 on Blackwell for reasoning LLMs", section
"Técnicas de preservação de acurácia: QuaRot, SpinQuant e ReSET": Hadamard /
Walsh-Hadamard rotations spread the outlier energy of a block evenly over its
32 elements before 4-bit quantization.  The rotation is defined here as fp32
butterflies of half-width 1, 2, 4, 8, 16 followed by one multiplication by
RN_fp32(1/sqrt(32)).
"""
from fractions import Fraction
import math

import numpy as np
import pytest

import oracle
from oracle import exact as ex
from fp8_quantization_block_b200 import synth

C32 = np.float32(1.0 / math.sqrt(32.0))


def sylvester(n: int) -> np.ndarray:
    """Sylvester Hadamard matrix by Kronecker products of [[1, 1], [1, -1]]."""
    h = np.array([[1]], dtype=np.int64)
    while h.shape[0] < n:
        h = np.kron(np.array([[1, 1], [1, -1]], dtype=np.int64), h)
    return h


def _bits(vals):
    return (np.asarray(vals, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_rotation_is_the_sylvester_hadamard_on_exact_inputs():
    # small integers: every butterfly sum is exact in fp32, so the only rounding
    # is the final product with c
    rng = np.random.default_rng(40)
    x = rng.integers(-64, 65, size=(8, 96)).astype(np.float32)
    y = oracle.rht32(_bits(x))
    H = sylvester(32)
    for j in range(3):
        blk = x[:, 32 * j:32 * (j + 1)].astype(np.int64)
        want = (blk @ H.T).astype(np.float32) * C32
        assert np.array_equal(y[:, 32 * j:32 * (j + 1)], want)


def test_rotation_of_a_basis_vector_and_of_a_constant_block():
    e = np.zeros((1, 32), np.float32)
    e[0, 5] = 1.0
    y = oracle.rht32(_bits(e))
    # column 5 of H32 times c: entries +-c
    assert np.array_equal(np.abs(y[0]), np.full(32, C32))
    assert np.array_equal(np.sign(y[0]).astype(np.int64), sylvester(32)[:, 5])
    ones = np.ones((1, 32), np.float32) * 2.0
    y = oracle.rht32(_bits(ones))
    assert y[0, 0] == np.float32(64.0) * C32 and np.all(y[0, 1:] == 0)


def test_rotation_error_bound_against_exact_arithmetic():
    x = synth.dit_activations(41, 4, 128)
    y = oracle.rht32(x)
    H = sylvester(32)
    inv = 1.0 / math.sqrt(32.0)
    for r in range(4):
        for j in range(4):
            blk = [ex.bf16(int(b)) for b in x[r, 32 * j:32 * (j + 1)]]
            l1 = float(sum(abs(v) for v in blk))
            for i in range(32):
                exact = float(sum(Fraction(int(H[i, k])) * blk[k] for k in range(32))) * inv
                # five rounded butterfly stages on partial sums bounded by ||x||_1, one product
                bound = (5 * l1 * inv + abs(exact)) * 2.0 ** -23
                assert abs(float(y[r, 32 * j + i]) - exact) <= bound


def test_rotation_preserves_energy():
    x = synth.student_t(42, 64, 512)
    y = oracle.rht32(x).astype(np.float64)
    xv = synth.bits_to_tensor(x).double().numpy()
    assert np.sum(y * y) == pytest.approx(np.sum(xv * xv), rel=1e-5)


@pytest.mark.parametrize("fmt", [0, 1, 2, 3])
def test_quantize_f32_tiny_matches_exhaustive(fmt):
    y = oracle.rht32(synth.tiny_pair()[0][:6, :128])
    M, K = y.shape
    codes, scales, g = oracle.quantize_f32(fmt, y)
    X = [[Fraction(float(v)) for v in row] for row in y]
    neg = [[bool(np.signbit(v)) for v in row] for row in y]
    ecodes, escales, eg = ex.quantize_values(fmt, X, neg)
    bs = ex.BLOCK[fmt]
    if fmt in (2, 3):
        c2 = codes.reshape(M, K // 2)
        un = np.empty((M, K), np.uint8)
        un[:, 0::2], un[:, 1::2] = c2 & 0xF, c2 >> 4
    else:
        un = codes.reshape(M, K)
    assert np.array_equal(un, np.array(ecodes, dtype=np.uint8))
    got_s = np.array([[scales[oracle.sf_offset(r, j, K // bs)] for j in range(K // bs)] for r in range(M)])
    assert np.array_equal(got_s, np.array(escales))
    if fmt == 3:
        assert Fraction(g) == eg


@pytest.mark.parametrize("fmt", [0, 2, 3])
def test_quantize_f32_equals_quantize_on_bf16_values(fmt):
    x = synth.sweep_tensor(43, 40, 512)
    xf = synth.bits_to_tensor(x).float().numpy()
    a = oracle.quantize(fmt, x)
    b = oracle.quantize_f32(fmt, xf)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and a[2] == b[2]


def test_rotation_improves_mxfp4_error_on_outlier_channels():
    # the page's claim: with outlier channels (the DiT activations carry 8
    # channels x30), rotating each 32-element block before MXFP4 lowers the
    # error (measured in the rotated domain, which is orthonormal up to fp32
    # rounding, so it equals the error of the de-rotated reconstruction)
    x = synth.dit_activations(44, 256, 1024)
    M, K = x.shape
    xv = synth.bits_to_tensor(x).double().numpy()
    c, s, _ = oracle.quantize(2, x)
    err_plain = np.sum((xv - oracle.dequantize_f64(2, c, s, 1.0, M, K)) ** 2)
    y = oracle.rht32(x)
    cr, sr, _ = oracle.quantize_f32(2, y)
    err_rot = np.sum((y.astype(np.float64) - oracle.dequantize_f64(2, cr, sr, 1.0, M, K)) ** 2)
    assert err_rot < 0.7 * err_plain
