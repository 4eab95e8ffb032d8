"""Oracle pins for MXFP4 with dynamic macro-block scaling (MBS, reading R21).

Page "Unveiling the Potential of Quantization with MXFP4: Strategies for
Quantization Error Reduction", section 2.B: besides the static variant (the
macro factor 1 + m/256 taken from the block maximum), a dynamic one whose
factor comes from a table built to minimise the quantization error.  The table
is not on the page; the oracle takes the error-minimising choice itself: per
1x128 macro block, the byte m with the smallest sum of squared errors of the
block's reconstruction (the terms added in element order in fp64), ties to the
smallest m.

Pinned against the exact Fraction quantizer of oracle/exact.py (each m's
squared error computed exactly), by invariants (never worse than the static
choice; exactly representable blocks come back with zero error) and by the
page's claim that the macro factor raises fidelity."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import exact as ex
from fp8_quantization_block_b200 import synth

MBS = 5


def _macro_blocks(bits, limit=None):
    """(row, macro index, exact values, sign bits, fp64 values) of every macro block."""
    M, K = bits.shape
    out = []
    for r in range(M):
        for mb in range(K // 128):
            b = bits[r, mb * 128:(mb + 1) * 128]
            vals = [ex.bf16(int(v)) for v in b]
            neg = [bool(int(v) & 0x8000) for v in b]
            f64 = np.array([oracle.bf16_to_double(int(v)) for v in b])
            out.append((r, mb, vals, neg, f64))
            if limit is not None and len(out) >= limit:
                return out
    return out


def _cases():
    rng = np.random.default_rng(7001)
    edge = synth.edge_rows(256)
    return [synth.sweep_tensor(7002, 2, 256), synth.student_t(7003, 2, 256), synth.dit_activations(7004, 2, 256),
            edge[:2], synth.to_bf16_bits(rng.normal(0, 1, (1, 128)) * np.where(np.arange(128) % 16 < 8, 1e3, 1e-3))]


@pytest.mark.parametrize("case", range(5))
def test_dynamic_mantissa_is_the_exact_error_minimum(case):
    bits = _cases()[case]
    for r, mb, vals, neg, f64 in _macro_blocks(bits, limit=4):
        exact = ex.mbs_dynamic_choice(vals, neg)
        m = oracle.mbs_dynamic_mantissa(f64)
        best = min(exact)
        # the fp64 sum adds exact terms; its rounding (at most 128 half-ulps) is
        # all that may separate the oracle's choice from the exact minimum
        slack = best * Fraction(128, 2 ** 52)
        assert exact[m] <= best + slack, (r, mb, m, float(exact[m]), float(best))
        # and no smaller m reaches the exact minimum by more than that slack
        assert all(exact[k] > best - slack for k in range(m)) or exact[m] == best
        # the oracle's fp64 sums agree with the exact ones for every m
        for k in (0, m, 255, 17, 128):
            e64 = oracle.mbs_macro_sse(f64, k)
            assert abs(Fraction(e64) - exact[k]) <= exact[k] * Fraction(128, 2 ** 52) + Fraction(0), (k, e64)


def test_dynamic_quantize_matches_exact_quantizer_for_its_choice():
    bits = np.vstack([synth.student_t(7010, 2, 256), synth.sweep_tensor(7011, 1, 256)])
    M, K = bits.shape
    codes, scales = oracle.quantize_mbs_dynamic(bits)
    macro = oracle.mbs_macro_bytes(scales, M, K)
    un = np.empty((M, K), np.uint8)
    c2 = codes.reshape(M, K // 2)
    un[:, 0::2], un[:, 1::2] = c2 & 0xF, c2 >> 4
    for r, mb, vals, neg, f64 in _macro_blocks(bits):
        m = int(macro[r, mb])
        assert m == oracle.mbs_dynamic_mantissa(f64)
        c, exps, _ = ex.mbs_quantize_macro(vals, m, neg)
        assert list(un[r, mb * 128:(mb + 1) * 128]) == c
        for jb in range(8):
            j = mb * 8 + jb
            assert scales[oracle.sf_offset(r, j, K // 16)] == exps[jb]


def test_dynamic_error_never_above_static():
    bits = np.vstack([synth.student_t(7020, 8, 1024), synth.dit_activations(7021, 8, 1024),
                      synth.sweep_tensor(7022, 8, 1024)])
    M, K = bits.shape
    cs, ss, _ = oracle.quantize(MBS, bits)
    cd, sd = oracle.quantize_mbs_dynamic(bits)
    xs = oracle.dequantize_f64(MBS, cs, ss, 1.0, M, K)
    xd = oracle.dequantize_f64(MBS, cd, sd, 1.0, M, K)
    x = np.array([[oracle.bf16_to_double(int(v)) for v in row] for row in bits])
    es = ((x - xs) ** 2).reshape(M, K // 128, 128).sum(axis=2)
    ed = ((x - xd) ** 2).reshape(M, K // 128, 128).sum(axis=2)
    assert np.all(ed <= es * (1 + 1e-12))
    assert np.any(ed < es)              # the search finds better factors somewhere


def test_representable_block_comes_back_exactly():
    rng = np.random.default_rng(7030)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    ran = 0
    for trial in range(6):
        # m a multiple of 8: (256 + m) q then has at most 8 significant bits, so
        # the block is exactly representable in bf16
        m0 = 8 * int(rng.integers(0, 32))
        f = 1 + m0 / 256.0
        q = rng.choice(grid, 128) * rng.choice([-1, 1], 128)
        for jb in range(8):
            q[jb * 16] = 6.0       # each base block reaches the top of the grid
        E = rng.integers(-6, 6, 8)
        x = np.concatenate([q[jb * 16:(jb + 1) * 16] * f * 2.0 ** E[jb] for jb in range(8)])
        # only values that bf16 holds exactly
        bits = (x.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
        f64 = np.array([oracle.bf16_to_double(int(v)) for v in bits])
        if not np.array_equal(f64, x):
            continue
        m = oracle.mbs_dynamic_mantissa(f64)
        assert oracle.mbs_macro_sse(f64, m) == 0.0
        assert m <= m0
        ran += 1
    assert ran >= 4


def test_dynamic_raises_qsnr_over_static():
    bits = synth.student_t(7040, 64, 1024)
    M, K = bits.shape
    cs, ss, _ = oracle.quantize(MBS, bits)
    cd, sd = oracle.quantize_mbs_dynamic(bits)
    qs = oracle.qsnr_db(bits, oracle.dequantize_f64(MBS, cs, ss, 1.0, M, K))[0]
    qd = oracle.qsnr_db(bits, oracle.dequantize_f64(MBS, cd, sd, 1.0, M, K))[0]
    assert qd >= qs
