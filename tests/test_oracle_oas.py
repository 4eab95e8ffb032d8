"""Oracle pins for MXFP4 with overflow-aware scaling (OAS) and for QSNR.

Page "Unveiling the Potential of Quantization with MXFP4: Strategies for
Quantization Error Reduction", section 2.A (OAS): the standard MX scale maps a
block's largest magnitude into (3, 6] of the E2M1 range; OAS maps it into
(3.5, 7], the elements above 6 saturating to 6.  Section 3/4 report fidelity
as QSNR (quantization signal-to-noise ratio, dB).
"""
from fractions import Fraction
import math

import numpy as np
import pytest

import oracle
from oracle import exact as ex
from fp8_quantization_block_b200 import synth

MXFP4 = 2


def _finite_positive_bf16():
    bits = np.arange(0x0001, 0x7F80, dtype=np.uint32)   # every positive finite bf16
    vals = (bits << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    return bits, vals


def test_oas_scale_maps_block_max_into_page_range():
    _, vals = _finite_positive_bf16()
    checked = 0
    for a in vals[::7]:          # a 1-in-7 sample of all ~32k values keeps this fast
        E = oracle.mx_scale_byte(a, 7.0)
        if 0 < E < 254:
            r = a / math.ldexp(1.0, E - 127)
            assert 3.5 < r <= 7.0, (a, E, r)
            checked += 1
    assert checked > 4000


def test_oas_is_ocp_minus_one_exactly_in_the_saturating_band():
    _, vals = _finite_positive_bf16()
    for a in vals[::5]:
        e_ocp = oracle.mx_scale_byte(a, 6.0)
        e_oas = oracle.mx_scale_byte(a, 7.0)
        if not (1 < e_ocp < 254):
            continue
        r = a / math.ldexp(1.0, e_ocp - 127)      # in (3, 6] by the OCP rule
        if 3.0 < r <= 3.5:
            assert e_oas == e_ocp - 1, (a, r)       # doubled: lands in (6, 7]
        else:
            assert e_oas == e_ocp, (a, r)


def test_oas_quantize_tiny_matches_exhaustive():
    A, _ = synth.tiny_pair()
    sub = np.vstack([A[:6, :128], synth.edge_rows(128), synth.tie_rows(128, MXFP4)])
    M, K = sub.shape
    codes, scales = oracle.quantize_oas(sub)
    ecodes, escales, _ = ex.quantize(MXFP4, sub, mx_threshold=Fraction(7))
    c2 = codes.reshape(M, K // 2)
    un = np.empty((M, K), np.uint8)
    un[:, 0::2], un[:, 1::2] = c2 & 0xF, c2 >> 4
    assert np.array_equal(un, np.array(ecodes, dtype=np.uint8))
    got_s = np.array([[scales[oracle.sf_offset(r, j, K // 32)] for j in range(K // 32)] for r in range(M)])
    assert np.array_equal(got_s, np.array(escales))


def test_oas_saturates_the_block_max_and_halves_the_step():
    # block max 13 (scaled by OCP into 3.25 with E = 129; by OAS into 6.5 with E = 128)
    vals = np.zeros((1, 32), dtype=np.float32)
    vals[0, 0], vals[0, 1], vals[0, 2] = 13.0, 1.0, -2.5
    bits = (vals.view(np.uint32) >> 16).astype(np.uint16)
    codes, scales = oracle.quantize_oas(bits)
    ocodes, oscales, _ = oracle.quantize(MXFP4, bits)
    assert oscales[0] == 129 and scales[0] == 128
    q = lambda c, i: (c[i // 2] >> (4 * (i % 2))) & 0xF
    assert q(codes, 0) == 7            # 6.5 saturates to 6 (code 7): 12 instead of 13
    assert q(ocodes, 0) == 5           # 3.25 -> 3 (code 5): 12 as well
    assert q(codes, 1) == 1            # 1/2 = 0.5 exactly under OAS (code 1)
    assert q(ocodes, 1) == 0           # 1/4 = 0.25 ties to 0 under OCP
    assert q(codes, 2) == 0xA          # -2.5/2 = -1.25: tie between 1 (code 2) and 1.5 -> even code 2, negative
    assert q(ocodes, 2) == 0x9         # -2.5/4 = -0.625 -> 0.5 (code 1), negative


# ------------------------------------------------------------ QSNR
def _bits(vals):
    return (np.asarray(vals, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_qsnr_hand_values():
    x = _bits([[1.0, 1.0]])
    db, sx, se = oracle.qsnr_db(x, np.array([[1.0, 0.5]]))
    assert sx == 2.0 and se == 0.25
    assert db == pytest.approx(10 * math.log10(8.0), abs=1e-12)
    db, _, se = oracle.qsnr_db(x, np.array([[1.0, 1.0]]))
    assert se == 0.0 and db == math.inf
    # a 10x larger error is exactly 20 dB worse
    db1, _, _ = oracle.qsnr_db(_bits([[4.0, -2.0, 1.0, 0.5]]), np.array([[4.0, -2.0, 1.0, 0.5625]]))
    db2, _, _ = oracle.qsnr_db(_bits([[4.0, -2.0, 1.0, 0.5]]), np.array([[4.0, -2.0, 1.0, 0.5 + 0.625]]))
    assert db1 - db2 == pytest.approx(20.0, abs=1e-9)


def test_qsnr_scale_invariant_for_mx():
    # scaling the input by a power of two scales the MX reconstruction by the same
    # power (the E8M0 exponent absorbs it): the QSNR does not change
    x = synth.gaussian_weights(31, 32, 256)
    xs = synth.to_bf16_bits(synth.bits_to_tensor(x).float().numpy() * 8.0)
    for quant in (lambda b: oracle.quantize(MXFP4, b)[:2], oracle.quantize_oas):
        c, s = quant(x)
        c2, s2 = quant(xs)
        d1, _, _ = oracle.qsnr_db(x, oracle.dequantize_f64(MXFP4, c, s, 1.0, 32, 256))
        d2, _, _ = oracle.qsnr_db(xs, oracle.dequantize_f64(MXFP4, c2, s2, 1.0, 32, 256))
        assert d1 == pytest.approx(d2, abs=1e-9)


def test_oas_does_not_lower_qsnr_on_gaussian_blocks():
    # the page's claim, on synthetic Gaussian data: OAS trades a small clipping
    # error on the block maximum for a finer step on the rest of the block
    x = synth.gaussian_weights(32, 256, 512)
    M, K = x.shape
    c, s, _ = oracle.quantize(MXFP4, x)
    co, so = oracle.quantize_oas(x)
    ocp, _, _ = oracle.qsnr_db(x, oracle.dequantize_f64(MXFP4, c, s, 1.0, M, K))
    oas, _, _ = oracle.qsnr_db(x, oracle.dequantize_f64(MXFP4, co, so, 1.0, M, K))
    cn, sn, gn = oracle.quantize(3, x)
    nv, _, _ = oracle.qsnr_db(x, oracle.dequantize_f64(3, cn, sn, gn, M, K))
    assert oas > ocp > 0
    assert nv > ocp
