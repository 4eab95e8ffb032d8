"""Oracle pins for MXFP4 with static macro-block scaling (MBS).

Page "Unveiling the Potential of Quantization with MXFP4: Strategies for
Quantization Error Reduction", section B (Macro Block Scaling): a higher-
precision factor (1 + m_MBS) with 8 mantissa bits on 1x128 macro blocks,
computed from the block maximum (the static variant) to normalise the
outliers, over the usual quantization in 1x16 blocks; sections 3-4: with it
MXFP4 comes within about 1 dB of NVFP4 in QSNR.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import exact as ex
from fp8_quantization_block_b200 import synth

MBS = 5


def _bits(vals):
    return (np.asarray(vals, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _unpack4(codes, M, K):
    c2 = codes.reshape(M, K // 2)
    un = np.empty((M, K), np.uint8)
    un[:, 0::2], un[:, 1::2] = c2 & 0xF, c2 >> 4
    return un


def test_static_mantissa_against_brute_force_and_hand_values():
    # hand values: 6 needs no factor; 7 = 6 * 299/256 rounded up (298/256 * 6 = 6.98 < 7)
    assert oracle.mbs_static_mantissa(6.0) == 0 and oracle.mbs_static_mantissa(0.0) == 0
    assert oracle.mbs_static_mantissa(7.0) == 43
    assert oracle.mbs_static_mantissa(12.0) == 0            # 6 * 2^1 exactly
    assert oracle.mbs_static_mantissa(11.99) == 0           # 6 * 511/256 < 11.99: next binade, m = 0
    rng = np.random.default_rng(80)
    for a in np.exp(rng.uniform(-40, 40, 400)):
        a = float(np.float32(a))
        assert oracle.mbs_static_mantissa(a) == ex.mbs_static_mantissa([Fraction(a)]), a


def test_static_mantissa_lands_the_macro_max_on_the_grid_top():
    # after dividing by 1 + m/256 the macro max sits in (6 * 2^e * 255/256, 6 * 2^e]
    rng = np.random.default_rng(81)
    for a in np.exp(rng.uniform(-30, 30, 300)):
        a = float(np.float32(a))
        m = oracle.mbs_static_mantissa(a)
        if m == 0:
            continue
        e = int(np.floor(np.log2(a / 6.0)))
        q = a / (1 + m / 256) / (6.0 * 2.0 ** e)
        assert 1 - 1 / 256 < q <= 1.0, (a, m, q)


def test_block_exponent_is_the_mx_rule_on_the_divided_block():
    rng = np.random.default_rng(82)
    for a, m in zip(np.exp(rng.uniform(-30, 30, 200)), rng.integers(0, 256, 200)):
        a = float(np.float32(a))
        E = oracle.mbs_block_exponent(a, int(m))
        f = 1 + Fraction(int(m), 256)
        assert Fraction(a) / (f * Fraction(2) ** (E - 127)) <= 6
        assert E == 0 or Fraction(a) / (f * Fraction(2) ** (E - 128)) > 6


def test_quantize_tiny_matches_exhaustive():
    A, _ = synth.tiny_pair()
    sub = np.vstack([A[:4, :256], synth.edge_rows(256), synth.tie_rows(256, 2)])
    M, K = sub.shape
    codes, scales, _ = oracle.quantize(MBS, sub)
    ecodes, escales, emacro = ex.quantize_mbs(sub)
    assert np.array_equal(_unpack4(codes, M, K), np.array(ecodes, dtype=np.uint8))
    got_s = np.array([[scales[oracle.sf_offset(r, j, K // 16)] for j in range(K // 16)] for r in range(M)])
    assert np.array_equal(got_s, np.array(escales))
    assert np.array_equal(oracle.mbs_macro_bytes(scales, M, K), np.array(emacro))


def test_macro_max_is_represented_almost_exactly():
    # one outlier per macro block: after the macro factor it maps to code 7 (6) of its block
    rng = np.random.default_rng(83)
    x = rng.normal(0, 1, (16, 512)).astype(np.float32)
    x[:, 37::128] = rng.uniform(20, 40, (16, 4)).astype(np.float32)
    bits = synth.to_bf16_bits(x)
    xv = synth.bits_to_tensor(bits).double().numpy()
    c, s, _ = oracle.quantize(MBS, bits)
    xh = oracle.dequantize_f64(MBS, c, s, 1.0, 16, 512)
    outl = np.abs(xv[:, 37::128])
    assert np.all(np.abs(xh[:, 37::128] - xv[:, 37::128]) <= outl / 256)
    # plain MXFP4 (E8M0 only) leaves up to a quarter of a binade on the same outliers
    c4, s4, _ = oracle.quantize(2, bits)
    x4 = oracle.dequantize_f64(2, c4, s4, 1.0, 16, 512)
    assert np.abs(x4[:, 37::128] - xv[:, 37::128]).max() > 8 * np.abs(xh[:, 37::128] - xv[:, 37::128]).max()


def test_mbs_with_all_mantissas_zero_is_mx_block16():
    # every macro max an exact 6 * 2^k: m = 0 everywhere, and the result equals
    # an E8M0 quantizer on 16-element blocks (checked exhaustively on the same rows)
    rng = np.random.default_rng(84)
    x = rng.normal(0, 1, (4, 256)).astype(np.float32)
    x[:, 0::128] = 6.0 * 2.0 ** rng.integers(-3, 4, (4, 2))
    x = np.clip(x, -5.9, 5.9)
    x[:, 0::128] = 6.0 * 2.0 ** 2
    bits = synth.to_bf16_bits(x)
    c, s, _ = oracle.quantize(MBS, bits)
    assert not oracle.mbs_macro_bytes(s, 4, 256).any()
    X = [[ex.bf16(int(b)) for b in row] for row in bits]
    neg = [[bool(int(b) & 0x8000) for b in row] for row in bits]
    ex.BLOCK[99], ex.GRIDS[99], ex.MAXELEM[99] = 16, ex.GRIDS[2], ex.MAXELEM[2]   # MX rule, block 16
    try:
        ecodes, escales, _ = ex.quantize_values(99, X, neg)
    finally:
        for d in (ex.BLOCK, ex.GRIDS, ex.MAXELEM):
            d.pop(99)
    assert np.array_equal(_unpack4(c, 4, 256), np.array(ecodes, dtype=np.uint8))
    got_s = np.array([[s[oracle.sf_offset(r, j, 16)] for j in range(16)] for r in range(4)])
    assert np.array_equal(got_s, np.array(escales))


def test_mbs_qsnr_between_mxfp4_and_nvfp4_gap_claim():
    # the page's claim on synthetic heavy-tailed activations: MBS lifts MXFP4's
    # QSNR toward NVFP4's
    x = synth.student_t(85, 256, 1024)
    M, K = x.shape
    db = {}
    for fmt in (2, 3, MBS):
        c, s, g = oracle.quantize(fmt, x)
        db[fmt], _, _ = oracle.qsnr_db(x, oracle.dequantize_f64(fmt, c, s, g, M, K))
    assert db[MBS] > db[2] + 1.0
    assert db[MBS] > db[3] - 1.5


def test_storage_sizes():
    M, K = 4096, 4096
    t = oracle.scales_bytes(MBS, M, K)
    assert t == M * K // 16 + M * K // 128               # tiles (one byte per 16) + one byte per 128
    bits = 8 * (oracle.codes_bytes(MBS, M, K) + t) / (M * K)
    assert bits == pytest.approx(4 + 8 / 16 + 8 / 128)   # 4.5625 bits/element
