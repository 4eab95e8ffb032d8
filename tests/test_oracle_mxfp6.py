"""Oracle pins for MXFP6 E3M2.

Page "Microscaling MXFP4/NVFP4 on Blackwell for reasoning LLMs", section
"Fundamentos matemáticos do formato MXFP4 e E8M0", format table: MXFP6 has
6-bit E3M2 elements and one 8-bit E8M0 scale per 32-element block, 6.25
effective bits per element.  The E3M2 bit layout is the OCP one (sign, three
exponent bits with bias 3, two mantissa bits, no infinities or NaN); here it
is pinned against an independent library implementation (ml_dtypes'
float6_e3m2fn) and the exhaustive Fraction checker.
"""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

import oracle
from oracle import exact as ex
from fp8_quantization_block_b200 import synth

MXFP6 = 4


def _lib_decode(code: int) -> float:
    return float(np.array([code], dtype=np.uint8).view(ml_dtypes.float6_e3m2fn)[0])


def test_e3m2_decode_every_code_matches_library():
    for c in range(64):
        assert oracle.decode("e3m2", c) == _lib_decode(c), c
    assert oracle.decode("e3m2", 0x1F) == 28.0 and oracle.decode("e3m2", 0x3F) == -28.0
    assert oracle.max_element(MXFP6) == 28.0
    # gradual underflow: the subnormal step (2^-4) equals the first binade's step
    assert oracle.decode("e3m2", 1) == 2.0 ** -4 and oracle.decode("e3m2", 5) - oracle.decode("e3m2", 4) == 2.0 ** -4


def test_e3m2_encode_matches_library_rne_and_exhaustive():
    rng = np.random.default_rng(60)
    pos = sorted({oracle.decode("e3m2", c) for c in range(32)})
    mids = [(a + b) / 2 for a, b in zip(pos, pos[1:])]
    vals = np.concatenate([rng.uniform(-28, 28, 4000), rng.normal(0, 0.3, 2000), mids, [-m for m in mids],
                           pos, [0.0, -0.0]]).astype(np.float32)
    lib = vals.astype(ml_dtypes.float6_e3m2fn).view(np.uint8) & 0x3F
    for v, want in zip(vals, lib):
        got = oracle.encode("e3m2", float(v))
        assert got == want, (v, got, want)
        assert got == ex.round_to_grid(Fraction(float(v)), ex.E3M2_GRID, 0x20, bool(np.signbit(v)))


def test_e3m2_encode_saturates_and_keeps_the_sign_of_zero():
    assert oracle.encode("e3m2", 1e6) == 0x1F and oracle.encode("e3m2", -30.0) == 0x3F
    assert oracle.encode("e3m2", 29.9) == 0x1F
    assert oracle.encode("e3m2", -1e-9) == 0x20 and oracle.encode("e3m2", 1e-9) == 0x00
    # exactly half of the smallest subnormal ties to the even code 0
    assert oracle.encode("e3m2", 2.0 ** -5) == 0x00 and oracle.encode("e3m2", 3 * 2.0 ** -5) == 0x02


def test_mxfp6_bits_per_element_is_the_pages_6_25():
    M, K = 4096, 4096
    bits = 8 * (oracle.codes_bytes(MXFP6, M, K) + oracle.scales_bytes(MXFP6, M, K)) / (M * K)
    assert bits == 6.25
    assert oracle.block_size(MXFP6) == 32
    assert oracle.codes_bytes(MXFP6, 1, 32) == 24      # 16 codes in 12 bytes


def test_mx_scale_rule_for_e3m2_maps_block_max_into_14_28():
    rng = np.random.default_rng(61)
    for a in np.exp(rng.uniform(-60, 60, 3000)):
        E = oracle.mx_scale_byte(float(a), 28.0)
        assert E == ex.mx_scale_byte([Fraction(float(a))], MXFP6)
        if 0 < E < 254:
            r = a / 2.0 ** (E - 127)
            assert 14.0 < r <= 28.0


def _unpack6(codes: np.ndarray, M: int, K: int) -> np.ndarray:
    """Code k of a row = bits 6k..6k+5 of the row's little-endian bit string."""
    rows = codes.reshape(M, K * 3 // 4)
    bitstr = np.unpackbits(rows, axis=1, bitorder="little")
    weights = 1 << np.arange(6)
    return (bitstr.reshape(M, K, 6) * weights).sum(axis=2).astype(np.uint8)


def test_quantize_tiny_matches_exhaustive():
    A, _ = synth.tiny_pair()
    sub = np.vstack([A[:6, :128], synth.edge_rows(128), synth.tie_rows(128, 0)])
    M, K = sub.shape
    codes, scales, _ = oracle.quantize(MXFP6, sub)
    ecodes, escales, _ = ex.quantize(MXFP6, sub)
    assert np.array_equal(_unpack6(codes, M, K), np.array(ecodes, dtype=np.uint8))
    got_s = np.array([[scales[oracle.sf_offset(r, j, K // 32)] for j in range(K // 32)] for r in range(M)])
    assert np.array_equal(got_s, np.array(escales))


def test_quantize_e3m2_midpoints_tie_to_even():
    # block max 28 pins E = 127 (scale 1): the other elements sit on E3M2 midpoints
    pos = sorted({oracle.decode("e3m2", c) for c in range(32)})
    mids = [(a + b) / 2 for a, b in zip(pos, pos[1:])]
    row = np.zeros(32, np.float32)
    row[0] = 28.0
    row[1:1 + len(mids)] = mids
    bits = (row.view(np.uint32) >> 16).astype(np.uint16)[None, :]
    assert np.array_equal(synth.bits_to_tensor(bits).float().numpy()[0], row)   # exact in bf16
    codes, scales, _ = oracle.quantize(MXFP6, bits)
    assert scales[0] == 127
    q = _unpack6(codes, 1, 32)[0]
    for i, m in enumerate(mids):
        lo = pos.index(max(p for p in pos if p < m))
        assert q[1 + i] == (lo if lo % 2 == 0 else lo + 1), (m, q[1 + i])


def test_roundtrip_of_representable_blocks():
    rng = np.random.default_rng(62)
    pos = np.array(sorted({oracle.decode("e3m2", c) for c in range(32)}))
    M, K = 16, 256
    vals = pos[rng.integers(0, 32, size=(M, K))] * np.where(rng.random((M, K)) < 0.5, -1, 1)
    vals[:, ::32] = 28.0                                     # every block reaches the format max
    e = rng.integers(-20, 20, size=(M, K // 32))
    x = (vals * np.repeat(2.0 ** e, 32, axis=1)).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    codes, scales, _ = oracle.quantize(MXFP6, bits)
    back = oracle.dequantize_f64(MXFP6, codes, scales, 1.0, M, K)
    assert np.array_equal(back, x.astype(np.float64))


def test_packing_roundtrip_through_dequantize_bf16():
    x = synth.sweep_tensor(63, 20, 256)
    codes, scales, _ = oracle.quantize(MXFP6, x)
    d64 = oracle.dequantize_f64(MXFP6, codes, scales, 1.0, 20, 256)
    d16 = oracle.dequantize_bf16(MXFP6, codes, scales, 1.0, 20, 256)
    assert np.array_equal(synth.bits_to_tensor(d16).double().numpy(), d64)   # every E3M2 * 2^k fits bf16
