"""Pins for the CPU oracle: it is checked against what the pages print, against
closed forms and invariants, against library routines (torch's float8 and bf16
casts, numpy matmul, scipy's normal CDF) and against exhaustive search in exact
arithmetic (oracle/exact.py) on tiny inputs.  No GPU is needed."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import oracle.exact as ex
from fp8_quantization_block_b200 import synth

E4M3, E5M2, MXFP4, NVFP4 = 0, 1, 2, 3


# ---------------------------------------------------------------- formats
def test_e2m1_values_match_page(facts):
    page = facts["e2m1_magnitudes"]["values"]
    pos = [oracle.decode("e2m1", c) for c in range(8)]
    neg = [oracle.decode("e2m1", c | 8) for c in range(8)]
    assert pos == page                      # ascending by code: layout s.ee.m, bias 1
    assert neg == [-v for v in page]
    assert math.copysign(1.0, neg[0]) == -1.0


def test_e8m0_every_byte(facts):
    bias = facts["e8m0"]["bias"]
    for E in range(255):
        assert Fraction(oracle.decode("e8m0", E)) == Fraction(2) ** (E - bias)
    assert math.isnan(oracle.decode("e8m0", 255))   # reading: 0xFF reserved as NaN


@pytest.mark.parametrize("name,tdtype,maxval", [("e4m3", torch.float8_e4m3fn, 448.0),
                                                ("e5m2", torch.float8_e5m2, 57344.0)])
def test_fp8_decode_all_codes_vs_torch(name, tdtype, maxval, facts):
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(tdtype).to(torch.float64).numpy()
    got = np.array([oracle.decode(name, c) for c in range(256)])
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.all(both_nan | (ref == got))
    assert np.array_equal(np.signbit(ref[~both_nan]), np.signbit(got[~both_nan]))
    finite = got[np.isfinite(got)]
    assert finite.max() == maxval
    if name == "e4m3":
        assert maxval == facts["e4m3_range"]["max"]
    # monotone over the positive codes
    pos = [oracle.decode(name, c) for c in range(0x7F if name == "e4m3" else 0x7C)]
    assert all(a < b for a, b in zip(pos, pos[1:]))


@pytest.mark.parametrize("name,tdtype,maxval", [("e4m3", torch.float8_e4m3fn, 448.0),
                                                ("e5m2", torch.float8_e5m2, 57344.0)])
def test_fp8_encode_vs_torch_rne(name, tdtype, maxval):
    rng = np.random.default_rng(11)
    # random magnitudes across the whole range, incl. subnormals, both signs
    mags = np.exp2(rng.uniform(-22 if name == "e4m3" else -20, math.log2(maxval), 20000))
    vals = (mags * rng.choice([-1.0, 1.0], mags.size)).astype(np.float32)
    # exact midpoints between neighbouring codes (fp32-representable): ties to even
    pos = np.array([oracle.decode(name, c) for c in range(0x7F if name == "e4m3" else 0x7C)])
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    vals = np.concatenate([vals, mids, -mids, np.array([0.0, -0.0], np.float32)])
    ref = torch.from_numpy(vals).to(tdtype).view(torch.uint8).numpy()
    got = np.array([oracle.encode(name, float(v)) for v in vals], dtype=np.uint8)
    assert np.array_equal(ref, got)


def test_fp8_encode_saturates():
    assert oracle.encode("e4m3", 1e6) == 0x7E and oracle.encode("e4m3", -500.0) == 0xFE
    assert oracle.encode("e5m2", 1e9) == 0x7B and oracle.encode("e5m2", -60000.0) == 0xFB


def test_e2m1_rne_hand_ties():
    # ties go to the even mantissa: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    cases = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0,
             0.2499: 0.0, 0.2501: 0.5, 5.0001: 6.0, 7.0: 6.0, 1e9: 6.0}
    for v, want in cases.items():
        c = oracle.encode("e2m1", v)
        assert oracle.decode("e2m1", c) == want, v
        cn = oracle.encode("e2m1", -v)
        assert cn == (c | 8)
    # zero keeps its sign
    assert oracle.encode("e2m1", -0.0) == 0x8 and oracle.encode("e2m1", -0.1) == 0x8
    assert oracle.encode("e2m1", 0.0) == 0x0


def test_e2m1_encode_vs_exhaustive():
    rng = np.random.default_rng(5)
    vals = list(rng.uniform(-8, 8, 3000)) + [k / 8 for k in range(-64, 65)]
    for v in vals:
        want = ex.round_to_grid(Fraction(v), ex.E2M1_GRID, 0x8, math.copysign(1.0, v) < 0)
        assert oracle.encode("e2m1", v) == want, v


def test_bf16_rne_vs_exhaustive_and_torch():
    allb = np.arange(0, 0x7F80, dtype=np.uint32)         # every non-negative finite bf16
    table = (allb << 16).view(np.float32).astype(np.float64)
    rng = np.random.default_rng(3)
    vals = np.concatenate([np.exp2(rng.uniform(-140, 127.9, 4000)),
                           (table[1:200] + table[:199]) / 2,          # subnormal midpoints
                           (table[20001:20200] + table[20000:20199]) / 2])
    for v in vals:
        i = np.searchsorted(table, v)
        lo, hi = table[i - 1], table[min(i, table.size - 1)]
        if table[i] == v:
            want = i
        elif v - lo < hi - v:
            want = i - 1
        elif v - lo > hi - v:
            want = i
        else:
            want = i - 1 if (i - 1) % 2 == 0 else i
        assert oracle.double_to_bf16(v) == want
        assert oracle.double_to_bf16(-v) == want | 0x8000
    f32 = np.exp2(rng.uniform(-130, 127, 5000)).astype(np.float32)
    ref = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.double_to_bf16(float(v)) for v in f32], dtype=np.uint16)
    assert np.array_equal(ref, got)
    assert oracle.double_to_bf16(3.4e38) == 0x7F80    # RNE overflow


# ------------------------------------------------------------- scale rules
def _blocks(rng, n, bs):
    out = []
    for i in range(n):
        e = rng.integers(-30, 30)
        blk = rng.standard_normal(bs) * 2.0 ** e
        if i % 5 == 0:
            blk[rng.integers(bs)] = 6.0 * 2.0 ** e           # exactly on the boundary
        if i % 7 == 0:
            blk[rng.integers(bs)] = np.nextafter(np.float32(6.0 * 2.0 ** e), np.float32(np.inf))
        if i % 11 == 0:
            blk[:] = 0.0
        out.append(synth.to_bf16_bits(blk))
    return out


@pytest.mark.parametrize("fmt", [E4M3, E5M2, MXFP4])
def test_mx_scale_rule_exhaustive(fmt):
    rng = np.random.default_rng(100 + fmt)
    maxelem = oracle.max_element(fmt)
    for bits in _blocks(rng, 300, 32):
        blk = [ex.bf16(int(b)) for b in bits]
        amax = max(abs(x) for x in blk)
        assert oracle.mx_scale_byte(float(amax), maxelem) == ex.mx_scale_byte(blk, fmt)


def test_scale_rule_matches_page_formula(facts):
    """E = ceil(log2(max_val / 6)) + 127 (evaluated in floating point away from
    integer boundaries, where the float log2 cannot flip the ceiling)."""
    rng = np.random.default_rng(7)
    m6 = facts["scale_rule"]["max_e2m1"]
    n = 0
    for amax in np.exp2(rng.uniform(-100, 100, 5000)):
        t = math.log2(amax / m6)
        if abs(t - round(t)) < 1e-9:
            continue
        n += 1
        assert oracle.mx_scale_byte(amax, m6) == math.ceil(t) + 127
    assert n > 4000


@pytest.mark.parametrize("fmt,lo,hi", [(MXFP4, 3.0, 6.0), (E4M3, 224.0, 448.0), (E5M2, 28672.0, 57344.0)])
def test_mx_mapped_range_invariant(fmt, lo, hi, facts):
    if fmt == MXFP4:
        r = facts["mx_mapped_range"]
        assert (lo, hi) == (r["low_exclusive"], r["high_inclusive"])
    rng = np.random.default_rng(200 + fmt)
    for amax in np.exp2(rng.uniform(-60, 60, 3000)):
        E = oracle.mx_scale_byte(amax, hi)
        if 0 < E < 254:
            ratio = amax / 2.0 ** (E - 127)
            assert lo < ratio <= hi


@pytest.mark.parametrize("fmt", [E4M3, E5M2, MXFP4])
def test_mx_roundtrip_representable_blocks(fmt):
    """Blocks of 2^e * q with q on the element grid (max element included) come back exactly."""
    rng = np.random.default_rng(300 + fmt)
    grid = {E4M3: [oracle.decode("e4m3", c) for c in range(0x7F)],
            E5M2: [oracle.decode("e5m2", c) for c in range(0x7C)],
            MXFP4: [oracle.decode("e2m1", c) for c in range(8)]}[fmt]
    M, K = 16, 128
    x = np.zeros((M, K))
    for r in range(M):
        for b in range(K // 32):
            e = int(rng.integers(-20, 20))
            q = rng.choice(grid, 32) * rng.choice([-1, 1], 32)
            q[rng.integers(32)] = grid[-1]
            x[r, b * 32:(b + 1) * 32] = q * 2.0 ** e
    bits = synth.to_bf16_bits(x)
    assert np.array_equal(synth.bits_to_tensor(bits).double().numpy(), x)   # bf16-exact inputs
    codes, scales, g = oracle.quantize(fmt, bits)
    back = oracle.dequantize_f64(fmt, codes, scales, g, M, K)
    assert np.array_equal(back, x)


def test_nvfp4_global_scale_closed_form_and_rounding():
    for k in range(-60, 60, 7):
        assert oracle.nvfp4_global_scale(2688.0 * 2.0 ** k) == 2.0 ** k
    assert oracle.nvfp4_global_scale(0.0) == 1.0
    rng = np.random.default_rng(9)
    for amax in np.exp2(rng.uniform(-120, 127, 2000)):
        amax = float(synth.bits_to_tensor(synth.to_bf16_bits(np.array([amax]))).double()[0])
        g = oracle.nvfp4_global_scale(amax)
        assert Fraction(g) == ex.nvfp4_global_scale(Fraction(amax))
        q = Fraction(amax) / 2688
        assert Fraction(g) >= q
        assert Fraction(float(np.nextafter(np.float32(g), np.float32(0)))) < q


def test_nvfp4_block_scale_exhaustive():
    rng = np.random.default_rng(13)
    for bits in _blocks(rng, 300, 16):
        blk = [ex.bf16(int(b)) for b in bits]
        amax = max(abs(x) for x in blk)
        g = float(np.float32(2.0 ** rng.uniform(-20, 5)))
        assert oracle.nvfp4_block_scale(float(amax), g) == ex.nvfp4_block_scale(blk, Fraction(g))


def test_nvfp4_max_block_scale_within_e4m3():
    bits = synth.student_t(3, 64, 256)
    codes, scales, g = oracle.quantize(NVFP4, bits)
    assert max(oracle.decode("e4m3", int(s)) for s in scales) <= 448.0
    amax = oracle.amax_bf16(bits)
    assert g == oracle.nvfp4_global_scale(amax)


def test_nvfp4_roundtrip_representable_blocks():
    """Blocks g * s * q, with some |q| = 6, return exactly (s, q)."""
    rng = np.random.default_rng(17)
    g = 2.0 ** -3
    M, K = 8, 64
    x = np.zeros((M, K))
    want_s = []
    for r in range(M):
        for b in range(K // 16):
            s_code = int(rng.integers(8, 0x70))
            s = oracle.decode("e4m3", s_code)
            q = rng.choice([0, 0.5, 1, 1.5, 2, 3, 4, 6], 16) * rng.choice([-1, 1], 16)
            q[rng.integers(16)] = 6.0
            x[r, b * 16:(b + 1) * 16] = g * s * q
            want_s.append(s_code)
    bits = synth.to_bf16_bits(x)
    assert np.array_equal(synth.bits_to_tensor(bits).double().numpy(), x)
    codes, scales, gg = oracle.quantize(NVFP4, bits, gscale=g)
    back = oracle.dequantize_f64(NVFP4, codes, scales, gg, M, K)
    assert np.array_equal(back, x)
    got_s = [int(scales[oracle.sf_offset(r, b, K // 16)]) for r in range(M) for b in range(K // 16)]
    assert got_s == want_s


@pytest.mark.parametrize("fmt", [E4M3, E5M2, MXFP4, NVFP4])
def test_quantize_tiny_matches_exhaustive(fmt):
    A, _ = synth.tiny_pair()
    sub = np.vstack([A[:6, :128], synth.edge_rows(128), synth.tie_rows(128, fmt)])
    codes, scales, g = oracle.quantize(fmt, sub)
    ecodes, escales, eg = ex.quantize(fmt, sub)
    M, K = sub.shape
    bs = ex.BLOCK[fmt]
    if fmt in (MXFP4, NVFP4):
        c2 = codes.reshape(M, K // 2)
        un = np.empty((M, K), np.uint8)
        un[:, 0::2], un[:, 1::2] = c2 & 0xF, c2 >> 4
    else:
        un = codes.reshape(M, K)
    assert np.array_equal(un, np.array(ecodes, dtype=np.uint8))
    got_s = np.array([[scales[oracle.sf_offset(r, j, K // bs)] for j in range(K // bs)] for r in range(M)])
    assert np.array_equal(got_s, np.array(escales))
    if fmt == NVFP4:
        assert Fraction(g) == eg


# ------------------------------------------------------------ storage
def test_bits_per_element_and_kv_bytes(facts):
    bpe = facts["bits_per_element"]
    M, K = 1024, 4096
    unpadded_scales = lambda fmt: M * K // oracle.block_size(fmt)
    mxfp4 = (oracle.codes_bytes(MXFP4, M, K) + unpadded_scales(MXFP4)) * 8 / (M * K)
    nvfp4 = (oracle.codes_bytes(NVFP4, M, K) + unpadded_scales(NVFP4)) * 8 / (M * K)
    mxfp8 = (oracle.codes_bytes(E4M3, M, K) + unpadded_scales(E4M3)) * 8 / (M * K)
    assert mxfp4 == bpe["mxfp4"]
    assert bpe["nvfp4_min"] <= nvfp4 <= bpe["nvfp4_max"]
    assert mxfp8 == bpe["fp8_e4m3"] + 8 / 32
    # when the row count is a multiple of 128 and K/bs of 4, padding is zero
    assert oracle.scales_bytes(MXFP4, M, K) == unpadded_scales(MXFP4)
    kv = facts["kv_cache_bytes_per_token"]
    per_token = 2 * kv["layers"] * kv["kv_heads"] * kv["head_dim"]
    assert per_token * 2 == kv["bf16_bytes"] and per_token * 1 == kv["fp8_bytes"]
    assert per_token * mxfp4 / 8 == kv["mxfp4_bytes"]
    assert mxfp4 / 8 == kv["mxfp4_bytes_per_element"]
    assert facts["block_sizes"]["nvfp4"] == oracle.block_size(NVFP4) == 16
    assert facts["block_sizes"]["mxfp8"] == oracle.block_size(E4M3) == 32


def test_scale_layout_is_a_permutation():
    for M, sf_cols in [(128, 4), (200, 6), (64, 16), (384, 12)]:
        padded_rows = -(-M // 128) * 128
        padded_cols = -(-sf_cols // 4) * 4
        offs = {oracle.sf_offset(r, c, sf_cols) for r in range(padded_rows) for c in range(padded_cols)}
        assert offs == set(range(padded_rows * padded_cols))


def test_dequant_bf16_is_one_rounding_of_f64():
    bits = synth.student_t(3, 32, 128)
    for fmt in (E4M3, E5M2, MXFP4, NVFP4):
        codes, scales, g = oracle.quantize(fmt, bits)
        d64 = oracle.dequantize_f64(fmt, codes, scales, g, 32, 128)
        d16 = oracle.dequantize_bf16(fmt, codes, scales, g, 32, 128)
        want = np.vectorize(oracle.double_to_bf16)(d64).astype(np.uint16)
        assert np.array_equal(d16, want)
        # dequantized values are within the format's relative half-spacing of the inputs
        x = synth.bits_to_tensor(bits).double().numpy()
        assert np.all(np.sign(d64) * np.sign(x) >= 0)


def test_nonfinite_input_rejected():
    bits = synth.tiny_pair()[0][:2, :64].copy()
    bits[0, 3] = 0x7F80
    with pytest.raises(ValueError):
        oracle.quantize(E4M3, bits)


# ---------------------------------------------------------------- GEMM
def test_gemm_f64_vs_exact_fractions():
    A, B = synth.tiny_pair()
    for fmt in (E4M3, MXFP4, NVFP4):
        ca, sa, ga = oracle.quantize(fmt, A)
        cb, sb, gb = oracle.quantize(fmt, B)
        Ad = oracle.dequantize_f64(fmt, ca, sa, ga, 64, 256)
        Bd = oracle.dequantize_f64(fmt, cb, sb, gb, 64, 256)
        rows, cols = [0, 5, 17, 63], [0, 9, 40, 63]
        C, Cabs = oracle.gemm_f64(Ad, Bd, rows=rows)
        exact = ex.gemm([[Fraction(v) for v in Ad[i]] for i in range(64)],
                        [[Fraction(v) for v in Bd[j]] for j in range(64)], rows=rows, cols=cols)
        for t, i in enumerate(rows):
            for u, j in enumerate(cols):
                err = abs(Fraction(C[t, j]) - exact[t][u])
                assert err <= Fraction(256 * 2.0 ** -53) * Fraction(Cabs[t, j])


def test_gemm_integer_values_match_numpy():
    rng = np.random.default_rng(21)
    A = rng.integers(-6, 7, (33, 128)).astype(np.float64)
    B = rng.integers(-6, 7, (17, 128)).astype(np.float64)
    C, Cabs = oracle.gemm_f64(A, B)
    assert np.array_equal(C, A @ B.T)
    assert np.array_equal(Cabs, np.abs(A) @ np.abs(B).T)


def test_tolerance_detects_planted_mistakes():
    A, B = synth.tiny_pair()
    ca, sa, ga = oracle.quantize(E4M3, A)
    cb, sb, gb = oracle.quantize(E4M3, B)
    Ad = oracle.dequantize_f64(E4M3, ca, sa, ga, 64, 256)
    Bd = oracle.dequantize_f64(E4M3, cb, sb, gb, 64, 256)
    C, Cabs = oracle.gemm_f64(Ad, Bd)
    c16 = synth.bits_to_tensor(np.vectorize(oracle.double_to_bf16)(C).astype(np.uint16)).double().numpy()
    assert oracle.gemm_tolerance_ok(c16, C, Cabs)[0]
    assert not oracle.gemm_tolerance_ok(C.T, C, Cabs)[0]                 # transposed output
    Cbad, _ = oracle.gemm_f64(Ad, -Bd)
    assert not oracle.gemm_tolerance_ok(Cbad, C, Cabs)[0]                 # sign slip
    Cdrop, _ = oracle.gemm_f64(Ad[:, :224].copy(), Bd[:, :224].copy())
    assert not oracle.gemm_tolerance_ok(Cdrop, C, Cabs)[0]                # dropped k-blocks


def test_gelu_against_normal_cdf():
    from scipy.special import ndtr
    x = np.linspace(-8, 8, 1001)
    y = oracle.gelu(x)
    assert np.allclose(y, x * ndtr(x), rtol=1e-14, atol=1e-15)
    assert np.allclose(y - oracle.gelu(-x), x, rtol=0, atol=1e-14)      # GELU(x) - GELU(-x) = x


def test_gelu_negative_tail_relative():
    """Far in the negative tail GELU(x) = x Phi(x) is tiny but far above the
    bf16 range's floor (about -1.0e-18 at x = -9), so it must keep its relative
    accuracy there, not cancel to zero.  Pinned by Laplace's asymptotic series
    of the normal tail, Phi(-t) = phi(t)/t * sum_n (-1)^n (2n-1)!! / t^(2n),
    summed to its smallest term (below 1e-15 of the sum for t >= 9), and by
    scipy's ndtr away from it."""
    from scipy.special import ndtr
    for t in (9.0, 9.5, 10.0, 12.0, 16.0, 20.0, 26.0, 30.0, 37.0):
        term, total, n = 1.0, 1.0, 0
        while True:
            nxt = -term * (2 * n + 1) / (t * t)
            if abs(nxt) >= abs(term):
                break
            term, n = nxt, n + 1
            total += term
        assert abs(term) < 1e-15
        phi = np.exp(-t * t / 2) / np.sqrt(2 * np.pi)
        want = -t * phi / t * total
        got = float(oracle.gelu(np.array([-t]))[0])
        assert got == pytest.approx(want, rel=1e-12), (t, got, want)
    # the rounding of x / sqrt(2) reaches the result multiplied by about x^2
    # (the log-derivative of exp(-x^2 / 2)): 1369 * 2^-52 = 3e-13 at x = -37
    x = np.linspace(-37, -1, 3601)
    assert np.all(np.abs(oracle.gelu(x) / (x * ndtr(x)) - 1) <= 4 * x * x * 2.0 ** -52)


def test_gelu_lipschitz_constant_of_the_fused_tolerance():
    """The fused GEMM tests bound GELU's error by 1.13 x the GEMM bound: the
    largest |GELU'| is Phi(sqrt 2) + sqrt 2 phi(sqrt 2) = 1.128904, below 1.13.
    Checked on the oracle's GELU by central differences on a fine grid."""
    from scipy.special import ndtr
    x = np.linspace(-10, 10, 400001)
    h = 1e-6
    d = (oracle.gelu(x + h) - oracle.gelu(x - h)) / (2 * h)
    s2 = np.sqrt(2.0)
    closed = ndtr(s2) + s2 * np.exp(-1.0) / np.sqrt(2 * np.pi)
    assert closed == pytest.approx(1.128904, abs=1e-6)
    assert np.max(np.abs(d)) == pytest.approx(closed, abs=1e-6)
    assert np.max(np.abs(d)) < 1.13


def test_ridge_point_arithmetic(facts):
    r = facts["roofline_ridge"]
    assert r["fp4_dense_tflops"] * 1e12 / (r["hbm_gbs"] * 1e9) == r["ridge_flop_per_byte"]
