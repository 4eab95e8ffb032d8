"""Exact-arithmetic (fractions.Fraction) brute-force checker for the C oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  It re-derives the
quantization of tiny inputs by exhaustive search instead of the C oracle's
closed-form steps, so that a slip in either (a wrong bias, a reversed tie, an
off-by-one in the scale rule, a transposed operand) shows up as a mismatch:

* element formats are decoded from their bit fields into exact Fractions and
  every rounding picks the nearest grid value by scanning the whole grid,
  ties to the even code;
* the MX block exponent is the smallest E in [0, 254] for which no element of
  the block exceeds the format's largest magnitude after division by
  2^(E - 127) (microscaling page, FAQ on how E8M0 picks the shared exponent);
* the NVFP4 block scale is the smallest of the 126 positive finite E4M3 values
  that keeps every element within 6 after division by g * s;
* the GEMM is an exact Fraction sum.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

E2M1_BITS, E4M3_BITS, E5M2_BITS, E3M2_BITS = (1, 2, 1), (1, 4, 3), (1, 5, 2), (1, 3, 2)


def _minifloat(code: int, ebits: int, mbits: int, bias: int) -> Fraction | None:
    s = (code >> (ebits + mbits)) & 1
    e = (code >> mbits) & ((1 << ebits) - 1)
    m = code & ((1 << mbits) - 1)
    if e == 0:
        mag = Fraction(m, 1 << mbits) * Fraction(2) ** (1 - bias)
    else:
        mag = (1 + Fraction(m, 1 << mbits)) * Fraction(2) ** (e - bias)
    return -mag if s else mag


def e2m1(code: int) -> Fraction:
    return _minifloat(code & 0xF, 2, 1, 1)


def e4m3(code: int) -> Fraction | None:
    if code & 0x7F == 0x7F:
        return None  # NaN
    return _minifloat(code, 4, 3, 7)


def e5m2(code: int) -> Fraction | None:
    if (code >> 2) & 0x1F == 0x1F:
        return None  # inf / NaN
    return _minifloat(code, 5, 2, 15)


def e3m2(code: int) -> Fraction:
    """OCP 6-bit E3M2: bias 3, every code finite."""
    return _minifloat(code & 0x3F, 3, 2, 3)


def bf16(bits: int) -> Fraction:
    s = (bits >> 15) & 1
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    assert e != 0xFF, "non-finite bf16"
    if e == 0:
        mag = Fraction(m, 128) * Fraction(2) ** -126
    else:
        mag = (1 + Fraction(m, 128)) * Fraction(2) ** (e - 127)
    return -mag if s else mag


# Positive finite grids: list of (value, code), increasing in value.
E2M1_GRID = [(e2m1(c), c) for c in range(8)]
E4M3_GRID = [(e4m3(c), c) for c in range(0x7F)]
E5M2_GRID = [(e5m2(c), c) for c in range(0x7C)]
E3M2_GRID = [(e3m2(c), c) for c in range(0x20)]
GRIDS = {0: (E4M3_GRID, 0x80), 1: (E5M2_GRID, 0x80), 2: (E2M1_GRID, 0x8), 3: (E2M1_GRID, 0x8),
         4: (E3M2_GRID, 0x20)}
MAXELEM = {0: Fraction(448), 1: Fraction(57344), 2: Fraction(6), 3: Fraction(6), 4: Fraction(28)}
BLOCK = {0: 32, 1: 32, 2: 32, 3: 16, 4: 32}
DECODE = {0: e4m3, 1: e5m2, 2: e2m1, 3: e2m1, 4: e3m2}


def round_to_grid(v: Fraction, grid, sign_bit: int, negative: bool) -> int:
    """Nearest grid magnitude to |v| by exhaustive scan, ties to the even code,
    saturating at the largest magnitude; the sign bit is kept for zero."""
    a = abs(v)
    best = None
    for val, code in grid:
        d = abs(a - val)
        if best is None or d < best[0] or (d == best[0] and code % 2 == 0):
            best = (d, code)
    if a > grid[-1][0]:
        best = (None, grid[-1][1])
    return best[1] | (sign_bit if negative else 0)


def mx_scale_byte(block: list[Fraction], fmt: int, threshold: Fraction | None = None) -> int:
    """Smallest E8M0 byte in [0, 254] after which no element exceeds
    `threshold` (the format's largest magnitude by default; 7 for MXFP4 with
    overflow-aware scaling), 254 if none does."""
    lim = MAXELEM[fmt] if threshold is None else threshold
    for E in range(0, 255):
        if all(abs(x) / Fraction(2) ** (E - 127) <= lim for x in block):
            return E
    return 254


def nvfp4_global_scale(amax_t: Fraction) -> Fraction:
    """Smallest fp32 value >= amax_t / 2688 (amax_t == 0 -> 1)."""
    if amax_t == 0:
        return Fraction(1)
    q = amax_t / 2688
    f = np.float32(float(q))
    while Fraction(float(f)) < q:
        f = np.nextafter(f, np.float32(np.inf))
    while True:
        p = np.nextafter(f, np.float32(0))
        if p > 0 and Fraction(float(p)) >= q:
            f = p
        else:
            break
    return Fraction(float(f))


def nvfp4_block_scale(block: list[Fraction], g: Fraction) -> int:
    if all(x == 0 for x in block):
        return 0
    for val, code in E4M3_GRID[1:]:
        if all(abs(x) <= 6 * g * val for x in block):
            return code
    return 0x7E


def quantize(fmt: int, bits: np.ndarray, g: Fraction | None = None, mx_threshold: Fraction | None = None):
    """Exact quantization of a tiny bf16 matrix (MX scales by the threshold
    rule above; elements by RNE onto the format's grid, saturating).

    Returns (codes[M][K] unpacked ints, scales[M][K/bs] ints, g)."""
    M, K = bits.shape
    X = [[bf16(int(bits[r, k])) for k in range(K)] for r in range(M)]
    neg = [[bool(int(bits[r, k]) & 0x8000) for k in range(K)] for r in range(M)]
    return quantize_values(fmt, X, neg, g, mx_threshold)


def quantize_values(fmt: int, X, neg, g: Fraction | None = None, mx_threshold: Fraction | None = None):
    """quantize() on exact values X[M][K] (Fractions) with sign flags neg[M][K]."""
    M, K = len(X), len(X[0])
    bs = BLOCK[fmt]
    grid, sbit = GRIDS[fmt]
    if fmt == 3 and g is None:
        g = nvfp4_global_scale(max(abs(x) for row in X for x in row))
    codes = [[0] * K for _ in range(M)]
    scales = [[0] * (K // bs) for _ in range(M)]
    for r in range(M):
        for j in range(K // bs):
            blk = X[r][j * bs:(j + 1) * bs]
            if fmt == 3:
                sc = nvfp4_block_scale(blk, g)
                denom = g * e4m3(sc)
            else:
                sc = mx_scale_byte(blk, fmt, mx_threshold)
                denom = Fraction(2) ** (sc - 127)
            scales[r][j] = sc
            for i, x in enumerate(blk):
                k = j * bs + i
                if denom == 0:
                    codes[r][k] = sbit if neg[r][k] else 0
                else:
                    codes[r][k] = round_to_grid(x / denom, grid, sbit, neg[r][k])
    return codes, scales, g


def mbs_static_mantissa(block: list[Fraction]) -> int:
    """Macro mantissa by brute force: e = floor(log2(alpha / 6)) found by
    scanning, then the smallest m in [0, 255] with alpha / (1 + m/256) <= 6 * 2^e
    (0 for an all-zero block or when none suffices)."""
    alpha = max(abs(x) for x in block)
    if alpha == 0:
        return 0
    e = next(e for e in range(-200, 200) if 6 * Fraction(2) ** e <= alpha < 6 * Fraction(2) ** (e + 1))
    for m in range(256):
        if alpha / (1 + Fraction(m, 256)) <= 6 * Fraction(2) ** e:
            return m
    return 0


def mbs_quantize_macro(block: list[Fraction], m: int, negative: list[bool]):
    """One macro block (128 exact values) quantized with macro mantissa m:
    per 16 the smallest E with every |x| / ((1 + m/256) 2^(E-127)) <= 6, the
    nearest E2M1 value of each quotient (ties to the even code).  Returns
    (codes[128], exponents[8], values xhat[128])."""
    f = 1 + Fraction(m, 256)
    codes, exps, xhat = [], [], []
    for jb in range(8):
        blk = block[jb * 16:(jb + 1) * 16]
        amax = max(abs(x) for x in blk)
        # the smallest E with amax <= 6 f 2^(E-127): a float estimate, settled exactly
        E = 0 if amax == 0 else min(254, max(0, math.ceil(math.log2(float(amax / (6 * f)))) + 127))
        while E > 0 and amax <= 6 * f * Fraction(2) ** (E - 1 - 127):
            E -= 1
        while E < 254 and amax > 6 * f * Fraction(2) ** (E - 127):
            E += 1
        exps.append(E)
        denom = f * Fraction(2) ** (E - 127)
        for i, x in enumerate(blk):
            c = round_to_grid(x / denom, E2M1_GRID, 0x8, negative[jb * 16 + i])
            codes.append(c)
            xhat.append(e2m1(c) * denom)
    return codes, exps, xhat


def mbs_dynamic_choice(block: list[Fraction], negative: list[bool]):
    """Every macro mantissa's exact squared error of the block: a list of 256
    Fractions sum (x - xhat)^2."""
    out = []
    for m in range(256):
        _, _, xhat = mbs_quantize_macro(block, m, negative)
        out.append(sum(((x - h) ** 2 for x, h in zip(block, xhat)), Fraction(0)))
    return out


def quantize_mbs(bits: np.ndarray):
    """MXFP4 with static macro-block scaling, exhaustively: per 128 elements m
    as above; per 16 the smallest E with every |x| / ((1 + m/256) 2^(E-127)) <= 6;
    elements the nearest E2M1 value of that quotient, ties to the even code.
    Returns (codes[M][K], scales[M][K/16], macro[M][K/128])."""
    M, K = bits.shape
    X = [[bf16(int(bits[r, k])) for k in range(K)] for r in range(M)]
    codes = [[0] * K for _ in range(M)]
    scales = [[0] * (K // 16) for _ in range(M)]
    macro = [[0] * (K // 128) for _ in range(M)]
    for r in range(M):
        for mb in range(K // 128):
            m = mbs_static_mantissa(X[r][mb * 128:(mb + 1) * 128])
            macro[r][mb] = m
            f = 1 + Fraction(m, 256)
            for jb in range(8):
                j = mb * 8 + jb
                blk = X[r][j * 16:(j + 1) * 16]
                E = next((E for E in range(255) if all(abs(x) / (f * Fraction(2) ** (E - 127)) <= 6 for x in blk)),
                         254)
                scales[r][j] = E
                denom = f * Fraction(2) ** (E - 127)
                for i, x in enumerate(blk):
                    codes[r][j * 16 + i] = round_to_grid(x / denom, E2M1_GRID, 0x8, bool(int(bits[r, j * 16 + i]) & 0x8000))
    return codes, scales, macro


def dequant(fmt: int, codes, scales, g: Fraction | None):
    bs = BLOCK[fmt]
    out = []
    for r, row in enumerate(codes):
        orow = []
        for k, c in enumerate(row):
            sc = scales[r][k // bs]
            if fmt == 3:
                s = g * e4m3(sc)
                v = e2m1(c)
            else:
                s = Fraction(2) ** (sc - 127)
                v = DECODE[fmt](c)
            orow.append(s * v)
        out.append(orow)
    return out


def gemm(A, B, rows=None, cols=None):
    rows = range(len(A)) if rows is None else rows
    cols = range(len(B)) if cols is None else cols
    return [[sum((a * b for a, b in zip(A[i], B[j])), Fraction(0)) for j in cols] for i in rows]
