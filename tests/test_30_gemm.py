"""GPU block-scaled GEMM parity against the fp64 oracle, through the C ABI.

The first tests pin the scale-factor layout the tensor core reads: operands of
all-ones codes with unit scales, except one scale byte doubled at a chosen
(row, scale column); exactly the outputs that block feeds must change, by the
amount the definition C = sum_k A_dq B_dq gives."""
import numpy as np
import pytest
import torch

import oracle
from fp8_quantization_block_b200 import mx, synth
from gpu_helpers import gemm_check, host, quantize_dev

pytestmark = pytest.mark.gpu
FMTS = [0, 1, 2, 3]

ONE_CODE = {0: 0x38, 1: 0x3C, 2: 0x2, 3: 0x2}           # 1.0 in E4M3 / E5M2 / E2M1
UNIT_SCALE = {0: 127, 1: 127, 2: 127, 3: 0x38}          # 2^0 (E8M0) / 1.0 (E4M3)
DOUBLE_SCALE = {0: 128, 1: 128, 2: 128, 3: 0x40}


def probe_operand(fmt, rows, K, hot=None):
    bs = oracle.block_size(fmt)
    if fmt in (2, 3):
        codes = np.full(rows * K // 2, ONE_CODE[fmt] | (ONE_CODE[fmt] << 4), dtype=np.uint8)
    else:
        codes = np.full(rows * K, ONE_CODE[fmt], dtype=np.uint8)
    scales = np.zeros(oracle.scales_bytes(fmt, rows, K), dtype=np.uint8)
    for r in range(rows):
        for j in range(K // bs):
            scales[oracle.sf_offset(r, j, K // bs)] = UNIT_SCALE[fmt]
    if hot is not None:
        scales[oracle.sf_offset(hot[0], hot[1], K // bs)] = DOUBLE_SCALE[fmt]
    return codes, scales


def to_mx(fmt, rows, K, codes, scales, g=1.0):
    t = mx.empty(fmt, rows, K)
    t.codes.copy_(torch.from_numpy(codes))
    t.scales.copy_(torch.from_numpy(scales))
    if t.gscale is not None:
        t.gscale.fill_(g)
    return t


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("side", ["A", "B"])
def test_scale_layout_probe(fmt, side):
    M, N, K = 256, 256, 512
    bs = oracle.block_size(fmt)
    hots = [(0, 0), (37, 1), (70, 2), (101, 3), (127, 5), (128 + 64 + 9, K // bs - 1), (200, 6)]
    for hot in hots:
        ca, sa = probe_operand(fmt, M, K, hot if side == "A" else None)
        cb, sb = probe_operand(fmt, N, K, hot if side == "B" else None)
        A, B = to_mx(fmt, M, K, ca, sa), to_mx(fmt, N, K, cb, sb)
        C = mx.gemm(A, B)
        torch.cuda.synchronize()
        mx.check_device_error()
        Ad = oracle.dequantize_f64(fmt, ca, sa, 1.0, M, K)
        Bd = oracle.dequantize_f64(fmt, cb, sb, 1.0, N, K)
        Cref, _ = oracle.gemm_f64(Ad, Bd)
        got = C.float().cpu().double().numpy()
        assert np.array_equal(got, Cref), (fmt, side, hot, np.argwhere(got != Cref)[:4])
        # exactly one row (A side) or column (B side) exceeds the base value K
        changed = np.argwhere(got != K)
        axis = 0 if side == "A" else 1
        assert set(changed[:, axis].tolist()) == {hot[0]}


def quantized_pair(fmt, A_bits, B_bits):
    qa, qb = quantize_dev(A_bits, fmt), quantize_dev(B_bits, fmt)
    ca, sa, ga = host(qa)
    cb, sb, gb = host(qb)
    Ad = oracle.dequantize_f64(fmt, ca, sa, ga, *A_bits.shape)
    Bd = oracle.dequantize_f64(fmt, cb, sb, gb, *B_bits.shape)
    return qa, qb, Ad, Bd


@pytest.mark.parametrize("fmt", FMTS)
def test_tiny_config(fmt):
    A_bits, B_bits = synth.tiny_pair()
    qa, qb, Ad, Bd = quantized_pair(fmt, A_bits, B_bits)
    C = mx.gemm(qa, qb)
    torch.cuda.synchronize()
    mx.check_device_error()
    ok, worst = gemm_check(C, Ad, Bd)
    assert ok, worst


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,N,K", [(200, 72, 384), (1, 28, 128), (130, 300, 256), (257, 129, 640), (64, 520, 1152)])
def test_ragged_shapes(fmt, M, N, K):
    A_bits = synth.sweep_tensor(1000 + M, M, K)
    B_bits = synth.gaussian_weights(2000 + N, N, K)
    qa, qb, Ad, Bd = quantized_pair(fmt, A_bits, B_bits)
    C = mx.gemm(qa, qb)
    torch.cuda.synchronize()
    mx.check_device_error()
    ok, worst = gemm_check(C, Ad, Bd)
    assert ok, worst


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,N,K", [(1, 300, 640), (17, 520, 384), (32, 257, 1152)])
def test_small_m_kernel(fmt, M, N, K):
    """At most 32 rows of A and more than 128 of B: the kernel loads 32-row A
    tiles and keeps a fifth stage of B.  The tensor core's rows past 32 read
    other shared memory; those accumulator rows must never reach C (ragged N,
    a K tail inside a stage, M = 1 and M = 32)."""
    A_bits = synth.sweep_tensor(5000 + M, M, K)
    B_bits = synth.gaussian_weights(6000 + N, N, K)
    qa, qb, Ad, Bd = quantized_pair(fmt, A_bits, B_bits)
    big = torch.full((M + 3, N + 8), 5.0, dtype=torch.bfloat16, device="cuda")
    C = big[:M, :N]
    mx.gemm(qa, qb, out=C)
    torch.cuda.synchronize()
    mx.check_device_error()
    ok, worst = gemm_check(C, Ad, Bd)
    assert ok, worst
    assert torch.all(big[M:] == 5.0) and torch.all(big[:, N:] == 5.0)


def test_output_row_pitch():
    fmt = 0
    A_bits, B_bits = synth.tiny_pair()
    qa, qb, Ad, Bd = quantized_pair(fmt, A_bits, B_bits)
    big = torch.full((64, 200), 7.0, dtype=torch.bfloat16, device="cuda")
    mx.gemm(qa, qb, out=big[:, :64])
    torch.cuda.synchronize()
    ok, worst = gemm_check(big[:, :64], Ad, Bd)
    assert ok, worst
    assert torch.all(big[:, 64:] == 7.0)


def test_dit_mxfp8_full_size_sampled_rows():
    X = synth.dit_activations()
    W = synth.gaussian_weights(2, 3072, 3072)
    qa, qb, Ad, Bd = quantized_pair(0, X, W)
    C = mx.gemm(qa, qb)
    torch.cuda.synchronize()
    mx.check_device_error()
    rows = np.sort(np.random.default_rng(1).choice(4096, 256, replace=False))
    ok, worst = gemm_check(C, Ad, Bd, rows=rows)
    assert ok, worst


def test_nvfp4_mlp_gemm1_sampled_rows():
    X = synth.student_t(3, 4608, 3072)
    W1 = synth.gaussian_weights(4, 12288, 3072)
    qa, qb, Ad, Bd = quantized_pair(3, X, W1)
    C = mx.gemm(qa, qb)
    torch.cuda.synchronize()
    mx.check_device_error()
    rows = np.sort(np.random.default_rng(2).choice(4608, 64, replace=False))
    ok, worst = gemm_check(C, Ad, Bd, rows=rows)
    assert ok, worst


@pytest.mark.parametrize("fmt", [2, 3])
@pytest.mark.parametrize("M", [1, 16, 128])
def test_skinny_weight_stream(fmt, M):
    X = synth.normal_with_outliers(np.random.default_rng(200 + M), (M, 8192), 0.0, 1.0)
    X = synth.to_bf16_bits(X)
    W = synth.gaussian_weights(7, 28672, 8192)
    qa, qb, Ad, Bd = quantized_pair(fmt, X, W)
    C = mx.gemm(qa, qb)
    torch.cuda.synchronize()
    mx.check_device_error()
    cols = np.random.default_rng(3).choice(28672, 2048, replace=False)
    ok, worst = gemm_check(C[:, torch.from_numpy(cols).cuda()], Ad, Bd[cols])
    assert ok, worst


def test_gemm_is_deterministic():
    A_bits, B_bits = synth.tiny_pair(M=300, N=520, K=1024)
    qa, qb = quantize_dev(A_bits, 3), quantize_dev(B_bits, 3)
    c1 = mx.gemm(qa, qb).clone()
    c2 = mx.gemm(qa, qb)
    torch.cuda.synchronize()
    assert torch.equal(c1.view(torch.int16), c2.view(torch.int16))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("pair", [0, 1])
def test_pair_and_single_cta_kernels(fmt, pair):
    """M > 128 runs on CTA pairs (256 x 256 tiles) by default; the single-CTA
    kernel (128 x 256 tiles) stays available.  Both against the oracle,
    including ragged M and N tails and a K tail inside a stage."""
    M, N, K = 333, 520, 640
    A_bits = synth.sweep_tensor(3000 + fmt, M, K)
    B_bits = synth.gaussian_weights(4000 + fmt, N, K)
    qa, qb, Ad, Bd = quantized_pair(fmt, A_bits, B_bits)
    try:
        assert mx.mx_debug_set(mx.MX_DEBUG_PAIR_GEMM, pair) == mx.MX_OK
        C = mx.gemm(qa, qb)
        torch.cuda.synchronize()
        mx.check_device_error()
    finally:
        mx.mx_debug_set(mx.MX_DEBUG_PAIR_GEMM, 1)
    ok, worst = gemm_check(C, Ad, Bd)
    assert ok, worst
