"""GPU quantize / dequantize parity: packed codes, tiled scales and the NVFP4
global scale are compared bit for bit with the CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from fp8_quantization_block_b200 import mx, synth
from gpu_helpers import assert_quant_equal, host, quantize_dev, to_dev

pytestmark = pytest.mark.gpu
FMTS = [0, 1, 2, 3]


@pytest.mark.parametrize("fmt", FMTS)
def test_tiny_pair(fmt):
    A, B = synth.tiny_pair()
    for bits in (A, B):
        assert_quant_equal(quantize_dev(bits, fmt), bits, fmt)


@pytest.mark.parametrize("fmt", FMTS)
def test_edge_and_tie_rows(fmt):
    bits = np.vstack([synth.edge_rows(256), synth.tie_rows(256, fmt)])
    assert_quant_equal(quantize_dev(bits, fmt), bits, fmt)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,K", [(1, 32), (200, 96), (129, 4096), (300, 160), (5, 2080)])
def test_ragged_shapes(fmt, M, K):
    bits = synth.sweep_tensor(7 + M, M, K)
    assert_quant_equal(quantize_dev(bits, fmt), bits, fmt)


@pytest.mark.parametrize("M,K", [(3, 48), (130, 208), (64, 16)])
def test_nvfp4_16_element_tails(M, K):
    bits = synth.student_t(11, M, K)
    assert_quant_equal(quantize_dev(bits, 3), bits, 3)


@pytest.mark.parametrize("g", [0.01, 1.0, 3.0e-6, 7.5])
def test_nvfp4_given_gscale(g):
    bits = synth.student_t(12, 96, 512)
    g32 = float(np.float32(g))
    q = quantize_dev(bits, 3, gscale=g32)
    assert_quant_equal(q, bits, 3, gscale=g32)
    assert float(q.gscale.cpu()[0]) == g32


@pytest.mark.parametrize("scale_exp", [-118, -125, 100])
def test_nvfp4_extreme_global_scales(scale_exp):
    # a whole tensor near the bottom of the bf16 range (g subnormal: the block
    # scale search walks the codes exactly) or near the top, g computed
    x = synth.bits_to_tensor(synth.student_t(14, 64, 512)).float().numpy() * np.float32(2.0 ** scale_exp)
    bits = synth.to_bf16_bits(x)
    assert_quant_equal(quantize_dev(bits, 3), bits, 3)


@pytest.mark.parametrize("g", [1e-39, 3e-36])
def test_nvfp4_given_tiny_gscale(g):
    # subnormal and tiny given g on ordinary data: most blocks saturate at s = 448
    bits = synth.student_t(15, 32, 256)
    g32 = float(np.float32(g))
    assert_quant_equal(quantize_dev(bits, 3, gscale=g32), bits, 3, gscale=g32)


@pytest.mark.parametrize("fmt", FMTS)
def test_row_pitch_larger_than_k(fmt):
    bits = synth.sweep_tensor(31, 70, 640)
    x = to_dev(bits)
    padded = torch.zeros((70, 704), dtype=torch.bfloat16, device="cuda")
    padded[:, :640] = x
    q = mx.quantize(padded[:, :640], fmt)
    torch.cuda.synchronize()
    assert_quant_equal(q, bits, fmt)


@pytest.mark.parametrize("fmt", FMTS)
def test_sweep_block(fmt):
    bits = synth.sweep_tensor(100, 2048, 4096)
    assert_quant_equal(quantize_dev(bits, fmt), bits, fmt)


def test_dit_activations_full_mxfp8():
    bits = synth.dit_activations()
    for fmt in (0, 1):
        assert_quant_equal(quantize_dev(bits, fmt), bits, fmt)


def test_mlp_activations_full_nvfp4():
    bits = synth.student_t(3, 4608, 3072)
    assert_quant_equal(quantize_dev(bits, 3), bits, 3)


@pytest.mark.parametrize("fmt", FMTS)
def test_largest_sweep_sampled_rows(fmt):
    """[262144 x 4096] (2^30 elements) drawn on the device by torch's seeded
    generator; codes of sampled rows (quantization is row-local given g)."""
    M, K = 262144, 4096
    gen = torch.Generator(device="cuda").manual_seed(110)
    x = torch.randn((M, K), generator=gen, device="cuda", dtype=torch.float32)
    mask = torch.rand((M, K), generator=gen, device="cuda") < 0.005
    x = torch.where(mask, x * 100, x).to(torch.bfloat16)
    del mask
    q = mx.quantize(x, fmt)
    torch.cuda.synchronize()
    mx.check_device_error()
    rng = np.random.default_rng(5)
    rows = np.sort(np.concatenate([rng.choice(M, 250, replace=False), [0, 127, 128, M - 1]]))
    xb = x[torch.from_numpy(rows).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
    g = None
    if fmt == 3:
        amax = float(x.abs().max().float().cpu())
        g = oracle.nvfp4_global_scale(amax)
        assert float(q.gscale.cpu()[0]) == g
    c, s, _ = oracle.quantize(fmt, xb, gscale=g)
    bs = oracle.block_size(fmt)
    row_bytes = K * (8 if fmt < 2 else 4) // 8
    gc = q.codes.view(M, row_bytes)[torch.from_numpy(rows).cuda()].cpu().numpy()
    gs = q.scales.cpu().numpy()
    for t, r in enumerate(rows):
        assert np.array_equal(gc[t], c[t * row_bytes:(t + 1) * row_bytes]), r
        got = [gs[oracle.sf_offset(int(r), j, K // bs)] for j in range(K // bs)]
        want = [s[oracle.sf_offset(t, j, K // bs)] for j in range(K // bs)]
        assert got == want, r
    del x


@pytest.mark.parametrize("fmt", FMTS)
def test_dequantize_bit_exact(fmt):
    bits = np.vstack([synth.sweep_tensor(40, 250, 512), synth.edge_rows(512)])
    q = quantize_dev(bits, fmt)
    d = mx.dequantize(q)
    torch.cuda.synchronize()
    c, s, g = host(q)
    want = oracle.dequantize_bf16(fmt, c, s, g, bits.shape[0], bits.shape[1])
    got = d.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, want)


def test_quantize_is_deterministic():
    bits = synth.student_t(3, 512, 3072)
    a = host(quantize_dev(bits, 3))
    b = host(quantize_dev(bits, 3))
    assert all(np.array_equal(u, v) for u, v in zip(a[:2], b[:2])) and a[2] == b[2]
