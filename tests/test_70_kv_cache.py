"""K/V-cache quantization at the shapes of an 80-layer, 8-KV-head, 128-dim
grouped-query-attention model (page "Microscaling MXFP4/NVFP4 on Blackwell",
section on KV-cache compression): codes and scales bit-exact with the oracle
for MXFP4 and MXFP8 E5M2, and the per-token byte counts the page prints."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from fp8_quantization_block_b200 import mx, synth
from gpu_helpers import assert_quant_equal, quantize_dev

LAYERS, HEADS, DIM = 80, 8, 128
ROWS_PER_TOKEN, K = 2 * LAYERS, HEADS * DIM
FACTS = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "microscaling_facts.json")))["kv_cache_bytes_per_token"]


def test_bytes_per_token_from_the_library_sizes():
    # one token's K and V for every layer is a [160 x 1024] matrix
    codes = mx.mx_codes_bytes(mx.MX_MXFP4, ROWS_PER_TOKEN, K)
    scales_unpadded = ROWS_PER_TOKEN * K // 32
    assert codes + scales_unpadded == FACTS["mxfp4_bytes"]            # 87,040 B
    assert mx.mx_codes_bytes(mx.MX_MXFP8_E5M2, ROWS_PER_TOKEN, K) == FACTS["fp8_bytes"]
    assert ROWS_PER_TOKEN * K * 2 == FACTS["bf16_bytes"]
    # many tokens: 128-row padding of the scale tiles vanishes (160 * 4 tokens = 640 rows)
    assert mx.mx_scales_bytes(mx.MX_MXFP4, 4 * ROWS_PER_TOKEN, K) == 4 * scales_unpadded


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", [mx.MX_MXFP4, mx.MX_MXFP8_E5M2, mx.MX_MXFP8_E4M3, mx.MX_NVFP4])
@pytest.mark.parametrize("tokens", [1, 3])
def test_kv_quantize_bit_exact(fmt, tokens):
    bits = synth.kv_cache(80 + tokens, tokens)
    assert bits.shape == (tokens * ROWS_PER_TOKEN, K)
    assert_quant_equal(quantize_dev(bits, fmt), bits, fmt)


@pytest.mark.gpu
def test_kv_dequantize_round_trip_matches_oracle():
    bits = synth.kv_cache(90, 2)
    q = quantize_dev(bits, mx.MX_MXFP4)
    got = mx.dequantize(q)
    torch.cuda.synchronize()
    c, s, g = oracle.quantize(mx.MX_MXFP4, bits)
    want = oracle.dequantize_bf16(mx.MX_MXFP4, c, s, g, *bits.shape)
    assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16), want)
