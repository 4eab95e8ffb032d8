"""Failure detection without faulting the GPU: the GEMM's producer is told to
issue nothing, so the consumers' bounded waits run out after a short limit,
the kernel returns early, and mx_check_device_error reports MX_ERR_TIMEOUT.
The context stays usable: a normal GEMM afterwards is correct."""
import numpy as np
import pytest
import torch

from fp8_quantization_block_b200 import mx, synth
from gpu_helpers import gemm_check, host, quantize_dev
import oracle

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_context_survives():
    A_bits, B_bits = synth.tiny_pair()
    qa, qb = quantize_dev(A_bits, 0), quantize_dev(B_bits, 0)
    torch.cuda.synchronize()
    assert mx.mx_check_device_error()[0] == mx.MX_OK
    try:
        assert mx.mx_debug_set(mx.MX_DEBUG_WAIT_LIMIT_NS, 50_000_000) == mx.MX_OK    # 50 ms
        assert mx.mx_debug_set(mx.MX_DEBUG_SKIP_PRODUCER, 1) == mx.MX_OK
        mx.gemm(qa, qb)
        status, info = mx.mx_check_device_error()
    finally:
        mx.mx_debug_set(mx.MX_DEBUG_SKIP_PRODUCER, 0)
        mx.mx_debug_set(mx.MX_DEBUG_WAIT_LIMIT_NS, 1_000_000_000)
    assert status == mx.MX_ERR_TIMEOUT, (status, info)
    assert info[0] & 1 and info[1] != 0 and info[3] >= 1
    assert mx.mx_check_device_error()[0] == mx.MX_OK          # the word was cleared
    # the context is still healthy
    C = mx.gemm(qa, qb)
    torch.cuda.synchronize()
    assert mx.mx_check_device_error()[0] == mx.MX_OK
    ca, sa, ga = host(qa)
    cb, sb, gb = host(qb)
    ok, worst = gemm_check(C, oracle.dequantize_f64(0, ca, sa, ga, 64, 256), oracle.dequantize_f64(0, cb, sb, gb, 64, 256))
    assert ok, worst


def test_error_word_starts_clean_and_status_strings():
    assert mx.mx_check_device_error()[0] == mx.MX_OK
    assert mx.mx_status_string(mx.MX_ERR_TIMEOUT) == "MX_ERR_TIMEOUT"
