"""Shared helpers for the GPU parity tests (marshalling only)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from fp8_quantization_block_b200 import mx, synth

FMT_NAMES = {0: "mxfp8_e4m3", 1: "mxfp8_e5m2", 2: "mxfp4", 3: "nvfp4"}


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return synth.bits_to_tensor(bits).cuda()


def quantize_dev(bits: np.ndarray, fmt: int, gscale: float | None = None):
    x = to_dev(bits)
    g = None if gscale is None else torch.tensor([gscale], dtype=torch.float32, device="cuda")
    q = mx.quantize(x, fmt, gscale=g)
    torch.cuda.synchronize()
    mx.check_device_error()
    return q


def host(q: mx.MxTensor):
    g = float(q.gscale.cpu()[0]) if q.gscale is not None else 1.0
    return q.codes.cpu().numpy(), q.scales.cpu().numpy(), g


def first_mismatch(a: np.ndarray, b: np.ndarray):
    idx = np.nonzero(a != b)[0]
    return None if idx.size == 0 else (int(idx[0]), int(a[idx[0]]), int(b[idx[0]]), int(idx.size))


def assert_quant_equal(q: mx.MxTensor, bits: np.ndarray, fmt: int, gscale: float | None = None):
    c, s, g = oracle.quantize(fmt, bits, gscale=gscale)
    gc, gs, gg = host(q)
    assert first_mismatch(gc, c) is None, f"codes differ: first (index, gpu, oracle, count) = {first_mismatch(gc, c)}"
    assert first_mismatch(gs, s) is None, f"scales differ: first (index, gpu, oracle, count) = {first_mismatch(gs, s)}"
    if fmt == 3:
        assert np.float32(gg) == np.float32(g), (gg, g)
    return c, s, g


def gemm_check(C: torch.Tensor, Ad: np.ndarray, Bd: np.ndarray, rows=None):
    Cref, Cabs = oracle.gemm_f64(Ad, Bd, rows=rows)
    Cg = C.float().cpu().double().numpy()
    if rows is not None:
        Cg = Cg[np.asarray(rows)]
    ok, worst = oracle.gemm_tolerance_ok(Cg, Cref, Cabs)
    return ok, worst
