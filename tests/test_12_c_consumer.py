"""A plain C99 program uses the library through include/mx.h alone (no C++,
no PyTorch): it must compile and link against libmx.so with warnings as
errors (CPU), and on the GPU its codes and scales must equal the oracle's and
its GEMM output must be within the oracle's tolerance."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from fp8_quantization_block_b200 import build as mxbuild
from fp8_quantization_block_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi", "mx_c_consumer.c")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def compile_consumer(out_dir: str) -> str:
    lib = mxbuild.build()
    exe = os.path.join(out_dir, "mx_c_consumer")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-O1", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), SRC, "-o", exe, "-L", os.path.dirname(lib), "-lmx",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-Wl,-rpath," + os.path.dirname(lib),
           "-Wl,-rpath," + os.path.join(CUDA, "lib64")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-3000:]
    return exe


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_consumer_compiles_and_links_as_c99(tmp_path):
    exe = compile_consumer(str(tmp_path))
    assert os.path.exists(exe)


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", [0, 2, 3])
def test_c_consumer_matches_the_oracle(tmp_path, fmt):
    exe = compile_consumer(str(tmp_path))
    A_bits, B_bits = synth.tiny_pair()
    M, K = A_bits.shape
    N = B_bits.shape[0]
    a_path, b_path = tmp_path / "a.bin", tmp_path / "b.bin"
    np.ascontiguousarray(A_bits, dtype="<u2").tofile(a_path)
    np.ascontiguousarray(B_bits, dtype="<u2").tofile(b_path)
    prefix = str(tmp_path / "out")
    res = subprocess.run([exe, str(fmt), str(M), str(N), str(K), str(a_path), str(b_path), prefix],
                         capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stdout + res.stderr
    codes = np.fromfile(prefix + ".codes", dtype=np.uint8)
    scales = np.fromfile(prefix + ".scales", dtype=np.uint8)
    g = float(np.fromfile(prefix + ".gscale", dtype=np.float32)[0])
    C = np.fromfile(prefix + ".c", dtype="<u2").reshape(M, N)
    ca, sa, ga = oracle.quantize(fmt, A_bits)
    assert np.array_equal(codes, ca) and np.array_equal(scales, sa)
    if fmt == 3:
        assert np.float32(g) == np.float32(ga)
    cb, sb, gb = oracle.quantize(fmt, B_bits)
    Ad = oracle.dequantize_f64(fmt, ca, sa, ga, M, K)
    Bd = oracle.dequantize_f64(fmt, cb, sb, gb, N, K)
    Cref, Cabs = oracle.gemm_f64(Ad, Bd)
    Cg = (C.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ok, worst = oracle.gemm_tolerance_ok(Cg, Cref, Cabs)
    assert ok, worst
