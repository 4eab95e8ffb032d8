"""Host-side helpers of bench.py, on the CPU: the kernel each GEMM shape runs
(named as the built library's kernel symbols), and the roofline object that
picks the tensor or the HBM bound by arithmetic intensity."""
import importlib.util
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PEAKS = {"hbm_gbs": 6537.3, "bf16_tflops": 1647.8, "bf16_tflops_sustained": 1379.4}


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="module")
def kernel_symbols():
    from fp8_quantization_block_b200 import build
    lib = build.build()
    if shutil.which("nm") is None:
        pytest.skip("nm not available")
    out = subprocess.run(["nm", "-C", lib], capture_output=True, text=True, check=True).stdout
    names = set()
    for line in out.splitlines():
        for kind in ("gemm_pair_kernel<", "gemm_kernel<"):
            i = line.find("mx::" + kind)
            if i >= 0:
                j = line.index(">", i)
                names.add(line[i + 4:j + 1])
    return names


SHAPES = [(4096, 3072), (4608, 12288), (16, 28672), (1, 300), (32, 257), (33, 4096), (128, 28672),
          (300, 100), (129, 129), (128, 129)]


@pytest.mark.parametrize("fmt", [0, 1, 2, 3, 4])
def test_kernel_names_are_built_kernels(bench, kernel_symbols, fmt):
    for M, N in SHAPES:
        for gelu in (False, True):
            for split in (False, True):
                name = bench.gemm_kernel_name(fmt, M, N, gelu, split)
                assert name in kernel_symbols, (fmt, M, N, name, sorted(kernel_symbols))


def test_kernel_choice_by_shape(bench):
    assert bench.gemm_kernel_name(0, 4096, 3072) == "gemm_pair_kernel<0, 6, 256, false>"
    assert bench.gemm_kernel_name(3, 4608, 12288) == "gemm_pair_kernel<3, 5, 256, false>"
    assert bench.gemm_kernel_name(3, 4608, 12288, gelu=True) == "gemm_pair_kernel<3, 7, 128, false>"
    assert bench.gemm_kernel_name(3, 4608, 12288, gelu=True, split=True) == "gemm_pair_kernel<3, 7, 128, false>"
    assert bench.gemm_kernel_name(4, 4096, 3072) == "gemm_pair_kernel<4, 6, 256, false>"
    assert bench.gemm_kernel_name(3, 16, 28672) == "gemm_kernel<3, 256, 5, 32, false>"
    assert bench.gemm_kernel_name(3, 16, 8192, split=True) == "gemm_kernel<3, 256, 5, 32, true>"
    assert bench.gemm_kernel_name(3, 128, 28672) == "gemm_kernel<3, 256, 4, 128, false>"
    assert bench.gemm_kernel_name(2, 300, 100) == "gemm_kernel<2, 128, 4, 128, false>"


def test_roofline_bound_follows_arithmetic_intensity(bench):
    # DiT MXFP8 GEMM: ~1600 FLOP per algorithmic byte, far above the ridge
    ts, tb = bench.tensor_peak(0, PEAKS, True), bench.tensor_peak(0, PEAKS, False)
    assert tb == pytest.approx(2 * 1647.8) and ts == pytest.approx(2 * 1379.4)
    clocks = {"sm_mhz": 1710.0, "sm_max_mhz": 1965.0}
    r = bench.gemm_roofline(0, 4096, 3072, 3072, 0.0397, PEAKS, tb, ts, clocks)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    flops = 2 * 4096 * 3072 * 3072
    assert r["achieved"] == pytest.approx(flops / 0.0397e-3 / 1e12, rel=1e-3)
    # the headline fraction is against the burst peak (the kernel is timed as a
    # short graph replay): 77.31 GFLOP / 39.7 us / (2 x 1647.8) = 0.59
    assert r["peak"] == pytest.approx(tb, rel=1e-3)
    assert r["frac"] == pytest.approx(flops / 0.0397e-3 / 1e12 / (2 * 1647.8), rel=1e-3)
    assert r["frac"] == pytest.approx(0.591, abs=2e-3)
    assert r["frac_of_sustained_peak"] == pytest.approx(r["achieved"] / ts, rel=1e-3)
    # clock-normalised: 39.7 us x 1710 / 1965 = 34.55 us
    assert r["clock_normalised_kernel_us"] == pytest.approx(39.7 * 1710 / 1965, abs=0.01)
    assert r["clock_normalised_frac"] == pytest.approx(flops / (39.7e-6 * 1710 / 1965) / 1e12 / tb, rel=1e-3)
    # without clock samples there is no clock-normalised figure
    assert "clock_normalised_frac" not in bench.gemm_roofline(0, 4096, 3072, 3072, 0.0397, PEAKS, tb, ts, None)
    # skinny NVFP4 weight stream: ~32 FLOP per byte, below the ridge
    ts, tb = bench.tensor_peak(3, PEAKS, True), bench.tensor_peak(3, PEAKS, False)
    r = bench.gemm_roofline(3, 16, 28672, 8192, 0.025, PEAKS, tb, ts, clocks)
    nbytes = bench.gemm_bytes(3, 16, 28672, 8192)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["algorithmic_bytes"] == nbytes
    # W: 28672 x 8192 codes at 4 bits plus one E4M3 scale per 16 (padded tiles), X and C small
    assert nbytes == 28672 * 8192 // 2 + 28672 * 8192 // 16 + 128 * 8192 // 16 + 16 * 8192 // 2 + 2 * 16 * 28672
    assert r["achieved"] == pytest.approx(nbytes / 0.025e-3 / 1e9, rel=1e-3)
    assert r["frac"] == pytest.approx(r["achieved"] / PEAKS["hbm_gbs"], rel=1e-3)


def test_result_line_keeps_the_contract(bench):
    """The GPU arm's JSON line built from fake device times: every key of the
    contract, whole-job value = world x per-replica work / slowest time, the
    roofline object of the dominant kernel, e2e with the copy bytes."""
    import argparse
    args = argparse.Namespace(steps=50, warmup=5, workload="dit_mxfp8")
    wl = bench.WORKLOADS["dit_mxfp8"]
    r = {"ms": 50 * 0.049, "f_ms": [0.0405] * 50, "f_ms_iso": [0.044] * 50, "two_ms": 0.052, "q_ms": 0.0099,
         "g_ms": 0.042, "e2e_ms": 50 * 0.55, "eager_ms": 50 * 0.048, "n_sets": 6,
         "per_set": 73_000_000, "h2d": 4096 * 3072 * 2, "d2h": 4096 * 3072 * 2,
         "clocks": {"sm_mhz": 1762.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}}
    for world in (1, 2):
        line = bench.result_line(args, wl, r, world)
        for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                  "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
            assert k in line, k
        flops = 2.0 * 4096 * 3072 * 3072
        assert line["n_gpus"] == world and line["steps"] == 50 and line["scaling"] == "weak"
        assert line["value"] == pytest.approx(world * flops * 50 / (r["ms"] * 1e-3) / 1e12, rel=1e-3)
        assert line["higher_is_better"] is True and line["vs_baseline"] is None
        assert line["config"]["workload"] == wl["name"]
        roof = line["roofline"]
        assert roof["bound"] == "tensor" and roof["kernel"] == "gemm_pair_kernel<0, 6, 256, false>"
        assert roof["kernel_us"] == pytest.approx(42.0)                  # the GEMM's own launches
        assert roof["frac"] == pytest.approx(roof["achieved"] / roof["peak"], rel=1e-3)
        assert roof["peak"] == pytest.approx(bench.tensor_peak(0, bench.measured_peaks()[0], False), rel=1e-3)
        assert roof["clock_normalised_kernel_us"] == pytest.approx(42.0 * 1762 / 1965, abs=0.01)
        assert roof["fused_call"]["us"] == pytest.approx(40.5)
        assert roof["fused_call"]["frac"] == pytest.approx(flops / 40.5e-6 / 1e12 / roof["peak"], rel=1e-3)
        assert "traffic" in roof
        assert set(line["e2e"]) >= {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
        assert line["e2e"]["h2d_bytes_per_step"] == r["h2d"]
        # the counter reset, the quantize kernel and the GEMM overlapping it
        assert line["gpu_launches"] == 3 * 50
        split = line["two_kernel_split"]
        assert split["step_us"] == pytest.approx(52.0) and split["gemm_us"] == pytest.approx(42.0)
        assert split["quantize_GB/s"] == pytest.approx(4096 * 3072 * 3.03125 / 9.9e-6 / 1e9, rel=1e-3)
    # the skinny workload's GEMM is reported against HBM
    args.workload = "skinny_nvfp4"
    line = bench.result_line(args, bench.WORKLOADS["skinny_nvfp4"], dict(r, f_ms=[0.025] * 50), 1)
    assert line["roofline"]["bound"] == "hbm" and line["roofline"]["unit"] == "GB/s"
    assert line["roofline"]["kernel"] == "gemm_kernel<3, 256, 5, 32, false>"
    # one band of X: the amax slot's clear, the amax pre-pass, the quantize kernel, the GEMM
    assert line["gpu_launches"] == 4 * 50
    json_line = __import__("json").dumps(line)
    assert "\n" not in json_line


def test_fused_launch_counts(bench):
    # MX formats: counter reset + quantize + GEMM with several bands, quantize + GEMM with one
    assert bench.fused_launches(0, 4096, 3072) == 3 and bench.fused_launches(2, 128, 8192) == 2
    # NVFP4 without g: the amax pre-pass (slot clear + amax) before the quantize ...
    assert bench.fused_launches(3, 16, 8192) == 4 and bench.fused_launches(3, 4608, 3072) == 4
    # ... except for an X of at most 16384 elements, whose amax the quantize kernel takes itself
    assert bench.fused_launches(3, 1, 8192) == 2 and bench.fused_launches(3, 1, 16384) == 2
    assert bench.fused_launches(3, 2, 16384) == 4


def test_extras_get_clock_normalised_fractions(bench):
    ex = {"mlp_nvfp4_gemm1": {"us": 81.5, "frac_tensor": 0.647}, "quantize_sweep": {"x": {"frac_hbm": 0.8}}}
    bench.add_clock_normalised(ex, {"sm_mhz": 1700.0, "sm_max_mhz": 1965.0})
    assert ex["mlp_nvfp4_gemm1"]["clock_normalised_frac_tensor"] == pytest.approx(0.647 * 1965 / 1700, abs=1e-3)
    assert "clock_normalised_frac_tensor" not in ex["quantize_sweep"]
    ex2 = {"g": {"frac_tensor": 0.5}}
    bench.add_clock_normalised(ex2, {"sm_mhz": None, "sm_max_mhz": None})
    assert "clock_normalised_frac_tensor" not in ex2["g"]
