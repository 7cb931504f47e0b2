"""The benchmark's reference arm (the oracle on the host cores) runs on a CPU
machine and prints one JSON line with the keys the benchmark contract names:
checked on the tiny workload so it takes seconds."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_16x16_fp32", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "tiny_16x16_fp32" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    # the step is a uniformly scaled-down sample: the rate and the sample time
    # describe the same work, the full-layer time is a separate estimate
    f = d["sample_fraction"]
    assert 0 < f <= 1
    assert abs(d["full_layer_ms_estimate"] * f - d["ms_per_step"]) <= 1e-6 * d["ms_per_step"]
    # the same config object as the GPU arm prints
    sys.path.insert(0, ROOT)
    import bench
    from quantized_conv3d_implicit_b200 import workloads
    assert d["config"] == json.loads(json.dumps(bench.workload_config(workloads.get("tiny_16x16_fp32"))))


def test_default_workload_is_the_largest_single_gpu_layer():
    from quantized_conv3d_implicit_b200 import workloads
    flops = {n: wl.flops for n, wl in workloads.WORKLOADS.items()}
    assert workloads.HEADLINE == max(flops, key=flops.get)
    crop = workloads.get("edge_full_96_bf16_d5")
    full = workloads.get(workloads.HEADLINE)
    assert crop.x_shape[3:] == full.x_shape[3:] and crop.cout == full.cout and crop.kernel == full.kernel


def test_warmup_below_three_is_refused():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--warmup", "2"],
                       capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert r.returncode != 0 and "warmup" in r.stderr
