"""bench.py's JSON line: the keys and types the benchmark contract requires.

The reference arm (the fp64 oracle on the host cores) runs on the CPU; the GPU arm runs
on a small case of the same kernel."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
             "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "e2e"}


def _run(args, timeout=900):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                         capture_output=True, text=True, timeout=timeout)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_reference_arm_line():
    d = _run(["--impl", "reference", "--steps", "2", "--warmup", "1", "--rows", "1024"])
    assert BASE_KEYS <= set(d)
    assert d["impl"] == "reference"
    assert d["unit"] == "GB/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["config"]["workload"].startswith("wan22_ln_B1_L176400_D5120")


@pytest.mark.gpu
def test_gpu_arm_line():
    d = _run(["--rows", "8192", "--steps", "20", "--warmup", "5", "--cpu-seconds", "1"])
    assert BASE_KEYS <= set(d)
    assert d["n_gpus"] == 1 and d["steps"] == 20 and d["warmup"] == 5
    assert d["scaling"] == "weak" and d["dtype"] == "bf16" and d["unit"] == "GB/s"
    rf = d["roofline"]
    assert rf["bound"] == "hbm" and rf["unit"] == "GB/s" and rf["peak"] > 0
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-3
    assert d["gpu_launches"] == 20
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert e["verified"] is True, e["verified"]      # host copies equal the device outputs
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["config"]["launch"] == "stream"
    cb = d["cpu_baseline"]
    assert cb["one_core"]["value"] > 0 and cb["one_core"]["rows_per_s"] > 0


@pytest.mark.gpu
def test_gpu_arm_flushed_small_case():
    # a launch-bound shape with L2 flushed before every timed launch
    d = _run(["--workload", "rms_fused_B1_L16_D5120", "--flush-l2", "--steps", "20", "--warmup", "5",
              "--no-e2e", "--no-cpu-baseline"])
    assert d["gpu_launches"] == 20 and d["value"] > 0
    assert d["config"]["l2"].startswith("flushed")


@pytest.mark.gpu
def test_gpu_arm_norm_only():
    d = _run(["--workload", "microbench_bcast_B1_L176400_D5120", "--spec", "ln_nss_now",
              "--rows", "4096", "--steps", "10", "--warmup", "3", "--cpu-seconds", "1"])
    assert d["config"]["spec"] == "ln_nss_now" and d["value"] > 0
    assert d["e2e"]["d2h_bytes_per_step"] == 4096 * 5120 * 2   # y only
    assert d["e2e"]["verified"] is True, d["e2e"]["verified"]


def test_kernel_digest_ignores_comments_only():
    # the recorded ncu traffic stays attached to the code it was measured on: comments
    # and layout do not change the digest, code does (string literals kept verbatim)
    sys.path.insert(0, ROOT)
    import bench
    base = 'x = a + b; // sum\nasm("add.f32 %0, %1; // not a comment");'
    assert bench._code_tokens(base) == bench._code_tokens(
        '/* block */ x = a +   b;\n\nasm("add.f32 %0, %1; // not a comment"); // more')
    assert bench._code_tokens(base) != bench._code_tokens(base.replace("a + b", "a - b"))
    assert bench._code_tokens(base) != bench._code_tokens(base.replace("// not a", "// NOT a"))
    assert bench._code_tokens("c = '\\''; // q") == "c = '\\'';"


@pytest.mark.gpu
def test_gpu_arm_dit_forward_mix():
    # one step = the 121 norm calls of a DiT forward (41 + 40 + 40) on the broadcast shape
    d = _run(["--dit-mix", "--rows", "4096", "--steps", "2", "--warmup", "3"])
    assert d["gpu_launches"] == 2 * 121
    assert sum(d["config"]["calls_per_step"].values()) == 121
    assert d["config"]["workload"].startswith("dit_forward_mix")
    assert d["roofline"]["launches_per_step"] == 121 and d["value"] > 0
    assert d["e2e"] is None and d["cpu_baseline"] is None
