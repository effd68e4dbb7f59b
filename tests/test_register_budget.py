"""Register budget of the hot kernel instances (host-only: nvcc and ptxas, no GPU).

A spill in the row kernel puts local-memory traffic on every element: an earlier layout
spilled 116 bytes in the WAN2.2-shaped instance and cost ~6% there. This test compiles the
instances the measured workloads use, in one small translation unit, and checks with
`-Xptxas -v` that none of them spills and that each fits the register share its CTA count
per SM allows.
"""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "rmsnorm_row_b200", "csrc")

# (D, IS_RMS, NORM_ONLY, HAS_GATE, HAS_WEIGHT, HAS_BIAS, AFFINE_F32, CACHED_MOD, label)
INSTANCES = [
    (5120, 0, 0, 1, 0, 0, 0, 0, "WAN2.2 LN, per-row scale/shift"),
    (5120, 0, 0, 1, 1, 0, 0, 0, "LN gate weight, per-row scale/shift"),
    (5120, 1, 0, 1, 1, 0, 0, 0, "RMS gate weight, per-row scale/shift"),
    (5120, 0, 0, 1, 1, 0, 0, 1, "frame gate: LN gate weight, per-frame scale/shift"),
    (5120, 0, 1, 0, 0, 0, 0, 1, "norm-only LN, broadcast scale/shift"),
    (10240, 0, 0, 1, 0, 0, 0, 0, "D=10240 LN gate, per-row scale/shift"),
    (10240, 1, 0, 0, 1, 0, 0, 0, "D=10240 RMS weight, per-row scale/shift"),
    (10240, 0, 1, 0, 0, 0, 0, 1, "D=10240 norm-only LN, broadcast scale/shift"),
]


def _b(v):
    return "true" if v else "false"


def _source():
    lines = ['#include "fused_norm_kernel.cuh"', "namespace fused_norm_impl {"]
    for D, rms, no, g, w, b, f32, cm, _ in INSTANCES:
        vpt = f"vpt_of<{D}>({_b(no)}, {_b(cm)}, {_b(w or b)})"
        lines.append(f"template cudaError_t launch_rows<{D}, {vpt}, {_b(rms)}, {_b(no)}, "
                     f"{_b(g)}, {_b(w)}, {_b(b)}, {_b(f32)}, {_b(cm)}>(const RowParams&, int64_t, "
                     f"cudaStream_t);")
    lines.append("}")
    return "\n".join(lines) + "\n"


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc")
def test_hot_instances_do_not_spill(tmp_path):
    src = tmp_path / "budget.cu"
    src.write_text(_source())
    out = subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                          "--expt-relaxed-constexpr", "-Xptxas", "-v", "-I", CSRC,
                          "-I", os.path.join(ROOT, "include"), "-c", str(src), "-o",
                          str(tmp_path / "budget.o")], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    report = {}
    current = None
    for line in out.stderr.splitlines():
        m = re.search(r"Compiling entry function '_ZN15fused_norm_impl15fused_norm_rowsILi(\d+)ELi(\d+)E"
                      r"((?:Lb[01]E)+)", line)
        if m:
            current = (int(m.group(1)), int(m.group(2)), tuple(int(c) for c in re.findall(r"Lb([01])E", m.group(3))))
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and current:
            report.setdefault(current, {})["spill"] = int(m.group(1)) + int(m.group(2))
        m = re.search(r"Used (\d+) registers", line)
        if m and current:
            report.setdefault(current, {})["regs"] = int(m.group(1))
            current = None
    assert len(report) == len(INSTANCES), sorted(report)
    for (D, vpt, flags), r in report.items():
        label = next(i[-1] for i in INSTANCES if (i[0],) + tuple(i[1:8]) == (D,) + flags)
        cached = flags[-1]
        threads = D // (8 * vpt)
        norm_only = flags[1]
        min_blocks = {(5120, 0): 5, (5120, 1): 6, (10240, 0): 2, (10240, 1): 3}[(D, cached)]
        if norm_only and cached:
            min_blocks = {5120: 12, 10240: 6}[D]
        assert r["spill"] == 0, f"{label}: {r['spill']} bytes of spills"
        assert r["regs"] * threads * min_blocks <= 65536, f"{label}: {r['regs']} registers"
