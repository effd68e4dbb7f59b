"""Benchmark of the fused residual / gate / norm / modulation kernel on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--spec NAME] [--rows L] [--graph | --flush-l2]
                    [--affine-fp32] [--dit-mix] [--no-e2e] [--no-cpu-baseline]
                    [--e2e-steps E] [--cpu-seconds S]

One step = one call of the op over the whole workload (every full tensor read or
written once). Default workload: WAN2.2-shaped LayerNorm, B=1 L=176400 D=5120 bf16,
gate (1,D), per-row scale/shift, no affine weight (the shape the pages' microbenchmark
uses: sglang PR #36349, section "Microbenchmark"). Inputs are seeded synthetic
bf16 values; they are larger than L2 (7.2 GB read per step), so no flush is needed
between steps (the small L=16 workloads can flush L2 before every launch: --flush-l2).

Metric: achieved HBM GB/s, counting the algorithmic bytes (each full tensor once,
broadcast operands once), also reported as rows/s and as a fraction of the measured
HBM copy bandwidth. Multi-GPU: one process per GPU. `python bench.py --gpus N` starts
the N ranks itself (under torch.distributed.run, on 127.0.0.1); started by torchrun
instead, it uses the ranks it is given. Each rank runs its own full-size problem (rows
are independent, nothing is exchanged), value = all ranks' bytes / max-over-ranks time
(weak scaling). With several ranks the pinned host buffers of the end-to-end number are
one copy per node in shared memory (the ranks run the same seeded problem), not one per
rank.

--impl reference times the fp64 CPU oracle (the only other implementation that
exists) on the host cores, on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
import synth.device  # noqa: E402

METRIC = "achieved HBM GB/s (% of B200 peak) and rows/s, fused LN L=176400 D=5120 bf16"
FALLBACK_HBM_GBS = 6650.0
KERNEL = "fused_norm_rows"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=50)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=synth.W4.name, choices=sorted(synth.WORKLOADS))
    p.add_argument("--rows", type=int, default=0, help="override L (profiling a smaller case)")
    p.add_argument("--spec", default="", help="specialisation of the workload (e.g. rms_gate_w); "
                   "default: the workload's first")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--flush-l2", action="store_true",
                   help="write a 512 MB buffer before every timed launch and time each launch "
                        "alone (for the small shapes, whose inputs otherwise stay in L2)")
    p.add_argument("--affine-fp32", action="store_true",
                   help="weight and bias as fp32 (used at full precision), as the pages' "
                        "microbenchmark passes them")
    p.add_argument("--dit-mix", action="store_true",
                   help="one step = the norm calls of one WAN2.2 DiT forward on the pages' "
                        "microbenchmark shape: 41 norm_scale_shift, 40 fused without affine, 40 "
                        "fused with fp32 weight and bias (use with a small --steps)")
    p.add_argument("--graph", action="store_true",
                   help="replay the timed launches from one CUDA graph (removes host launch "
                        "overhead; for the launch-bound small shapes)")
    return p.parse_args()


def pick_spec(w, args):
    if not args.spec:
        return w.specs[0]
    for sp in w.specs:
        if sp.name == args.spec:
            return sp
    raise SystemExit(f"{w.name} has no specialisation {args.spec!r}; "
                     f"choose from {[sp.name for sp in w.specs]}")


def workload(args):
    w = synth.WORKLOADS[args.workload]
    if args.rows:
        F = w.F
        if F and args.rows % F:
            raise SystemExit(f"--rows must be a multiple of {F} for {w.name}")
        w = synth.scaled(w, args.rows)
    return w


def config_dict(w, spec, n, affine_fp32=False):
    lay = {op: w.layout(op) for op in ("gate", "scale", "shift")}
    return {"workload": w.name, "spec": spec.name, "B": w.B, "L": w.L, "D": w.D, "frames": w.F or None,
            "norm": "rms" if spec.is_rms else "layer", "has_gate": spec.has_gate,
            "has_weight": spec.has_weight, "has_bias": spec.has_bias,
            "affine_dtype": ("fp32" if affine_fp32 else "bf16") if (spec.has_weight or spec.has_bias) else None,
            "layouts": lay, "eps": w.eps,
            "parallelism": f"rows per rank, {n} independent problem(s)" if n > 1 else "single GPU",
            "l2": "inputs larger than L2 (no flush needed)" if w.algorithmic_bytes(spec) > 4 * 126e6
                  else "L2-resident (small case)"}


def _code_tokens(src: str) -> str:
    """C/C++ source with comments removed and whitespace runs collapsed (string and
    character literals kept verbatim): what the compiler sees, not how it is annotated."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_digest():
    """sha256 over the kernel sources' code (comments and layout excluded), so that a
    recorded ncu measurement stays attached to the code it was taken on."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "rmsnorm_row_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh", ".h")):
            h.update(name.encode())
            h.update(_code_tokens(open(os.path.join(csrc, name), encoding="utf-8").read()).encode())
    return h.hexdigest()


def recorded_traffic(w, spec):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel source; otherwise None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", text)
    if not m or m.group(1) != kernel_source_digest():
        return None
    m = re.search(rf"^{re.escape(w.name)}\s+traffic_bytes_per_launch:\s*([0-9]+)", text, re.M)
    return int(m.group(1)) if m else None


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def physical_gpus(n_local):
    """nvidia-smi ids of the first n_local visible GPUs (CUDA_VISIBLE_DEVICES may
    renumber or hide devices)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").strip()
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        return ids[:n_local]
    return [str(i) for i in range(n_local)]


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_ids):
        self.lines, self.proc, self.gpu_ids = [], None, gpu_ids

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", ",".join(str(i) for i in self.gpu_ids), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        return self.summary()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ our arm

def run_ours(args):
    import torch
    import torch.distributed as dist

    import rmsnorm_row_b200 as fn

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    if args.dit_mix:   # inputs for all three ops of the mix: fused with fp32 w and b reads them all
        args.workload, args.spec, args.affine_fp32 = "microbench_bcast_B1_L176400_D5120", "ln_gate_w_b", True
        args.no_e2e = args.no_cpu_baseline = True
    w = workload(args)
    spec = pick_spec(w, args)
    bytes_step = w.algorithmic_bytes(spec)
    norm = "rms" if spec.is_rms else "layer"

    # Inputs: generated into pinned host buffers (these are also the e2e host inputs),
    # then copied to the device once. Several ranks share one copy per node.
    bufs = cuda_host_buffers(torch, dist, world, local, dev)
    host = {}
    for name in ("x", "residual", "gate", "scale", "shift", "weight", "bias"):
        if name == "gate" and not spec.has_gate or name == "weight" and not spec.has_weight \
                or name == "bias" and not spec.has_bias \
                or name in ("residual", "gate") and spec.norm_only:
            continue
        if name in ("weight", "bias") and args.affine_fp32:
            t = bufs.get(f"in_{name}", 2 * w.D,
                         lambda a, name=name: a.view(np.float32).__setitem__(slice(None), w.generate_f32(name)))
            host[name] = t.view(torch.float32).view(w.D)
            continue
        n = 1 if name in ("weight", "bias") else w.stored_rows(name)
        t = bufs.get(f"in_{name}", n * w.D, lambda a, name=name: w.generate(name, out=a.reshape(-1, w.D)))
        host[name] = t.view(torch.bfloat16).view(synth.device.operand_view_shape(w, name))
    d = {k: v.to(dev) for k, v in host.items()}
    y = torch.empty((w.B, w.L, w.D), dtype=torch.bfloat16, device=dev)
    r = None if spec.norm_only else torch.empty_like(y)
    stream = torch.cuda.current_stream(dev)

    # The C arguments are marshalled once; each step is one fused_norm_launch call
    # (the tensor-level API marshals the same arguments on every call, which costs
    # ~15 us of host time and dominates the launch-bound small shapes).
    args_c = fn.build_args(d["x"], d.get("residual"), d.get("gate"), d.get("weight"), d.get("bias"),
                           d["scale"], d["shift"], y, r)
    affine_fp32 = bool(args.affine_fp32 and (spec.has_weight or spec.has_bias))
    if affine_fp32:   # fp32 weight / bias: 4 bytes per channel instead of 2
        bytes_step += 2 * w.D * (int(spec.has_weight) + int(spec.has_bias))
    handle = fn.api._handle(w.D, spec.is_rms, spec.has_gate, spec.has_weight, spec.has_bias,
                            spec.norm_only, w.eps, affine_fp32)

    # (handle, C arguments, launches per step); one step launches each of them that often
    calls = [(handle, args_c, 1)]
    mix = None
    if args.dit_mix:
        nss = synth.Spec(False, False, False, norm_only=True)
        fused = synth.Spec(False, True, False)
        h_nss = fn.api._handle(w.D, False, False, False, False, True, w.eps, False)
        h_fused = fn.api._handle(w.D, False, True, False, False, False, w.eps, False)
        a_nss = fn.build_args(d["x"], None, None, None, None, d["scale"], d["shift"], y, None)
        a_fused = fn.build_args(d["x"], d["residual"], d["gate"], None, None, d["scale"], d["shift"], y, r)
        calls = [(h_nss, a_nss, 41), (h_fused, a_fused, 40), (handle, args_c, 40)]
        bytes_step = 41 * w.algorithmic_bytes(nss) + 40 * w.algorithmic_bytes(fused) + 40 * bytes_step
        mix = {"norm_scale_shift (LN, no affine)": 41, "fused (LN, gate, no affine)": 40,
               "fused (LN, gate, fp32 weight and bias)": 40}
    per_step = sum(c[2] for c in calls)

    def step():
        for h_, a_, count in calls:
            for _ in range(count):
                st = fn.fused_norm_launch(h_, a_, int(stream.cuda_stream))
                if st != fn.FN_OK:
                    raise fn.FusedNormError(st, "fused_norm_launch", fn.fused_norm_status_string(st))

    # one call through the tensor-level API first: same result as the prebuilt launch
    if spec.norm_only:
        fn.norm_scale_shift(d["x"], d.get("weight"), d.get("bias"), d["scale"], d["shift"], norm,
                            w.eps, out=y, stream=stream)
    else:
        fn.fused_residual_norm_scale_shift(d["residual"], d["x"], d.get("gate"), d.get("weight"),
                                           d.get("bias"), d["scale"], d["shift"], norm, w.eps,
                                           out=y, residual_out=r, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)

    # rank 0 samples every GPU of this node that the job uses
    local_world = int(os.environ.get("LOCAL_WORLD_SIZE", str(world)))
    sampler = ClockSampler(physical_gpus(local_world)) if rank == 0 else None
    if sampler:
        sampler.start()
        t_end = time.time() + 1.0       # keep the GPU busy while nvidia-smi starts
        while time.time() < t_end:
            step()
        torch.cuda.synchronize(dev)

    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    launches = 0
    graph = None
    if args.graph:
        # capture the K timed launches (no per-step events inside a graph)
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            stream_saved, stream = stream, cap
            with torch.cuda.graph(graph, stream=cap):
                for _ in range(K):
                    step()
            stream = stream_saved
        torch.cuda.synchronize(dev)
        graph.replay()
        torch.cuda.synchronize(dev)
    if args.flush_l2 and graph is not None:
        raise SystemExit("--flush-l2 and --graph are exclusive")
    scratch = torch.empty(128 << 20, dtype=torch.int32, device=dev) if args.flush_l2 else None
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)] if args.flush_l2 else None
    barrier()
    torch.cuda.synchronize(dev)
    ev[0].record(stream)
    if graph is not None:
        with torch.cuda.stream(stream):
            graph.replay()
        launches = K * per_step
        ev[K].record(stream)
    elif scratch is not None:
        for i in range(K):
            scratch.zero_()           # 512 MB written: the inputs leave the 126 MB L2
            starts[i].record(stream)
            step()
            launches += per_step
            ev[i + 1].record(stream)
    else:
        for i in range(K):
            step()
            launches += per_step
            ev[i + 1].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop() if sampler else None
    if graph is not None:
        per = [ev[0].elapsed_time(ev[K]) / K] * K
    elif scratch is not None:
        per = [starts[i].elapsed_time(ev[i + 1]) for i in range(K)]
    else:
        per = [ev[i].elapsed_time(ev[i + 1]) for i in range(K)]
    total_ms = sum(per) if scratch is not None else ev[0].elapsed_time(ev[K])
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms = float(t.item())
    ms_step = total_ms / K

    # e2e: the same op through the public API with host buffers; every step copies
    # its inputs in from pinned memory and its outputs back, in row chunks on three
    # streams so copies in, compute and copies out overlap.
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, spec, host, d, dev, world, local, fn, torch, dist, y, r, bufs)
        e2e["host_buffers"] = bufs.kind

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, spec, host, args.cpu_seconds)

    if rank == 0:
        peak, peak_kind = measured_peak()
        kernel_ms = statistics.mean(per)
        achieved = bytes_step / (kernel_ms * 1e-3) / 1e9
        value = world * bytes_step / (ms_step * 1e-3) / 1e9
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded normal draws, WAN2.2 shapes; no model weights)",
            "config": dict(config_dict(w, spec, world, affine_fp32), launch="cuda_graph" if graph is not None else "stream",
                           **({"workload": f"dit_forward_mix_{w.name}", "calls_per_step": mix,
                               "spec": None} if mix else {}),
                           **({"l2": "flushed before every timed launch (512 MB write, outside the "
                                     "per-launch events)"} if scratch is not None else {})),
            "rows_per_s": round(world * w.rows * per_step / (ms_step * 1e-3), 1),
            "pct_of_peak": round(100.0 * value / world / peak, 2),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                         "peak_kind": f"{peak_kind} (HBM copy bandwidth)", "unit": "GB/s",
                         "frac": round(achieved / peak, 4),
                         "traffic": recorded_traffic(w, spec), "kernel": KERNEL,
                         "algorithmic_bytes_per_launch": bytes_step // per_step if per_step == 1 else None,
                         "algorithmic_bytes_per_step": bytes_step, "launches_per_step": per_step,
                         "kernel_ms_mean": round(kernel_ms, 5),
                         "kernel_ms_median": round(statistics.median(per), 5)},
            "clocks": clocks,
            "gpu_launches": launches,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    bufs.close()
    if world > 1:
        dist.destroy_process_group()


class HostBuffers:
    """Pinned host buffers (int16 elements). One rank: private pinned tensors. Several
    ranks on one node: one copy per node in POSIX shared memory, created and filled by
    local rank 0 and registered as pinned memory by every rank (all ranks run the same
    seeded problem, so they read the same inputs and write the same output bytes).
    Falls back to private buffers when /dev/shm cannot hold them.

    barrier() and all_min(flag) are the job's collectives; pin(ptr, nbytes) -> bool and
    unpin(ptr) register host memory with the GPU driver."""

    def __init__(self, torch, world, local, run_id, barrier, all_min, pin, unpin, shm="/dev/shm"):
        self.torch, self.world, self.local, self.run = torch, world, local, run_id
        self.barrier, self.all_min, self.pin, self.unpin, self.shm = barrier, all_min, pin, unpin, shm
        self.kind = "private pinned (one rank)" if world == 1 else "node-shared pinned"
        self.maps, self.registered, self.paths = [], [], []

    def get(self, tag, n, fill=None):
        torch = self.torch
        if self.world == 1 or not self.kind.startswith("node-shared"):
            t = torch.empty(n, dtype=torch.int16, pin_memory=torch.cuda.is_available())
            if fill is not None:
                fill(t.numpy().view(np.uint16))
            return t
        import mmap
        path = os.path.join(self.shm, f"fused_norm_bench_{self.run}_{tag}")
        nbytes = n * 2
        ok = True
        if self.local == 0:
            try:
                st = os.statvfs(self.shm)
                ok = st.f_bavail * st.f_frsize > nbytes + (256 << 20)
            except OSError:
                ok = False
        if not self.all_min(ok):
            self.kind = "private pinned (shared memory too small for a node-shared copy)"
            return self.get(tag, n, fill)
        if self.local == 0:
            fd = os.open(path, os.O_CREAT | os.O_EXCL | os.O_RDWR, 0o600)
            os.ftruncate(fd, nbytes)
            mm = mmap.mmap(fd, nbytes)
            os.close(fd)
            self.paths.append(path)
            if fill is not None:
                fill(np.frombuffer(mm, dtype=np.uint16))
        self.barrier()
        if self.local != 0:
            fd = os.open(path, os.O_RDWR)
            mm = mmap.mmap(fd, nbytes)
            os.close(fd)
        self.maps.append(mm)
        t = torch.from_numpy(np.frombuffer(mm, dtype=np.int16))
        if self.pin(t.data_ptr(), nbytes):
            self.registered.append(t.data_ptr())
        else:
            self.kind = "node-shared (pinning refused: pageable copies)"
        self.barrier()
        if self.local == 0:
            os.unlink(path)                  # every rank has mapped it; the mappings stay valid
            self.paths.remove(path)
        return t

    def close(self):
        for ptr in self.registered:
            self.unpin(ptr)
        self.registered = []
        for path in self.paths:
            try:
                os.unlink(path)
            except OSError:
                pass


def cuda_host_buffers(torch, dist, world, local, dev):
    """HostBuffers wired to NCCL collectives and cudaHostRegister."""
    def all_min(flag):
        t = torch.tensor([1 if flag else 0], dtype=torch.int32, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MIN)
        return bool(t.item())
    rt = torch.cuda.cudart()
    return HostBuffers(torch, world, local,
                       os.environ.get("TORCHELASTIC_RUN_ID") or os.environ.get("MASTER_PORT", "0"),
                       barrier=lambda: dist.barrier(device_ids=[local]), all_min=all_min,
                       pin=lambda ptr, nbytes: int(rt.cudaHostRegister(ptr, nbytes, 0)) == 0,
                       unpin=lambda ptr: rt.cudaHostUnregister(ptr))


def run_e2e(args, w, spec, host, d, dev, world, local, fn, torch, dist, y_ref=None, r_ref=None, bufs=None):
    norm = "rms" if spec.is_rms else "layer"
    rows = w.rows
    chunk = 4096
    n_out = w.B * w.L * w.D
    hy = bufs.get("out_y", n_out).view(torch.bfloat16).view(w.B, w.L, w.D)
    hr = None if spec.norm_only else bufs.get("out_r", n_out).view(torch.bfloat16).view(w.B, w.L, w.D)
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    dy = torch.empty((w.B, w.L, w.D), dtype=torch.bfloat16, device=dev)
    dr = None if spec.norm_only else torch.empty_like(dy)
    per_row = {k: (w.layout(k) == "row") for k in ("gate", "scale", "shift")}
    flat = lambda t: t.view(-1, w.D)
    h2d_bytes = sum(v.numel() * 2 for v in host.values())
    d2h_bytes = (hy.numel() + (0 if hr is None else hr.numel())) * 2

    n_chunks = (rows + chunk - 1) // chunk
    kernel_done = [None] * n_chunks   # chunk c's kernel of the previous step
    copied_out = [None] * n_chunks    # chunk c's copy-out of the previous step

    def one():
        # broadcast / per-frame operands: one small copy per step (after every kernel
        # of the previous step that reads them)
        with torch.cuda.stream(s_in):
            if kernel_done[-1] is not None:
                s_in.wait_event(kernel_done[-1])
            for k in ("gate", "scale", "shift", "weight", "bias"):
                if k in host and not per_row.get(k, False):
                    d[k].copy_(host[k], non_blocking=True)
        for c, r0 in enumerate(range(0, rows, chunk)):
            r1 = min(rows, r0 + chunk)
            with torch.cuda.stream(s_in):
                if kernel_done[c] is not None:      # inputs of chunk c no longer read
                    s_in.wait_event(kernel_done[c])
                for k in ("x", "residual") + tuple(k for k in ("gate", "scale", "shift") if per_row.get(k)):
                    if k in host:
                        flat(d[k])[r0:r1].copy_(flat(host[k])[r0:r1], non_blocking=True)
                e_in = torch.cuda.Event()
                e_in.record(s_in)
            s_cmp.wait_event(e_in)
            if copied_out[c] is not None:           # outputs of chunk c already on the host
                s_cmp.wait_event(copied_out[c])
            sub = lambda t, k: (flat(t)[r0:r1].view(1, r1 - r0, w.D) if per_row.get(k, True) else t)
            # a chunk of tokens is a (1, n, D) problem when B == 1 and there is no frame axis
            if spec.norm_only:
                fn.norm_scale_shift(
                    sub(d["x"], "x"), d.get("weight"), d.get("bias"), sub(d["scale"], "scale"),
                    sub(d["shift"], "shift"), norm, w.eps,
                    out=flat(dy)[r0:r1].view(1, r1 - r0, w.D), stream=s_cmp)
            else:
                fn.fused_residual_norm_scale_shift(
                    sub(d["residual"], "residual"), sub(d["x"], "x"),
                    sub(d["gate"], "gate") if "gate" in d else None, d.get("weight"), d.get("bias"),
                    sub(d["scale"], "scale"), sub(d["shift"], "shift"), norm, w.eps,
                    out=flat(dy)[r0:r1].view(1, r1 - r0, w.D),
                    residual_out=flat(dr)[r0:r1].view(1, r1 - r0, w.D), stream=s_cmp)
            e_c = torch.cuda.Event()
            e_c.record(s_cmp)
            kernel_done[c] = e_c
            s_out.wait_event(e_c)
            with torch.cuda.stream(s_out):
                flat(hy)[r0:r1].copy_(flat(dy)[r0:r1], non_blocking=True)
                if hr is not None:
                    flat(hr)[r0:r1].copy_(flat(dr)[r0:r1], non_blocking=True)
                e_o = torch.cuda.Event()
                e_o.record(s_out)
            copied_out[c] = e_o

    if w.B != 1 or w.F:
        return {"value": None, "unit": "GB/s", "note": "e2e chunking implemented for B=1 without frames"}
    one()
    torch.cuda.synchronize(dev)
    K = max(1, args.e2e_steps)
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for _ in range(K):
        one()
    # the last step's results must be on the host
    s_in.wait_stream(s_out)
    t1.record(s_in)
    torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1) / K
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item())
    return {"value": round(world * w.algorithmic_bytes(spec) / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(ms, 3), "steps": K, "h2d_bytes_per_step": h2d_bytes,
            "d2h_bytes_per_step": d2h_bytes,
            "verified": _same_rows(torch, w, hy, hr, y_ref, r_ref, chunk),
            "how": "pinned host inputs copied in and outputs copied out every step, 4096-row "
                   "chunks pipelined over copy-in / compute / copy-out streams"}


def _same_rows(torch, w, hy, hr, y_ref, r_ref, chunk):
    """Whether the outputs copied back to the host equal, bit for bit, the device outputs of
    the timed launches (same inputs, deterministic kernel) on sampled rows: the first and
    last row of every 16th chunk, the first and last chunk whole, the middle row. Reports,
    never raises: the check must not cost the benchmark its line."""
    if y_ref is None:
        return None
    try:
        rows = w.rows
        pick = set(range(min(chunk, rows))) | set(range(max(rows - chunk, 0), rows)) | {rows // 2}
        for c0 in range(0, rows, 16 * chunk):
            pick |= {c0, min(rows, c0 + chunk) - 1}
        idx = torch.tensor(sorted(pick), dtype=torch.long)
        pairs = [(hy, y_ref)] + ([(hr, r_ref)] if hr is not None and r_ref is not None else [])
        for host_t, dev_t in pairs:
            a = host_t.view(-1, w.D)[idx].view(torch.int16)
            b = dev_t.view(-1, w.D)[idx.to(dev_t.device)].cpu().view(torch.int16)
            if not torch.equal(a, b):
                return False
        return True
    except Exception as exc:  # reported, not raised
        return f"not checked: {type(exc).__name__}: {exc}"[:200]


# ------------------------------------------------------------------ oracle (CPU)

def _oracle_rows(w, spec, host_np, r0, r1):
    import oracle
    n = r1 - r0
    st = (n * w.D, 0, w.D)
    bst = lambda k: st if w.layout(k) == "row" else (0, 0, 0)
    sl = lambda k: host_np[k][r0:r1] if w.layout(k) == "row" else host_np[k]
    return oracle.fused_norm(1, n, w.D, x=host_np["x"][r0:r1], x_st=st,
                             residual=None if spec.norm_only else host_np["residual"][r0:r1],
                             res_st=None if spec.norm_only else st,
                             gate=sl("gate") if spec.has_gate else None,
                             gate_st=bst("gate") if spec.has_gate else None,
                             weight=host_np.get("weight"), bias=host_np.get("bias"),
                             scale=sl("scale"), scale_st=bst("scale"), shift=sl("shift"),
                             shift_st=bst("shift"), is_rms=spec.is_rms, norm_only=spec.norm_only,
                             eps=w.eps)


def cpu_baseline(w, spec, host, seconds):
    """The oracle, as it stands, on the leading rows of the same inputs until about
    `seconds` of wall time have passed (bounded sample)."""
    import oracle
    if w.B != 1 or w.F:
        return None
    host_np = {k: (v.numpy() if v.dtype == torch_float32() else
                   v.view(torch_int16()).numpy().view(np.uint16).reshape(-1, w.D)) for k, v in host.items()}
    per_row_bytes = w.algorithmic_bytes(spec) / w.rows
    done, t0, chunk = 0, time.time(), 1024
    while time.time() - t0 < seconds and done < w.rows:
        r1 = min(w.rows, done + chunk)
        _oracle_rows(w, spec, host_np, done, r1)
        done = r1
    el = time.time() - t0
    cores = oracle.num_threads()
    # the same oracle on one core, over a 4096-row slice
    n1 = min(4096, w.rows)
    oracle.set_num_threads(1)
    try:
        t1 = time.time()
        _oracle_rows(w, spec, host_np, 0, n1)
        el1 = time.time() - t1
    finally:
        oracle.set_num_threads(cores)
    return {"value": round(done * per_row_bytes / el / 1e9, 4), "unit": "GB/s",
            "rows_per_s": round(done / el, 1), "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"first {done} of {w.rows} rows of the same workload ({el:.1f} s)",
            "one_core": {"value": round(n1 * per_row_bytes / el1 / 1e9, 4), "unit": "GB/s",
                         "rows_per_s": round(n1 / el1, 1), "sample": f"first {n1} rows"}}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def torch_int16():
    import torch
    return torch.int16


def torch_float32():
    import torch
    return torch.float32


def run_reference(args):
    """The fp64 oracle on the host cores, K timed steps of a bounded row sample."""
    import oracle
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    w = workload(args)
    spec = pick_spec(w, args)
    if w.B != 1 or w.F:
        print(json.dumps({"impl": "reference", "unavailable": "reference arm implemented for B=1 workloads"}))
        return
    per_row_bytes = w.algorithmic_bytes(spec) / w.rows
    # size the per-step sample so warm-up + timed steps take about 2 minutes
    budget_s = 120.0
    probe_rows = 512
    names = ["x", "scale", "shift"] + ([] if spec.norm_only else ["residual"]) + \
        (["gate"] if spec.has_gate and not spec.norm_only else []) + \
        (["weight"] if spec.has_weight else []) + (["bias"] if spec.has_bias else [])

    def gen(rows):
        out = {}
        for name in names:
            if name in ("weight", "bias") and args.affine_fp32:
                out[name] = w.generate_f32(name)
                continue
            per_token = name in ("x", "residual") or (name not in ("weight", "bias") and w.layout(name) == "row")
            out[name] = w.generate(name, np.arange(rows if per_token else 1, dtype=np.int64))
        return out

    probe = gen(probe_rows)
    t0 = time.time()
    _oracle_rows(w, spec, probe, 0, probe_rows)
    t_row = (time.time() - t0) / probe_rows
    steps = args.steps + max(args.warmup, 0)
    rows = int(max(64, min(w.rows, budget_s / max(steps, 1) / max(t_row, 1e-9))))
    data = gen(rows)
    for _ in range(args.warmup):
        _oracle_rows(w, spec, data, 0, rows)
    t0 = time.time()
    for _ in range(args.steps):
        _oracle_rows(w, spec, data, 0, rows)
    el = time.time() - t0
    ms = el / max(args.steps, 1) * 1e3
    value = rows * per_row_bytes / (ms * 1e-3) / 1e9
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded normal draws, WAN2.2 shapes)", "impl": "reference",
            "config": config_dict(w, spec, 1, bool(args.affine_fp32 and (spec.has_weight or spec.has_bias))),
            "rows_per_s": round(rows / (ms * 1e-3), 1),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": f"first {rows} of {w.rows} rows per step"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def free_port():
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def launch_ranks(args):
    """`--gpus N` (N > 1) without a torchrun environment: start the N ranks under
    torch.distributed.run on this node and return their exit status. Host-side work
    (generating the node-shared inputs, the CPU legs) runs on local rank 0 alone, so
    every rank keeps the whole host's OpenMP pool."""
    env = dict(os.environ)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1", f"--master-port={free_port()}",
           os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.run(cmd, env=env).returncode


def main():
    args = parse()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(launch_ranks(args))
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
