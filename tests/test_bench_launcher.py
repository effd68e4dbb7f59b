"""bench.py with several ranks, on the CPU: the self-launch of `--gpus N` and the
node-shared host buffers (gloo ranks stand in for the NCCL ones; pinning is a no-op).
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_launches_its_own_ranks():
    # plain `python bench.py --gpus 2` (no torchrun environment): bench starts the two
    # ranks itself; rank 0 alone prints the one JSON line, the other exits 0
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "2", "--warmup", "1", "--rows", "512"],
                         cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, shm, outdir):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)

    def all_min(flag):
        t = torch.tensor([1 if flag else 0], dtype=torch.int32)
        dist.all_reduce(t, op=dist.ReduceOp.MIN)
        return bool(t.item())

    pinned = []
    bufs = bench.HostBuffers(torch, world, rank, f"t{port}", barrier=dist.barrier, all_min=all_min,
                             pin=lambda p, n: pinned.append((p, n)) or True, unpin=lambda p: None,
                             shm=shm)
    n = 4096

    def fill(a):
        a[:] = np.arange(n, dtype=np.uint16) * 7

    inp = bufs.get("in_x", n, fill)
    out = bufs.get("out_y", n)
    dist.barrier()                                            # rank 0 has unlinked the names
    leftovers = [f for f in os.listdir(shm) if f.startswith(f"fused_norm_bench_t{port}")] \
        if os.path.isdir(shm) else []
    if rank == 1:
        out[:] = torch.arange(n, dtype=torch.int16) * 3     # written by one rank ...
    dist.barrier()
    seen_out = out.numpy().copy()                             # ... seen by every rank
    res = {"kind": bufs.kind, "inp_ok": bool(np.array_equal(inp.numpy().view(np.uint16),
                                                             np.arange(n, dtype=np.uint16) * 7)),
           "out_ok": bool(np.array_equal(seen_out, np.arange(n, dtype=np.int16) * 3)),
           "pinned": len(pinned), "leftovers": leftovers}
    bufs.close()
    with open(os.path.join(outdir, f"r{rank}.json"), "w") as f:
        json.dump(res, f)
    dist.destroy_process_group()


def _run(shm, tmp_path):
    world = 2
    mp.start_processes(_rank, args=(world, _free_port(), shm, str(tmp_path)), nprocs=world,
                       start_method="spawn")
    return [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]


def test_node_shared_host_buffers(tmp_path):
    shm = tmp_path / "shm"
    shm.mkdir()
    for r in _run(str(shm), tmp_path):
        assert r["kind"] == "node-shared pinned"
        assert r["inp_ok"] and r["out_ok"], r       # one copy: filled once, written once
        assert r["pinned"] == 2                     # every rank registers both buffers
        assert r["leftovers"] == []                 # names unlinked once every rank mapped them
    assert os.listdir(shm) == []


def test_private_buffers_when_shared_memory_is_unusable(tmp_path):
    res = _run(str(tmp_path / "missing"), tmp_path)
    for r in res:
        assert r["kind"].startswith("private pinned"), r
        assert r["inp_ok"] and r["pinned"] == 0
    # private copies: rank 1's write lands in its own buffer only
    assert res[1]["out_ok"] and not res[0]["out_ok"]
