"""Multi-process row sharding on the CPU (gloo, world size 2).

Rows are independent, so a problem split across ranks by rows_shards / shard_args
must give, row for row, exactly the result of the unsplit problem. Each rank here
runs its shard through the oracle (addresses in the shard arguments are byte offsets
into host buffers), rank 0 gathers the pieces and compares them with the whole
problem bitwise. The shard arguments also pass the library's host-side validation.
The benchmark's max-over-ranks timing reduction is exercised the same way.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

LAYOUTS = ["bcast", "row", "frame", "batch"]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _problem(B, L, D, F, layout, seed):
    import synth
    rng = np.random.default_rng(seed)
    from helpers import f32_to_bf16_bits_rne

    def rnd(n, sd=1.0):
        return f32_to_bf16_bits_rne((sd * rng.normal(size=(n, D))).astype(np.float32)).reshape(-1)

    n_op = synth.layout_rows(layout, B, L, F)
    bufs = {"x": rnd(B * L), "residual": rnd(B * L), "gate": rnd(n_op, .5), "scale": rnd(n_op, .1),
            "shift": rnd(n_op, .1), "weight": rnd(1, .1) + 0}
    st = synth.layout_strides(layout, B, L, D, F)
    return bufs, st


def _args_for(B, L, D, F, st, with_bases):
    """fn_args whose pointers are byte offsets from per-buffer bases."""
    import rmsnorm_row_b200 as fn
    a = fn.fn_args()
    a.B, a.L, a.tokens_per_frame = B, L, (L // F if F else 0)
    base = with_bases
    row = (L * D, 0, D)
    a.x = fn.fn_operand(base["x"], *row)
    a.residual = fn.fn_operand(base["residual"], *row)
    a.gate = fn.fn_operand(base["gate"], *st)
    a.scale = fn.fn_operand(base["scale"], *st)
    a.shift = fn.fn_operand(base["shift"], *st)
    a.weight = base["weight"]
    a.y, a.y_stride_b, a.y_stride_l = base["y"], L * D, D
    a.r, a.r_stride_b, a.r_stride_l = base["r"], L * D, D
    return a


def _run_oracle_on(a, bufs, bases, D):
    """Oracle call on host buffers addressed like `a` (byte offsets from `bases`)."""
    import oracle
    off = lambda name, ptr: (ptr - bases[name]) // 2
    def view(name, o):
        return bufs[name][off(name, o.ptr):]
    res = oracle.fused_norm(
        a.B, a.L, D, x=view("x", a.x), x_st=(a.x.stride_b, a.x.stride_f, a.x.stride_l),
        residual=view("residual", a.residual),
        res_st=(a.residual.stride_b, a.residual.stride_f, a.residual.stride_l),
        gate=view("gate", a.gate), gate_st=(a.gate.stride_b, a.gate.stride_f, a.gate.stride_l),
        weight=bufs["weight"], scale=view("scale", a.scale),
        scale_st=(a.scale.stride_b, a.scale.stride_f, a.scale.stride_l),
        shift=view("shift", a.shift), shift_st=(a.shift.stride_b, a.shift.stride_f, a.shift.stride_l),
        tokens_per_frame=a.tokens_per_frame)
    return res


def _worker(rank, world, port, B, L, D, F, q):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), OMP_NUM_THREADS="2")
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        for layout in LAYOUTS:
            # token splits need not align to frames without a frame axis
            _one_layout(rank, world, layout, B, L, D, F if layout == "frame" else 0, q)
    finally:
        dist.destroy_process_group()


def _one_layout(rank, world, layout, B, L, D, F, q):
    if True:
        import rmsnorm_row_b200 as fn
        from rmsnorm_row_b200.shard import shard_args
        bufs, st = _problem(B, L, D, F, layout, seed=7)
        GB = 1 << 34
        bases = {k: (i + 1) * GB for i, k in enumerate(["x", "residual", "gate", "scale", "shift",
                                                          "weight", "y", "r"])}
        full = _args_for(B, L, D, F, st, bases)
        mine = shard_args(full, world, rank)
        # the library takes D in {5120, 10240}: validate the same split at D = 5120
        import synth
        Dk = 5120
        st_k = synth.layout_strides(layout, B, L, Dk, F)
        _, h = fn.fused_norm_create(fn.fn_config(D=Dk, has_gate=1, has_weight=1, eps=1e-6))
        ok_valid = fn.fused_norm_validate(h, shard_args(_args_for(B, L, Dk, F, st_k, bases),
                                                        world, rank)) == fn.FN_OK
        part = _run_oracle_on(mine, bufs, bases, D)
        y_off = (mine.y - bases["y"]) // 2
        payload = torch.from_numpy(np.concatenate([part["y"].reshape(-1), part["r"].reshape(-1)]).astype(np.int32))
        meta = torch.tensor([y_off, mine.B, mine.L, int(ok_valid)], dtype=torch.int64)
        metas = [torch.zeros(4, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(metas, meta)
        n_max = torch.tensor([payload.numel()], dtype=torch.int64)
        dist.all_reduce(n_max, op=dist.ReduceOp.MAX)
        padded = torch.zeros(int(n_max.item()), dtype=torch.int32)
        padded[:payload.numel()] = payload
        outs = [torch.zeros_like(padded) for _ in range(world)]
        dist.all_gather(outs, padded)
        # max-over-ranks timing reduction, as in the benchmark
        t = torch.tensor([float(rank + 1)], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            whole = _run_oracle_on(full, bufs, bases, D)
            y_all = np.full(B * L * D, -1, dtype=np.int64)
            r_all = np.full(B * L * D, -1, dtype=np.int64)
            for m, o in zip(metas, outs):
                yo, b, l = int(m[0]), int(m[1]), int(m[2])
                n = b * l * D
                y_p, r_p = o[:n].numpy().reshape(b, l, D), o[n:].numpy().reshape(b, l, D)
                for bi in range(b):
                    for li in range(l):
                        dst = yo + bi * L * D + li * D
                        y_all[dst:dst + D] = y_p[bi, li]
                        r_all[dst:dst + D] = r_p[bi, li]
            same = (np.array_equal(y_all, whole["y"].reshape(-1).astype(np.int64)) and
                    np.array_equal(r_all, whole["r"].reshape(-1).astype(np.int64)))
            q.put((layout, same, all(int(m[3]) for m in metas), float(t.item())))


@pytest.mark.parametrize("B,L,F", [(2, 24, 3), (1, 24, 6), (3, 12, 2)])
def test_row_sharding_world2_matches_whole(B, L, F):
    world, D = 2, 64
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, B, L, D, F, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for _ in LAYOUTS:
        layout, same, valid, tmax = q.get(timeout=10)
        assert same, f"{layout}: sharded result differs from the whole problem"
        assert valid, f"{layout}: a shard failed host-side validation"
        assert tmax == float(world)


def test_row_shards_cover_rows_and_respect_frames():
    from rmsnorm_row_b200.shard import row_shards
    assert row_shards(4, 10, 2) == [(0, 2, 0, 10), (2, 4, 0, 10)]
    assert row_shards(1, 176400, 8, 8400)[0] == (0, 1, 0, 16800)
    for (B, L, W, T) in [(1, 176400, 8, 8400), (3, 100, 4, 0), (1, 7, 3, 0), (2, 49 * 3600, 8, 3600)]:
        sh = row_shards(B, L, W, T)
        assert len(sh) == W
        covered = sum((b1 - b0) * (l1 - l0) for b0, b1, l0, l1 in sh)
        assert covered == B * L
        if T:
            assert all(l0 % T == 0 and l1 % T == 0 for _, _, l0, l1 in sh)
