"""Row sharding of one problem across ranks (one process per GPU).

Every row of the op is independent (its statistics are taken over its own D
channels), so splitting the B*L rows across GPUs is exact and needs no exchange:
each rank launches the same kernel on its slice, with offset pointers. Broadcast,
per-batch and per-frame operands are read, not split, except that an offset along
the token or batch axis moves their pointers too.

Shards are whole batches when the batch count divides evenly across ranks,
otherwise token ranges [l0, l1) of every batch; with a frame axis, token ranges
start and end on frame boundaries, so each shard's frames are whole and its
tokens_per_frame is unchanged.
"""
from __future__ import annotations

from typing import List, Tuple

from . import _abi


def row_shards(B: int, L: int, world: int, tokens_per_frame: int = 0) -> List[Tuple[int, int, int, int]]:
    """(b0, b1, l0, l1) for each rank: batches [b0, b1) x tokens [l0, l1)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    if B % world == 0 and B >= world:
        per = B // world
        return [(r * per, (r + 1) * per, 0, L) for r in range(world)]
    unit = tokens_per_frame if tokens_per_frame > 0 else 1
    if L % unit:
        raise ValueError("tokens_per_frame must divide L")
    units = L // unit
    out = []
    for r in range(world):
        u0 = (units * r) // world
        u1 = (units * (r + 1)) // world
        out.append((0, B, u0 * unit, u1 * unit))
    return out


def _offset_operand(o: _abi.fn_operand, b0: int, l0: int, tpf: int) -> _abi.fn_operand:
    if not o.ptr:
        return _abi.fn_operand(None, o.stride_b, o.stride_f, o.stride_l)
    f0 = l0 // tpf if tpf > 0 else 0
    elems = b0 * o.stride_b + f0 * o.stride_f + l0 * o.stride_l
    return _abi.fn_operand(o.ptr + 2 * elems, o.stride_b, o.stride_f, o.stride_l)


def shard_args(a: _abi.fn_args, world: int, rank: int) -> _abi.fn_args:
    """fn_args of this rank's shard of the problem `a` (pointers offset, sizes cut)."""
    b0, b1, l0, l1 = row_shards(a.B, a.L, world, a.tokens_per_frame)[rank]
    s = _abi.fn_args.from_buffer_copy(a)
    s.B, s.L = b1 - b0, l1 - l0
    tpf = a.tokens_per_frame
    for name in ("x", "residual", "gate", "scale", "shift"):
        setattr(s, name, _offset_operand(getattr(a, name), b0, l0, tpf))
    if a.y:
        s.y = a.y + 2 * (b0 * a.y_stride_b + l0 * a.y_stride_l)
    if a.r:
        s.r = a.r + 2 * (b0 * a.r_stride_b + l0 * a.r_stride_l)
    return s
