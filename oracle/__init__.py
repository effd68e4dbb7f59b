"""fp64 CPU oracle for the fused residual / gate / norm / modulation row op.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package. The GPU library never
loads it and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, one OpenMP loop over rows);
this module only marshals numpy arrays to it. Arrays hold bf16 bit patterns as
``uint16``. What the oracle computes, and the pages it follows, is stated in the
header of ``oracle.c``: sglang PR #36349 "[AMD][Diffusion] Migrate FlyDSL fused
norm kernels to the v0.3.0 stable API" (section "Microbenchmark") and sglang PR
#33144 (sections "Modifications", "Accuracy Tests" and "Known gaps").

Every function here is pinned by the CPU tests in ``tests/test_oracle_pins.py``
(closed forms, invariants, exact high-precision brute force on tiny rows, and
torch's CPU layer_norm / rms_norm as a library special case).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# ORACLE_LIB names another build of oracle.c; the mutation tests use it to load
# copies with planted mistakes and check that the pins catch them.
_LIB_PATH = os.environ.get("ORACLE_LIB") or os.path.join(_HERE, "liboracle.so")
_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        from oracle.build import build

        build()
    lib = ctypes.CDLL(_LIB_PATH)
    i64, dbl, vp = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_double.restype = dbl
    lib.oracle_bf16_rne.argtypes = [dbl]
    lib.oracle_bf16_rne.restype = ctypes.c_uint16
    lib.oracle_fused_norm.argtypes = [i64, i64, i64, i64, ctypes.c_int, ctypes.c_int, dbl] + [vp] * 20
    lib.oracle_fused_norm.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
    lib.oracle_set_num_threads.restype = None
    _lib = lib
    return lib


def bf16_rne(v: float) -> int:
    """fp64 value -> bf16 bit pattern, round to nearest even (single rounding)."""
    return int(_load().oracle_bf16_rne(float(v)))


def bf16_to_double(bits: int) -> float:
    return float(_load().oracle_bf16_to_double(int(bits) & 0xFFFF))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads for the row loop of later calls (OpenMP)."""
    _load().oracle_set_num_threads(int(n))


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _st(st: Optional[Sequence[int]], n: int = 3):
    if st is None:
        return None
    a = np.asarray(list(st), dtype=np.int64)
    assert a.shape == (n,)
    return a


def _bf16_array(a):
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _f32_array(a):
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    assert a.dtype == np.float32, a.dtype
    return a


def fused_norm(B: int, L: int, D: int, *, x, x_st, scale, scale_st, shift, shift_st,
               residual=None, res_st=None, gate=None, gate_st=None, weight=None, bias=None,
               is_rms: bool = False, norm_only: bool = False, eps: float = 1e-6,
               tokens_per_frame: int = 0, want_n: bool = False, want_stats: bool = False):
    """Run the oracle over all B*L rows.

    Operand arrays are flat-indexable uint16 buffers addressed with strides
    {stride_b, stride_f, stride_l} in elements (0 = broadcast). weight and bias are
    (D,) uint16 bf16 bit patterns or (D,) float32 arrays. Returns a dict with
    ``y`` (B, L, D) uint16, ``r`` (B, L, D) uint16 or None, and optionally ``n``
    (B, L, D) float64 (the normalised value before the affine step) and ``stats``
    (B*L, 3) float64 (mean or 0, variance or mean-square, 1/sqrt(. + eps)).
    """
    lib = _load()
    x, residual, gate = _bf16_array(x), _bf16_array(residual), _bf16_array(gate)
    w16 = _bf16_array(weight) if weight is not None and np.asarray(weight).dtype == np.uint16 else None
    b16 = _bf16_array(bias) if bias is not None and np.asarray(bias).dtype == np.uint16 else None
    w32 = _f32_array(weight) if weight is not None and w16 is None else None
    b32 = _f32_array(bias) if bias is not None and b16 is None else None
    scale, shift = _bf16_array(scale), _bf16_array(shift)
    y = np.empty((B, L, D), dtype=np.uint16)
    r = None if norm_only else np.empty((B, L, D), dtype=np.uint16)
    out_st = np.asarray([L * D, D], dtype=np.int64)
    n = np.empty((B, L, D), dtype=np.float64) if want_n else None
    stats = np.empty((B * L, 3), dtype=np.float64) if want_stats else None
    zero3 = np.zeros(3, dtype=np.int64)
    keep = [_st(x_st), _st(res_st) if res_st is not None else zero3,
            _st(gate_st) if gate_st is not None else zero3, _st(scale_st), _st(shift_st)]
    rc = lib.oracle_fused_norm(
        B, L, D, tokens_per_frame, int(bool(is_rms)), int(bool(norm_only)), float(eps),
        _p(x), _p(keep[0]), _p(residual), _p(keep[1]), _p(gate), _p(keep[2]),
        _p(w16), _p(b16), _p(w32), _p(b32), _p(scale), _p(keep[3]), _p(shift), _p(keep[4]),
        _p(y), _p(out_st), _p(r), _p(out_st), _p(n), _p(stats))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return {"y": y, "r": r, "n": n, "stats": stats}


def run_workload_rows(w, spec, flat_rows: np.ndarray, *, want_n: bool = False,
                      want_stats: bool = False):
    """Oracle outputs for selected tokens of a synthetic workload.

    The tokens' operand rows are drawn from the seeded generator and laid out as a
    compact per-row problem (B=1, L=len(flat_rows)); broadcast, per-batch and
    per-frame operands are gathered by the generator's own layout recipe. The
    arithmetic is the oracle's, unchanged.
    """
    flat_rows = np.asarray(flat_rows, dtype=np.int64)
    n_tok, D = len(flat_rows), w.D
    row_st = (n_tok * D, 0, D)

    def gather(op):
        return w.generate(op, w.token_rows(op, flat_rows))

    x = w.generate("x", flat_rows)
    residual = None if spec.norm_only else w.generate("residual", flat_rows)
    gate = gather("gate") if (spec.has_gate and not spec.norm_only) else None
    weight = w.generate("weight", np.zeros(1, dtype=np.int64)) if spec.has_weight else None
    bias = w.generate("bias", np.zeros(1, dtype=np.int64)) if spec.has_bias else None
    return fused_norm(
        1, n_tok, D, x=x, x_st=row_st, residual=residual,
        res_st=row_st if residual is not None else None, gate=gate,
        gate_st=row_st if gate is not None else None, weight=weight, bias=bias,
        scale=gather("scale"), scale_st=row_st, shift=gather("shift"), shift_st=row_st,
        is_rms=spec.is_rms, norm_only=spec.norm_only, eps=w.eps, want_n=want_n,
        want_stats=want_stats)
