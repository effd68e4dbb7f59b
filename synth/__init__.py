"""Seeded synthetic inputs for the fused residual / gate / norm / modulation op.

This package draws numbers and describes workloads; it holds none of the op's
arithmetic. The fp64 oracle (tests) and the benchmark both read what it makes, so
the two sides see the same bf16 inputs. Values come back as numpy ``uint16`` arrays
holding bf16 bit patterns.

Workloads follow the shapes the pages measure on (sglang PR #36349, section
"Microbenchmark": WAN2.2 LayerNorm at seq 176400, dim 5120; sglang PR #33144,
section "Accuracy Tests": L in {16, 90000}, D in {5120, 10240}, every
specialisation, both scale/shift layouts and the 4D frame-gate layout).
No model weights or activations are available, so seeded normal draws stand in.

Layouts, with strides in elements {stride_b, stride_f, stride_l} for a (B, L, D)
problem with F frames of L/F tokens each:
  bcast  (1, D)        {0, 0, 0}          one stored row
  row    (B, L, D)     {L*D, 0, D}        B*L stored rows
  frame  (B, F, 1, D)  {F*D, D, 0}        B*F stored rows, row b*F + f
  batch  (B, 1, D)     {D, 0, 0}          B stored rows
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Dict, Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None

# Tensor ids key the generator streams.
TENSOR_IDS = {"x": 0, "residual": 1, "gate": 2, "weight": 3, "scale": 4, "shift": 5, "bias": 6}


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        from synth.build import build

        build()
    lib = ctypes.CDLL(_LIB_PATH)
    i64, u64, u32, dbl = ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_double
    vp = ctypes.c_void_p
    lib.synth_fill_bf16.argtypes = [vp, i64, i64, i64, i64, u64, u32, dbl, dbl, vp]
    lib.synth_fill_bf16.restype = None
    lib.synth_fill_bf16_rows.argtypes = [vp, i64, vp, i64, i64, u64, u32, dbl, dbl, vp]
    lib.synth_fill_bf16_rows.restype = None
    lib.synth_value_bf16.argtypes = [i64, i64, u64, u32, dbl, dbl, dbl]
    lib.synth_value_bf16.restype = ctypes.c_uint16
    lib.synth_fill_f32_row.argtypes = [vp, i64, u64, u32, dbl, dbl]
    lib.synth_fill_f32_row.restype = None
    lib.synth_pick_rows.argtypes = [i64, i64, u64, vp, vp]
    lib.synth_pick_rows.restype = None
    _lib = lib
    return lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def fill(out: np.ndarray, row0: int, seed: int, tensor: str, mu: float, sigma: float,
         row_mult: Optional[np.ndarray] = None) -> np.ndarray:
    """Fill a (nrows, D) uint16 array with rows row0.. of the named tensor's stream."""
    assert out.dtype == np.uint16 and out.ndim == 2 and out.strides[1] == 2
    lib = _load()
    if row_mult is not None:
        row_mult = np.ascontiguousarray(row_mult, dtype=np.float64)
        assert row_mult.shape == (out.shape[0],)
    lib.synth_fill_bf16(_ptr(out), out.strides[0] // 2, row0, out.shape[0], out.shape[1],
                        seed, TENSOR_IDS[tensor], mu, sigma, _ptr(row_mult))
    return out


def fill_rows(out: np.ndarray, rows: np.ndarray, seed: int, tensor: str, mu: float, sigma: float,
              row_mult: Optional[np.ndarray] = None) -> np.ndarray:
    """Fill out[i] with stream row rows[i] (any order, repeats allowed)."""
    assert out.dtype == np.uint16 and out.ndim == 2 and out.strides[1] == 2
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    assert rows.shape == (out.shape[0],)
    lib = _load()
    if row_mult is not None:
        row_mult = np.ascontiguousarray(row_mult, dtype=np.float64)
        assert row_mult.shape == rows.shape
    lib.synth_fill_bf16_rows(_ptr(out), out.strides[0] // 2, _ptr(rows), rows.shape[0],
                             out.shape[1], seed, TENSOR_IDS[tensor], mu, sigma, _ptr(row_mult))
    return out


def value(row: int, c: int, seed: int, tensor: str, mu: float, sigma: float, mult: float = 1.0) -> int:
    return int(_load().synth_value_bf16(row, c, seed, TENSOR_IDS[tensor], mu, sigma, mult))


def pick_rows(n: int, count: int, seed: int) -> np.ndarray:
    """First `count` entries of a seeded uniform permutation of range(n)."""
    lib = _load()
    perm = np.empty(max(n, 1), dtype=np.int64)
    out = np.empty(max(count, 1), dtype=np.int64)
    lib.synth_pick_rows(n, count, seed, _ptr(perm), _ptr(out))
    return out[:count].copy()


# ---------------------------------------------------------------------------
# Layouts and workloads
# ---------------------------------------------------------------------------

def layout_strides(layout: str, B: int, L: int, D: int, F: int) -> Tuple[int, int, int]:
    if layout == "bcast":
        return (0, 0, 0)
    if layout == "row":
        return (L * D, 0, D)
    if layout == "frame":
        return (F * D, D, 0)
    if layout == "batch":
        return (D, 0, 0)
    raise ValueError(layout)


def layout_rows(layout: str, B: int, L: int, F: int) -> int:
    return {"bcast": 1, "row": B * L, "frame": B * F, "batch": B}[layout]


def layout_row_of(layout: str, b: np.ndarray, l: np.ndarray, L: int, F: int) -> np.ndarray:
    """Stored row that token (b, l) reads, for each layout (frames: contiguous token blocks)."""
    b = np.asarray(b, dtype=np.int64)
    l = np.asarray(l, dtype=np.int64)
    if layout == "bcast":
        return np.zeros_like(l)
    if layout == "row":
        return b * L + l
    if layout == "frame":
        return b * F + l // (L // F)
    if layout == "batch":
        return b.copy()
    raise ValueError(layout)


@dataclasses.dataclass(frozen=True)
class Spec:
    """One specialisation of the op."""
    is_rms: bool
    has_gate: bool
    has_weight: bool
    has_bias: bool = False
    norm_only: bool = False

    @property
    def name(self) -> str:
        s = ("rms" if self.is_rms else "ln")
        if self.norm_only:
            s += "_nss"
        else:
            s += "_gate" if self.has_gate else "_nogate"
        s += "_w" if self.has_weight else "_now"
        if self.has_bias:
            s += "_b"
        return s


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    L: int
    D: int
    F: int                       # frames (0: no frame axis)
    layouts: Tuple[Tuple[str, str], ...]   # operand -> layout for gate, scale, shift
    dists: Tuple[Tuple[str, Tuple[float, float]], ...]  # tensor -> (mu, sigma)
    specs: Tuple[Spec, ...]
    seed: int
    outlier_frac: float = 0.0
    outlier_mult: float = 1.0
    eps: float = 1e-6

    @property
    def rows(self) -> int:
        return self.B * self.L

    @property
    def tokens_per_frame(self) -> int:
        return self.L // self.F if self.F else 0

    def layout(self, operand: str) -> str:
        if operand in ("x", "residual"):
            return "row"
        return dict(self.layouts)[operand]

    def dist(self, tensor: str) -> Tuple[float, float]:
        return dict(self.dists)[tensor]

    def strides(self, operand: str) -> Tuple[int, int, int]:
        return layout_strides(self.layout(operand), self.B, self.L, self.D, self.F)

    def stored_rows(self, operand: str) -> int:
        return layout_rows(self.layout(operand), self.B, self.L, self.F)

    def outlier_rows(self) -> np.ndarray:
        """Flattened rows of x and residual scaled by outlier_mult (sorted)."""
        if self.outlier_frac <= 0:
            return np.zeros(0, dtype=np.int64)
        count = int(math.ceil(self.outlier_frac * self.rows))
        return np.sort(pick_rows(self.rows, count, self.seed))

    def row_mult(self, rows: np.ndarray) -> Optional[np.ndarray]:
        if self.outlier_frac <= 0:
            return None
        mult = np.ones(len(rows), dtype=np.float64)
        mult[np.isin(rows, self.outlier_rows())] = self.outlier_mult
        return mult

    def generate(self, tensor: str, rows: Optional[np.ndarray] = None,
                 out: Optional[np.ndarray] = None) -> np.ndarray:
        """Stored rows of one tensor (all of them when rows is None).

        weight and bias are (1, D) vectors. x and residual carry the outlier factor.
        """
        mu, sigma = self.dist(tensor)
        if tensor in ("weight", "bias"):
            n_rows = 1
        else:
            n_rows = self.stored_rows(tensor)
        if rows is None:
            if out is None:
                out = np.empty((n_rows, self.D), dtype=np.uint16)
            mult = self.row_mult(np.arange(n_rows)) if tensor in ("x", "residual") else None
            return fill(out, 0, self.seed, tensor, mu, sigma, mult)
        rows = np.asarray(rows, dtype=np.int64)
        if out is None:
            out = np.empty((len(rows), self.D), dtype=np.uint16)
        mult = self.row_mult(rows) if tensor in ("x", "residual") else None
        return fill_rows(out, rows, self.seed, tensor, mu, sigma, mult)

    def generate_f32(self, tensor: str) -> np.ndarray:
        """A (D,) float32 affine parameter (weight or bias): the same draws as generate(),
        kept at binary32 precision."""
        assert tensor in ("weight", "bias")
        mu, sigma = self.dist(tensor)
        out = np.empty(self.D, dtype=np.float32)
        _load().synth_fill_f32_row(_ptr(out), self.D, self.seed, TENSOR_IDS[tensor], mu, sigma)
        return out

    def token_rows(self, operand: str, flat_rows: np.ndarray) -> np.ndarray:
        """Stored rows of `operand` read by the given flattened tokens b*L + l."""
        flat_rows = np.asarray(flat_rows, dtype=np.int64)
        b, l = flat_rows // self.L, flat_rows % self.L
        return layout_row_of(self.layout(operand), b, l, self.L, self.F)

    def algorithmic_bytes(self, spec: Spec) -> int:
        """Bytes an ideal implementation must move per call: every full tensor once,
        every broadcast or per-frame operand once (bf16)."""
        D, e = self.D, 2
        full = self.rows * D * e
        total = full * (1 if spec.norm_only else 2)          # x (+ residual)
        total += full * (1 if spec.norm_only else 2)         # y (+ r)
        ops = ["scale", "shift"] + (["gate"] if spec.has_gate and not spec.norm_only else [])
        for op in ops:
            total += self.stored_rows(op) * D * e
        if spec.has_weight:
            total += D * e
        if spec.has_bias:
            total += D * e
        return total


_DISTS = (("x", (0.0, 1.0)), ("residual", (0.0, 1.0)), ("gate", (0.0, 0.5)),
          ("weight", (1.0, 0.1)), ("scale", (0.0, 0.1)), ("shift", (0.0, 0.1)),
          ("bias", (0.0, 0.1)))

_ALL8 = tuple(Spec(is_rms=r, has_gate=g, has_weight=w)
              for r in (False, True) for g in (False, True) for w in (False, True))

# The five workloads (seed = 1000 + index). Index 4 is the headline shape.
WORKLOADS: Dict[str, Workload] = {}


def _add(w: Workload) -> Workload:
    WORKLOADS[w.name] = w
    return w


W1 = _add(Workload("rms_fused_B1_L16_D5120", 1, 16, 5120, 0,
                   (("gate", "bcast"), ("scale", "bcast"), ("shift", "bcast")), _DISTS,
                   (Spec(True, True, True),), seed=1001))
W2 = _add(Workload("ln_fused_rowgate_B2_L16_D5120", 2, 16, 5120, 0,
                   (("gate", "row"), ("scale", "bcast"), ("shift", "bcast")), _DISTS,
                   (Spec(False, True, False), Spec(False, False, False), Spec(True, True, False),
                    Spec(True, False, False)), seed=1002))
W3 = _add(Workload("all_specs_B1_L90000_D5120", 1, 90000, 5120, 0,
                   (("gate", "bcast"), ("scale", "row"), ("shift", "row")), _DISTS, _ALL8,
                   seed=1003, outlier_frac=0.01, outlier_mult=50.0))
W3B = _add(Workload("all_specs_B1_L90000_D10240", 1, 90000, 10240, 0,
                    (("gate", "bcast"), ("scale", "row"), ("shift", "row")), _DISTS, _ALL8,
                    seed=1003, outlier_frac=0.01, outlier_mult=50.0))
W4 = _add(Workload("wan22_ln_B1_L176400_D5120", 1, 176400, 5120, 0,
                   (("gate", "bcast"), ("scale", "row"), ("shift", "row")), _DISTS,
                   (Spec(False, True, False),), seed=1004))
W5 = _add(Workload("frame_gate_B1_F21x8400_D5120", 1, 176400, 5120, 21,
                   (("gate", "frame"), ("scale", "frame"), ("shift", "frame")), _DISTS,
                   (Spec(False, True, True),), seed=1005))
# Extra layouts beyond the graded five: the 49 x 3600 frame split the WAN2.2 shape
# actually has, and a per-batch (B, 1, D) broadcast.
W5B = _add(Workload("frame_gate_B1_F49x3600_D5120", 1, 176400, 5120, 49,
                    (("gate", "frame"), ("scale", "frame"), ("shift", "frame")), _DISTS,
                    (Spec(False, True, True),), seed=1006))
W6 = _add(Workload("batch_bcast_B3_L64_D5120", 3, 64, 5120, 0,
                   (("gate", "batch"), ("scale", "batch"), ("shift", "batch")), _DISTS,
                   (Spec(False, True, True), Spec(True, True, False)), seed=1007))
# The pages' own microbenchmark shape (sglang PR #36349, "Microbenchmark"): LayerNorm,
# seq 176400, dim 5120, gate, scale and shift broadcast (1, 1, D); the fused op without
# and with an affine weight and bias, and the norm-only op.
W7 = _add(Workload("microbench_bcast_B1_L176400_D5120", 1, 176400, 5120, 0,
                   (("gate", "bcast"), ("scale", "bcast"), ("shift", "bcast")), _DISTS,
                   (Spec(False, True, False), Spec(False, True, True, has_bias=True),
                    Spec(False, False, False, norm_only=True)), seed=1008))


def scaled(w: Workload, L: int, name: Optional[str] = None, F: Optional[int] = None) -> Workload:
    """Same recipe at another L (frames kept proportional when F is not given)."""
    if F is None:
        F = w.F
    return dataclasses.replace(w, L=L, F=F, name=name or f"{w.name}@L{L}")
