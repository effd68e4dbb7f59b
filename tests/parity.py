"""GPU-versus-oracle comparison helpers for the parity tests.

Pass criterion, per output tensor (y and r, bf16): at least 99.99% of elements within
1 ulp of the oracle's bf16 value (ulp distance = difference of the order-preserving
integer images of the two bit patterns, +0 == -0), and max |gpu - oracle| <= 2e-2.
The kernel's r is the correctly rounded exact residual + gate * x, as is the
oracle's, so r is required to match bit for bit.
"""
from __future__ import annotations

import dataclasses
from typing import Dict

import numpy as np
import torch

import oracle
import rmsnorm_row_b200 as fn
import synth
from synth.device import to_bits, upload
from helpers import bf16_bits_to_f64, ulp_distance

ULP_FRAC = 0.9999
MAX_ABS = 2e-2


@dataclasses.dataclass
class Tally:
    n: int = 0
    hist: Dict[int, int] = dataclasses.field(default_factory=dict)
    max_abs: float = 0.0
    exact: int = 0

    def add(self, gpu: np.ndarray, ref: np.ndarray):
        d = ulp_distance(gpu, ref).ravel()
        vals, counts = np.unique(np.minimum(d, 1000), return_counts=True)
        for v, c in zip(vals.tolist(), counts.tolist()):
            self.hist[v] = self.hist.get(v, 0) + c
        self.n += d.size
        self.exact += int(np.count_nonzero(d == 0))
        diff = np.abs(bf16_bits_to_f64(gpu) - bf16_bits_to_f64(ref))
        if diff.size:
            self.max_abs = max(self.max_abs, float(np.nanmax(diff)))

    @property
    def within1(self) -> float:
        return (self.hist.get(0, 0) + self.hist.get(1, 0)) / max(self.n, 1)

    def ok(self) -> bool:
        return self.within1 >= ULP_FRAC and self.max_abs <= MAX_ABS

    def __str__(self):
        return (f"n={self.n} exact={self.exact / max(self.n, 1):.6f} within1={self.within1:.6f} "
                f"max_abs={self.max_abs:.3g} hist={dict(sorted(self.hist.items()))}")


def run_gpu(w: synth.Workload, spec: synth.Spec, dev: Dict[str, torch.Tensor], *, out=None,
            residual_out=None):
    """One call through the binding (and so through the C ABI)."""
    norm = "rms" if spec.is_rms else "layer"
    weight = dev["weight"] if spec.has_weight else None
    bias = dev["bias"] if spec.has_bias else None
    if spec.norm_only:
        y = fn.norm_scale_shift(dev["x"], weight, bias, dev["scale"], dev["shift"], norm, w.eps,
                                out=out)
        return y, None
    return fn.fused_residual_norm_scale_shift(
        dev["residual"], dev["x"], dev["gate"] if spec.has_gate else None, weight, bias,
        dev["scale"], dev["shift"], norm, w.eps, out=out, residual_out=residual_out)


def compare_rows(w: synth.Workload, spec: synth.Spec, y: torch.Tensor, r, rows: np.ndarray,
                 ty: Tally, tr: Tally, chunk: int = 8192):
    """Compare the given flattened rows of y (and r) with the oracle, chunk by chunk."""
    yf = y.view(-1, w.D)
    rf = None if r is None else r.view(-1, w.D)
    for i in range(0, len(rows), chunk):
        sel = rows[i:i + chunk]
        idx = torch.from_numpy(sel).to(y.device)
        ref = oracle.run_workload_rows(w, spec, sel)
        ty.add(to_bits(yf.index_select(0, idx)), ref["y"][0])
        if rf is not None:
            tr.add(to_bits(rf.index_select(0, idx)), ref["r"][0])


def check_workload(w: synth.Workload, spec: synth.Spec, device, rows=None, dev=None):
    """Upload, run once, compare (all rows unless given). Returns (tally_y, tally_r)."""
    dev = dev if dev is not None else upload(w, spec, device)
    y, r = run_gpu(w, spec, dev)
    torch.cuda.synchronize(device)
    rows = np.arange(w.rows, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    ty, tr = Tally(), Tally()
    compare_rows(w, spec, y, r, rows, ty, tr)
    return ty, tr
