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
from synth.device import to_bits
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
        gpu = np.asarray(gpu, dtype=np.uint16).ravel()
        ref = np.asarray(ref, dtype=np.uint16).ravel()
        self.n += gpu.size
        differ = np.flatnonzero(gpu != ref)
        # +0 and -0 are the same value: distance 0, but not counted as bit-exact
        n_same = gpu.size - differ.size
        self.exact += n_same
        self.hist[0] = self.hist.get(0, 0) + n_same
        if differ.size:
            g, r = gpu[differ], ref[differ]
            d = ulp_distance(g, r)
            vals, counts = np.unique(np.minimum(d, 1000), return_counts=True)
            for v, c in zip(vals.tolist(), counts.tolist()):
                self.hist[v] = self.hist.get(v, 0) + c
            diff = np.abs(bf16_bits_to_f64(g) - bf16_bits_to_f64(r))
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


OPERANDS = ("x", "residual", "gate", "scale", "shift", "weight", "bias")


def host_inputs(w: synth.Workload, names=OPERANDS):
    """Every stored row of the named tensors, generated once (uint16 bf16 bits)."""
    return {n: w.generate(n) for n in names}


def upload_host(w: synth.Workload, host, device):
    """Device copies (bf16, operand view shapes) of host_inputs() arrays."""
    from synth.device import operand_view_shape
    out = {}
    for n, a in host.items():
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
        out[n] = t.to(device).view(operand_view_shape(w, n))
    return out


def oracle_rows(w: synth.Workload, spec: synth.Spec, host, flat_rows: np.ndarray):
    """Oracle outputs for the given tokens, gathered from host_inputs() arrays as a
    compact per-row problem (operand rows picked by the generator's layout recipe)."""
    n, D = len(flat_rows), w.D
    st = (n * D, 0, D)
    pick = lambda op: host[op][w.token_rows(op, flat_rows)]
    return oracle.fused_norm(
        1, n, D, x=host["x"][flat_rows], x_st=st,
        residual=None if spec.norm_only else host["residual"][flat_rows],
        res_st=None if spec.norm_only else st,
        gate=pick("gate") if (spec.has_gate and not spec.norm_only) else None,
        gate_st=st if (spec.has_gate and not spec.norm_only) else None,
        weight=(host["weight"].reshape(-1) if host["weight"].dtype == np.float32 else host["weight"])
        if spec.has_weight else None,
        bias=(host["bias"].reshape(-1) if host["bias"].dtype == np.float32 else host["bias"])
        if spec.has_bias else None,
        scale=pick("scale"), scale_st=st, shift=pick("shift"), shift_st=st,
        is_rms=spec.is_rms, norm_only=spec.norm_only, eps=w.eps)


def compare_rows(w: synth.Workload, spec: synth.Spec, y: torch.Tensor, r, rows: np.ndarray,
                 ty: Tally, tr: Tally, host=None, chunk: int = 8192):
    """Compare the given flattened rows of y (and r) with the oracle, chunk by chunk."""
    yf = y.view(-1, w.D)
    rf = None if r is None else r.view(-1, w.D)
    for i in range(0, len(rows), chunk):
        sel = rows[i:i + chunk]
        idx = torch.from_numpy(sel).to(y.device)
        ref = oracle_rows(w, spec, host, sel) if host is not None else \
            oracle.run_workload_rows(w, spec, sel)
        ty.add(to_bits(yf.index_select(0, idx)), ref["y"][0])
        if rf is not None:
            tr.add(to_bits(rf.index_select(0, idx)), ref["r"][0])


def check_workload(w: synth.Workload, spec: synth.Spec, device, rows=None, dev=None, host=None):
    """Run once through the binding and compare with the oracle (all rows unless given).

    Inputs come from `host` (host_inputs()) when given, else from the generator; the
    device copies from `dev` when given, else from an upload. Returns (tally_y, tally_r).
    """
    if host is None and dev is None:
        host = host_inputs(w)
    if dev is None:
        dev = upload_host(w, host, device)
    y, r = run_gpu(w, spec, dev)
    torch.cuda.synchronize(device)
    rows = np.arange(w.rows, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    ty, tr = Tally(), Tally()
    compare_rows(w, spec, y, r, rows, ty, tr, host=host)
    return ty, tr
