"""GPU parity: the CUDA kernels (called through the C ABI via the binding) against
the fp64 oracle on the same seeded inputs.

Workloads are the pages' test matrix and WAN2.2 shapes (sglang PR #33144,
"Accuracy Tests": every is_rms x has_gate x has_weight, both scale/shift layouts,
D in {5120, 10240}, L in {16, 90000}, the 4D frame-gate layout; sglang PR #36349,
"Microbenchmark": LayerNorm at seq 176400, dim 5120). Pass criterion: see
tests/parity.py (>= 99.99% of y within 1 bf16 ulp, max |err| <= 2e-2, r bit-exact).
"""
import numpy as np
import pytest
import torch

import rmsnorm_row_b200 as fn
import synth
from parity import Tally, check_workload, host_inputs, upload_host

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _assert(ty: Tally, tr: Tally, label: str):
    print(f"\n{label}\n  y: {ty}\n  r: {tr}")
    assert ty.ok(), f"{label}: y fails the tolerance: {ty}"
    if tr.n:
        assert tr.exact == tr.n, f"{label}: r not bit-exact: {tr}"


def test_gpu_available():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    cap = torch.cuda.get_device_capability(0)
    assert cap[0] >= 10, f"sm_100a kernels need compute capability 10.x, got {cap}"


# ---- small configs: every element -------------------------------------------

def test_rms_fused_B1_L16():
    w = synth.W1
    _assert(*check_workload(w, w.specs[0], DEV), w.name)


@pytest.mark.parametrize("spec", synth.W2.specs, ids=lambda s: s.name)
def test_ln_fused_rowgate_B2_L16(spec):
    w = synth.W2
    _assert(*check_workload(w, spec, DEV), f"{w.name}/{spec.name}")


@pytest.mark.parametrize("D", [5120, 10240])
@pytest.mark.parametrize("spec", synth._ALL8, ids=lambda s: s.name)
def test_all_specs_ragged_L(D, spec):
    # L = 1237 (odd), B = 2: several thousand rows across both batches, outliers included
    base = synth.W3 if D == 5120 else synth.W3B
    w = synth.scaled(base, 1237)
    w = synth.dataclasses.replace(w, B=2, name=f"{w.name}_B2")
    _assert(*check_workload(w, spec, DEV), f"{w.name}/{spec.name}")


@pytest.mark.parametrize("D", [5120, 10240])
@pytest.mark.parametrize("spec", [synth.Spec(False, True, True, has_bias=True),
                                  synth.Spec(True, False, False, has_bias=True),
                                  synth.Spec(False, False, True, norm_only=True),
                                  synth.Spec(True, False, False, norm_only=True),
                                  synth.Spec(False, False, True, has_bias=True, norm_only=True)],
                         ids=lambda s: s.name)
def test_bias_and_norm_only(D, spec):
    base = synth.W3 if D == 5120 else synth.W3B
    w = synth.scaled(base, 777)
    _assert(*check_workload(w, spec, DEV), f"{w.name}/{spec.name}")


@pytest.mark.parametrize("w", [synth.W6, synth.scaled(synth.W5, 420, F=21),
                               synth.scaled(synth.W5B, 490, F=49)], ids=lambda w: w.name)
def test_extra_layouts(w):
    for spec in w.specs:
        _assert(*check_workload(w, spec, DEV), f"{w.name}/{spec.name}")


@pytest.mark.parametrize("D", [5120, 10240])
@pytest.mark.parametrize("layouts", [("bcast", "bcast", "bcast"), ("batch", "batch", "bcast"),
                                     ("frame", "frame", "frame"), ("row", "frame", "bcast"),
                                     ("row", "bcast", "row"), ("bcast", "row", "bcast")],
                         ids=lambda l: "-".join(l))
def test_modulation_layouts(D, layouts):
    # scale and shift broadcast, per batch or per frame run the instances that fetch them
    # from L1 as they are used; one of them per token runs the instances that load them
    # with x. L = 531 = 9 frames of 59 tokens.
    base = synth.W3 if D == 5120 else synth.W3B
    w = synth.scaled(base, 531)
    w = synth.dataclasses.replace(w, B=2, F=9 if "frame" in layouts else 0,
                                  layouts=(("gate", layouts[0]), ("scale", layouts[1]),
                                           ("shift", layouts[2])),
                                  name=f"{w.name}_B2_{'-'.join(layouts)}")
    for spec in (synth.Spec(False, True, False), synth.Spec(True, True, True),
                 synth.Spec(False, False, True, has_bias=True),
                 synth.Spec(True, False, True, norm_only=True)):
        _assert(*check_workload(w, spec, DEV), f"{w.name}/{spec.name}")


# ---- full-size configs --------------------------------------------------------

@pytest.mark.parametrize("D", [5120, 10240])
def test_all_specs_B1_L90000_full(D):
    w = synth.W3 if D == 5120 else synth.W3B
    # inputs generated and uploaded once; each specialisation reads what it needs
    host = host_inputs(w, ("x", "residual", "gate", "scale", "shift", "weight"))
    dev = upload_host(w, host, DEV)
    for spec in w.specs:
        _assert(*check_workload(w, spec, DEV, dev=dev, host=host), f"{w.name}/{spec.name}")
    del dev
    torch.cuda.empty_cache()


def _full_size(w):
    spec = w.specs[0]
    host = host_inputs(w, ("x", "residual", "gate", "scale", "shift", "weight"))
    dev = upload_host(w, host, DEV)
    ty, tr = check_workload(w, spec, DEV, dev=dev, host=host)
    del dev, host
    torch.cuda.empty_cache()
    _assert(ty, tr, f"{w.name}/{spec.name}")


def test_wan22_ln_B1_L176400_full():
    _full_size(synth.W4)


def test_frame_gate_B1_F21x8400_full():
    _full_size(synth.W5)


def test_frame_gate_B1_F49x3600_full():
    _full_size(synth.W5B)


@pytest.mark.parametrize("spec", synth.W7.specs, ids=lambda s: s.name)
def test_microbench_bcast_B1_L176400_full(spec):
    w = synth.W7
    host = host_inputs(w, ("x", "residual", "gate", "scale", "shift", "weight", "bias"))
    dev = upload_host(w, host, DEV)
    ty, tr = check_workload(w, spec, DEV, dev=dev, host=host)
    del dev, host
    torch.cuda.empty_cache()
    _assert(ty, tr, f"{w.name}/{spec.name}")


# ---- fp32 affine parameters ----------------------------------------------------------

@pytest.mark.parametrize("D", [5120, 10240])
@pytest.mark.parametrize("layouts", [("bcast", "row", "row"), ("bcast", "bcast", "bcast"),
                                     ("frame", "frame", "frame")], ids=lambda l: "-".join(l))
@pytest.mark.parametrize("spec", [synth.Spec(False, True, True, has_bias=True),
                                  synth.Spec(True, True, True, has_bias=True),
                                  synth.Spec(True, False, True),
                                  synth.Spec(False, True, True),
                                  synth.Spec(False, False, False, has_bias=True),
                                  synth.Spec(True, False, True, has_bias=True, norm_only=True)],
                         ids=lambda s: s.name)
def test_fp32_affine(D, layouts, spec):
    # weight and bias as fp32 (the same draws as the bf16 ones, kept at 24 bits), used at
    # full precision on both sides. Per-row scale/shift run the instances that load them
    # with x; broadcast and per-frame ones the instances that fetch them from L1 (with a
    # CTA count of their own for an fp32 bias). L = 531 = 9 frames of 59 tokens.
    from parity import oracle_rows
    base = synth.W3 if D == 5120 else synth.W3B
    w = synth.scaled(base, 531)
    w = synth.dataclasses.replace(w, F=9 if "frame" in layouts else 0,
                                  layouts=(("gate", layouts[0]), ("scale", layouts[1]),
                                           ("shift", layouts[2])),
                                  name=f"{w.name}_{'-'.join(layouts)}")
    host = host_inputs(w)
    dev = upload_host(w, host, DEV)
    w32 = torch.from_numpy(w.generate_f32("weight")).to(DEV) if spec.has_weight else None
    b32 = torch.from_numpy(w.generate_f32("bias")).to(DEV) if spec.has_bias else None
    norm = "rms" if spec.is_rms else "layer"
    if spec.norm_only:
        y, r = fn.norm_scale_shift(dev["x"], w32, b32, dev["scale"], dev["shift"], norm, w.eps), None
    else:
        y, r = fn.fused_residual_norm_scale_shift(dev["residual"], dev["x"],
                                                  dev["gate"] if spec.has_gate else None, w32, b32,
                                                  dev["scale"], dev["shift"], norm, w.eps)
    torch.cuda.synchronize()
    host32 = dict(host)
    host32["weight"] = w.generate_f32("weight")
    host32["bias"] = w.generate_f32("bias")
    ref = oracle_rows(w, spec, host32, np.arange(w.rows))
    from synth.device import to_bits
    ty, tr = Tally(), Tally()
    ty.add(to_bits(y).reshape(-1, D), ref["y"][0])
    if r is not None:
        tr.add(to_bits(r).reshape(-1, D), ref["r"][0])
    _assert(ty, tr, f"{w.name}/{spec.name}/fp32-affine")
    assert ty.exact == ty.n
