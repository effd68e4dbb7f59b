"""Host-side checks of the C ABI: the library loads without a GPU, exports every
function include/fused_norm.h declares, and applies every argument rule before any
launch. Nothing here makes a CUDA call: create / validate / plan / get_config /
status_string are host-only, and launch returns before touching CUDA when the
arguments are rejected. Device pointers below are fake, aligned addresses that are
never dereferenced.
"""
import ctypes
import os
import re
import subprocess

import pytest

import rmsnorm_row_b200 as fn
from rmsnorm_row_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fused_norm.h")
OK, INV, UNS, MIS = fn.FN_OK, fn.FN_ERR_INVALID_ARG, fn.FN_ERR_UNSUPPORTED, fn.FN_ERR_MISALIGNED


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:fn_status|const char\*|int)\s+(fused_norm_\w+)\s*\(", text, re.M)))


def test_header_functions_are_exported():
    names = declared_functions()
    assert len(names) >= 9
    assert sorted(names) == sorted(_abi.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(\w+)$", out, re.M))
    for n in names:
        assert n in exported, n
        assert hasattr(fn.load(), n)


def test_struct_layouts_match_header():
    # The header's structs are plain C; check the sizes ctypes sees against a C compile.
    src = (f'#include "{HEADER}"\n#include <stdio.h>\n#include <stddef.h>\n'
           'int main(){printf("%zu %zu %zu %zu %zu\\n", sizeof(fn_config), sizeof(fn_operand),'
           ' sizeof(fn_args), offsetof(fn_args, weight), offsetof(fn_args, r_stride_l));return 0;}')
    exe = os.path.join(ROOT, "_build_sizes_probe")
    try:
        subprocess.run(["gcc", "-x", "c", "-", "-o", exe], input=src, text=True, check=True)
        got = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()
    finally:
        if os.path.exists(exe):
            os.remove(exe)
    want = [ctypes.sizeof(_abi.fn_config), ctypes.sizeof(_abi.fn_operand), ctypes.sizeof(_abi.fn_args),
            _abi.fn_args.weight.offset, _abi.fn_args.r_stride_l.offset]
    assert [int(v) for v in got] == want


def cfg(D=5120, is_rms=0, gate=1, weight=0, bias=0, norm_only=0, eps=1e-6, affine_fp32=0):
    return fn.fn_config(D=D, is_rms=is_rms, has_gate=gate, has_weight=weight, has_bias=bias,
                        norm_only=norm_only, affine_fp32=affine_fp32, eps=eps)


def make(D=5120, is_rms=0, gate=1, weight=0, bias=0, norm_only=0, eps=1e-6, affine_fp32=0):
    st, h = fn.fused_norm_create(cfg(D, is_rms, gate, weight, bias, norm_only, eps, affine_fp32))
    assert st == OK
    return h


BASE = 0x7F0000000000
MB = 1 << 24


def valid_args(B=2, L=8, D=5120, gate=True, weight=False, bias=False, norm_only=False, tpf=0):
    """Per-row x/residual/scale/shift, broadcast gate, outputs (B, L, D); buffers spaced
    by max(16 MB, one full tensor)."""
    MB = max(1 << 24, ((B * L * D * 2) + 0xFFFF) & ~0xFFFF)
    a = fn.fn_args()
    a.B, a.L, a.tokens_per_frame = B, L, tpf
    row = (L * D, 0, D)
    a.x = fn.fn_operand(BASE + 0 * MB, *row)
    if not norm_only:
        a.residual = fn.fn_operand(BASE + 1 * MB, *row)
    if gate:
        a.gate = fn.fn_operand(BASE + 2 * MB, 0, 0, 0)
    a.scale = fn.fn_operand(BASE + 3 * MB, *row)
    a.shift = fn.fn_operand(BASE + 4 * MB, *row)
    if weight:
        a.weight = BASE + 5 * MB
    if bias:
        a.bias = BASE + 6 * MB
    a.y, a.y_stride_b, a.y_stride_l = BASE + 7 * MB, L * D, D
    if not norm_only:
        a.r, a.r_stride_b, a.r_stride_l = BASE + 8 * MB, L * D, D
    return a


# ---------------------------------------------------------------- create

@pytest.mark.parametrize("D,want", [(5120, OK), (10240, OK), (4096, UNS), (5128, UNS), (0, UNS), (-5120, UNS)])
def test_create_D(D, want):
    st, h = fn.fused_norm_create(cfg(D=D))
    assert st == want
    if h:
        fn.fused_norm_destroy(h)


@pytest.mark.parametrize("args", [
    (5120, 2, 1, 0, 0, 0, 1e-6), (5120, 0, -1, 0, 0, 0, 1e-6), (5120, 0, 1, 3, 0, 0, 1e-6),
    (5120, 0, 1, 0, 0, 1, 1e-6),            # norm-only with a gate
    (5120, 0, 1, 0, 0, 0, -1e-6), (5120, 0, 1, 0, 0, 0, float("nan")), (5120, 0, 1, 0, 0, 0, float("inf")),
    (5120, 0, 1, 0, 0, 0, 1e-6, 1),         # fp32 affine without weight or bias
    (5120, 0, 1, 1, 0, 0, 1e-6, 2),         # affine_fp32 not a flag
])
def test_create_rejects(args):
    st, h = fn.fused_norm_create(cfg(*args))
    assert st == INV and h is None


def test_create_null_and_config_roundtrip():
    assert fn.load().fused_norm_create(None, None) == INV
    h = make(D=10240, is_rms=1, gate=0, weight=1, bias=1, affine_fp32=1)
    st, c = fn.fused_norm_get_config(h)
    assert st == OK and (c.D, c.is_rms, c.has_gate, c.has_weight, c.has_bias, c.affine_fp32) == (10240, 1, 0, 1, 1, 1)
    assert c.eps == 1e-6
    assert fn.fused_norm_destroy(h) == OK
    assert fn.fused_norm_destroy(None) == OK


def test_status_strings():
    for s in (OK, INV, UNS, MIS, fn.FN_ERR_CUDA, 99):
        assert isinstance(fn.fused_norm_status_string(s), str) and fn.fused_norm_status_string(s)


# ---------------------------------------------------------------- validate

def test_valid_args_pass_and_plan():
    h = make()
    a = valid_args()
    assert fn.fused_norm_validate(h, a) == OK
    st, grid, block, smem = fn.fused_norm_plan(h, a)
    # one CTA per row; a whole number of warps, each thread owning whole 16-byte vectors
    assert (st, grid, smem) == (OK, 16, 0)
    assert block % 32 == 0 and 5120 % (8 * block) == 0
    h2 = make(D=10240)
    st, grid, block, smem = fn.fused_norm_plan(h2, valid_args(D=10240, B=1, L=90000))
    assert (st, grid) == (OK, 90000)
    assert block % 32 == 0 and 10240 % (8 * block) == 0


@pytest.mark.parametrize("D", [5120, 10240])
@pytest.mark.parametrize("norm_only", [0, 1])
@pytest.mark.parametrize("bcast", [False, True])
@pytest.mark.parametrize("weight", [0, 1])
def test_plan_follows_the_instance(D, norm_only, bcast, weight):
    # scale and shift broadcast (stride_l 0) select the instances that re-read them from
    # cache, whose launch shape may differ; the plan reports the block the launch uses
    h = make(D=D, gate=0 if norm_only else 1, norm_only=norm_only, weight=weight)
    a = valid_args(D=D, B=1, L=1000, gate=not norm_only, weight=bool(weight), norm_only=bool(norm_only))
    if bcast:
        a.scale.stride_b = a.scale.stride_l = a.shift.stride_b = a.shift.stride_l = 0
    st, grid, block, smem = fn.fused_norm_plan(h, a)
    assert (st, grid, smem) == (OK, 1000, 0)
    want = {5120: 128, 10240: 320}[D]
    if norm_only and bcast:
        # norm-only with cached modulation: 10 vectors per thread, except with an affine
        # operand at D = 5120 (5 vectors)
        want = 128 if (D == 5120 and weight) else D // 80
    assert block == want


def _mut(**kw):
    a = valid_args()
    for k, v in kw.items():
        obj = a
        parts = k.split("__")
        for p in parts[:-1]:
            obj = getattr(obj, p)
        setattr(obj, parts[-1], v)
    return a


@pytest.mark.parametrize("change,want", [
    (dict(B=-1), INV), (dict(L=-3), INV), (dict(tokens_per_frame=-2), INV),
    (dict(tokens_per_frame=3), INV),                               # 3 does not divide L = 8
    (dict(x__stride_f=5120), INV),                                 # stride_f without a frame axis
    (dict(x__ptr=None), INV), (dict(scale__ptr=None), INV), (dict(shift__ptr=None), INV),
    (dict(y=None), INV), (dict(r=None), INV), (dict(residual__ptr=None), INV),
    (dict(gate__ptr=None), INV),                                   # has_gate but no gate
    (dict(weight=BASE + 5 * MB), INV),                             # weight without has_weight
    (dict(bias=BASE + 6 * MB), INV),
    (dict(x__stride_l=-5120), INV), (dict(y_stride_l=-5120), INV),
    (dict(x__ptr=BASE + 2), MIS), (dict(gate__ptr=BASE + 2 * MB + 8), MIS),
    (dict(y=BASE + 7 * MB + 4), MIS), (dict(r=BASE + 8 * MB + 2), MIS),
    (dict(x__stride_l=5124), MIS), (dict(scale__stride_b=40964), MIS), (dict(y_stride_l=5124), MIS),
    (dict(y_stride_l=4096), INV),                                  # y rows overlap each other
    (dict(r_stride_b=5120 * 4), INV),                              # r batches overlap
    (dict(y=BASE + 0 * MB), INV),                                  # y aliases x
    (dict(y=BASE + 3 * MB + 4096), INV),                           # y overlaps scale
    (dict(r=BASE + 7 * MB), INV),                                  # r aliases y
    (dict(r=BASE + 2 * MB), INV),                                  # r overlaps the gate
    (dict(r=BASE + 1 * MB + 16), INV),                             # r overlaps residual, not in place
    (dict(r=BASE + 1 * MB, r_stride_l=10240, r_stride_b=81920), INV),  # same base, other strides
])
def test_validate_rejects(change, want):
    h = make()
    a = _mut(**change)
    assert fn.fused_norm_validate(h, a) == want
    # launch applies the same rules first and never reaches CUDA for these
    assert fn.fused_norm_launch(h, a, 0) == want


def test_in_place_residual_is_allowed():
    h = make()
    a = _mut(r=BASE + 1 * MB)          # r == residual, same strides
    assert fn.fused_norm_validate(h, a) == OK


def test_empty_problem_is_a_no_op():
    h = make()
    for B, L in ((0, 8), (2, 0), (0, 0)):
        a = fn.fn_args()
        a.B, a.L = B, L                  # every pointer NULL: nothing is read
        assert fn.fused_norm_validate(h, a) == OK
        assert fn.fused_norm_launch(h, a, 0) == OK


def test_frame_layout_and_broadcast_batch():
    h = make(weight=1)
    a = valid_args(weight=True, tpf=400, L=8400, B=1)
    a.gate = fn.fn_operand(BASE + 2 * MB, 21 * 5120, 5120, 0)
    a.scale = fn.fn_operand(BASE + 3 * MB, 21 * 5120, 5120, 0)
    a.shift = fn.fn_operand(BASE + 4 * MB, 0, 5120, 0)
    a.x = fn.fn_operand(BASE + 20 * MB, 8400 * 5120, 0, 5120)
    a.residual = fn.fn_operand(BASE + 120 * MB, 8400 * 5120, 0, 5120)
    a.y, a.y_stride_b, a.y_stride_l = BASE + 220 * MB, 8400 * 5120, 5120
    a.r, a.r_stride_b, a.r_stride_l = BASE + 320 * MB, 8400 * 5120, 5120
    assert fn.fused_norm_validate(h, a) == OK
    a.tokens_per_frame = 0           # frame strides need a frame axis
    assert fn.fused_norm_validate(h, a) == INV


def test_norm_only_rules():
    h = make(gate=0, norm_only=1, weight=1, bias=1)
    a = valid_args(gate=False, norm_only=True, weight=True, bias=True)
    assert fn.fused_norm_validate(h, a) == OK
    a.residual = fn.fn_operand(BASE + 1 * MB, 8 * 5120, 0, 5120)
    assert fn.fused_norm_validate(h, a) == INV
    a = valid_args(gate=False, norm_only=True, weight=True, bias=True)
    a.r, a.r_stride_b, a.r_stride_l = BASE + 8 * MB, 8 * 5120, 5120
    assert fn.fused_norm_validate(h, a) == INV


def test_extent_overflow_is_rejected():
    h = make()
    a = valid_args(B=1, L=1 << 40)
    a.x.stride_l = a.residual.stride_l = a.scale.stride_l = a.shift.stride_l = 5120
    assert fn.fused_norm_validate(h, a) == INV


def test_row_count_limit():
    # one CTA per row with 32-bit row indices: B * L must stay below 2^31
    h = make()
    assert fn.fused_norm_validate(h, valid_args(B=1, L=(1 << 31) - 1)) == OK
    assert fn.fused_norm_validate(h, valid_args(B=1, L=1 << 31)) == INV
    assert fn.fused_norm_validate(h, valid_args(B=2, L=1 << 30)) == INV
    assert fn.fused_norm_validate(h, valid_args(B=3, L=(1 << 31) // 3)) == OK


def test_null_handle_and_args():
    assert fn.load().fused_norm_validate(None, None) == INV
    h = make()
    assert fn.load().fused_norm_validate(h, None) == INV


def test_fp32_affine_extent_in_overlap_rules():
    # fp32 weight spans 4*D bytes: y placed right after a bf16-sized weight overlaps it
    h16, h32 = make(weight=1), make(weight=1, affine_fp32=1)
    a = valid_args(weight=True)
    a.y = a.weight + 5120 * 2
    a.y_stride_b, a.y_stride_l = 8 * 5120, 5120
    assert fn.fused_norm_validate(h16, a) == OK
    assert fn.fused_norm_validate(h32, a) == INV


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    # no fallback: without the built library every entry point raises, naming the build step
    from rmsnorm_row_b200 import _abi
    monkeypatch.setattr(_abi, "_lib", None)
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "libfused_norm.so"))
    with pytest.raises(ImportError, match="rmsnorm_row_b200.build"):
        _abi.fused_norm_version()
    with pytest.raises(ImportError, match="no fallback"):
        _abi.fused_norm_create(_abi.fn_config(D=5120, eps=1e-6))
