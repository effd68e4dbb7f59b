"""GPU checks of the launch contract: which error a launch reports, which device it runs
on, that each call runs the CUDA kernel, and that one handle serves every launch shape.

* fused_norm_launch reports the status of its own launch only. An error left pending in
  the caller's CUDA runtime (here: torch's, by an invalid cudaSetDevice, a host-side
  argument error that touches no GPU) is neither returned as FN_ERR_CUDA nor cleared.
* The tensor-level API runs on its inputs' device whichever device is current (needs
  two GPUs; skipped otherwise).
* A CUDA activity trace shows exactly one fused_norm_rows kernel per call, nothing else.
* One handle launched with different L, frame counts and operand layouts matches the
  oracle bit for bit each time.
* Launches captured into a CUDA graph replay to the eager results.
* fused_norm_plan reports the grid and block that the launch uses, instance by instance.
"""
import ctypes

import pytest
import torch

import rmsnorm_row_b200 as fn
from rmsnorm_row_b200 import _abi

pytestmark = pytest.mark.gpu


def _rand(shape, seed, device, sd=1.0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (sd * torch.randn(shape, generator=g)).to(torch.bfloat16).to(device)


def _caller_runtime():
    """The CUDA runtime library torch loaded into this process (same instance)."""
    torch.cuda.init()
    with open("/proc/self/maps") as f:
        for line in f:
            path = line.split()[-1]
            if "libcudart.so" in path:
                rt = ctypes.CDLL(path)
                for name in ("cudaGetLastError", "cudaPeekAtLastError", "cudaSetDevice"):
                    getattr(rt, name).restype = ctypes.c_int
                rt.cudaSetDevice.argtypes = [ctypes.c_int]
                return rt
    pytest.skip("torch's CUDA runtime is not a separate shared library in this process")


def test_launch_neither_reports_nor_clears_a_pending_error():
    dev = torch.device("cuda:0")
    B, L, D = 1, 64, 5120
    x, res = _rand((B, L, D), 1, dev), _rand((B, L, D), 2, dev)
    gate, scale, shift = (_rand((1, 1, D), s, dev, 0.1) for s in (3, 4, 5))
    y = torch.empty_like(x)
    r = torch.empty_like(x)
    args = fn.build_args(x, res, gate, None, None, scale, shift, y, r)
    cfg = _abi.fn_config(D=D, is_rms=0, has_gate=1, has_weight=0, has_bias=0, norm_only=0,
                         affine_fp32=0, eps=1e-6)
    st, h = _abi.fused_norm_create(cfg)
    assert st == fn.FN_OK
    stream = int(torch.cuda.current_stream(dev).cuda_stream)
    rt = _caller_runtime()
    try:
        rt.cudaGetLastError()                       # start clean
        injected = rt.cudaSetDevice(1 << 20)        # no such device: cudaErrorInvalidDevice
        assert injected != 0
        assert rt.cudaPeekAtLastError() == injected
        # nothing but ctypes calls between the injection and the checks
        assert _abi.fused_norm_launch(h, args, stream) == fn.FN_OK
        assert _abi.fused_norm_last_cuda_error() == 0
        assert rt.cudaPeekAtLastError() == injected  # still pending, for its owner to read
        assert rt.cudaGetLastError() == injected
        assert rt.cudaGetLastError() == 0
        torch.cuda.synchronize(dev)
        ref_y, ref_r = fn.fused_residual_norm_scale_shift(res, x, gate, None, None, scale, shift,
                                                          "layer", 1e-6)
        torch.cuda.synchronize(dev)
        assert torch.equal(y.view(torch.int16), ref_y.view(torch.int16))
        assert torch.equal(r.view(torch.int16), ref_r.view(torch.int16))
    finally:
        _abi.fused_norm_destroy(h)


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs two GPUs")
def test_api_runs_on_the_inputs_device():
    d1 = torch.device("cuda:1")
    B, L, D = 2, 33, 5120
    x, res = _rand((B, L, D), 11, d1), _rand((B, L, D), 12, d1)
    gate, scale, shift = _rand((B, L, D), 13, d1, 0.5), _rand((1, D), 14, d1, 0.1), _rand((1, D), 15, d1, 0.1)
    with torch.cuda.device(d1):
        want_y, want_r = fn.fused_residual_norm_scale_shift(res, x, gate, None, None, scale, shift)
        want_n = fn.norm_scale_shift(x, None, None, scale, shift, "rms")
        torch.cuda.synchronize(d1)
    torch.cuda.set_device(0)
    y, r = fn.fused_residual_norm_scale_shift(res, x, gate, None, None, scale, shift)
    n = fn.norm_scale_shift(x, None, None, scale, shift, "rms")
    assert torch.cuda.current_device() == 0
    torch.cuda.synchronize(d1)
    assert torch.equal(y.view(torch.int16), want_y.view(torch.int16))
    assert torch.equal(r.view(torch.int16), want_r.view(torch.int16))
    assert torch.equal(n.view(torch.int16), want_n.view(torch.int16))


def test_every_call_runs_the_cuda_kernel():
    # the pages' tests count dispatches to prove there is no silent fallback; here the
    # CUDA activity trace of a few calls must show exactly one fused_norm_rows kernel per
    # call and nothing else
    try:
        from torch.profiler import ProfilerActivity, profile
    except ImportError:
        pytest.skip("torch.profiler unavailable")
    dev = torch.device("cuda:0")
    B, L, D = 1, 96, 5120
    x, res = _rand((B, L, D), 21, dev), _rand((B, L, D), 22, dev)
    gate, scale, shift = (_rand((1, 1, D), s, dev, 0.1) for s in (23, 24, 25))
    y = torch.empty_like(x)
    r = torch.empty_like(x)
    n = torch.empty_like(x)
    torch.cuda.synchronize(dev)
    calls = 3
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        for _ in range(calls):
            fn.fused_residual_norm_scale_shift(res, x, gate, None, None, scale, shift, "layer", 1e-6,
                                               out=y, residual_out=r)
            fn.norm_scale_shift(x, None, None, scale, shift, "rms", 1e-6, out=n)
        torch.cuda.synchronize(dev)
    kernels = [e.name for e in prof.events() if e.device_type.name == "CUDA"]
    if not kernels:
        pytest.skip("no CUDA activity recorded (tracing unavailable)")
    ours = [k for k in kernels if "fused_norm_rows" in k]
    assert len(ours) == 2 * calls, kernels
    assert len(kernels) == len(ours), kernels


def test_one_handle_serves_every_length_and_layout():
    # a handle fixes only the specialisation; L, B, frames and operand strides are launch
    # arguments (the pages test that one compiled kernel is reused across L and layouts)
    import numpy as np
    import synth
    from parity import Tally, compare_rows, host_inputs, upload_host
    dev = torch.device("cuda:0")
    cfg = _abi.fn_config(D=5120, is_rms=0, has_gate=1, has_weight=1, has_bias=0, norm_only=0,
                         affine_fp32=0, eps=1e-6)
    st, h = _abi.fused_norm_create(cfg)
    assert st == fn.FN_OK
    spec = synth.Spec(False, True, True)
    try:
        for L, F, layouts in ((16, 0, ("bcast", "row", "row")), (531, 9, ("frame", "frame", "frame")),
                              (1237, 0, ("row", "bcast", "bcast"))):
            w = synth.dataclasses.replace(synth.scaled(synth.W3, L), F=F,
                                          layouts=(("gate", layouts[0]), ("scale", layouts[1]),
                                                   ("shift", layouts[2])), name=f"reuse_L{L}")
            host = host_inputs(w)
            d = upload_host(w, host, dev)
            y = torch.empty((w.B, w.L, w.D), dtype=torch.bfloat16, device=dev)
            r = torch.empty_like(y)
            args = fn.build_args(d["x"], d["residual"], d["gate"], d["weight"], None, d["scale"],
                                 d["shift"], y, r)
            assert _abi.fused_norm_launch(h, args, int(torch.cuda.current_stream(dev).cuda_stream)) == fn.FN_OK
            torch.cuda.synchronize(dev)
            ty, tr = Tally(), Tally()
            compare_rows(w, spec, y, r, np.arange(w.rows), ty, tr, host=host)
            assert ty.exact == ty.n and tr.exact == tr.n, (L, layouts, str(ty), str(tr))
    finally:
        _abi.fused_norm_destroy(h)


def test_launches_replay_from_a_cuda_graph():
    # the library launches on the caller's stream and allocates nothing, so its launches
    # can be captured into a CUDA graph and replayed; the replay gives the eager bits
    dev = torch.device("cuda:0")
    B, L, D = 2, 40, 5120
    x, res = _rand((B, L, D), 31, dev), _rand((B, L, D), 32, dev)
    gate, scale, shift = _rand((B, L, D), 33, dev, 0.5), _rand((1, D), 34, dev, 0.1), _rand((1, D), 35, dev, 0.1)
    weight = (1 + _rand((D,), 36, dev, 0.1).float()).to(torch.bfloat16)
    want_y, want_r = fn.fused_residual_norm_scale_shift(res, x, gate, weight, None, scale, shift, "rms")
    want_n = fn.norm_scale_shift(x, weight, None, scale, shift, "layer")
    y, r, n = torch.empty_like(x), torch.empty_like(x), torch.empty_like(x)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(cap), torch.cuda.graph(graph, stream=cap):
        fn.fused_residual_norm_scale_shift(res, x, gate, weight, None, scale, shift, "rms", out=y,
                                           residual_out=r, stream=cap)
        fn.norm_scale_shift(x, weight, None, scale, shift, "layer", out=n, stream=cap)
    for _ in range(2):
        y.zero_(), r.zero_(), n.zero_()
        graph.replay()
        torch.cuda.synchronize(dev)
        for got, want in ((y, want_y), (r, want_r), (n, want_n)):
            assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    del graph


def _kernel_launches(prof, tmp_path):
    """(name, grid, block) of each fused_norm_rows kernel in a profiler trace."""
    import json
    path = tmp_path / "trace.json"
    prof.export_chrome_trace(str(path))
    events = json.load(open(path)).get("traceEvents", [])
    out = []
    for e in events:
        if e.get("cat") == "kernel" and "fused_norm_rows" in e.get("name", ""):
            a = e.get("args", {})
            if "grid" not in a or "block" not in a:
                pytest.skip("the trace does not record launch dimensions")
            out.append((e["name"], tuple(a["grid"]), tuple(a["block"])))
    return out


@pytest.mark.parametrize("D", [5120, 10240])
@pytest.mark.parametrize("case", ["fused_row", "fused_bcast", "nss_bcast", "nss_bcast_w",
                                  "nss_bcast_wb_f32", "nss_row"])
def test_plan_matches_the_launch(D, case, tmp_path):
    # the launch shape (threads per row) differs by instance; fused_norm_plan must report
    # the grid and block the launch really uses, and the block must hold D / 8 vectors
    # (the kernel's second template argument is the vectors per thread)
    import re
    from torch.profiler import ProfilerActivity, profile
    dev = torch.device("cuda:0")
    B, L = 1, 37
    x = _rand((B, L, D), 41, dev)
    norm_only = case.startswith("nss")
    res = None if norm_only else _rand((B, L, D), 42, dev)
    gate = None if norm_only else _rand((1, 1, D), 43, dev, 0.5)
    per_row = case.endswith("_row")
    shape = (B, L, D) if per_row else (1, 1, D)
    scale, shift = _rand(shape, 44, dev, 0.1), _rand(shape, 45, dev, 0.1)
    weight = bias = None
    if case == "nss_bcast_w":
        weight = (1 + _rand((D,), 46, dev, 0.1).float()).to(torch.bfloat16)
    if case == "nss_bcast_wb_f32":
        weight = 1 + _rand((D,), 46, dev, 0.1).float()
        bias = _rand((D,), 47, dev, 0.1).float()
    y = torch.empty_like(x)
    r = None if norm_only else torch.empty_like(x)
    args = fn.build_args(x, res, gate, weight, bias, scale, shift, y, r)
    cfg = _abi.fn_config(D=D, is_rms=0, has_gate=int(gate is not None), has_weight=int(weight is not None),
                         has_bias=int(bias is not None), norm_only=int(norm_only),
                         affine_fp32=int(weight is not None and weight.dtype == torch.float32), eps=1e-6)
    st, h = _abi.fused_norm_create(cfg)
    assert st == fn.FN_OK
    try:
        st, grid, block, smem = _abi.fused_norm_plan(h, args)
        assert st == fn.FN_OK and smem == 0
        stream = int(torch.cuda.current_stream(dev).cuda_stream)
        torch.cuda.synchronize(dev)
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            assert _abi.fused_norm_launch(h, args, stream) == fn.FN_OK
            torch.cuda.synchronize(dev)
        launches = _kernel_launches(prof, tmp_path)
        if not launches:
            pytest.skip("no CUDA activity recorded (tracing unavailable)")
        assert len(launches) == 1, launches
        name, g, b = launches[0]
        assert g == (grid, 1, 1) and b == (block, 1, 1), (name, g, b, grid, block)
        m = re.search(r"fused_norm_rows<(\d+), (\d+),", name)
        assert m and int(m.group(1)) == D and block * 8 * int(m.group(2)) == D, name
    finally:
        _abi.fused_norm_destroy(h)
