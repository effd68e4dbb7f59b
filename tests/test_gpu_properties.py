"""GPU checks that need no oracle run, or that pin the kernel to exact values:
hand-derived worked cases, closed forms and identities (constant rows, scale = -1,
gate = 0, gate-free = unit gate), the unfused composition (norm of the returned r
gives the same y), bitwise determinism and in-place residual update, edge shapes
(empty, single row, ragged, padded strides) with guard bands, and argument errors
leaving outputs untouched. All calls go through the C ABI via the binding.
"""
import numpy as np
import pytest
import torch

import golden_cases
import oracle
import rmsnorm_row_b200 as fn
import synth
from helpers import ulp_distance
from parity import Tally
from synth.device import from_bits, to_bits, upload

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def bf(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).to(DEV)


def rand_bf16(shape, sd=1.0, mu=0.0, seed=0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (mu + sd * torch.randn(shape, generator=g)).to(torch.bfloat16).to(DEV)


def bits(t):
    return to_bits(t)


# ---- hand-derived worked cases (tests/golden/hand_cases.txt), tiled ----------------

@pytest.mark.parametrize("D", [5120, 10240])
@pytest.mark.parametrize("case", golden_cases.load(), ids=lambda c: c["name"])
def test_hand_cases_exact(case, D):
    c = golden_cases.tiled(case, D)
    L = 3  # several identical rows
    t = lambda k: from_bits(np.tile(c[k], (1, L, 1)), DEV)
    res, x = t("residual"), t("x")
    gate = None if c["gate"] is None else from_bits(c["gate"].reshape(1, 1, D), DEV)
    scale, shift = t("scale"), t("shift")
    y, r = fn.fused_residual_norm_scale_shift(res, x, gate, None, None, scale, shift,
                                              "rms" if c["is_rms"] else "layer", 1e-6)
    torch.cuda.synchronize()
    assert np.array_equal(bits(r)[0], np.tile(c["want_r"], (L, 1)))
    assert np.array_equal(bits(y)[0], np.tile(c["want_y"], (L, 1)))


# ---- closed forms and identities ------------------------------------------------------

@pytest.mark.parametrize("D", [5120, 10240])
@pytest.mark.parametrize("op", ["norm_only", "fused"])
def test_y_is_rounded_once(D, op):
    # RMSNorm, eps = 0, rows of +-1: n = +-1 exactly and y = n (1 + 2^-8) + 2^-40. The
    # positive elements lie just above the bf16 midpoint 1 + 2^-8 by less than float32
    # resolution and must round up to 1 + 2^-7 (0x3F81), not to the float32 tie and then
    # to the even 1.0; the negative ones round to -1.0 (0xBF80).
    L = 4
    row = torch.tensor([1.0, -1.0] * (D // 2))
    v = row.repeat(1, L, 1).to(torch.bfloat16).to(DEV)
    scale = torch.full((1, 1, D), 2.0 ** -8).to(torch.bfloat16).to(DEV)
    shift = torch.full((1, 1, D), 2.0 ** -40).to(torch.bfloat16).to(DEV)
    if op == "norm_only":
        y = fn.norm_scale_shift(v, None, None, scale, shift, "rms", 0.0)
    else:
        y, _ = fn.fused_residual_norm_scale_shift(v, torch.zeros_like(v), None, None, None, scale,
                                                  shift, "rms", 0.0)
    torch.cuda.synchronize()
    want = np.where(row.numpy() > 0, 0x3F81, 0xBF80).astype(np.uint16)
    assert np.array_equal(bits(y)[0], np.tile(want, (L, 1)))


@pytest.mark.parametrize("D", [5120, 10240])
def test_constant_rows_give_shift_exactly(D):
    L = 64
    vals = torch.tensor([0.0, 1.0, -3.5, 0.15625, 96.0, 1e-3, -250.0, 7.0] * 8)[:L]
    res = vals.view(1, L, 1).expand(1, L, D).to(torch.bfloat16).contiguous().to(DEV)
    x = rand_bf16((1, L, D), seed=1)
    gate = torch.zeros((1, 1, D), dtype=torch.bfloat16, device=DEV)
    scale, shift = rand_bf16((1, L, D), 0.1, seed=2), rand_bf16((1, L, D), 0.1, seed=3)
    y, r = fn.fused_residual_norm_scale_shift(res, x, gate, None, None, scale, shift, "layer", 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(r.view(torch.int16), res.view(torch.int16))          # gate = 0: r = residual
    assert (ulp_distance(bits(y), bits(shift)) == 0).all()                  # n = 0: y = shift


@pytest.mark.parametrize("is_rms", [False, True])
def test_scale_minus_one_and_gate_identities(is_rms):
    D, L = 5120, 40
    norm = "rms" if is_rms else "layer"
    res, x = rand_bf16((1, L, D), seed=4), rand_bf16((1, L, D), seed=5)
    gate = rand_bf16((1, 1, D), 0.5, seed=6)
    shift = rand_bf16((1, L, D), 0.1, seed=7)
    minus1 = torch.full((1, 1, D), -1.0, dtype=torch.bfloat16, device=DEV)
    y, _ = fn.fused_residual_norm_scale_shift(res, x, gate, None, None, minus1, shift, norm, 1e-6)
    assert (ulp_distance(bits(y), bits(shift)) == 0).all()
    scale = rand_bf16((1, L, D), 0.1, seed=8)
    ones = torch.ones((1, 1, D), dtype=torch.bfloat16, device=DEV)
    y1, r1 = fn.fused_residual_norm_scale_shift(res, x, None, None, None, scale, shift, norm, 1e-6)
    y2, r2 = fn.fused_residual_norm_scale_shift(res, x, ones, None, None, scale, shift, norm, 1e-6)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(r1.view(torch.int16), r2.view(torch.int16))


@pytest.mark.parametrize("spec", [synth.Spec(False, True, False), synth.Spec(True, True, True),
                                  synth.Spec(False, False, True, has_bias=True)], ids=lambda s: s.name)
def test_unfused_composition(spec):
    # norm of the returned r, computed by the kernel as a gate-free call with x = 0 and
    # again as a norm-only call, gives bitwise the same y as the fused call.
    w = synth.scaled(synth.W3, 300)
    dev = upload(w, spec, DEV)
    norm = "rms" if spec.is_rms else "layer"
    y, r = fn.fused_residual_norm_scale_shift(dev["residual"], dev["x"], dev["gate"] if spec.has_gate else None,
                                              dev["weight"], dev["bias"], dev["scale"], dev["shift"], norm, 1e-6)
    zeros = torch.zeros_like(dev["x"])
    y2, r2 = fn.fused_residual_norm_scale_shift(r, zeros, None, dev["weight"], dev["bias"],
                                                dev["scale"], dev["shift"], norm, 1e-6)
    y3 = fn.norm_scale_shift(r, dev["weight"], dev["bias"], dev["scale"], dev["shift"], norm, 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(r2.view(torch.int16), r.view(torch.int16))
    assert torch.equal(y2.view(torch.int16), y.view(torch.int16))
    assert torch.equal(y3.view(torch.int16), y.view(torch.int16))


def test_determinism_and_in_place_residual():
    w = synth.scaled(synth.W4, 2048)
    spec = w.specs[0]
    dev = upload(w, spec, DEV)
    y1, r1 = fn.fused_residual_norm_scale_shift(dev["residual"], dev["x"], dev["gate"], None, None,
                                                dev["scale"], dev["shift"], "layer", 1e-6)
    y2, r2 = fn.fused_residual_norm_scale_shift(dev["residual"], dev["x"], dev["gate"], None, None,
                                                dev["scale"], dev["shift"], "layer", 1e-6)
    res_copy = dev["residual"].clone()
    y3, r3 = fn.fused_residual_norm_scale_shift(res_copy, dev["x"], dev["gate"], None, None,
                                                dev["scale"], dev["shift"], "layer", 1e-6,
                                                residual_out=res_copy)
    torch.cuda.synchronize()
    assert r3.data_ptr() == res_copy.data_ptr()
    for a, b in ((y1, y2), (r1, r2), (y1, y3), (r1, res_copy)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


# ---- edge shapes, strides and guard bands --------------------------------------------

def _padded(B, L, D, pad, fill):
    """A (B, L, D) view into a bigger buffer with padded rows and canaries around it."""
    G = 4096  # guard elements on each side
    buf = torch.full((2 * G + B * L * (D + pad),), fill, dtype=torch.int16, device=DEV)
    view = buf[G:G + B * L * (D + pad)].view(B, L, D + pad)[:, :, :D].view(torch.bfloat16)
    return buf, view, G


@pytest.mark.parametrize("B,L", [(1, 1), (3, 5), (2, 1), (1, 7)])
@pytest.mark.parametrize("D", [5120, 10240])
def test_edge_shapes_padded_outputs_and_guards(B, L, D):
    res, x = rand_bf16((B, L, D), seed=11), rand_bf16((B, L, D), seed=12)
    gate = rand_bf16((B, 1, D), 0.5, seed=13)                   # per batch
    scale, shift = rand_bf16((B, L, D), 0.1, seed=14), rand_bf16((1, 1, D), 0.1, seed=15)
    weight = rand_bf16((D,), 0.1, 1.0, seed=16)
    canary = 0x5A5A
    ybuf, y, G = _padded(B, L, D, 64, canary)
    rbuf, r, _ = _padded(B, L, D, 128, canary)
    fn.fused_residual_norm_scale_shift(res, x, gate, weight, None, scale, shift, "layer", 1e-6,
                                       out=y, residual_out=r)
    torch.cuda.synchronize()
    for buf, pad in ((ybuf, 64), (rbuf, 128)):
        host = buf.cpu().numpy()
        assert (host[:G] == canary).all() and (host[-G:] == canary).all()
        body = host[G:len(host) - G].reshape(B, L, D + pad)
        assert (body[:, :, D:] == canary).all()
    # values against the oracle
    xs, rs = bits(x), bits(res)
    ref = oracle.fused_norm(B, L, D, x=xs, x_st=(L * D, 0, D), residual=rs, res_st=(L * D, 0, D),
                            gate=bits(gate), gate_st=(D, 0, 0), weight=bits(weight),
                            scale=bits(scale), scale_st=(L * D, 0, D), shift=bits(shift),
                            shift_st=(0, 0, 0))
    ty, tr = Tally(), Tally()
    ty.add(bits(y.contiguous()), ref["y"])
    tr.add(bits(r.contiguous()), ref["r"])
    assert ty.ok(), str(ty)
    assert tr.exact == tr.n, str(tr)


def test_empty_problem_launches_nothing():
    D = 5120
    x = torch.empty((0, 16, D), dtype=torch.bfloat16, device=DEV)
    s = torch.zeros((1, 1, D), dtype=torch.bfloat16, device=DEV)
    y, r = fn.fused_residual_norm_scale_shift(x.clone(), x, None, None, None, s, s, "layer", 1e-6)
    assert y.shape == (0, 16, D) and r.shape == (0, 16, D)


def test_rejected_call_leaves_outputs_untouched():
    D, L = 5120, 4
    res, x = rand_bf16((1, L, D), seed=21), rand_bf16((1, L, D), seed=22)
    s = torch.zeros((1, 1, D), dtype=torch.bfloat16, device=DEV)
    y = torch.full((1, L, D), 3.0, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(fn.FusedNormError) as ei:   # y aliases x
        fn.fused_residual_norm_scale_shift(res, x, None, None, None, s, s, "layer", 1e-6, out=x)
    assert ei.value.status == fn.FN_ERR_INVALID_ARG
    raw = torch.zeros(L * D + 8, dtype=torch.bfloat16, device=DEV)
    mis = raw[1:1 + L * D].view(1, L, D)                          # 2-byte offset
    with pytest.raises(fn.FusedNormError) as ei:
        fn.fused_residual_norm_scale_shift(res, mis, None, None, None, s, s, "layer", 1e-6, out=y)
    assert ei.value.status == fn.FN_ERR_MISALIGNED
    torch.cuda.synchronize()
    assert (y.float() == 3.0).all()
    with pytest.raises(TypeError):
        fn.fused_residual_norm_scale_shift(res.float(), x, None, None, None, s, s)
    with pytest.raises(fn.FusedNormError) as ei:
        fn.fused_residual_norm_scale_shift(res[..., :4096].contiguous(), x[..., :4096].contiguous(),
                                           None, None, None, s[..., :4096].contiguous(),
                                           s[..., :4096].contiguous())
    assert ei.value.status == fn.FN_ERR_UNSUPPORTED


# ---- rounding-boundary and statistics stress ------------------------------------------

def _near_cancelling_problem(D, L, seed, offset=0.0, spread=1.0, is_rms=False):
    """Rows where shift nearly cancels n * (1 + scale) (so y is tiny and sits close to
    rounding boundaries), with a mean offset and spread per row; built from the oracle's
    own n on CPU."""
    from helpers import f32_to_bf16_bits_rne
    rng = np.random.default_rng(seed)
    def bfbits(a):
        return f32_to_bf16_bits_rne(np.asarray(a, dtype=np.float32))
    res = bfbits(offset + spread * rng.normal(size=(1, L, D)))
    x = bfbits(rng.normal(size=(1, L, D)))
    gate = bfbits(0.5 * rng.normal(size=(1, 1, D)))
    scale = bfbits(0.3 * rng.normal(size=(1, L, D)))
    zeros = np.zeros((1, L, D), np.uint16)
    st = (L * D, 0, D)
    base = oracle.fused_norm(1, L, D, x=x, x_st=st, residual=res, res_st=st, gate=gate,
                             gate_st=(0, 0, 0), scale=zeros, scale_st=st, shift=zeros, shift_st=st,
                             is_rms=is_rms, want_n=True)
    from helpers import bf16_bits_to_f64
    s = bf16_bits_to_f64(scale)
    target = -base["n"] * (1.0 + s) * (1.0 + 1e-3 * rng.normal(size=(1, L, D)))
    shift = bfbits(target)
    return res, x, gate, scale, shift


@pytest.mark.parametrize("is_rms", [False, True])
@pytest.mark.parametrize("offset,spread", [(0.0, 1.0), (1000.0, 0.01), (0.0, 1e-3), (-3.0, 40.0)])
def test_near_cancellation_and_offsets_bit_exact(is_rms, offset, spread):
    D, L = 5120, 96
    res, x, gate, scale, shift = _near_cancelling_problem(D, L, 31, offset, spread, is_rms)
    dev = lambda a: from_bits(a, DEV)
    y, r = fn.fused_residual_norm_scale_shift(dev(res), dev(x), dev(gate), None, None, dev(scale),
                                              dev(shift), "rms" if is_rms else "layer", 1e-6)
    torch.cuda.synchronize()
    st = (L * D, 0, D)
    ref = oracle.fused_norm(1, L, D, x=x, x_st=st, residual=res, res_st=st, gate=gate,
                            gate_st=(0, 0, 0), scale=scale, scale_st=st, shift=shift, shift_st=st,
                            is_rms=is_rms)
    ty, tr = Tally(), Tally()
    ty.add(bits(y), ref["y"])
    tr.add(bits(r), ref["r"])
    print(f"\nnear-cancellation offset={offset} spread={spread} rms={is_rms}\n  y: {ty}\n  r: {tr}")
    assert tr.exact == tr.n
    assert ty.hist.get(0, 0) == ty.n, f"y not bit-exact: {ty}"


@pytest.mark.parametrize("D", [5120, 10240])
@pytest.mark.parametrize("op", ["fused", "norm_only"])
@pytest.mark.parametrize("is_rms", [False, True])
@pytest.mark.parametrize("offset,spread", [(1000.0, 1.0), (1000.0, 0.01), (-3.0e4, 1.0), (0.0, 1e-3)])
def test_offset_rows_with_broadcast_modulation_bit_exact(D, op, is_rms, offset, spread):
    # broadcast scale and shift run the instances that re-read them from cache (for
    # norm-only at D=10240 with 256 threads per row); rows whose mean dwarfs their spread
    # take the centred second pass, which re-reads the row from memory
    from helpers import f32_to_bf16_bits_rne
    L = 40
    rng = np.random.default_rng(7 + D + int(is_rms))
    bfbits = lambda a: f32_to_bf16_bits_rne(np.asarray(a, dtype=np.float32))
    base = bfbits(offset + spread * rng.normal(size=(1, L, D)))
    x = bfbits(rng.normal(size=(1, L, D))) if op == "fused" else base
    gate = bfbits(0.5 * rng.normal(size=(1, 1, D)))
    scale = bfbits(0.3 * rng.normal(size=(1, 1, D)))
    shift = bfbits(0.1 * rng.normal(size=(1, 1, D)))
    weight = bfbits(1 + 0.1 * rng.normal(size=D))
    dev = lambda a: from_bits(a, DEV)
    norm = "rms" if is_rms else "layer"
    st, b0 = (L * D, 0, D), (0, 0, 0)
    if op == "fused":
        y, r = fn.fused_residual_norm_scale_shift(dev(base), dev(x), dev(gate), dev(weight), None,
                                                  dev(scale), dev(shift), norm, 1e-6)
        ref = oracle.fused_norm(1, L, D, x=x, x_st=st, residual=base, res_st=st, gate=gate, gate_st=b0,
                                weight=weight, scale=scale, scale_st=b0, shift=shift, shift_st=b0,
                                is_rms=is_rms)
    else:
        y = fn.norm_scale_shift(dev(x), dev(weight), None, dev(scale), dev(shift), norm, 1e-6)
        r = None
        ref = oracle.fused_norm(1, L, D, x=x, x_st=st, weight=weight, scale=scale, scale_st=b0,
                                shift=shift, shift_st=b0, is_rms=is_rms, norm_only=True)
    torch.cuda.synchronize()
    assert np.array_equal(bits(y), ref["y"]), "y not bit-exact"
    if r is not None:
        assert np.array_equal(bits(r), ref["r"]), "r not bit-exact"
    if (offset, spread) == (1000.0, 1.0) and not is_rms:
        # the case is built so that some rows take the centred pass (mean^2 > 2^20 var > 0)
        from helpers import bf16_bits_to_f64
        v = bf16_bits_to_f64(ref["r"] if r is not None else x).reshape(L, D)
        mu, var = v.mean(axis=1), v.var(axis=1)
        assert np.any((mu * mu > 2.0 ** 20 * var) & (var > 0))


@pytest.mark.parametrize("D", [5120, 10240])
@pytest.mark.parametrize("is_rms", [False, True])
def test_special_values_propagate_like_the_oracle(D, is_rms):
    # IEEE propagation with no special handling: a NaN in x, an infinity in the residual
    # and a residual + gate * x that overflows bf16 poison their own rows (r at that
    # element; y through the statistics: all NaN for a NaN, and for LayerNorm's
    # inf - inf; RMSNorm's 1/sqrt(inf) = 0 leaves y = shift but inf * 0 at the element);
    # the other rows are untouched. NaN payloads may differ, so NaN positions are
    # compared as a mask and every other element bit for bit.
    from helpers import f32_to_bf16_bits_rne
    L = 8
    rng = np.random.default_rng(99 + D)
    bfbits = lambda a: f32_to_bf16_bits_rne(np.asarray(a, dtype=np.float32))
    res = bfbits(rng.normal(size=(1, L, D)))
    x = bfbits(rng.normal(size=(1, L, D)))
    gate = bfbits(0.5 * rng.normal(size=(1, 1, D)))
    scale = bfbits(0.1 * rng.normal(size=(1, L, D)))
    shift = bfbits(0.1 * rng.normal(size=(1, L, D)))
    x[0, 0, 17] = 0x7FC0                      # NaN
    res[0, 1, 3] = 0x7F80                     # +inf
    gate[0, 0, 5] = 0x3F80                    # 1.0
    res[0, 2, 5] = x[0, 2, 5] = 0x7F7F        # bf16 max: the sum overflows to +inf
    dev = lambda a: from_bits(a, DEV)
    y, r = fn.fused_residual_norm_scale_shift(dev(res), dev(x), dev(gate), None, None, dev(scale),
                                              dev(shift), "rms" if is_rms else "layer", 1e-6)
    torch.cuda.synchronize()
    st = (L * D, 0, D)
    ref = oracle.fused_norm(1, L, D, x=x, x_st=st, residual=res, res_st=st, gate=gate,
                            gate_st=(0, 0, 0), scale=scale, scale_st=st, shift=shift, shift_st=st,
                            is_rms=is_rms)

    def nan_mask(b):
        b = np.asarray(b, dtype=np.uint16)
        return ((b & 0x7F80) == 0x7F80) & ((b & 0x7F) != 0)

    for got, want in ((bits(y), ref["y"]), (bits(r), ref["r"])):
        got, want = got.reshape(L, D), want.reshape(L, D)
        assert np.array_equal(nan_mask(got), nan_mask(want))
        keep = ~nan_mask(want)
        assert np.array_equal(got[keep], want[keep])
    ry = bits(y).reshape(L, D)
    assert nan_mask(ry[0]).all()              # a NaN reaches every statistic
    if not is_rms:
        assert nan_mask(ry[1:3]).all()        # inf - inf in the variance
    assert not nan_mask(ry[3:]).any()         # the other rows are finite
    rr = bits(r).reshape(L, D)
    assert rr[1, 3] == 0x7F80 and rr[2, 5] == 0x7F80 and nan_mask(rr[0, 17])


@pytest.mark.parametrize("D", [5120, 10240])
@pytest.mark.parametrize("is_rms", [False, True])
def test_zero_spread_with_zero_eps_matches_the_oracle(D, is_rms):
    # eps = 0 on rows with no spread (LayerNorm: a constant row; RMSNorm: a zero row):
    # 1/sqrt(0) = inf and 0 * inf = NaN on both sides; rows with spread stay finite
    from helpers import f32_to_bf16_bits_rne
    L = 4
    rng = np.random.default_rng(5 + D)
    bfbits = lambda a: f32_to_bf16_bits_rne(np.asarray(a, dtype=np.float32))
    x = bfbits(rng.normal(size=(1, L, D)))
    x[0, 0, :] = 0x0000 if is_rms else 0x4040    # 0.0 or 3.0 across the row
    scale = bfbits(0.1 * rng.normal(size=(1, 1, D)))
    shift = bfbits(0.1 * rng.normal(size=(1, 1, D)))
    dev = lambda a: from_bits(a, DEV)
    y = fn.norm_scale_shift(dev(x), None, None, dev(scale), dev(shift), "rms" if is_rms else "layer", 0.0)
    torch.cuda.synchronize()
    ref = oracle.fused_norm(1, L, D, x=x, x_st=(L * D, 0, D), scale=scale, scale_st=(0, 0, 0),
                            shift=shift, shift_st=(0, 0, 0), is_rms=is_rms, norm_only=True, eps=0.0)
    got, want = bits(y).reshape(L, D), ref["y"].reshape(L, D)
    nan = lambda b: ((b & 0x7F80) == 0x7F80) & ((b & 0x7F) != 0)
    assert nan(want[0]).all() and nan(got[0]).all()
    assert np.array_equal(got[1:], want[1:])
