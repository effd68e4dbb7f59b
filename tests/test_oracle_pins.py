"""Pins for the fp64 oracle, on the CPU.

The oracle is only trusted once it is tied to something other than itself. Each
test here checks it against what the mathematics or a library fixes: closed forms,
invariants, exact high-precision brute force on tiny rows, all 65536 bf16 patterns,
and torch's CPU layer_norm / rms_norm. A plausible slip in the oracle (a dropped
term, a wrong sign, eps outside the sqrt, a transposed operand, a wrong frame index,
double rounding) fails at least one of them.

Semantics under test (sglang PR #36349 "[AMD][Diffusion] Migrate FlyDSL fused norm
kernels to the v0.3.0 stable API", section "Microbenchmark"; sglang PR #33144, same
title, sections "Modifications" and "Accuracy Tests"): r = residual + gate * x;
LayerNorm or RMSNorm of r with eps inside the square root; optional affine weight
(and bias); y = n * (1 + scale) + shift; y and r returned in bf16.
"""
from fractions import Fraction

import mpmath
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import bf16_bits_to_f64, f32_to_bf16_bits_rne

mpmath.mp.dps = 60
EPS = 1e-6


def exact_bits(vals):
    """bf16 bit patterns of values that must be exactly representable in bf16."""
    f = np.asarray(vals, dtype=np.float64)
    b = f32_to_bf16_bits_rne(f.astype(np.float32))
    assert np.array_equal(bf16_bits_to_f64(b), f, equal_nan=True), "value not exact in bf16"
    return b


def one_row(r_vals, *, scale=None, shift=None, weight=None, bias=None, is_rms=False,
            x_vals=None, gate_vals=None, eps=EPS, norm_only=False):
    """Run the oracle on one row whose residual is r_vals (x = 0 unless given)."""
    D = len(r_vals)
    z = np.zeros(D)
    res = exact_bits(r_vals)
    x = exact_bits(z if x_vals is None else x_vals)
    gate = None if gate_vals is None else exact_bits(gate_vals)
    sc = exact_bits(z if scale is None else scale)
    sh = exact_bits(z if shift is None else shift)
    w = None if weight is None else exact_bits(weight)
    b = None if bias is None else exact_bits(bias)
    st = (D, 0, D)
    if norm_only:
        return oracle.fused_norm(1, 1, D, x=res, x_st=st, scale=sc, scale_st=st, shift=sh,
                                 shift_st=st, weight=w, bias=b, is_rms=is_rms, norm_only=True,
                                 eps=eps, want_n=True, want_stats=True)
    return oracle.fused_norm(1, 1, D, x=x, x_st=st, residual=res, res_st=st, gate=gate,
                             gate_st=st if gate is not None else None, weight=w, bias=b,
                             scale=sc, scale_st=st, shift=sh, shift_st=st, is_rms=is_rms,
                             eps=eps, want_n=True, want_stats=True)


def nearest_bf16_ok(y_exact, bits):
    """True when `bits` is the bf16 nearest to y_exact (ties to even), judged by comparing
    against both neighbours in exact arithmetic; independent of any rounding code."""
    v = Fraction(bf16_bits_to_f64(np.array([bits]))[0])
    lo = Fraction(bf16_bits_to_f64(np.array([(bits - 1) & 0xFFFF]))[0])
    hi = Fraction(bf16_bits_to_f64(np.array([(bits + 1) & 0xFFFF]))[0])
    d = abs(y_exact - v)
    for nb in (lo, hi):
        dn = abs(y_exact - nb)
        if dn < d:
            return False
        if dn == d and (bits & 1):
            return False   # a tie must land on the even pattern
    return True


# --------------------------------------------------------------------------
# bf16 conversions
# --------------------------------------------------------------------------

def test_bf16_to_double_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_to_double(int(b)) for b in bits])
    ok = np.isnan(ref) == np.isnan(got)
    both = ~np.isnan(ref)
    assert ok.all()
    assert np.array_equal(got[both], ref[both])
    assert np.array_equal(np.signbit(got[both]), np.signbit(ref[both]))


def test_bf16_rne_matches_torch_on_float32_values():
    # For binary32 inputs one rounding is the whole story, so torch's float -> bf16
    # (round to nearest even) is an independent reference.
    rng = np.random.default_rng(7)
    u = rng.integers(0, 2**32, size=200_000, dtype=np.uint64).astype(np.uint32)
    f = u.view(np.float32)
    f = f[np.isfinite(f)]
    f = np.concatenate([f, np.float32([0.0, -0.0, 1e-45, -1e-45, 1.1754944e-38, 3.3895314e38,
                                       3.3961776e38, 3.4028235e38, -3.4028235e38])])
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_rne(float(v)) for v in f], dtype=np.uint16)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("base_bits", [0x3F80, 0x3F81, 0x4000, 0x0001, 0x0080, 0x7F7E, 0xBF80, 0xC123])
def test_bf16_rne_ties_and_near_ties_in_double(base_bits):
    # Midpoints between adjacent bf16 values, and points 2^-40 of a quantum either side:
    # a double-rounding oracle (fp64 -> fp32 -> bf16) gets the near-ties wrong.
    a = Fraction(bf16_bits_to_f64(np.array([base_bits]))[0])
    b = Fraction(bf16_bits_to_f64(np.array([base_bits + 1]))[0])
    mid = (a + b) / 2
    tiny = (b - a) * Fraction(1, 2**40)
    even = base_bits if base_bits % 2 == 0 else base_bits + 1
    away_from_zero = base_bits + 1      # |b| > |a| for these patterns
    toward_zero = base_bits
    assert oracle.bf16_rne(float(mid)) == even
    assert oracle.bf16_rne(float(mid + tiny)) == away_from_zero
    assert oracle.bf16_rne(float(mid - tiny)) == toward_zero


def test_bf16_rne_specials():
    assert oracle.bf16_rne(float("inf")) == 0x7F80
    assert oracle.bf16_rne(float("-inf")) == 0xFF80
    assert oracle.bf16_rne(0.0) == 0x0000
    assert oracle.bf16_rne(-0.0) == 0x8000
    nan = oracle.bf16_rne(float("nan"))
    assert (nan & 0x7F80) == 0x7F80 and (nan & 0x7F) != 0
    mx = float(Fraction(2**127) * (2 - Fraction(1, 128)))
    half_q = 2.0 ** (127 - 8)
    assert oracle.bf16_rne(mx) == 0x7F7F
    assert oracle.bf16_rne(mx + half_q) == 0x7F80          # tie rounds to even = infinity
    assert oracle.bf16_rne(mx + half_q * (1 - 2**-30)) == 0x7F7F
    assert oracle.bf16_rne(2.0 ** -133) == 0x0001          # smallest subnormal
    assert oracle.bf16_rne(2.0 ** -134) == 0x0000          # tie -> even (zero)
    assert oracle.bf16_rne(2.0 ** -134 * (1 + 2**-20)) == 0x0001
    assert oracle.bf16_rne(-3 * 2.0 ** -134) == 0x8002     # tie between 1 and 2 quanta -> 2


def test_special_values_follow_ieee():
    # c15: no special handling. A NaN reaches every statistic of its row; an infinity
    # gives LayerNorm inf - inf (NaN everywhere) but RMSNorm 1/sqrt(inf) = 0, so each
    # finite element's n is exactly 0 and y = shift, and the infinite element 0 * inf = NaN
    D = 16
    nan = lambda b: ((np.asarray(b) & 0x7F80) == 0x7F80) & ((np.asarray(b) & 0x7F) != 0)
    rng = np.random.default_rng(3)
    vals = exact_bits(np.round(rng.normal(size=D) * 8) / 8)
    shift = np.round(rng.normal(size=D) * 16) / 64
    scale = np.round(rng.normal(size=D) * 16) / 64
    for is_rms in (False, True):
        res = bf16_bits_to_f64(vals).copy()
        res[3] = np.nan
        out = one_row(res, scale=scale, shift=shift, is_rms=is_rms)
        assert nan(out["y"]).all() and nan(out["r"][0, 0, 3])
    res = bf16_bits_to_f64(vals).copy()
    res[5] = np.inf
    out = one_row(res, scale=scale, shift=shift, is_rms=False)
    assert nan(out["y"]).all() and out["r"][0, 0, 5] == 0x7F80
    out = one_row(res, scale=scale, shift=shift, is_rms=True)
    y = out["y"].reshape(-1)
    assert nan(y[5])
    keep = np.arange(D) != 5
    assert np.array_equal(y[keep], exact_bits(shift)[keep])
    # an overflowing residual + gate * x is an infinity in r
    big = float(Fraction(2**127) * (2 - Fraction(1, 128)))   # bf16 max
    res = bf16_bits_to_f64(vals).copy()
    xs = np.zeros(D)
    res[7], xs[7] = big, big
    out = one_row(res, x_vals=xs, gate_vals=np.ones(D), scale=scale, shift=shift, is_rms=True)
    assert out["r"][0, 0, 7] == 0x7F80 and nan(out["y"][0, 0, 7])


# --------------------------------------------------------------------------
# P1 constant rows, P2 +-a rows
# --------------------------------------------------------------------------

@pytest.mark.parametrize("c", [0.0, 1.0, -3.5, 0.15625, 96.0])
def test_p1_constant_row_layernorm_gives_shift_exactly(c):
    D = 64
    rng = np.random.default_rng(1)
    shift = bf16_bits_to_f64(f32_to_bf16_bits_rne(rng.normal(size=D).astype(np.float32)))
    scale = bf16_bits_to_f64(f32_to_bf16_bits_rne(rng.normal(size=D).astype(np.float32)))
    out = one_row([c] * D, scale=scale, shift=shift)
    assert np.all(out["n"] == 0.0)
    assert np.array_equal(out["y"][0, 0], exact_bits(shift))
    assert out["stats"][0, 0] == c and out["stats"][0, 1] == 0.0


@pytest.mark.parametrize("c", [1.0, -3.5, 0.001953125, 96.0])
def test_p1_constant_row_rms(c):
    D = 32
    out = one_row([c] * D, is_rms=True)
    want = mpmath.mpf(c) / mpmath.sqrt(mpmath.mpf(c) ** 2 + mpmath.mpf(EPS))
    assert np.allclose(out["n"][0, 0], float(want), rtol=1e-15, atol=0)


@pytest.mark.parametrize("is_rms", [False, True])
@pytest.mark.parametrize("a", [1.0, 0.25, 7.0, 0.0009765625])
def test_p2_plus_minus_a_row(is_rms, a):
    D = 40
    vals = np.array([a if i % 2 == 0 else -a for i in range(D)])
    out = one_row(vals, is_rms=is_rms)
    mag = mpmath.mpf(a) / mpmath.sqrt(mpmath.mpf(a) ** 2 + mpmath.mpf(EPS))
    want = np.where(vals > 0, float(mag), -float(mag))
    assert np.allclose(out["n"][0, 0], want, rtol=1e-15, atol=0)
    # unit RMS of n up to the eps factor a^2 / (a^2 + eps)
    assert abs(np.mean(out["n"][0, 0] ** 2) - float(mag**2)) < 1e-14


# --------------------------------------------------------------------------
# P3 moments on random and outlier rows (statistics computed independently by numpy)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("is_rms", [False, True])
def test_p3_moments_on_synthetic_rows(is_rms):
    w = synth.scaled(synth.W3, 2000)
    rows = np.concatenate([np.arange(40), w.outlier_rows()[:20]])
    spec = synth.Spec(is_rms=is_rms, has_gate=True, has_weight=False)
    out = oracle.run_workload_rows(w, spec, rows, want_n=True, want_stats=True)
    r = bf16_bits_to_f64(out["r"][0])
    n = out["n"][0]
    mean_r = r.mean(axis=1, dtype=np.float64)
    if is_rms:
        ms = np.mean(r * r, axis=1)
        np.testing.assert_allclose(np.mean(n * n, axis=1), ms / (ms + EPS), rtol=1e-12)
        np.testing.assert_allclose(n, r / np.sqrt(ms + EPS)[:, None], rtol=1e-13, atol=1e-15)
    else:
        var = np.var(r, axis=1)
        assert np.all(np.abs(n.mean(axis=1)) < 1e-12)
        np.testing.assert_allclose(np.var(n, axis=1), var / (var + EPS), rtol=1e-12)
        np.testing.assert_allclose(out["stats"][:, 0], mean_r, rtol=1e-13, atol=1e-15)
    # the outlier rows are really scaled by 50 (their spread is ~50x the others)
    sd = r.std(axis=1)
    assert np.all(sd[40:] > 20 * np.median(sd[:40]))


# --------------------------------------------------------------------------
# P4 identities of the modulation and gate wiring
# --------------------------------------------------------------------------

def _rand_bf16(rng, n, mu=0.0, sd=1.0):
    return bf16_bits_to_f64(f32_to_bf16_bits_rne((mu + sd * rng.normal(size=n)).astype(np.float32)))


def test_p4_modulation_identities():
    D = 96
    rng = np.random.default_rng(3)
    r = _rand_bf16(rng, D)
    s = _rand_bf16(rng, D, 0, 0.1)
    t = _rand_bf16(rng, D, 0, 0.1)
    base = one_row(r)                                   # scale = shift = 0
    n = base["n"][0, 0]
    assert all(nearest_bf16_ok(Fraction(v), int(b)) for v, b in zip(n, base["y"][0, 0]))
    shift_only = one_row(r, shift=t)
    assert all(nearest_bf16_ok(Fraction(v) + Fraction(tt), int(b))
               for v, tt, b in zip(n, t, shift_only["y"][0, 0]))
    scale_only = one_row(r, scale=s)
    assert all(nearest_bf16_ok(Fraction(v) * (1 + Fraction(ss)), int(b))
               for v, ss, b in zip(n, s, scale_only["y"][0, 0]))
    minus_one = one_row(r, scale=[-1.0] * D, shift=t)
    assert np.array_equal(minus_one["y"][0, 0], exact_bits(t))


def test_p4_affine_weight_and_bias():
    D = 48
    rng = np.random.default_rng(4)
    r, wt, bs = _rand_bf16(rng, D), _rand_bf16(rng, D, 1, 0.1), _rand_bf16(rng, D, 0, 0.1)
    s, t = _rand_bf16(rng, D, 0, 0.1), _rand_bf16(rng, D, 0, 0.1)
    out = one_row(r, weight=wt, bias=bs, scale=s, shift=t)
    n = out["n"][0, 0]
    for i in range(D):
        want = (Fraction(n[i]) * Fraction(wt[i]) + Fraction(bs[i])) * (1 + Fraction(s[i])) + Fraction(t[i])
        # fp64 evaluation of the same expression can sit one fp64 rounding away; accept
        # the bf16 nearest to the exact value unless the exact value is within 1e-12 of a tie
        if not nearest_bf16_ok(want, int(out["y"][0, 0, i])):
            b = int(out["y"][0, 0, i])
            v = Fraction(bf16_bits_to_f64(np.array([b]))[0])
            assert abs(abs(want - v) - abs(float(v) * 2**-9)) < 1e-12 * abs(float(v))
    # weight alone with scale = shift = 0 equals n * w
    only_w = one_row(r, weight=wt)
    assert all(nearest_bf16_ok(Fraction(n[i]) * Fraction(wt[i]), int(only_w["y"][0, 0, i]))
               for i in range(D))


def test_p4_gate_wiring():
    D = 64
    rng = np.random.default_rng(5)
    res, x, g = _rand_bf16(rng, D), _rand_bf16(rng, D), _rand_bf16(rng, D, 0, 0.5)
    zero_gate = one_row(res, x_vals=x, gate_vals=np.zeros(D))
    assert np.array_equal(zero_gate["r"][0, 0], exact_bits(res))
    zero_x = one_row(res, x_vals=np.zeros(D), gate_vals=g)
    assert np.array_equal(zero_x["r"][0, 0], exact_bits(res))
    no_gate = one_row(res, x_vals=x)
    unit_gate = one_row(res, x_vals=x, gate_vals=np.ones(D))
    assert np.array_equal(no_gate["r"], unit_gate["r"])
    assert np.array_equal(no_gate["y"], unit_gate["y"])
    gated = one_row(res, x_vals=x, gate_vals=g)
    for i in range(D):
        exact = Fraction(res[i]) + Fraction(g[i]) * Fraction(x[i])
        assert nearest_bf16_ok(exact, int(gated["r"][0, 0, i]))
    # swapping x and residual is not a symmetry once the gate is not 1
    swapped = one_row(x, x_vals=res, gate_vals=g)
    assert not np.array_equal(swapped["r"], gated["r"])


def test_residual_rounding_near_tie_from_a_tiny_residual():
    # gate * x = 1.75 * 0.578125 = 259/256, a midpoint between two bf16 values. A
    # residual of -2^-40 or +2^-40 decides the direction; 0 leaves a tie (-> even).
    D = 8
    g, x = [1.75] * D, [0.578125] * D
    for res, want in ((0.0, 1.015625), (2.0 ** -40, 1.015625), (-(2.0 ** -40), 1.0078125)):
        out = one_row([res] * D, x_vals=x, gate_vals=g)
        assert np.all(bf16_bits_to_f64(out["r"][0, 0]) == want)


def test_y_is_rounded_once():
    # RMSNorm with eps = 0 of a row of +-1 gives n = +-1 exactly, so y = n (1 + s) + t is
    # known exactly. With s = 2^-8 and t = 2^-40, y = 1 + 2^-8 + 2^-40 lies just above the
    # bf16 midpoint 1 + 2^-8 (between 1 and 1 + 2^-7), by far less than float32
    # resolution: one rounding gives 1 + 2^-7 (0x3F81); rounding through float32 first
    # lands on the tie and then on the even neighbour 1.0 (0x3F80). The negative
    # elements sit just inside the midpoint and round to -1.0 either way.
    D = 8
    r = np.array([1.0, -1.0] * (D // 2))
    out = one_row(r, scale=np.full(D, 2.0 ** -8), shift=np.full(D, 2.0 ** -40), is_rms=True,
                  eps=0.0)
    assert np.array_equal(out["n"].reshape(D), r)
    y = out["y"].reshape(D)
    assert np.array_equal(y, np.where(r > 0, 0x3F81, 0xBF80).astype(np.uint16))


def test_norm_only_equals_fused_with_zero_x():
    D = 80
    rng = np.random.default_rng(6)
    v, s, t, wt = _rand_bf16(rng, D), _rand_bf16(rng, D, 0, .1), _rand_bf16(rng, D, 0, .1), _rand_bf16(rng, D, 1, .1)
    for is_rms in (False, True):
        a = one_row(v, scale=s, shift=t, weight=wt, is_rms=is_rms, norm_only=True)
        b = one_row(v, scale=s, shift=t, weight=wt, is_rms=is_rms)
        assert a["r"] is None
        assert np.array_equal(a["y"], b["y"])
        assert np.array_equal(b["r"][0, 0], exact_bits(v))


# --------------------------------------------------------------------------
# P5 invariances (bf16-exact shifts and powers-of-two scales)
# --------------------------------------------------------------------------

def test_p5_shift_and_scale_invariance():
    D = 128
    rng = np.random.default_rng(8)
    base = rng.integers(-60, 61, size=D).astype(np.float64)     # exact in bf16
    n0 = one_row(base)["n"][0, 0]
    n_shift = one_row(base + 64.0)["n"][0, 0]                   # still exact (|.| <= 124)
    np.testing.assert_allclose(n_shift, n0, rtol=0, atol=1e-14)
    var = np.var(base)
    for alpha in (4.0, 0.25):
        n_a = one_row(base * alpha)["n"][0, 0]
        factor = np.sqrt(var + EPS) / np.sqrt(var + EPS / alpha**2)   # eps does not scale
        np.testing.assert_allclose(n_a, n0 * factor, rtol=1e-14, atol=1e-15)
        r_a = one_row(base * alpha, is_rms=True)["n"][0, 0]
        r_0 = one_row(base, is_rms=True)["n"][0, 0]
        ms = np.mean(base**2)
        np.testing.assert_allclose(r_a, r_0 * np.sqrt(ms + EPS) / np.sqrt(ms + EPS / alpha**2),
                                   rtol=1e-14, atol=1e-15)


# --------------------------------------------------------------------------
# P6 brute force on tiny rows, exact rationals + 60-digit square roots
# --------------------------------------------------------------------------

def _exact_n(vals, is_rms):
    fr = [Fraction(v) for v in vals]
    D = len(fr)
    if is_rms:
        second = sum(v * v for v in fr) / D
        mu = Fraction(0)
    else:
        mu = sum(fr) / D
        second = sum(v * v for v in fr) / D - mu * mu    # E[v^2] - E[v]^2, exact in rationals
    rho = 1 / mpmath.sqrt(mpmath.mpf(second.numerator) / second.denominator + mpmath.mpf(EPS))
    return [(mpmath.mpf((v - mu).numerator) / (v - mu).denominator) * rho for v in fr]


@pytest.mark.parametrize("D", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("is_rms", [False, True])
def test_p6_tiny_rows_brute_force(D, is_rms):
    rng = np.random.default_rng(100 + D)
    for _ in range(20):
        vals = _rand_bf16(rng, D, 0, 2.0)
        s, t = _rand_bf16(rng, D, 0, 0.1), _rand_bf16(rng, D, 0, 0.1)
        out = one_row(vals, scale=s, shift=t, is_rms=is_rms)
        want_n = _exact_n(vals, is_rms)
        for i in range(D):
            assert abs(out["n"][0, 0, i] - float(want_n[i])) <= 4e-16 * max(1.0, abs(float(want_n[i])))
            y_exact = want_n[i] * (1 + mpmath.mpf(s[i])) + mpmath.mpf(t[i])
            fy = Fraction(mpmath.nstr(y_exact, 50)) if y_exact != 0 else Fraction(0)
            b = int(out["y"][0, 0, i])
            if not nearest_bf16_ok(fy, b):
                # only acceptable when the exact value sits within fp64 noise of a tie
                v = Fraction(bf16_bits_to_f64(np.array([b]))[0])
                nb = [Fraction(bf16_bits_to_f64(np.array([(b + k) & 0xFFFF]))[0]) for k in (-1, 1)]
                gaps = [abs(abs(fy - v) - abs(fy - q)) for q in nb]
                assert min(gaps) < Fraction(1, 10**12) * max(abs(fy), Fraction(1, 10**30))


def test_p6_d1_and_d2_closed_forms():
    out = one_row([3.25])
    assert out["n"][0, 0, 0] == 0.0
    p, q = 1.5, -0.75
    out = one_row([p, q])
    h = (p - q) / 2
    want = float(mpmath.mpf(h) / mpmath.sqrt(mpmath.mpf(h) ** 2 + mpmath.mpf(EPS)))
    np.testing.assert_allclose(out["n"][0, 0], [want, -want], rtol=1e-15)


# --------------------------------------------------------------------------
# P8 library special case: torch CPU layer_norm / rms_norm in fp64
# --------------------------------------------------------------------------

@pytest.mark.parametrize("is_rms", [False, True])
def test_p8_matches_torch_norms(is_rms):
    w = synth.scaled(synth.W3B, 400)
    rows = np.arange(64)
    rows = np.concatenate([rows, w.outlier_rows()[:8]])
    spec = synth.Spec(is_rms=is_rms, has_gate=True, has_weight=False)
    out = oracle.run_workload_rows(w, spec, rows, want_n=True)
    r = torch.from_numpy(bf16_bits_to_f64(out["r"][0]))
    if is_rms:
        ref = torch.nn.functional.rms_norm(r, (w.D,), eps=EPS)
    else:
        ref = torch.nn.functional.layer_norm(r, (w.D,), eps=EPS)
    np.testing.assert_allclose(out["n"][0], ref.numpy(), rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# Operand resolution: strides for broadcast, per-row, per-frame and per-batch layouts
# --------------------------------------------------------------------------

@pytest.mark.parametrize("layouts", [("bcast",) * 3, ("row",) * 3, ("frame",) * 3, ("batch",) * 3,
                                     ("row", "frame", "bcast"), ("batch", "row", "frame"),
                                     ("bcast", "batch", "row")], ids=lambda l: "-".join(l))
def test_operand_layouts_match_explicit_gather(layouts):
    # gate, scale and shift each resolved through its own strides (mixed layouts catch an
    # operand read through another operand's strides)
    B, F, T, D = 2, 3, 4, 16
    L = F * T
    rng = np.random.default_rng(9)

    def rnd(n, sd=1.0):
        return f32_to_bf16_bits_rne((sd * rng.normal(size=(n, D))).astype(np.float32))

    n_stored = {"bcast": 1, "row": B * L, "frame": B * F, "batch": B}
    st = {op: synth.layout_strides(lay, B, L, D, F) for op, lay in zip(("gate", "scale", "shift"), layouts)}
    x, res = rnd(B * L), rnd(B * L)
    gate, sc, sh = (rnd(n_stored[lay], sd) for lay, sd in zip(layouts, (.5, .1, .1)))
    row_st = (L * D, 0, D)
    got = oracle.fused_norm(B, L, D, x=x, x_st=row_st, residual=res, res_st=row_st, gate=gate,
                            gate_st=st["gate"], scale=sc, scale_st=st["scale"], shift=sh,
                            shift_st=st["shift"], tokens_per_frame=T if "frame" in layouts else 0)

    def which(layout, b, l):   # the stored row token (b, l) reads, written out per layout
        return {"bcast": 0, "row": b * L + l, "frame": b * F + l // T, "batch": b}[layout]

    idx = [np.array([which(lay, b, l) for b in range(B) for l in range(L)]) for lay in layouts]
    want = oracle.fused_norm(1, B * L, D, x=x, x_st=(0, 0, D), residual=res, res_st=(0, 0, D),
                             gate=gate[idx[0]], gate_st=(0, 0, D), scale=sc[idx[1]],
                             scale_st=(0, 0, D), shift=sh[idx[2]], shift_st=(0, 0, D))
    assert np.array_equal(got["y"].reshape(-1, D), want["y"].reshape(-1, D))
    assert np.array_equal(got["r"].reshape(-1, D), want["r"].reshape(-1, D))


def test_oracle_rejects_bad_arguments():
    D = 8
    a = np.zeros((1, D), np.uint16)
    st = (D, 0, D)
    with pytest.raises(ValueError):
        oracle.fused_norm(1, 3, D, x=a, x_st=st, residual=a, res_st=st, scale=a, scale_st=st,
                          shift=a, shift_st=st, tokens_per_frame=2)


# --------------------------------------------------------------------------
# fp32 affine parameters (used as given, not cast to bf16)
# --------------------------------------------------------------------------

def test_fp32_affine_equal_to_bf16_when_representable():
    D = 64
    rng = np.random.default_rng(12)
    r, s, t = _rand_bf16(rng, D), _rand_bf16(rng, D, 0, .1), _rand_bf16(rng, D, 0, .1)
    wt, bs = _rand_bf16(rng, D, 1, .1), _rand_bf16(rng, D, 0, .1)   # bf16-exact values
    a = one_row(r, scale=s, shift=t, weight=wt, bias=bs)
    st = (D, 0, D)
    b = oracle.fused_norm(1, 1, D, x=exact_bits(np.zeros(D)), x_st=st, residual=exact_bits(r), res_st=st,
                          weight=wt.astype(np.float32), bias=bs.astype(np.float32),
                          scale=exact_bits(s), scale_st=st, shift=exact_bits(t), shift_st=st, eps=EPS)
    assert np.array_equal(a["y"], b["y"])


def test_fp32_affine_against_exact_rationals():
    D = 48
    rng = np.random.default_rng(13)
    r, s, t = _rand_bf16(rng, D), _rand_bf16(rng, D, 0, .1), _rand_bf16(rng, D, 0, .1)
    wt = (1 + 0.1 * rng.normal(size=D)).astype(np.float32)          # 24-bit values
    bs = (0.1 * rng.normal(size=D)).astype(np.float32)
    st = (D, 0, D)
    out = oracle.fused_norm(1, 1, D, x=exact_bits(np.zeros(D)), x_st=st, residual=exact_bits(r),
                            res_st=st, weight=wt, bias=bs, scale=exact_bits(s), scale_st=st,
                            shift=exact_bits(t), shift_st=st, eps=EPS, want_n=True)
    n = out["n"][0, 0]
    nonexact = 0
    for i in range(D):
        want = (Fraction(n[i]) * Fraction(float(wt[i])) + Fraction(float(bs[i]))) * (1 + Fraction(s[i])) + Fraction(t[i])
        if not nearest_bf16_ok(want, int(out["y"][0, 0, i])):
            nonexact += 1
    assert nonexact == 0
    # and the fp32 values really carry more than bf16 precision here
    assert not np.array_equal(bf16_bits_to_f64(f32_to_bf16_bits_rne(wt)), wt.astype(np.float64))
