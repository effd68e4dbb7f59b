"""The kernel's rounding rule for y, emulated on the CPU with exact IEEE arithmetic.

The kernel evaluates y = n (1 + scale) + shift in fp32 with the fp64 row statistics
rounded to fp32, together with a bound B = 8 u P on its error (u = 2^-24,
P = |1+s| (|w| kappa + |n w| + |b|) + |shift|, kappa = |mean| rho). It widens y to the
interval [RD(y - B), RU(y + B)] (ends rounded down and up) and takes the bf16 rounding
of the upper end when both ends round to the same bf16 value; every other element is
recomputed in fp64. This test replays those fp32 operations one by one (numpy float32
arithmetic rounds each operation to nearest; fused multiply-adds are done exactly and
rounded once, to nearest or in the stated direction) and checks, over rows built to be
hard (means far above the spread, tiny and huge spreads, shift nearly cancelling
n (1 + scale)), that every element the rule lets through rounds exactly like the fp64
evaluation of the formula (round to odd into fp32, then to nearest even), as the
fallback path computes it.

It exercises the design of the check, not the compiled kernel (the GPU parity tests do
that); it shares nothing with the oracle.
"""
import numpy as np

F32 = np.float32


def _bf16_rne(a: np.ndarray) -> np.ndarray:
    """float32 array -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return (((u + 0x7FFF + ((u >> 16) & 1)) >> 16) & 0xFFFF).astype(np.uint16)


def _to_bf16_values(x) -> np.ndarray:
    """Round float64 samples to bf16 and return them as float64 values."""
    bits = _bf16_rne(np.asarray(x, dtype=np.float64).astype(np.float32)).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def _f32_round_odd_then_f32(x: np.ndarray, err: np.ndarray) -> np.ndarray:
    """x + err (x = RN64 of an exact value, err its exact remainder) rounded once to
    float32: round to odd at fp64 precision, then to nearest float32 (53 >= 24 + 2)."""
    x = np.asarray(x, dtype=np.float64)
    # truncation toward zero of the exact value, at fp64 precision
    away = (err != 0) & (np.sign(err) != np.sign(x)) & (x != 0)
    trunc = np.where(away, np.nextafter(x, 0.0), x)
    inexact = err != 0
    bits = trunc.view(np.uint64) | inexact.astype(np.uint64)
    return bits.view(np.float64).astype(np.float32)


def _fma_exact(a, b, c):
    """a * b + c for float32 operands as (RN64 value, exact remainder)."""
    p = a.astype(np.float64) * b.astype(np.float64)      # exact: 24 + 24 bits
    c64 = c.astype(np.float64)
    s = p + c64                                          # TwoSum: exact remainder
    bp = s - c64
    err = (p - bp) + (c64 - (s - bp))
    return s, err


def _fma32(a, b, c) -> np.ndarray:
    """fmaf: a * b + c for float32 operands with a single rounding to nearest float32."""
    return _f32_round_odd_then_f32(*_fma_exact(a, b, c))


def _fma32_directed(a, b, c, up: bool) -> np.ndarray:
    """fmaf with one rounding toward +inf (up) or -inf: __fmaf_ru / __fmaf_rd."""
    s, err = _fma_exact(a, b, c)
    f = s.astype(np.float32)
    diff = s - f.astype(np.float64)                      # exact (f is within an fp32 ulp of s)
    sign = np.where(diff != 0, np.sign(diff), np.sign(err))   # sign of exact - f
    if up:
        return np.where(sign > 0, np.nextafter(f, np.float32(np.inf)), f).astype(np.float32)
    return np.where(sign < 0, np.nextafter(f, np.float32(-np.inf)), f).astype(np.float32)


def _bf16_from_double(v: np.ndarray) -> np.ndarray:
    """The fallback's rounding: round to odd into float32, then to nearest even bf16."""
    f = v.astype(np.float32)
    f64 = f.astype(np.float64)
    # f is RN; the remainder v - f is exact in fp64 for |v| in float32 range
    return _bf16_rne(_f32_round_odd_then_f32(f64, v - f64))


def _fast_path(v, s, t, w, b, mu, rho, k=F32(2.0 ** -21)):
    """The kernel's fp32 evaluation of y, its interval and its decision: returns the
    bf16 result of the fast path and whether the element goes to the fp64 path."""
    neg_mu = F32(-mu)
    rho32 = F32(rho)
    kappa = F32(abs(neg_mu) * rho32)
    n = (v.astype(F32) + neg_mu) * rho32
    nw = n * w.astype(F32) if w is not None else n
    nb = nw + b.astype(F32) if b is not None else nw
    a = s.astype(F32) + F32(1)
    t32 = t.astype(F32)
    y = _fma32(nb, a, t32)
    if w is not None:
        inner = _fma32(np.abs(w.astype(F32)), np.full_like(nw, kappa), np.abs(nw))
    else:
        inner = kappa + np.abs(nw)
    if b is not None:
        inner = inner + np.abs(b.astype(F32))
    p = _fma32(np.abs(a), inner, np.abs(t32))
    lo = _fma32_directed(p, np.full_like(p, -k), y, up=False)
    hi = _fma32_directed(p, np.full_like(p, k), y, up=True)
    out = _bf16_rne(hi)
    return out, _bf16_rne(lo) != out


def _fp64_formula(v, s, t, w, b, mu, rho):
    """The formula in fp64, in the fallback's order."""
    n = (v - mu) * rho
    if w is not None:
        n = n * w
    if b is not None:
        n = n + b
    return n * (1.0 + s) + t


def _rows(rng, trials, D):
    """Rows of (v, s, t, w, b, mean, rho, kind); kind is "cancel" when the shift nearly
    cancels n (1 + scale), "offset" when the mean exceeds one spread (the larger the
    ratio, the less the fp32 subtraction resolves and the more the rule sends to fp64),
    else "centred" (the shape of the workloads' activations)."""
    for trial in range(trials):
        spread = 10.0 ** rng.uniform(-3, 3)
        offset = rng.choice([0.0, 1.0, 100.0, 1e4, 1e5]) * rng.normal()
        v = _to_bf16_values(offset + spread * rng.normal(size=D))
        s = _to_bf16_values(rng.choice([0.1, 1.0, 3.0]) * rng.normal(size=D))
        w = _to_bf16_values(1 + 0.1 * rng.normal(size=D)) if trial % 2 else None
        b = _to_bf16_values(0.1 * rng.normal(size=D)) if trial % 3 == 0 else None
        mu = float(np.mean(v))
        rho = 1.0 / np.sqrt(float(np.var(v)) + 1e-6)
        if trial % 3 == 1:      # shift nearly cancels n (1 + scale)
            n = (v - mu) * rho * (w if w is not None else 1.0) + (b if b is not None else 0.0)
            t = _to_bf16_values(-(n * (1 + s)) * (1 + 1e-3 * rng.normal(size=D)))
        else:
            t = _to_bf16_values(rng.choice([0.1, 1.0, 10.0]) * rng.normal(size=D))
        kind = ("cancel" if trial % 3 == 1 else
                "offset" if abs(mu) > np.sqrt(float(np.var(v))) else "centred")
        yield v, s, t, w, b, mu, rho, kind


def test_fma_emulation_rounds_once():
    # 2^36 + 1 = 1774001 * 38737, so a * b = 2^-24 + 2^-60 exactly and a * b + 1 lies just
    # above the float32 tie 1 + 2^-24: one rounding gives 1 + 2^-23, while rounding to fp64
    # first lands on the tie and then rounds to even (1.0)
    a = np.array([1774001 * 2.0 ** -44], dtype=np.float32)
    b = np.array([38737 * 2.0 ** -16], dtype=np.float32)
    one = np.array([1.0], dtype=np.float32)
    assert float(a[0]) * 2 ** 44 == 1774001 and float(b[0]) * 2 ** 16 == 38737
    assert (a.astype(np.float64) * b.astype(np.float64) + 1.0).astype(np.float32)[0] == 1.0
    assert _fma32(a, b, one)[0] == np.float32(1 + 2.0 ** -23)
    assert _fma32(-a, b, -one)[0] == np.float32(-(1 + 2.0 ** -23))
    # exactly on the tie: nearest even
    c = np.array([2.0 ** -24], dtype=np.float32)
    assert _fma32(c, one, one)[0] == np.float32(1.0)
    assert _fma32(c, np.array([3.0], dtype=np.float32), one)[0] == np.float32(1 + 2.0 ** -22)


def test_directed_fma_emulation():
    # 1 + 2^-30: rounds down to 1, up to 1 + 2^-23; an exact result stays put
    one = np.array([1.0], dtype=np.float32)
    tiny = np.array([2.0 ** -30], dtype=np.float32)
    assert _fma32_directed(tiny, one, one, up=False)[0] == np.float32(1.0)
    assert _fma32_directed(tiny, one, one, up=True)[0] == np.float32(1 + 2.0 ** -23)
    assert _fma32_directed(-tiny, one, one, up=False)[0] == np.float32(1 - 2.0 ** -24)
    assert _fma32_directed(-tiny, one, one, up=True)[0] == np.float32(1.0)
    half = np.array([0.5], dtype=np.float32)
    for up in (False, True):
        assert _fma32_directed(half, half, one, up=up)[0] == np.float32(1.25)


def test_interval_rule_never_lets_a_misrounding_through():
    rng = np.random.default_rng(20260)
    D = 4096
    total = {"centred": 0, "offset": 0, "cancel": 0}
    flagged = dict(total)
    for v, s, t, w, b, mu, rho, kind in _rows(rng, 300, D):
        fast, near = _fast_path(v, s, t, w, b, mu, rho)
        ok = ~near
        want = _bf16_from_double(_fp64_formula(v, s, t, w, b, mu, rho)[ok])
        bad = np.flatnonzero(fast[ok] != want)
        assert bad.size == 0, (f"fast path misrounds {bad.size} elements, e.g. v={v[ok][bad[0]]!r} "
                               f"s={s[ok][bad[0]]!r} t={t[ok][bad[0]]!r}")
        total[kind] += D
        flagged[kind] += int(near.sum())
    # every kind of row is represented
    assert min(total.values()) >= 20 * D, total
    # on centred rows the rule sends only a small share of elements to the fp64 path
    assert flagged["centred"] / total["centred"] < 2e-3, flagged["centred"] / total["centred"]


def test_interval_rule_detects_a_tight_bound():
    # with the bound divided by 64 the rule must let misroundings through on the same
    # rows (the check above would catch a bound that is too small)
    rng = np.random.default_rng(20260)
    D = 4096
    misrounded = 0
    for v, s, t, w, b, mu, rho, _ in _rows(rng, 60, D):
        fast, near = _fast_path(v, s, t, w, b, mu, rho, k=F32(2.0 ** -27))
        ok = ~near
        want = _bf16_from_double(_fp64_formula(v, s, t, w, b, mu, rho)[ok])
        misrounded += int((fast[ok] != want).sum())
    assert misrounded > 0
