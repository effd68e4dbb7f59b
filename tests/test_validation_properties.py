"""What fused_norm_validate's acceptance guarantees, checked on random calls (host only).

The kernel writes every output row from one CTA and reads its inputs freely, so an
accepted call must have: output rows that never share a byte (y rows among themselves,
r rows among themselves, y against r), and no output byte that any input row or the
affine vectors occupy, except r aliasing the residual element for element (the in-place
update, where each element is read and then written by the same thread). Hypothesis
draws small problems (the row count is what matters; D is the real 5120) with strides
and base addresses chosen to make overlaps likely; every accepted call is checked by
enumerating the byte interval of each row.
"""
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import rmsnorm_row_b200 as fn

D = 5120
ROW = 2 * D                    # bytes in one bf16 row
BASE = 1 << 40                 # dummy device addresses (never dereferenced on the host)


def _intervals(ptr, sb, sf, sl, B, L, tpf, nbytes=ROW):
    out = []
    for b in range(B):
        for l in range(L):
            f = l // tpf if tpf else 0
            start = ptr + 2 * (b * sb + f * sf + l * sl)
            out.append(((b, l), start, start + nbytes))
    return out


def _disjoint(a, b):
    return a[2] <= b[1] or b[2] <= a[1]


strides = st.sampled_from([0, 8, D // 2, D, D + 8, 2 * D, 3 * D, 7 * D])
offsets = st.sampled_from([0, 8, 16, ROW // 2, ROW, 2 * ROW, 5 * ROW, 13 * ROW])
REGION = 1 << 30               # far larger than any extent drawn here


@st.composite
def calls(draw):
    B = draw(st.integers(1, 3))
    L = draw(st.integers(1, 6))
    tpf = draw(st.sampled_from([0] + [t for t in range(1, L + 1) if L % t == 0]))
    names = ("x", "residual", "gate", "scale", "shift", "y", "r", "weight")

    def place(i):
        # its own region, or (sometimes) another buffer's region, so overlaps are possible
        region = draw(st.integers(0, len(names) - 1)) if draw(st.integers(0, 3)) == 0 else i
        return BASE + region * REGION + draw(offsets)

    ops = {}
    for i, name in enumerate(names[:5]):
        ops[name] = (place(i), draw(strides), draw(strides) if tpf else 0, draw(strides))
    y = (place(5), draw(strides), draw(strides))
    if draw(st.integers(0, 3)) == 0:     # propose the in-place residual update
        p, sb, _, sl = ops["residual"]
        r = (p, sb, sl)
        ops["residual"] = (p, sb, 0, sl)
    else:
        r = (place(6), draw(strides), draw(strides))
    w = place(7)
    return B, L, tpf, ops, y, r, w


def _args(B, L, tpf, ops, y, r, w):
    a = fn.fn_args()
    a.B, a.L, a.tokens_per_frame = B, L, tpf
    for name, (p, sb, sf, sl) in ops.items():
        setattr(a, name, fn.fn_operand(p, sb, sf, sl))
    a.weight = w
    a.y, a.y_stride_b, a.y_stride_l = y
    a.r, a.r_stride_b, a.r_stride_l = r
    return a


_handle = None


def _h():
    global _handle
    if _handle is None:
        st_, h = fn.fused_norm_create(fn.fn_config(D=D, has_gate=1, has_weight=1, eps=1e-6))
        assert st_ == fn.FN_OK
        _handle = h
    return _handle


@settings(max_examples=4000, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(calls())
def test_accepted_calls_have_no_write_hazards(call):
    B, L, tpf, ops, y, r, w = call
    status = fn.fused_norm_validate(_h(), _args(*call))
    if status != fn.FN_OK:
        return
    ys = _intervals(y[0], y[1], 0, y[2], B, L, 0)
    rs = _intervals(r[0], r[1], 0, r[2], B, L, 0)
    ins = {name: _intervals(p, sb, sf, sl, B, L, tpf) for name, (p, sb, sf, sl) in ops.items()}
    ins["weight"] = [((0, 0), w, w + ROW)]
    # output rows: pairwise disjoint within y, within r, and between y and r
    for outs in (ys, rs):
        for i in range(len(outs)):
            for j in range(i + 1, len(outs)):
                assert _disjoint(outs[i], outs[j]), ("output rows overlap", outs[i], outs[j])
    for a in ys:
        for b in rs:
            assert _disjoint(a, b), ("y and r overlap", a, b)
    # no output byte is an input byte, except r on the residual element for element
    for name, rows in ins.items():
        for o in ys:
            for i in rows:
                assert _disjoint(o, i), ("y overlaps", name, o, i)
        for o in rs:
            for i in rows:
                if _disjoint(o, i):
                    continue
                assert name == "residual" and o[0] == i[0] and o[1] == i[1], ("r overlaps", name, o, i)


def test_generator_reaches_accepted_and_rejected_calls():
    # the strategy is only useful if both outcomes occur often
    seen = {"ok": 0, "rejected": 0, "ok_in_place": 0}

    @settings(max_examples=1500, deadline=None)
    @given(calls())
    def probe(call):
        ok = fn.fused_norm_validate(_h(), _args(*call)) == fn.FN_OK
        seen["ok" if ok else "rejected"] += 1
        if ok and call[5][0] == call[3]["residual"][0]:
            seen["ok_in_place"] += 1

    probe()
    assert seen["ok"] >= 30 and seen["rejected"] >= 30 and seen["ok_in_place"] >= 5, seen
