"""The oracle reproduces the hand-derived worked cases in tests/golden/, bit for bit,
at the pattern's own width and tiled to the kernel widths 5120 and 10240; and its
outputs on small seeded workloads still match the digests recorded by
tests/golden/make_golden.py (a change to the oracle's arithmetic shows up here)."""
import json
import os

import numpy as np
import pytest

import oracle
import golden_cases
from golden.make_golden import digest_cases

CASES = golden_cases.load()


def _run(case):
    D = len(case["residual"])
    st = (D, 0, D)
    return oracle.fused_norm(1, 1, D, x=case["x"], x_st=st, residual=case["residual"],
                             res_st=st, gate=case["gate"],
                             gate_st=st if case["gate"] is not None else None,
                             scale=case["scale"], scale_st=st, shift=case["shift"], shift_st=st,
                             is_rms=case["is_rms"], eps=1e-6)


@pytest.mark.parametrize("width", [None, 5120, 10240])
@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_hand_case(case, width):
    c = case if width is None else golden_cases.tiled(case, width)
    out = _run(c)
    assert np.array_equal(out["r"][0, 0], c["want_r"])
    assert np.array_equal(out["y"][0, 0], c["want_y"])


def test_oracle_digests_unchanged():
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_digests.json")
    stored = json.load(open(path))
    assert digest_cases() == stored["digests"]
