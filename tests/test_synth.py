"""The seeded input generator: reproducible, sliceable, and drawing the stated
distributions; the workload byte counts match the stated algorithmic traffic."""
import math

import numpy as np
import pytest

import synth
from helpers import bf16_bits_to_f64


def test_slices_match_full_fill():
    w = synth.scaled(synth.W3, 300)
    full = w.generate("x")
    part = synth.fill(np.empty((50, w.D), np.uint16), 120, w.seed, "x", 0.0, 1.0,
                      w.row_mult(np.arange(120, 170)))
    assert np.array_equal(full[120:170], part)
    rows = np.array([5, 299, 0, 5, 77])
    assert np.array_equal(w.generate("x", rows), full[rows])
    for (r, c) in [(0, 0), (5, 1), (77, 5119), (299, 4000)]:
        mult = 50.0 if r in set(w.outlier_rows()) else 1.0
        assert synth.value(r, c, w.seed, "x", 0.0, 1.0, mult) == full[r, c]


def test_streams_are_distinct_and_seeded():
    w = synth.W1
    a = w.generate("scale")
    b = w.generate("shift")
    assert not np.array_equal(a, b)
    w2 = synth.W2
    assert not np.array_equal(w.generate("x"), w2.generate("x")[:16])
    assert np.array_equal(w.generate("x"), w.generate("x"))


@pytest.mark.parametrize("tensor,mu,sd", [("x", 0, 1), ("residual", 0, 1), ("gate", 0, .5),
                                          ("weight", 1, .1), ("scale", 0, .1), ("shift", 0, .1)])
def test_distributions(tensor, mu, sd):
    v = bf16_bits_to_f64(synth.fill(np.empty((64, 5120), np.uint16), 0, 42, tensor, mu, sd))
    assert abs(v.mean() - mu) < 5 * sd / math.sqrt(v.size) + 1e-3 * abs(mu)
    assert abs(v.std() / sd - 1) < 0.01
    # roughly normal: ~68.3% within one standard deviation
    assert abs(np.mean(np.abs(v - mu) < sd) - 0.6827) < 0.01


def test_outlier_rows():
    w = synth.W3
    rows = w.outlier_rows()
    assert len(rows) == 900 and len(set(rows.tolist())) == 900
    assert rows.min() >= 0 and rows.max() < w.rows
    x = bf16_bits_to_f64(w.generate("x", rows[:10]))
    plain = bf16_bits_to_f64(synth.fill_rows(np.empty((10, w.D), np.uint16), rows[:10], w.seed, "x", 0.0, 1.0))
    np.testing.assert_allclose(x, plain * 50.0, rtol=2 ** -7)


def test_layout_strides_and_rows():
    assert synth.layout_strides("bcast", 1, 10, 8, 0) == (0, 0, 0)
    assert synth.layout_strides("row", 2, 10, 8, 0) == (80, 0, 8)
    assert synth.layout_strides("frame", 2, 10, 8, 5) == (40, 8, 0)
    assert synth.layout_strides("batch", 2, 10, 8, 0) == (8, 0, 0)
    w = synth.W5
    toks = np.array([0, 8399, 8400, 176399])
    assert synth.W5.token_rows("gate", toks).tolist() == [0, 0, 1, 20]


def test_algorithmic_bytes():
    assert synth.W4.algorithmic_bytes(synth.W4.specs[0]) == 10_838_026_240
    assert synth.W1.algorithmic_bytes(synth.W1.specs[0]) == 696_320
    assert synth.W5.algorithmic_bytes(synth.W5.specs[0]) == 7_225_999_360
    assert synth.W3.algorithmic_bytes(synth.Spec(False, True, True)) == 5_529_620_480
    assert synth.W3B.algorithmic_bytes(synth.Spec(False, True, True)) == 11_059_240_960
    assert synth.W2.algorithmic_bytes(synth.Spec(False, True, False)) == 1_658_880
    assert synth.W2.algorithmic_bytes(synth.Spec(False, False, False)) == 1_331_200
