"""Reader for tests/golden/hand_cases.txt (hand-derived worked cases)."""
import os

import numpy as np

from helpers import bf16_bits_to_f64, f32_to_bf16_bits_rne

PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_cases.txt")
KEYS = ("norm", "residual", "x", "gate", "scale", "shift", "want_r", "want_y")


def _bits(tokens):
    f = np.array([float(t) for t in tokens], dtype=np.float64)
    b = f32_to_bf16_bits_rne(f.astype(np.float32))
    if not np.array_equal(bf16_bits_to_f64(b), f):
        raise ValueError(f"golden value not exact in bf16: {tokens}")
    return b


def load():
    cases, cur = [], None
    for line in open(PATH):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("case "):
            cur = {"name": line.split(None, 1)[1]}
            cases.append(cur)
            continue
        key, _, rest = line.partition(":")
        key, toks = key.strip(), rest.split()
        assert key in KEYS, key
        if key == "norm":
            cur["is_rms"] = toks[0] == "rms"
        elif toks == ["-"]:
            cur[key] = None
        else:
            cur[key] = _bits(toks)
    for c in cases:
        assert all(k in c for k in KEYS[1:]) and "is_rms" in c, c["name"]
    return cases


def tiled(case, D):
    """The case's pattern repeated to D channels (D must be a multiple of its length)."""
    P = len(case["residual"])
    assert D % P == 0
    out = dict(case)
    for k in KEYS[1:]:
        if case[k] is not None:
            out[k] = np.tile(case[k], D // P)
    return out
