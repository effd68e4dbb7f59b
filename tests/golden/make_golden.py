"""Write tests/golden/oracle_digests.json: sha256 of the oracle's outputs on small
seeded slices of every workload and specialisation.

Calls only the oracle and the seeded input generator. Rerun it only when a change
to the oracle's arithmetic is justified by the pages (and say which passage in the
commit message); the digest test fails until then.
"""
import hashlib
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

ROWS = 24


def _slice_rows(w):
    rows = list(range(0, min(w.rows, ROWS // 2)))
    rows += list(range(max(w.rows - ROWS // 2, 0), w.rows))
    rows += [int(r) for r in w.outlier_rows()[:4]]
    return np.array(sorted(set(rows)), dtype=np.int64)


def digest_cases():
    out = {}
    for w in synth.WORKLOADS.values():
        rows = _slice_rows(w)
        specs = list(w.specs) + [synth.Spec(False, False, True, has_bias=True),
                                 synth.Spec(True, False, True, norm_only=True)]
        for spec in specs:
            res = oracle.run_workload_rows(w, spec, rows)
            h = hashlib.sha256(res["y"].tobytes())
            if res["r"] is not None:
                h.update(res["r"].tobytes())
            out[f"{w.name}/{spec.name}"] = h.hexdigest()
    return out


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_digests.json")
    with open(path, "w") as f:
        json.dump({"rows_per_case": ROWS, "digests": digest_cases()}, f, indent=1, sort_keys=True)
    print(path)
