"""Write tests/golden/small_case.json from the fp64 oracle (regression fixture).

The pages print no worked numeric example for the gated delta rule, so this
file holds no page values: it is the oracle's own output on a small seeded
case, written by this script (which calls only ``oracle/``), so that any later
change to the oracle's arithmetic shows up as a diff in review.

Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402


def case():
    rng = np.random.default_rng(2024)
    T, nqk, nv, dk, dv = 10, 1, 2, 4, 3
    q = np.round(rng.standard_normal((T, nqk, dk)), 3)
    k = np.round(rng.standard_normal((T, nqk, dk)), 3)
    v = np.round(rng.standard_normal((T, nv, dv)), 3)
    g = -np.round(rng.uniform(0.0, 1.0, (T, nv)), 3)
    beta = np.round(rng.uniform(0.0, 1.0, (T, nv)), 3)
    s0 = np.round(0.1 * rng.standard_normal((2, nv, dk, dv)), 3)
    cu = np.array([0, 7, 10], dtype=np.int32)
    return dict(q=q, k=k, v=v, g=g, beta=beta, initial_state=s0, cu_seqlens=cu)


def main():
    c = case()
    out, sf = oracle.recurrent(**c)
    doc = {
        "what": "oracle.recurrent on case() of make_golden.py (two sequences, GQA 1:2)",
        "inputs": {k: (v.tolist() if v is not None else None) for k, v in c.items()},
        "out": out.tolist(),
        "final_state": sf.tolist(),
    }
    with open(os.path.join(HERE, "small_case.json"), "w") as f:
        json.dump(doc, f, indent=1)


if __name__ == "__main__":
    main()
