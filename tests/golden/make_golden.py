"""Writes oracle_small.json: small seeded cases and the oracle's outputs for them.

Calls only the oracle.  The file is a regression pin: any later change to the
oracle's arithmetic that moves these values must say, in its commit message,
which passage of the pages (or which reading of it) justifies the change.
Run from the repository root:  python tests/golden/make_golden.py
"""

import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))

from oracle import attention_bwd_ref, attention_fwd_ref  # noqa: E402


def main():
    rng = np.random.default_rng(20240601)
    cases = []
    for name, (n, d, scale, causal) in {
        "n5_d3_noncausal": (5, 3, 0.6, False),
        "n7_d4_causal": (7, 4, 0.5, True),
        "n9_d2_causal_stress": (9, 2, 2.0, True),
    }.items():
        q, k, v, do = (np.round(rng.standard_normal((1, 2, n, d)), 3) for _ in range(4))
        o, lse = attention_fwd_ref(q, k, v, scale, causal)
        dq, dk, dv = attention_bwd_ref(q, k, v, do, scale, causal)
        cases.append({
            "name": name, "scale": scale, "causal": causal,
            "q": q.tolist(), "k": k.tolist(), "v": v.tolist(), "do": do.tolist(),
            "o": o.tolist(), "lse": lse.tolist(), "dq": dq.tolist(), "dk": dk.tolist(), "dv": dv.tolist(),
        })
    out = {
        "source": "tests/golden/make_golden.py (oracle only); inputs rounded to 3 decimals",
        "cases": cases,
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=0)
        f.write("\n")


if __name__ == "__main__":
    main()
