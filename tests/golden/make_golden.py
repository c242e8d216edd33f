"""Write tests/golden/oracle_small.json: small seeded inputs and the fp64 oracle's outputs.

A regression fixture: it calls only the oracle package, so a later change to the oracle's
arithmetic shows up as a diff here (and must be justified by the passage it follows).
Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402

CASES = [
    # name, B, H, T, dk, dv, key scale, with S0, seed
    ("unit_scale", 1, 2, 6, 4, 3, 1.0, True, 11),
    ("stiff_keys", 1, 1, 5, 3, 3, 30.0, False, 12),
    ("tiny_keys", 2, 1, 4, 2, 5, 1e-4, True, 13),
]


def draw(B, H, T, dk, dv, scale, s0, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, T, dk))
    k = scale * rng.standard_normal((B, H, T, dk))
    v = rng.standard_normal((B, H, T, dv))
    beta = rng.uniform(0.0, 1.0, (B, H, T))
    S0 = rng.standard_normal((B, H, dk, dv)) if s0 else None
    return q, k, v, beta, S0


def main():
    out = []
    for name, B, H, T, dk, dv, scale, s0, seed in CASES:
        q, k, v, beta, S0 = draw(B, H, T, dk, dv, scale, s0, seed)
        o, ST = oracle.fwd(q, k, v, beta, S0, threads=1)
        rec = {"name": name, "shape": [B, H, T, dk, dv]}
        for key, arr in (("q", q), ("k", k), ("v", v), ("beta", beta), ("S0", S0),
                         ("o", o), ("S_T", ST)):
            rec[key] = None if arr is None else [float(x) for x in np.ravel(arr)]
        out.append(rec)
    with open(os.path.join(HERE, "oracle_small.json"), "w") as f:
        json.dump({"source": "tests/golden/make_golden.py (fp64 oracle, row convention)",
                   "cases": out}, f, indent=0)


if __name__ == "__main__":
    main()
