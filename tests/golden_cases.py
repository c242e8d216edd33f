"""Loader for the stored oracle fixtures in tests/golden/."""
import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_all():
    with open(os.path.join(GOLDEN, "oracle_small.json")) as f:
        data = json.load(f)
    cases = []
    for rec in data["cases"]:
        B, H, T, dk, dv = rec["shape"]
        shapes = {"q": (B, H, T, dk), "k": (B, H, T, dk), "v": (B, H, T, dv),
                  "beta": (B, H, T), "S0": (B, H, dk, dv), "o": (B, H, T, dv),
                  "S_T": (B, H, dk, dv)}
        case = {"name": rec["name"]}
        for key, shp in shapes.items():
            case[key] = None if rec[key] is None else np.array(rec[key], np.float64).reshape(shp)
        cases.append(case)
    return cases
