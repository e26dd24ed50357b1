"""Reader for the hand-computed fixtures under tests/golden/."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, rest = line.split(":", 1)
            vals[key.strip()] = np.array([float(x) for x in rest.split()], dtype=np.float64)
    N = int(vals.pop("N")[0])
    T = int(vals.pop("T")[0])
    out = {"N": N, "T": T}
    for key, arr in vals.items():
        if key in ("s0", "sT", "dsT", "ds0"):
            out[key] = arr.reshape(1, 1, N, N)
        else:
            out[key] = arr.reshape(1, T, 1, N)
    return out
