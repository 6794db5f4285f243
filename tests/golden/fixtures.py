"""Reader for the hand-worked text fixtures in this directory.

Each fixture is `name value value ...` lines; `#` starts a comment line.
"""

import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def load(name: str) -> dict:
    out = {}
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = np.array([float(v) for v in vals], dtype=np.float64)
    return out
