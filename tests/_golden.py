"""Reader for the hand-worked fixtures in tests/golden (``key = values`` lines,
rows separated by ``|``, ``#`` starts a comment)."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name: str) -> dict:
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = (s.strip() for s in line.split("=", 1))
            rows = [[float(x) for x in r.split()] for r in val.split("|")]
            arr = np.array(rows[0] if len(rows) == 1 else rows, dtype=np.float64)
            out[key] = float(arr[0]) if arr.shape == (1,) else arr
    return out
