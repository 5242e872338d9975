"""Reader for the worked-example fixtures under tests/golden/.

Each fixture is a text file: '#' lines hold the citation and the reading of the
example; every other line is ``name = numbers`` with ';' between matrix rows.
"""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_golden(name: str) -> dict:
    out = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = (s.strip() for s in line.split("=", 1))
            rows = [[float(x) for x in r.split()] for r in val.split(";")]
            a = np.array(rows, dtype=np.float64)
            out[key] = a[0] if a.shape[0] == 1 else a
    return out
