"""Reader for the hand-worked fixtures under tests/golden/.

Each fixture is ``key: value`` lines; values are Python literals in which the
name ``e`` stands for Euler's number, so closed-form entries such as
``(e+3)/(e+1)`` are evaluated here, not by the oracle.
"""
import math
import os

import numpy as np

from gqe_inputs import Dims

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name: str) -> dict:
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            key, val = key.strip(), val.strip()
            if key == "dims":
                kv = dict(tok.split("=") for tok in val.split())
                out["dims"] = Dims(**{k: int(v) for k, v in kv.items()})
            else:
                out[key] = np.asarray(eval(val, {"__builtins__": {}}, {"e": math.e}), dtype=np.float64)
    return out
