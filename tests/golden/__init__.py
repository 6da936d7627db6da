"""Reader for the hand-worked fixtures in this folder.

Each fixture is a text file of ``name: values`` lines; ``|`` separates rows
and ``#`` starts a comment that states the source passage and the derivation.
"""

import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def load(name: str) -> dict:
    out = {}
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = line.split(":", 1)
            rows = [r.split() for r in val.split("|")]
            conv = [[float(int(x, 16)) if x.startswith("0x") else float(x) for x in r] for r in rows]
            out[key.strip()] = np.array(conv[0] if len(conv) == 1 else conv, dtype=np.float64)
    return out
