"""Reader of the hand-worked cases under tests/golden/ (text: '#' comment
lines carry the source and the derivation, then 'key: values' lines)."""

import os

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name):
    out = {}
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, rest = line.partition(":")
            vals = rest.split()
            out[key.strip()] = [int(v, 16) if v.startswith("0x") else float(v) for v in vals]
    return out
