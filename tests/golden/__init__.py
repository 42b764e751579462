"""Hand-worked fixtures. Each file states the passage it follows and the derivation."""

import os

HERE = os.path.dirname(os.path.abspath(__file__))


def read_fixture(name):
    """Parse 'key: v v | v v' lines into dict of lists of float rows."""
    out = {}
    with open(os.path.join(HERE, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, rest = line.partition(":")
            rows = [[float(v) for v in part.split()] for part in rest.split("|")]
            out[key.strip()] = rows
    return out
