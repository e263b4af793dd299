"""Golden fixtures: small text files written out by hand from the pages' definitions, each
with its citation in its header."""

import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def load(name):
    """Parse a fixture: '#' lines are comments, 'key v v v' lines are metadata, bare rows of
    numbers form the matrix."""
    meta, rows = {}, []
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if parts[0][0].isalpha():
                meta[parts[0]] = [float(p) if "." in p else int(p) for p in parts[1:]]
            else:
                rows.append([float(p) if "." in p else int(p) for p in parts])
    return meta, (np.array(rows) if rows else None)
