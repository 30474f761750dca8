"""Readers for the text fixtures under tests/golden/ (comment lines start with '#')."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_table(name):
    """Return (meta dict from '# key value' lines, int64 matrix of the data rows)."""
    meta, rows = {}, []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line:
                continue
            if line.startswith("#"):
                parts = line[1:].split()
                if len(parts) == 2 and parts[1].lstrip("-").isdigit():
                    meta[parts[0]] = int(parts[1])
                continue
            rows.append([int(x) for x in line.split()])
    return meta, np.array(rows, dtype=np.int64)
