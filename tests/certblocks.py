"""Reader of tests/golden/certificate_blocks.txt (adversarial blocks for the certified fast score)."""
import os

import numpy as np

PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "certificate_blocks.txt")


def load():
    """[(kind, g float32, f_lo, n_offsets, x float32[16])]"""
    rows = []
    with open(PATH) as fh:
        for ln in fh:
            if ln.startswith("#") or not ln.strip():
                continue
            t = ln.split()
            rows.append((t[0], np.float32(float.fromhex(t[1])), int(t[2]), int(t[3]),
                         np.array([float.fromhex(v) for v in t[4:20]], np.float32)))
    return rows
