"""Reader of tests/golden/q6k_single_byte_probes.txt (hand-derived Q6_K element map).

Builds each probe's 210-byte super-block from its byte assignments and expands its expected
256 dequantized values.  No Q6_K arithmetic lives here: the expected values are the file's.
"""

import os

import numpy as np

PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "q6k_single_byte_probes.txt")
_FIELDS = {"ql": (0, 128), "qh": (128, 64), "sc": (192, 16)}


def _block(assignments):
    b = np.zeros(210, np.uint8)
    b[192:208] = 1                      # every scale 1
    b[208:210] = (0x00, 0x3C)           # d = 1.0, little endian
    for a in assignments.split():
        name, val = a.split("=")
        v = int(val, 16)
        if name == "d":
            b[208], b[209] = v & 0xFF, v >> 8
            continue
        field, idx = name.rstrip("]").split("[")
        off, size = _FIELDS[field]
        i = int(idx)
        assert 0 <= i < size and 0 <= v <= 0xFF, a
        b[off + i] = v
    return b


def load():
    """[(name, block uint8[210], expected float64[256])] in file order."""
    probes = []
    with open(PATH) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, assign, default, over = (p.strip() for p in line.split("|"))
            exp = np.full(256, float(default))
            for item in over.split():
                where, val = item.split("=")
                lo, _, hi = where.partition("-")
                exp[int(lo):int(hi or lo) + 1] = float(val)
            probes.append((name, _block(assign), exp))
    return probes
