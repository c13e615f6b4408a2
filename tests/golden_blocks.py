"""Parser for ``tests/golden/blocks_handworked.txt`` (no arithmetic)."""

import numpy as np

from conftest import read_golden


def handworked_blocks():
    """List of dicts {name, type, x (float16[32]), scale_bits (int), q or bytes}."""
    out = []
    cur = None
    for line in read_golden("blocks_handworked.txt"):
        tok = line.split()
        if tok[0] == "block":
            cur = {"name": tok[1], "type": tok[2]}
            out.append(cur)
        elif tok[0] == "x":
            cur["x"] = np.array([float(v) for v in tok[1:]], dtype=np.float16)
        elif tok[0] == "scale":
            cur["scale_bits"] = int(tok[1], 16)
        elif tok[0] == "q":
            cur["q"] = np.array([int(v) for v in tok[1:]], dtype=np.int8)
        elif tok[0] == "bytes":
            cur["bytes"] = np.array([int(v, 16) for v in tok[1:]], dtype=np.uint8)
    for b in out:
        assert b["x"].shape == (32,)
    return out
