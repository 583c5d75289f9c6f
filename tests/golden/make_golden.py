"""Write tests/golden/gta_tiny_oracle.txt from the fp64 oracle.

The pages print no worked numeric example, so this fixture is not a pin: it
freezes the seeded tiny GTA workload (batch 2, h_q 8, two tied groups, d_h 64,
rope 32, context 128, page size 16, scale 1/8) and the oracle's answer on it,
so that a later change to the generator or to the oracle's arithmetic shows up
as a diff.  It calls only the input generator and oracle/.
"""
import hashlib
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from kv_cache_paged_b200 import workload as wl  # noqa: E402
from oracle import oracle as orc  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "gta_tiny_oracle.txt")


def digest(inp):
    h = hashlib.sha256()
    for a in (inp.seqlens, inp.block_table, inp.q, inp.caches["tied_cache"], inp.caches["rope_cache"]):
        h.update(np.ascontiguousarray(a).tobytes())
    return h.hexdigest()


def render():
    inp = wl.make_workload("gta_tiny")
    out, lse, _ = orc.decode_inputs(inp, threads=1)
    lines = ["# fp64 oracle on the seeded tiny GTA workload (see make_golden.py)",
             f"inputs_sha256 {digest(inp)}"]
    for b in range(inp.B):
        for h in range(inp.h_q):
            lines.append(f"lse {b} {h} {lse[b, 0, h]:.17e}")
            lines.append(f"out {b} {h} " + " ".join(f"{v:.17e}" for v in out[b, 0, h]))
    return "\n".join(lines) + "\n"


if __name__ == "__main__":
    with open(OUT, "w") as f:
        f.write(render())
    print("wrote", OUT)
