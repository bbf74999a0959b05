"""Write tests/golden/tiny_oracle.json: the oracle's results on the tiny configuration
(4x8x8 tokens, 2 heads, D = 64, fp32 source, seed 0, drawn at sharpness 4; selections at
thresholds 0.5 to 0.99, the lower ones keeping strict subsets of the four kv blocks), kept as
a regression fixture for the oracle itself.

The pages print no worked example with numbers for block masses, selections or attention
outputs, so no stored value here comes from them: every value is written by this script,
which calls only the oracle and the seeded input generator.  The fixture catches a later
change to the oracle's arithmetic; the oracle's correctness is pinned separately (closed
forms, invariants, brute force, library routines).

    python tests/golden/make_golden.py
"""
import json
import math
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from block_sparse_attention_25_b200 import synth  # noqa: E402
from oracle import bsa_oracle as O  # noqa: E402

SHARPNESS = 4.0
TAUS = (0.5, 0.7, 0.8, 0.9, 0.99)


def compute():
    wl = synth.WORKLOADS["tiny"]
    g = O.Grid(wl.T, wl.H, wl.W, wl.Tp, wl.Hp, wl.Wp)
    q, k, v = synth.draw_qkv(wl, sharpness=SHARPNESS)
    qt, kt, vt = (O.permute_forward(x.double().numpy(), g) for x in (q, k, v))
    scale = 1.0 / math.sqrt(wl.head_dim)
    mass = O.block_mass(qt, kt, g, wl.q_block, 64, scale)
    out = {"workload": wl.name, "sharpness": SHARPNESS, "scale": scale,
           "mass": [float(x) for x in mass.reshape(-1)], "mass_shape": list(mass.shape),
           "selections": {}}
    rows = mass.astype(np.float32).reshape(-1, mass.shape[-1])
    for tau in TAUS:
        rp, ci = O.topp_select(rows, tau)
        out["selections"][str(tau)] = {"row_ptr": [int(x) for x in rp],
                                       "col_idx": [int(x) for x in ci]}
    rp, ci = O.topp_select(rows, 0.99)
    o, lse = O.masked_attention(qt, kt, vt, g, wl.q_block, 64, rp, ci, scale)
    out["attention_0.99"] = {
        "sum": float(o.sum()), "sum_sq": float((o * o).sum()),
        "row0": [float(x) for x in o[0, 0, 0]],
        "lse_finite_sum": float(lse[np.isfinite(lse)].sum()),
    }
    return out


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_oracle.json"), "w") as f:
        json.dump(compute(), f, indent=1)
        f.write("\n")
    print("wrote", os.path.join(HERE, "tiny_oracle.json"))
