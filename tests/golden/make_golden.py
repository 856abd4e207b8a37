"""Writes oracle_tiny.json, a frozen record of the oracle on one tiny case.

The pages print no worked example for any step of the path, so this fixture
is not a value from the pages: it freezes the oracle's own output (this script
calls only the oracle and the seeded input generator) so that any later change
to the oracle's arithmetic is visible in the CPU tests.

Run: python -m tests.golden.make_golden
"""
import json
import math
import os

import numpy as np

from oracle import ssa_oracle as O
from block_sparse_attention_ssa_b200.inputs import make_qkv, make_upstream

CASE = dict(B=1, Hq=2, Hkv=1, N=32, d=4, s=8, k=2, seed=2024, alpha=10.0)


def compute():
    c = CASE
    t = make_qkv(c["B"], c["Hq"], c["Hkv"], c["N"], c["d"], c["s"], c["seed"])
    Q, K, V = (t[x].astype(np.float64) for x in ("Q", "K", "V"))
    scale = 1.0 / math.sqrt(c["d"])
    idx = O.select_blocks(O.block_scores(Q, K, c["s"], scale), c["k"])
    g = make_upstream(Q.shape, c["seed"] + 1).astype(np.float64)
    dQ, dK, dV, l_align, f = O.ssa_backward(Q, K, V, idx, c["s"], scale, None, g, c["alpha"])
    return {
        "case": c,
        "idx": idx.tolist(),
        "delta": f["delta"].ravel().tolist(),
        "lse_full": f["lse_full"].ravel().tolist(),
        "lse_sel": f["lse_sel"].ravel().tolist(),
        "h_full_row0": f["h_full"][0, :, -1].ravel().tolist(),
        "h_sparse_row0": f["h_sparse"][0, :, -1].ravel().tolist(),
        "dQ_sum": dQ.sum(axis=(0, 2)).ravel().tolist(),
        "dK_sum": dK.sum(axis=(0, 2)).ravel().tolist(),
        "dV_sum": dV.sum(axis=(0, 2)).ravel().tolist(),
        "l_align": l_align,
    }


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json")
    with open(out, "w") as fh:
        json.dump(compute(), fh, indent=1)
    print("wrote", out)
