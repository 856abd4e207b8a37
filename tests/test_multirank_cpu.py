"""Multi-rank host logic on CPU (gloo, world size 2).

Each rank takes its kv-head shard of one problem, runs the path on it (the
fp64 oracle stands in for the kernels on CPU) with alpha rescaled for its
share of the elements, and the ranks exchange results.  The gathered outputs
and gradients, and the all-reduced alignment loss, must equal the unsharded
problem's."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_attention_ssa_b200 import shard
from block_sparse_attention_ssa_b200.inputs import make_qkv, make_upstream

CFG = dict(B=1, Hq=6, Hkv=3, N=64, d=8, s=16, k=2, alpha=10.0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    c = CFG
    t = make_qkv(c["B"], c["Hq"], c["Hkv"], c["N"], c["d"], c["s"], 99)
    g = make_upstream((c["B"], c["Hq"], c["N"], c["d"]), 98)
    return t["Q"].astype(np.float64), t["K"].astype(np.float64), t["V"].astype(np.float64), g.astype(np.float64)


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import ssa_oracle as O
        c = CFG
        Q, K, V, g = _problem()
        group = c["Hq"] // c["Hkv"]
        lo, hi = shard.kv_head_range(c["Hkv"], world, rank)
        q, k, v = shard.shard_views(Q, K, V, group, lo, hi)
        gl = g[:, lo * group:hi * group]
        scale = 1 / math.sqrt(c["d"])
        idx = O.select_blocks(O.block_scores(q, k, c["s"], scale), c["k"])
        m_local, m_global = q.size, Q.size
        a_loc = shard.local_alpha(c["alpha"], m_local, m_global)
        dQ, dK, dV, l_loc, f = O.ssa_backward(q, k, v, idx, c["s"], scale, None, gl, a_loc)

        def allsum(x):
            t = torch.tensor([x], dtype=torch.float64)
            dist.all_reduce(t)
            return float(t.item())

        l_glob = shard.combine_align_loss(l_loc, m_local, m_global, allsum)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), lo=lo, hi=hi, h_full=f["h_full"], delta=f["delta"],
                 idx=idx, dQ=dQ, dK=dK, dV=dV, l_glob=l_glob)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_kv_head_range_partitions_exactly():
    for Hkv in (1, 3, 8, 13):
        for world in (1, 2, 3, 8):
            got = [h for r in range(world) for h in range(*shard.kv_head_range(Hkv, world, r))]
            assert got == list(range(Hkv))
    with pytest.raises(ValueError):
        shard.kv_head_range(8, 2, 2)


def test_two_ranks_match_unsharded(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    from oracle import ssa_oracle as O
    c = CFG
    Q, K, V, g = _problem()
    group = c["Hq"] // c["Hkv"]
    scale = 1 / math.sqrt(c["d"])
    idx = O.select_blocks(O.block_scores(Q, K, c["s"], scale), c["k"])
    dQ, dK, dV, l_align, f = O.ssa_backward(Q, K, V, idx, c["s"], scale, None, g, c["alpha"])
    for r in range(world):
        z = np.load(tmp_path / f"rank{r}.npz")
        lo, hi = int(z["lo"]), int(z["hi"])
        hq = slice(lo * group, hi * group)
        np.testing.assert_array_equal(z["idx"], idx[:, hq])
        np.testing.assert_allclose(z["h_full"], f["h_full"][:, hq], atol=1e-13)
        np.testing.assert_allclose(z["delta"], f["delta"][:, hq], atol=1e-13)
        np.testing.assert_allclose(z["dQ"], dQ[:, hq], atol=1e-12)
        np.testing.assert_allclose(z["dK"], dK[:, lo:hi], atol=1e-12)
        np.testing.assert_allclose(z["dV"], dV[:, lo:hi], atol=1e-12)
        assert float(z["l_glob"]) == pytest.approx(l_align, rel=1e-12)
