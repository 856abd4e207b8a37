"""The kv-head shard of the path, run through the C ABI on one GPU.

A problem is split into two kv-head ranges, as two ranks would hold it
(block_sparse_attention_ssa_b200.shard): each shard passes strided views of
its heads (base offsets into the full Q, K, V, and the outputs written
straight into views of full-size h_full / h_sparse / dQ / dK / dV buffers) to
the same entry points, with alpha rescaled to its share of the elements.
The shards' selections, outputs and gradients must equal the unsharded
call's bit for bit (every (batch, kv head) group is independent and the
kernels are deterministic; with two equal shards the rescaled alpha and
element count are exact), and the combined alignment loss must equal the
unsharded one and the oracle's."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_ssa_b200 import api, shard
from oracle import ssa_oracle as O
from tests.gpu_util import TOL, case_inputs, ensure_library, f64, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    return ensure_library()


def _dense_fwd(dims):
    f = api.alloc_forward(dims)
    return {k: f[k] for k in ("scores", "idx", "lse_full", "lse_sel", "delta")}


@pytest.mark.parametrize("B,Hq,Hkv,N,d,s,k", [(2, 8, 4, 1024, 128, 64, 4), (1, 8, 2, 1024, 64, 16, 8)])
def test_two_kv_head_shards_match_unsharded(B, Hq, Hkv, N, d, s, k):
    world, alpha = 2, 10.0
    g = Hq // Hkv
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 5150 + d, "bf16")
    ones = torch.ones_like(dev["Q"])

    # unsharded
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, "bf16")
    ws = api.alloc_workspace(dims)
    ref = api.alloc_forward(dims)
    api.forward(dims, dev["Q"], dev["K"], dev["V"], ref, ws)
    ref_g = api.alloc_backward(dims)
    api.backward(dims, dev["Q"], dev["K"], dev["V"], ref, None, ones, alpha, ref_g, ws)

    # two shards writing into views of full-size buffers
    hf = torch.full_like(ref["h_full"], float("nan"))
    hs = torch.full_like(ref["h_sparse"], float("nan"))
    dQ = torch.full_like(ref_g["dQ"], float("nan"))
    dK = torch.full_like(ref_g["dK"], float("nan"))
    dV = torch.full_like(ref_g["dV"], float("nan"))
    m_global = B * Hq * N * d
    loss_parts = []
    for rank in range(world):
        lo, hi = shard.kv_head_range(Hkv, world, rank)
        q, kk, v = shard.shard_views(dev["Q"], dev["K"], dev["V"], g, lo, hi)
        hq = slice(lo * g, hi * g)
        sd = api.make_dims(B, (hi - lo) * g, hi - lo, N, d, s, k, "bf16")
        sws = api.alloc_workspace(sd)
        loc = _dense_fwd(sd)
        loc["h_full"], loc["h_sparse"] = hf[:, hq], hs[:, hq]
        api.forward(sd, q, kk, v, loc, sws)
        m_local = B * (hi - lo) * g * N * d
        grads = {"dQ": dQ[:, hq], "dK": dK[:, lo:hi], "dV": dV[:, lo:hi],
                 "align_loss": torch.empty(1, dtype=torch.float32, device="cuda")}
        api.backward(sd, q, kk, v, loc, None, ones[:, hq], shard.local_alpha(alpha, m_local, m_global), grads, sws)
        torch.cuda.synchronize()
        for key in ("idx", "lse_full", "lse_sel", "delta"):
            assert torch.equal(loc[key], ref[key][:, hq]), (rank, key)
        loss_parts.append((float(grads["align_loss"].item()), m_local))
    assert api.ssa_device_status() == api.SSA_OK

    for got, want in ((hf, ref["h_full"]), (hs, ref["h_sparse"]), (dQ, ref_g["dQ"]), (dK, ref_g["dK"]),
                      (dV, ref_g["dV"])):
        assert torch.equal(got, want)
    # rank 0's view of the one scalar all-reduce (the other rank's share added)
    others = sum(l_r * m_r / m_global for l_r, m_r in loss_parts[1:])
    loss = shard.combine_align_loss(loss_parts[0][0], loss_parts[0][1], m_global, lambda x: x + others)
    assert loss == pytest.approx(float(ref_g["align_loss"].item()), rel=1e-5)

    # the oracle on the whole problem
    scale = 1.0 / math.sqrt(d)
    idx = ref["idx"].cpu().numpy()
    dQo, dKo, dVo, l_align, f = O.ssa_backward(host["Q"], host["K"], host["V"], idx, s, scale, None,
                                               np.ones((B, Hq, N, d)), alpha)
    tol = TOL["bf16"]
    assert np.abs(f64(hf) - f["h_full"]).max() <= tol["out"]
    assert np.abs(f64(hs) - f["h_sparse"]).max() <= tol["out"]
    assert rel_l2(f64(dQ), dQo) < tol["grad"]
    assert rel_l2(f64(dK), dKo) < tol["grad"]
    assert rel_l2(f64(dV), dVo) < tol["grad"]
    assert loss == pytest.approx(l_align, rel=2e-2, abs=1e-6)
