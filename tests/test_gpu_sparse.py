"""GPU parity of the sparse stream alone (ssa_fwd_sparse, ssa_bwd_sparse)
against the fp64 oracle (oracle.forward_sparse / backward_sparse), through
the C ABI.

Cases cover both block sizes, GQA, both dtypes and head dims, a ragged last
128-row query tile, selections computed by the path and given selections
(rows without their diagonal block, duplicates, -1 padding, a query block
that attends nothing), and blocks that no query selects holding NaN, which
the sparse forward must never read.  Tolerances as for the dual stream."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_ssa_b200 import api
from block_sparse_attention_ssa_b200.inputs import make_upstream
from oracle import ssa_oracle as O
from tests.gpu_util import TOL, case_inputs, compare_selection, custom_idx, ensure_library, f64, rel_l2, upload

pytestmark = pytest.mark.gpu

# name: B, Hq, Hkv, N, d, s, k, dtype
CASES = {
    "bf16_gqa_odd_blocks": (1, 4, 1, 576, 128, 64, 4, "bf16"),
    "bf16_s128": (1, 2, 1, 768, 128, 128, 3, "bf16"),
    "bf16_gqa4_long": (1, 8, 2, 1536, 128, 64, 6, "bf16"),
    "bf16_full_budget": (1, 2, 1, 512, 128, 64, 16, "bf16"),
    "bf16_diag_only": (1, 2, 2, 512, 128, 64, 1, "bf16"),
    "bf16_d64": (2, 2, 2, 448, 64, 64, 3, "bf16"),
    "f32_gqa_d128": (1, 4, 2, 384, 128, 64, 3, "f32"),
    "f32_d64_s128": (1, 2, 1, 512, 64, 128, 2, "f32"),
}


@pytest.fixture(scope="module", autouse=True)
def lib():
    return ensure_library()


def _selection(dims, dev, host, s, k, scale):
    """The path's own selection, replaced by the oracle's on near-tie rows."""
    ws = api.alloc_workspace(dims)
    out = api.alloc_forward(dims)
    api.ssa_block_scores(dims, dev["Q"], dev["K"], out["scores"], ws)
    api.ssa_select_topk(dims, out["scores"], out["idx"])
    torch.cuda.synchronize()
    ora_scores = O.block_scores(host["Q"], host["K"], s, scale)
    ora_idx = O.select_blocks(ora_scores, k)
    if compare_selection(out["idx"].cpu().numpy(), ora_idx, ora_scores):
        out["idx"].copy_(torch.from_numpy(ora_idx))
    return out["idx"], ora_idx, ws


def _fwd_sparse(dims, dev, idx):
    B, Hq, N, d = dims.B, dims.Hq, dims.N, dims.d
    hs = torch.full((B, Hq, N, d), float("nan"), dtype=dims.torch_dtype, device="cuda")
    lse = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device="cuda")
    api.ssa_fwd_sparse(dims, dev["Q"], dev["K"], dev["V"], idx, hs, lse)
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    return hs, lse


def _check_fwd(hs, lse, ora, dt):
    tol = TOL[dt]
    err = np.abs(f64(hs) - ora["h_sparse"]).max()
    assert err <= tol["out"], ("h_sparse", err)
    fin = np.isfinite(ora["lse_sel"])
    got = f64(lse)
    assert np.array_equal(np.isfinite(got), fin)
    assert np.all(got[~fin] == -np.inf)
    if fin.any():
        assert np.abs(got[fin] - ora["lse_sel"][fin]).max() <= tol["lse"]


@pytest.mark.parametrize("name", list(CASES))
def test_fwd_sparse_matches_oracle(name):
    B, Hq, Hkv, N, d, s, k, dt = CASES[name]
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 707, dt)
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, dt)
    scale = 1 / math.sqrt(d)
    idx, ora_idx, _ = _selection(dims, dev, host, s, k, scale)
    hs, lse = _fwd_sparse(dims, dev, idx)
    _check_fwd(hs, lse, O.forward_sparse(host["Q"], host["K"], host["V"], ora_idx, s, scale), dt)


@pytest.mark.parametrize("cfg", [(1, 4, 2, 1024, 128, 64, 5), (1, 2, 1, 1152, 128, 64, 4),
                                 (1, 2, 2, 1024, 128, 128, 3), (1, 2, 1, 512, 64, 64, 3)])
def test_fwd_sparse_given_selection(cfg):
    """Selections that differ between neighbouring query blocks (so a 128-row
    query tile pairs blocks only one half selected), rows without their
    diagonal block, duplicates, padding and one query block with nothing."""
    B, Hq, Hkv, N, d, s, k = cfg
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 808, "bf16")
    n = N // s
    idx = custom_idx(B, Hq, n, k, seed=N + 7 * k, drop_diag_frac=0.3, pad_frac=0.2)
    idx[0, 0, n // 2] = -1
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, "bf16")
    hs, lse = _fwd_sparse(dims, dev, torch.from_numpy(idx).cuda())
    _check_fwd(hs, lse, O.forward_sparse(host["Q"], host["K"], host["V"], idx, s, 1 / math.sqrt(d)), "bf16")
    assert torch.all(hs[0, 0, (n // 2) * s:(n // 2 + 1) * s].float() == 0)


@pytest.mark.parametrize("s,dt", [(64, "bf16"), (128, "bf16"), (64, "f32")])
def test_fwd_sparse_never_reads_unselected_blocks(s, dt):
    """K and V of blocks that no query block selects are NaN on the device; the
    sparse forward loads only selected blocks, so its outputs stay finite and
    equal the oracle's on clean inputs."""
    B, Hq, Hkv, N, d, k = 1, 4, 2, 1536, 128, 4
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 909, dt)
    n = N // s
    idx = custom_idx(B, Hq, n, k, seed=31 + s)
    poisoned = [3, n // 2, n - 2]
    for j in poisoned:
        idx[idx == j] = -1
    for j in poisoned:
        dev["K"][:, :, j * s:(j + 1) * s] = float("nan")
        dev["V"][:, :, j * s:(j + 1) * s] = float("nan")
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, dt)
    hs, lse = _fwd_sparse(dims, dev, torch.from_numpy(idx).cuda())
    assert torch.isfinite(hs.float()).all()
    _check_fwd(hs, lse, O.forward_sparse(host["Q"], host["K"], host["V"], idx, s, 1 / math.sqrt(d)), dt)


@pytest.mark.parametrize("name", ["bf16_gqa_odd_blocks", "bf16_s128", "bf16_gqa4_long", "bf16_diag_only",
                                  "bf16_d64", "f32_gqa_d128"])
def test_bwd_sparse_matches_oracle(name):
    B, Hq, Hkv, N, d, s, k, dt = CASES[name]
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 606, dt)
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, dt)
    scale = 1 / math.sqrt(d)
    idx, ora_idx, ws = _selection(dims, dev, host, s, k, scale)
    hs, lse = _fwd_sparse(dims, dev, idx)
    g = make_upstream((B, Hq, N, d), 41)
    grads = api.alloc_backward(dims)
    api.ssa_bwd_sparse(dims, dev["Q"], dev["K"], dev["V"], idx, hs, lse, upload(g, dt), grads["dQ"], grads["dK"],
                       grads["dV"], ws)
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    from tests.gpu_util import oracle_view
    dQ, dK, dV = O.backward_sparse(host["Q"], host["K"], host["V"], ora_idx, s, scale,
                                   oracle_view(g, dt).astype(np.float64))
    for key, got, ref in (("dQ", grads["dQ"], dQ), ("dK", grads["dK"], dK), ("dV", grads["dV"], dV)):
        err = rel_l2(f64(got), ref)
        assert err < TOL[dt]["grad"], (key, err)


@pytest.mark.parametrize("cfg", [(1, 4, 2, 1024, 128, 64, 5), (1, 4, 1, 1024, 128, 128, 3)])
def test_bwd_sparse_given_selection(cfg):
    """Backward under given selections, including keys that no query attends
    (their dK and dV must be exactly zero) and a query block with nothing."""
    B, Hq, Hkv, N, d, s, k = cfg
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 505, "bf16")
    n = N // s
    idx = custom_idx(B, Hq, n, k, seed=N * 5 + k, drop_diag_frac=0.3, pad_frac=0.2)
    unused = [2, n - 3]
    for j in unused:
        idx[idx == j] = -1
    idx[0, 1, n // 2] = -1
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, "bf16")
    ws = api.alloc_workspace(dims)
    idx_d = torch.from_numpy(idx).cuda()
    hs, lse = _fwd_sparse(dims, dev, idx_d)
    g = make_upstream((B, Hq, N, d), 43)
    grads = api.alloc_backward(dims)
    for key in ("dQ", "dK", "dV"):
        grads[key].fill_(float("nan"))
    api.ssa_bwd_sparse(dims, dev["Q"], dev["K"], dev["V"], idx_d, hs, lse, upload(g, "bf16"), grads["dQ"],
                       grads["dK"], grads["dV"], ws)
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    from tests.gpu_util import oracle_view
    dQ, dK, dV = O.backward_sparse(host["Q"], host["K"], host["V"], idx, s, 1 / math.sqrt(d),
                                   oracle_view(g, "bf16").astype(np.float64))
    for key, got, ref in (("dQ", grads["dQ"], dQ), ("dK", grads["dK"], dK), ("dV", grads["dV"], dV)):
        err = rel_l2(f64(got), ref)
        assert err < TOL["bf16"]["grad"], (key, err)
    for j in unused:
        assert torch.all(grads["dK"][:, :, j * s:(j + 1) * s].float() == 0)
        assert torch.all(grads["dV"][:, :, j * s:(j + 1) * s].float() == 0)
    assert torch.all(grads["dQ"][0, 1, (n // 2) * s:(n // 2 + 1) * s].float() == 0)
