"""GPU parity at the pages' small block sizes (16 and 32 tokens; [digest]
"Model Architecture Configuration": block size 16, 16 blocks), where a 64 x 64
CUDA-core tile spans several query and key blocks and every element goes to
the selected or the dropped set on its own.  Each entry point of the path is
compared with the fp64 oracle: block scores and selection, the dual forward,
the dropped mass (with and without the full log-sum-exp), the sparse stream
alone forward and backward, the dual backward on both primaries, and the
decode step.  Includes the pages' model shape (g = 16 query heads per kv
head, d = 64).  Tolerances as elsewhere."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_ssa_b200 import api
from block_sparse_attention_ssa_b200.inputs import make_upstream
from oracle import ssa_oracle as O
from tests.gpu_util import (TOL, case_inputs, compare_selection, custom_idx, ensure_library, f64, oracle_view,
                            rel_l2, upload)

pytestmark = pytest.mark.gpu

# name: B, Hq, Hkv, N, d, s, k, dtype
CASES = {
    "f32_s16_d64": (1, 4, 2, 512, 64, 16, 16, "f32"),
    "bf16_s16_g16_d64": (1, 16, 1, 768, 64, 16, 16, "bf16"),
    "bf16_s32_d128": (2, 4, 2, 768, 128, 32, 6, "bf16"),
    "f32_s16_d128_k4": (1, 2, 1, 640, 128, 16, 4, "f32"),
    # a ragged last 128-row tile (576 = 4.5 x 128) with g = 8 (two head chunks)
    "bf16_s16_ragged_g8_d64": (1, 8, 1, 576, 64, 16, 8, "bf16"),
    "bf16_s32_ragged_d128": (1, 2, 1, 704, 128, 32, 5, "bf16"),
    # block 16 at d = 128 with g = 4 and a ragged last 128-row tile
    "bf16_s16_d128_g4": (1, 8, 2, 960, 128, 16, 16, "bf16"),
}


@pytest.fixture(scope="module", autouse=True)
def lib():
    return ensure_library()


def _forward(name, seed=515):
    B, Hq, Hkv, N, d, s, k, dt = CASES[name]
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, seed, dt)
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, dt)
    ws = api.alloc_workspace(dims)
    out = api.alloc_forward(dims)
    api.ssa_block_scores(dims, dev["Q"], dev["K"], out["scores"], ws)
    api.ssa_select_topk(dims, out["scores"], out["idx"])
    scale = 1 / math.sqrt(d)
    torch.cuda.synchronize()
    ora_scores = O.block_scores(host["Q"], host["K"], s, scale)
    ora_idx = O.select_blocks(ora_scores, k)
    if compare_selection(out["idx"].cpu().numpy(), ora_idx, ora_scores):
        out["idx"].copy_(torch.from_numpy(ora_idx))
    api.ssa_fwd_dual(dims, dev["Q"], dev["K"], dev["V"], out["idx"], out["h_full"], out["h_sparse"],
                     out["lse_full"], out["lse_sel"], out["delta"])
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    ora = O.forward_dual(host["Q"], host["K"], host["V"], ora_idx, s, scale)
    return dict(dims=dims, dev=dev, host=host, out=out, ws=ws, ora=ora, ora_idx=ora_idx, scale=scale,
                cfg=CASES[name])


@pytest.mark.parametrize("name", list(CASES))
def test_forward_dual_small_blocks(name):
    r = _forward(name)
    tol = TOL[r["cfg"][7]]
    for key in ("h_full", "h_sparse", "delta"):
        err = np.abs(f64(r["out"][key]) - r["ora"][key]).max()
        assert err <= tol["out"], (key, err)
    for key in ("lse_full", "lse_sel"):
        assert np.abs(f64(r["out"][key]) - r["ora"][key]).max() <= tol["lse"], key


@pytest.mark.parametrize("name", list(CASES))
def test_dropped_mass_small_blocks(name):
    r = _forward(name)
    tol = TOL[r["cfg"][7]]["out"]
    for lse in (r["out"]["lse_full"], None):
        delta = torch.full_like(r["out"]["delta"], float("nan"))
        api.ssa_dropped_mass(r["dims"], r["dev"]["Q"], r["dev"]["K"], r["out"]["idx"], lse, delta, r["ws"])
        torch.cuda.synchronize()
        assert np.abs(f64(delta) - r["ora"]["delta"]).max() <= tol


@pytest.mark.parametrize("name", list(CASES))
def test_sparse_alone_small_blocks(name):
    r = _forward(name)
    B, Hq, Hkv, N, d, s, k, dt = r["cfg"]
    dims, dev, host = r["dims"], r["dev"], r["host"]
    hs = torch.full_like(r["out"]["h_sparse"], float("nan"))
    lse = torch.full_like(r["out"]["lse_sel"], float("nan"))
    api.ssa_fwd_sparse(dims, dev["Q"], dev["K"], dev["V"], r["out"]["idx"], hs, lse)
    torch.cuda.synchronize()
    ora = O.forward_sparse(host["Q"], host["K"], host["V"], r["ora_idx"], s, r["scale"])
    assert np.abs(f64(hs) - ora["h_sparse"]).max() <= TOL[dt]["out"]
    assert np.abs(f64(lse) - ora["lse_sel"]).max() <= TOL[dt]["lse"]
    g = make_upstream((B, Hq, N, d), 47)
    grads = api.alloc_backward(dims)
    api.ssa_bwd_sparse(dims, dev["Q"], dev["K"], dev["V"], r["out"]["idx"], hs, lse, upload(g, dt), grads["dQ"],
                       grads["dK"], grads["dV"], r["ws"])
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    dQ, dK, dV = O.backward_sparse(host["Q"], host["K"], host["V"], r["ora_idx"], s, r["scale"],
                                   oracle_view(g, dt).astype(np.float64))
    for key, got, ref in (("dQ", grads["dQ"], dQ), ("dK", grads["dK"], dK), ("dV", grads["dV"], dV)):
        assert rel_l2(f64(got), ref) < TOL[dt]["grad"], key


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("primary", ["sparse", "full"])
def test_backward_dual_small_blocks(name, primary):
    r = _forward(name)
    B, Hq, Hkv, N, d, s, k, dt = r["cfg"]
    g = make_upstream((B, Hq, N, d), 53)
    gd = upload(g, dt)
    gf, gs = (gd, None) if primary == "full" else (None, gd)
    grads = api.alloc_backward(r["dims"])
    api.backward(r["dims"], r["dev"]["Q"], r["dev"]["K"], r["dev"]["V"], r["out"], gf, gs, 10.0, grads, r["ws"])
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    go = oracle_view(g, dt).astype(np.float64)
    ogf, ogs = (go, None) if primary == "full" else (None, go)
    dQ, dK, dV, l_align, _ = O.ssa_backward(r["host"]["Q"], r["host"]["K"], r["host"]["V"], r["ora_idx"], s,
                                            r["scale"], ogf, ogs, 10.0, fwd=r["ora"])
    for key, got, ref in (("dQ", grads["dQ"], dQ), ("dK", grads["dK"], dK), ("dV", grads["dV"], dV)):
        assert rel_l2(f64(got), ref) < TOL[dt]["grad"], key
    assert float(grads["align_loss"].item()) == pytest.approx(l_align, rel=5e-2 if dt == "bf16" else 1e-4)


@pytest.mark.parametrize("s,d,dt", [(16, 64, "f32"), (16, 64, "bf16"), (32, 128, "bf16"), (16, 128, "bf16")])
def test_given_selection_mixed_tiles(s, d, dt):
    """Random selections at blocks of 16 and 32 (rows without their diagonal
    block, duplicates, padding): most 64 x 64 tiles mix selected and dropped
    pairs inside a row and between rows."""
    B, Hq, Hkv, N, k = 1, 4, 2, 512, 6
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 616, dt)
    n = N // s
    idx = custom_idx(B, Hq, n, k, seed=77 + s + d, drop_diag_frac=0.3, pad_frac=0.2)
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, dt)
    out = api.alloc_forward(dims)
    ws = api.alloc_workspace(dims)
    out["idx"] = torch.from_numpy(idx).cuda()
    api.ssa_fwd_dual(dims, dev["Q"], dev["K"], dev["V"], out["idx"], out["h_full"], out["h_sparse"],
                     out["lse_full"], out["lse_sel"], out["delta"])
    gf, gs = make_upstream((B, Hq, N, d), 61), make_upstream((B, Hq, N, d), 62)
    grads = api.alloc_backward(dims)
    api.backward(dims, dev["Q"], dev["K"], dev["V"], out, upload(gf, dt), upload(gs, dt), 10.0, grads, ws)
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    scale = 1 / math.sqrt(d)
    dQ, dK, dV, _, ora = O.ssa_backward(host["Q"], host["K"], host["V"], idx, s, scale,
                                        oracle_view(gf, dt).astype(np.float64),
                                        oracle_view(gs, dt).astype(np.float64), 10.0)
    for key in ("h_full", "h_sparse", "delta"):
        assert np.abs(f64(out[key]) - ora[key]).max() <= TOL[dt]["out"], key
    for key in ("lse_full", "lse_sel"):
        fin = np.isfinite(ora[key])
        got = f64(out[key])
        assert np.array_equal(np.isfinite(got), fin), key
        assert np.abs(got[fin] - ora[key][fin]).max() <= TOL[dt]["lse"], key
    for key, got, ref in (("dQ", grads["dQ"], dQ), ("dK", grads["dK"], dK), ("dV", grads["dV"], dV)):
        assert rel_l2(f64(got), ref) < TOL[dt]["grad"], key


@pytest.mark.parametrize("s,d", [(16, 64), (32, 128)])
def test_sparse_alone_never_reads_unselected_small_blocks(s, d):
    """Blocks that no query selects hold NaN in K and V on the device while
    their neighbours inside the same 64-key tile are selected: the sparse
    stream alone must neither read nor weigh them."""
    B, Hq, Hkv, N, k = 1, 4, 2, 1024, 5
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 929, "bf16")
    n = N // s
    idx = custom_idx(B, Hq, n, k, seed=5 + s)
    poisoned = [1, 9, n // 2 + 1, n - 3]
    for j in poisoned:
        idx[idx == j] = -1
        dev["K"][:, :, j * s:(j + 1) * s] = float("nan")
        dev["V"][:, :, j * s:(j + 1) * s] = float("nan")
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, "bf16")
    hs = torch.full((B, Hq, N, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device="cuda")
    api.ssa_fwd_sparse(dims, dev["Q"], dev["K"], dev["V"], torch.from_numpy(idx).cuda(), hs, lse)
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    assert torch.isfinite(hs.float()).all()
    ora = O.forward_sparse(host["Q"], host["K"], host["V"], idx, s, 1 / math.sqrt(d))
    assert np.abs(f64(hs) - ora["h_sparse"]).max() <= TOL["bf16"]["out"]
    fin = np.isfinite(ora["lse_sel"])
    assert np.array_equal(np.isfinite(f64(lse)), fin)
    assert np.abs(f64(lse)[fin] - ora["lse_sel"][fin]).max() <= TOL["bf16"]["lse"]


@pytest.mark.parametrize("s,d,g", [(16, 64, 4), (32, 64, 1), (16, 128, 2), (32, 128, 2)])
def test_sparse_alone_small_blocks_given_selection(s, d, g):
    """Given selections at blocks of 16 and 32: rows without their diagonal
    block, duplicate entries, -1 padding, and one query block that attends
    nothing (its h_sparse is zero and its lse_sel is -inf)."""
    B, Hkv, N, k = 1, 2, 1088, 7
    Hq = g * Hkv
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 939 + s + d, "bf16")
    n = N // s
    idx = custom_idx(B, Hq, n, k, seed=17 + s + d, drop_diag_frac=0.3, pad_frac=0.3)
    idx[0, 1, n // 2] = -1
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, "bf16")
    hs = torch.full((B, Hq, N, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device="cuda")
    api.ssa_fwd_sparse(dims, dev["Q"], dev["K"], dev["V"], torch.from_numpy(idx).cuda(), hs, lse)
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    ora = O.forward_sparse(host["Q"], host["K"], host["V"], idx, s, 1 / math.sqrt(d))
    assert np.abs(f64(hs) - ora["h_sparse"]).max() <= TOL["bf16"]["out"]
    fin = np.isfinite(ora["lse_sel"])
    assert not fin[0, 1, (n // 2) * s:(n // 2 + 1) * s].any()
    assert np.array_equal(np.isfinite(f64(lse)), fin)
    assert np.all(f64(lse)[~fin] == -np.inf)
    assert np.abs(f64(lse)[fin] - ora["lse_sel"][fin]).max() <= TOL["bf16"]["lse"]
    assert torch.all(hs[0, 1, (n // 2) * s:(n // 2 + 1) * s].float() == 0)
    g_up = make_upstream((B, Hq, N, d), 53)
    grads = api.alloc_backward(dims)
    ws = api.alloc_workspace(dims)
    api.ssa_bwd_sparse(dims, dev["Q"], dev["K"], dev["V"], torch.from_numpy(idx).cuda(), hs, lse,
                       upload(g_up, "bf16"), grads["dQ"], grads["dK"], grads["dV"], ws)
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    dQ, dK, dV = O.backward_sparse(host["Q"], host["K"], host["V"], idx, s, 1 / math.sqrt(d),
                                   oracle_view(g_up, "bf16").astype(np.float64))
    for key, got, ref in (("dQ", grads["dQ"], dQ), ("dK", grads["dK"], dK), ("dV", grads["dV"], dV)):
        assert rel_l2(f64(got), ref) < TOL["bf16"]["grad"], key


def _skewed_idx(B, H, n, k, seed):
    """Every query block keeps key blocks 0 and 1 (with its diagonal and
    random others): the dK/dV lists of those two key blocks hold every query
    block, many pairs per warp."""
    rng = np.random.Generator(np.random.PCG64(seed))
    idx = np.full((B, H, n, k), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(n):
                if i + 1 <= k:
                    row = list(range(i + 1))
                else:
                    rest = rng.choice(np.arange(2, i), size=k - 3, replace=False).tolist()
                    row = sorted([0, 1, i] + rest)
                idx[b, h, i, :len(row)] = row
    return idx


@pytest.mark.parametrize("s,d", [(16, 64), (32, 128)])
def test_sparse_alone_skewed_selection(s, d):
    """The sparse stream alone when a few key blocks are chosen by every query
    block, whole-problem parity of h_sparse, lse_sel, dQ, dK, dV."""
    B, Hq, Hkv, N, k = 1, 4, 2, 2048, 5
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 951 + s, "bf16")
    n = N // s
    idx = _skewed_idx(B, Hq, n, k, 61 + s)
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, "bf16")
    idx_d = torch.from_numpy(idx).cuda()
    hs = torch.full((B, Hq, N, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device="cuda")
    api.ssa_fwd_sparse(dims, dev["Q"], dev["K"], dev["V"], idx_d, hs, lse)
    g_up = make_upstream((B, Hq, N, d), 59)
    grads = api.alloc_backward(dims)
    ws = api.alloc_workspace(dims)
    api.ssa_bwd_sparse(dims, dev["Q"], dev["K"], dev["V"], idx_d, hs, lse, upload(g_up, "bf16"), grads["dQ"],
                       grads["dK"], grads["dV"], ws)
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    scale = 1 / math.sqrt(d)
    ora = O.forward_sparse(host["Q"], host["K"], host["V"], idx, s, scale)
    assert np.abs(f64(hs) - ora["h_sparse"]).max() <= TOL["bf16"]["out"]
    assert np.abs(f64(lse) - ora["lse_sel"]).max() <= TOL["bf16"]["lse"]
    dQ, dK, dV = O.backward_sparse(host["Q"], host["K"], host["V"], idx, s, scale,
                                   oracle_view(g_up, "bf16").astype(np.float64))
    for key, got, ref in (("dQ", grads["dQ"], dQ), ("dK", grads["dK"], dK), ("dV", grads["dV"], dV)):
        assert rel_l2(f64(got), ref) < TOL["bf16"]["grad"], key
    for j in (0, 1):  # the two key blocks every query block chose
        rows = slice(j * s, (j + 1) * s)
        assert rel_l2(f64(grads["dK"][:, :, rows]), dK[:, :, rows]) < TOL["bf16"]["grad"], ("dK", j)
        assert rel_l2(f64(grads["dV"][:, :, rows]), dV[:, :, rows]) < TOL["bf16"]["grad"], ("dV", j)


def test_sparse_alone_max_blocks_block16():
    """The largest block count at block 16 (n = 2048, N = 32768): the
    selection bit sets and dK/dV lists at full width; sampled query blocks of
    h_sparse, lse_sel and dQ, and the last key block's dK, dV (only the last
    query block can select it)."""
    B, Hq, Hkv, N, d, s, k = 1, 2, 1, 32768, 64, 16, 16
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 961, "bf16")
    n = N // s
    idx = custom_idx(B, Hq, n, k, seed=67, drop_diag_frac=0.1, pad_frac=0.1)
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, "bf16")
    idx_d = torch.from_numpy(idx).cuda()
    hs = torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    api.ssa_fwd_sparse(dims, dev["Q"], dev["K"], dev["V"], idx_d, hs, lse)
    g_up = make_upstream((B, Hq, N, d), 71)
    grads = api.alloc_backward(dims)
    ws = api.alloc_workspace(dims)
    api.ssa_bwd_sparse(dims, dev["Q"], dev["K"], dev["V"], idx_d, hs, lse, upload(g_up, "bf16"), grads["dQ"],
                       grads["dK"], grads["dV"], ws)
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    scale = 1 / math.sqrt(d)
    g64 = oracle_view(g_up, "bf16").astype(np.float64)
    for h, i in ((0, 0), (1, 5), (0, 777), (1, 1500), (0, n - 1), (1, n - 1)):
        N1 = (i + 1) * s
        sl = (slice(0, 1), slice(h, h + 1))
        f = O.forward_sparse(host["Q"][sl + (slice(0, N1),)], host["K"][:, :, :N1], host["V"][:, :, :N1],
                             idx[sl + (slice(0, i + 1),)], s, scale, qblocks=[i])
        rows = slice(i * s, N1)
        assert np.abs(f64(hs[0, h, rows]) - f["h_sparse"][0, 0, rows]).max() <= TOL["bf16"]["out"], (h, i)
        if np.isfinite(f["lse_sel"][0, 0, rows]).all():
            assert np.abs(f64(lse[0, h, rows]) - f["lse_sel"][0, 0, rows]).max() <= TOL["bf16"]["lse"], (h, i)
        dQ, _, _ = O.backward_sparse(host["Q"][sl + (slice(0, N1),)], host["K"][:, :, :N1], host["V"][:, :, :N1],
                                     idx[sl + (slice(0, i + 1),)], s, scale, g64[sl + (slice(0, N1),)],
                                     qblocks=[i])
        assert rel_l2(f64(grads["dQ"][0, h, rows]), dQ[0, 0, rows]) < TOL["bf16"]["grad"], (h, i)
    _, dK, dV = O.backward_sparse(host["Q"], host["K"], host["V"], idx, s, scale, g64, qblocks=[n - 1])
    rows = slice((n - 1) * s, N)
    assert rel_l2(f64(grads["dK"][0, 0, rows]), dK[0, 0, rows]) < TOL["bf16"]["grad"]
    assert rel_l2(f64(grads["dV"][0, 0, rows]), dV[0, 0, rows]) < TOL["bf16"]["grad"]


def test_decode_block16():
    """Decode at block 16 across several block boundaries, against the oracle."""
    B, Hq, Hkv, N, d, s, k = 1, 8, 2, 512, 64, 16, 16
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 717, "f32")
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, "f32")
    st = api.alloc_decode(dims)
    ws = api.alloc_workspace(dims)
    t0 = 16 * 17 + 5
    api.ssa_decode_prefill(dims, dev["Q"], dev["K"], t0, st["qsum"], st["kbar"])
    scale = 1 / math.sqrt(d)
    for t in range(t0, t0 + 60):
        i = t // s
        api.ssa_decode_step(dims, dev["Q"][:, :, t:t + 1], dev["K"], dev["V"], t, st["qsum"], st["kbar"], st["h"],
                            st["lse"], st["idx"], ws)
        torch.cuda.synchronize()
        gidx = st["idx"].cpu().numpy()
        oidx = O.decode_select(host["Q"][:, :, i * s:t + 1], host["K"], t, s, k, scale, n_cache=N // s)
        assert np.array_equal(gidx, oidx), t
        h_ref, lse_ref = O.decode_attend(host["Q"][:, :, t], host["K"], host["V"], t, s, oidx, scale)
        assert np.abs(f64(st["h"])[:, :, 0] - h_ref).max() <= TOL["f32"]["out"], t
        assert np.abs(f64(st["lse"]) - lse_ref).max() <= TOL["f32"]["lse"], t
