"""GPU parity: each step of the path, called through the C ABI, against the
fp64 oracle on the same seeded inputs.  Sizes span several tiles and odd block
counts (a ragged last 128-row query tile), GQA, both head dims, both block
sizes and the degenerate budgets.

Tolerances (from the stated targets): outputs and delta 2e-2 absolute for bf16
inputs and 1e-4 for fp32; gradients 5e-2 relative-L2 for bf16 and 1e-4 for
fp32; selections bit-exact except near ties (gap < 1e-4 relative), which are
logged and compared downstream under the oracle's indices."""
import functools
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_ssa_b200 import api
from block_sparse_attention_ssa_b200.inputs import make_scores, make_upstream
from oracle import ssa_oracle as O
from tests.gpu_util import (TOL, case_inputs, compare_selection, custom_idx, ensure_library, f64,
                            oracle_view, rel_l2, upload)

pytestmark = pytest.mark.gpu

# name: B, Hq, Hkv, N, d, s, k, dtype
CASES = {
    "f32_mha_d64": (1, 2, 2, 512, 64, 64, 4, "f32"),
    "f32_gqa_d128": (1, 4, 2, 384, 128, 64, 3, "f32"),
    "f32_many_blocks": (1, 1, 1, 2112, 64, 64, 5, "f32"),
    "bf16_gqa_odd_blocks": (1, 4, 1, 576, 128, 64, 4, "bf16"),
    "bf16_s128": (1, 2, 1, 768, 128, 128, 3, "bf16"),
    "bf16_d64_b2": (2, 2, 2, 448, 64, 64, 3, "bf16"),
    "bf16_full_budget": (1, 2, 1, 512, 128, 64, 16, "bf16"),
    "bf16_diag_only": (1, 2, 2, 512, 128, 64, 1, "bf16"),
    "bf16_gqa4_long": (1, 8, 2, 1536, 128, 64, 6, "bf16"),
}


@pytest.fixture(scope="module", autouse=True)
def lib():
    return ensure_library()


@functools.lru_cache(maxsize=None)
def run_case(name, seed=101):
    B, Hq, Hkv, N, d, s, k, dt = CASES[name]
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, seed, dt)
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, dt)
    ws = api.alloc_workspace(dims)
    out = api.alloc_forward(dims)
    api.ssa_block_scores(dims, dev["Q"], dev["K"], out["scores"], ws)
    api.ssa_select_topk(dims, out["scores"], out["idx"])
    scale = 1 / math.sqrt(d)
    ora_scores = O.block_scores(host["Q"], host["K"], s, scale)
    ora_idx = O.select_blocks(ora_scores, k)
    torch.cuda.synchronize()
    near = compare_selection(out["idx"].cpu().numpy(), ora_idx, ora_scores)
    if near:
        print(f"{name}: {len(near)} near-tie rows, comparing under the oracle's indices")
        out["idx"].copy_(torch.from_numpy(ora_idx))
    api.ssa_fwd_dual(dims, dev["Q"], dev["K"], dev["V"], out["idx"], out["h_full"], out["h_sparse"],
                     out["lse_full"], out["lse_sel"], out["delta"])
    torch.cuda.synchronize()
    ora = O.forward_dual(host["Q"], host["K"], host["V"], ora_idx, s, scale)
    return dict(dims=dims, dev=dev, host=host, out=out, ws=ws, ora=ora, ora_idx=ora_idx,
                ora_scores=ora_scores, scale=scale, cfg=CASES[name])


@pytest.mark.parametrize("name", list(CASES))
def test_block_scores(name):
    r = run_case(name)
    got = f64(r["out"]["scores"])
    ref = r["ora_scores"]
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin)
    assert np.all(got[~fin] == -np.inf)
    scale = max(1.0, np.abs(ref[fin]).max())
    np.testing.assert_allclose(got[fin], ref[fin], rtol=1e-5, atol=1e-5 * scale)


@pytest.mark.parametrize("name", list(CASES))
def test_forward_dual(name):
    r = run_case(name)
    dt = r["cfg"][7]
    tol = TOL[dt]
    o, ora = r["out"], r["ora"]
    for key in ("h_full", "h_sparse", "delta"):
        err = np.abs(f64(o[key]) - ora[key]).max()
        assert err <= tol["out"], (key, err)
    for key in ("lse_full", "lse_sel"):
        err = np.abs(f64(o[key]) - ora[key]).max()
        assert err <= tol["lse"], (key, err)


def test_full_budget_gives_identical_streams():
    r = run_case("bf16_full_budget")
    o = r["out"]
    assert torch.equal(o["h_full"], o["h_sparse"])
    assert torch.all(o["delta"] == 0)
    assert torch.equal(o["lse_full"], o["lse_sel"])


def test_diag_only_budget():
    r = run_case("bf16_diag_only")
    idx = r["out"]["idx"].cpu().numpy()
    n = idx.shape[2]
    assert np.array_equal(idx[..., 0], np.broadcast_to(np.arange(n), idx.shape[:3]))


@pytest.mark.parametrize("ties", [0.0, 0.3, 0.9])
@pytest.mark.parametrize("n,k", [(16, 4), (77, 9), (512, 64), (1024, 16), (300, 300)])
def test_select_topk_bit_exact(n, k, ties):
    """Same fp32 scores on both sides (the decision is taken in the same
    precision), so the selection must match bit for bit, ties included."""
    S = make_scores(2, 3, n, seed=n * 7 + k, tie_frac=ties)
    dims = api.make_dims(2, 3, 3, n * 64, 64, 64, k, "f32")
    idx = torch.empty((2, 3, n, min(k, n)), dtype=torch.int32, device="cuda")
    api.ssa_select_topk(dims, torch.from_numpy(S).cuda(), idx)
    torch.cuda.synchronize()
    ref = O.select_blocks(S.astype(np.float64), k)
    assert np.array_equal(idx.cpu().numpy(), ref)


@pytest.mark.parametrize("name", ["f32_gqa_d128", "bf16_gqa_odd_blocks", "bf16_s128", "bf16_d64_b2",
                                  "bf16_gqa4_long"])
@pytest.mark.parametrize("primary", ["sparse", "full"])
def test_backward(name, primary):
    r = run_case(name)
    B, Hq, Hkv, N, d, s, k, dt = r["cfg"]
    dims, dev, host, out = r["dims"], r["dev"], r["host"], r["out"]
    g = make_upstream((B, Hq, N, d), 77)
    g_dev = upload(g, dt)
    g_host = oracle_view(g, dt).astype(np.float64)
    alpha = 10.0
    gf, gs = (g_dev, None) if primary == "full" else (None, g_dev)
    grads = api.alloc_backward(dims)
    api.backward(dims, dev["Q"], dev["K"], dev["V"], out, gf, gs, alpha, grads, r["ws"])
    torch.cuda.synchronize()
    ogf, ogs = (g_host, None) if primary == "full" else (None, g_host)
    dQ, dK, dV, l_align, _ = O.ssa_backward(host["Q"], host["K"], host["V"], r["ora_idx"], s, r["scale"],
                                            ogf, ogs, alpha, fwd=r["ora"])
    tol = TOL[dt]["grad"]
    for name_, got, ref in (("dQ", grads["dQ"], dQ), ("dK", grads["dK"], dK), ("dV", grads["dV"], dV)):
        err = rel_l2(f64(got), ref)
        assert err < tol, (name_, err)
    lt = 1e-4 if dt == "f32" else 5e-2
    assert float(grads["align_loss"].item()) == pytest.approx(l_align, rel=lt)


def test_backward_alignment_only_fp32():
    """No upstream gradient: all of dQ, dK, dV comes from the two stop-gradient
    MSE terms (fp32, so h_full - h_sparse is not blurred by output rounding)."""
    r = run_case("f32_gqa_d128")
    B, Hq, Hkv, N, d, s, k, dt = r["cfg"]
    grads = api.alloc_backward(r["dims"])
    alpha = 1000.0
    api.backward(r["dims"], r["dev"]["Q"], r["dev"]["K"], r["dev"]["V"], r["out"], None, None, alpha, grads, r["ws"])
    torch.cuda.synchronize()
    dQ, dK, dV, l_align, _ = O.ssa_backward(r["host"]["Q"], r["host"]["K"], r["host"]["V"], r["ora_idx"], s,
                                            r["scale"], None, None, alpha, fwd=r["ora"])
    for got, ref in ((grads["dQ"], dQ), (grads["dK"], dK), (grads["dV"], dV)):
        assert rel_l2(f64(got), ref) < 1e-3


@pytest.mark.parametrize("name", ["f32_mha_d64", "bf16_gqa_odd_blocks", "bf16_s128"])
@pytest.mark.parametrize("given_lse", [False, True])
def test_dropped_mass(name, given_lse):
    r = run_case(name)
    dt = r["cfg"][7]
    delta = torch.empty_like(r["out"]["delta"])
    lse = r["out"]["lse_full"] if given_lse else None
    api.ssa_dropped_mass(r["dims"], r["dev"]["Q"], r["dev"]["K"], r["out"]["idx"], lse, delta, r["ws"])
    torch.cuda.synchronize()
    ref = O.dropped_mass(r["host"]["Q"], r["host"]["K"], r["ora_idx"], r["cfg"][5], r["scale"])
    assert np.abs(f64(delta) - ref).max() <= TOL[dt]["out"]


@pytest.mark.parametrize("name", ["f32_gqa_d128", "bf16_gqa_odd_blocks"])
def test_align_mse(name):
    r = run_case(name)
    dt = r["cfg"][7]
    loss = torch.empty(2, dtype=torch.float32, device="cuda")
    api.ssa_align_mse(r["dims"], r["out"]["h_full"], r["out"]["h_sparse"], loss, r["ws"])
    torch.cuda.synchronize()
    l_sp, l_cm = O.align_losses(r["ora"]["h_full"], r["ora"]["h_sparse"])
    rt = 1e-4 if dt == "f32" else 5e-2
    assert loss[0].item() == pytest.approx(l_sp, rel=rt)
    assert loss[1].item() == pytest.approx(l_cm, rel=rt)


def test_strided_layout_matches_contiguous():
    """Q/K/V as [B, N, H, d] buffers viewed as [B, H, N, d] (non-contiguous
    strides) give the same outputs as contiguous copies."""
    r = run_case("bf16_gqa_odd_blocks")
    dims, dev, out = r["dims"], r["dev"], r["out"]
    strided = {k: v.transpose(1, 2).contiguous().transpose(1, 2) for k, v in dev.items()}
    assert strided["Q"].stride(2) != dims.d
    o2 = api.alloc_forward(dims)
    h_f = torch.empty((dims.B, dims.N, dims.Hq, dims.d), dtype=torch.bfloat16, device="cuda").transpose(1, 2)
    o2["h_full"] = h_f
    api.forward(dims, strided["Q"], strided["K"], strided["V"], o2, r["ws"])
    torch.cuda.synchronize()
    assert torch.equal(o2["idx"], out["idx"])
    assert torch.equal(o2["h_full"], out["h_full"])
    assert torch.equal(o2["h_sparse"], out["h_sparse"])
    assert torch.equal(o2["delta"], out["delta"])


def test_deterministic():
    r = run_case("bf16_gqa4_long")
    dims, dev, out = r["dims"], r["dev"], r["out"]
    o2 = api.alloc_forward(dims)
    api.forward(dims, dev["Q"], dev["K"], dev["V"], o2, r["ws"])
    g = torch.ones_like(out["h_sparse"])
    g1, g2 = api.alloc_backward(dims), api.alloc_backward(dims)
    api.backward(dims, dev["Q"], dev["K"], dev["V"], out, None, g, 10.0, g1, r["ws"])
    api.backward(dims, dev["Q"], dev["K"], dev["V"], out, None, g, 10.0, g2, r["ws"])
    torch.cuda.synchronize()
    for key in ("idx", "h_full", "h_sparse", "delta", "lse_full", "lse_sel"):
        assert torch.equal(o2[key], out[key]), key
    for key in ("dQ", "dK", "dV", "align_loss"):
        assert torch.equal(g1[key], g2[key]), key


def test_empty_batch_is_noop():
    dims = api.make_dims(0, 4, 2, 512, 128, 64, 4, "bf16")
    e = torch.empty((0, 4, 512, 128), dtype=torch.bfloat16, device="cuda")
    o = api.alloc_forward(dims)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    api.forward(dims, e, e[:, :2], e[:, :2], o, ws)
    torch.cuda.synchronize()


def test_unsupported_shape_raises():
    dims = api.make_dims(1, 2, 2, 1000, 128, 64, 4, "bf16")
    x = torch.zeros((1, 2, 1000, 128), dtype=torch.bfloat16, device="cuda")
    o = {k: torch.zeros(1, device="cuda") for k in ("lse_full", "lse_sel", "delta")}
    with pytest.raises(api.SsaError) as ei:
        api.ssa_fwd_dual(dims, x, x, x, torch.zeros(1, dtype=torch.int32, device="cuda"), x, x,
                         o["lse_full"], o["lse_sel"], o["delta"])
    assert ei.value.code == api.SSA_ERR_UNSUPPORTED


@pytest.mark.parametrize("cfg", [(1, 4, 2, 1024, 128, 64, 5), (1, 2, 1, 1152, 128, 64, 4),
                                 (1, 2, 2, 1024, 128, 128, 3)])
@pytest.mark.parametrize("extra", ["plain", "no_diag"])
def test_forward_custom_selection(cfg, extra):
    """Given selections (not computed by the path): mixed tiles, rows without
    their diagonal block, duplicated entries and -1 padding."""
    B, Hq, Hkv, N, d, s, k = cfg
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 303, "bf16")
    n = N // s
    idx = custom_idx(B, Hq, n, k, seed=N + k, drop_diag_frac=0.3 if extra == "no_diag" else 0.0,
                      pad_frac=0.2 if extra == "no_diag" else 0.0)
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, "bf16")
    out = api.alloc_forward(dims)
    api.ssa_fwd_dual(dims, dev["Q"], dev["K"], dev["V"], torch.from_numpy(idx).cuda(), out["h_full"],
                     out["h_sparse"], out["lse_full"], out["lse_sel"], out["delta"])
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    ora = O.forward_dual(host["Q"], host["K"], host["V"], idx, s, 1 / math.sqrt(d))
    for key in ("h_full", "h_sparse", "delta"):
        err = np.abs(f64(out[key]) - ora[key]).max()
        assert err <= TOL["bf16"]["out"], (key, err)
    fin = np.isfinite(ora["lse_sel"])
    assert np.array_equal(np.isfinite(f64(out["lse_sel"])), fin)
    assert np.abs(f64(out["lse_sel"])[fin] - ora["lse_sel"][fin]).max() <= TOL["bf16"]["lse"]
    assert np.abs(f64(out["lse_full"]) - ora["lse_full"]).max() <= TOL["bf16"]["lse"]


@pytest.mark.parametrize("s", [64, 128])
def test_forward_large_logits(s):
    """Logits with a wide range (keys scaled up, one late block boosted) make
    the running max jump by far more than the rescale threshold mid-row."""
    B, Hq, Hkv, N, d, k = 1, 2, 1, 1024, 128, 4
    from block_sparse_attention_ssa_b200.inputs import make_qkv
    t = make_qkv(B, Hq, Hkv, N, d, s, 404)
    t["K"] *= 3.0
    t["K"][:, :, 5 * s:6 * s] *= 2.5
    host = {x: oracle_view(t[x], "bf16") for x in ("Q", "K", "V")}
    dev = {x: upload(t[x], "bf16") for x in ("Q", "K", "V")}
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, "bf16")
    ws = api.alloc_workspace(dims)
    out = api.alloc_forward(dims)
    api.forward(dims, dev["Q"], dev["K"], dev["V"], out, ws)
    torch.cuda.synchronize()
    ora_scores = O.block_scores(host["Q"], host["K"], s, 1 / math.sqrt(d))
    ora_idx = O.select_blocks(ora_scores, k)
    if compare_selection(out["idx"].cpu().numpy(), ora_idx, ora_scores):
        out["idx"].copy_(torch.from_numpy(ora_idx))
        api.ssa_fwd_dual(dims, dev["Q"], dev["K"], dev["V"], out["idx"], out["h_full"], out["h_sparse"],
                         out["lse_full"], out["lse_sel"], out["delta"])
        torch.cuda.synchronize()
    ora = O.forward_dual(host["Q"], host["K"], host["V"], ora_idx, s, 1 / math.sqrt(d))
    for key in ("h_full", "h_sparse", "delta"):
        err = np.abs(f64(out[key]) - ora[key]).max()
        assert err <= TOL["bf16"]["out"], (key, err)
    assert np.abs(f64(out["lse_full"]) - ora["lse_full"]).max() <= 2e-2


@pytest.mark.parametrize("cfg", [(1, 4, 2, 1024, 128, 64, 5), (1, 2, 1, 1152, 128, 64, 4),
                                 (1, 4, 1, 1024, 128, 128, 3)])
@pytest.mark.parametrize("extra", ["plain", "no_diag"])
def test_backward_custom_selection(cfg, extra):
    """Backward under given selections (tiles selected for one query block and
    dropped for its neighbour, rows without their diagonal block), with
    upstream gradients on both streams and the alignment term."""
    B, Hq, Hkv, N, d, s, k = cfg
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 505, "bf16")
    n = N // s
    idx = custom_idx(B, Hq, n, k, seed=N * 3 + k, drop_diag_frac=0.3 if extra == "no_diag" else 0.0,
                      pad_frac=0.2 if extra == "no_diag" else 0.0)
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, "bf16")
    ws = api.alloc_workspace(dims)
    out = api.alloc_forward(dims)
    out["idx"] = torch.from_numpy(idx).cuda()
    api.ssa_fwd_dual(dims, dev["Q"], dev["K"], dev["V"], out["idx"], out["h_full"], out["h_sparse"],
                     out["lse_full"], out["lse_sel"], out["delta"])
    gf = make_upstream((B, Hq, N, d), 61)
    gs = make_upstream((B, Hq, N, d), 62)
    grads = api.alloc_backward(dims)
    api.backward(dims, dev["Q"], dev["K"], dev["V"], out, upload(gf, "bf16"), upload(gs, "bf16"), 10.0, grads, ws)
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    dQ, dK, dV, l_align, _ = O.ssa_backward(host["Q"], host["K"], host["V"], idx, s, 1 / math.sqrt(d),
                                            oracle_view(gf, "bf16").astype(np.float64),
                                            oracle_view(gs, "bf16").astype(np.float64), 10.0)
    for name_, got, ref in (("dQ", grads["dQ"], dQ), ("dK", grads["dK"], dK), ("dV", grads["dV"], dV)):
        err = rel_l2(f64(got), ref)
        assert err < TOL["bf16"]["grad"], (name_, err)


def test_backward_alignment_only_bf16():
    """bf16 path with no upstream gradient: every gradient comes from the
    alignment terms, whose h_full - h_sparse is formed from bf16 outputs."""
    r = run_case("bf16_gqa_odd_blocks")
    B, Hq, Hkv, N, d, s, k, dt = r["cfg"]
    grads = api.alloc_backward(r["dims"])
    alpha = 1000.0
    api.backward(r["dims"], r["dev"]["Q"], r["dev"]["K"], r["dev"]["V"], r["out"], None, None, alpha, grads, r["ws"])
    torch.cuda.synchronize()
    dQ, dK, dV, l_align, _ = O.ssa_backward(r["host"]["Q"], r["host"]["K"], r["host"]["V"], r["ora_idx"], s,
                                            r["scale"], None, None, alpha, fwd=r["ora"])
    for name_, got, ref in (("dQ", grads["dQ"], dQ), ("dK", grads["dK"], dK), ("dV", grads["dV"], dV)):
        err = rel_l2(f64(got), ref)
        assert err < TOL["bf16"]["grad"], (name_, err)
