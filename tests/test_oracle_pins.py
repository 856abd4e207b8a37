"""Pins of the fp64 oracle against facts the pages and the mathematics fix.

Each test is chosen so that a plausible slip in the oracle (a dropped 1/s in
the pooling, a wrong scale, an off-by-one in the causal or block mask, a
transposed operand, a lost stop-gradient, a wrong GQA head mapping) fails it.
None of these tests calls the CUDA path.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import ssa_oracle as O
from block_sparse_attention_ssa_b200.inputs import make_qkv, make_scores, make_upstream

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny(B=1, Hq=2, Hkv=1, N=32, d=4, s=8, seed=7, plant="exp1"):
    t = make_qkv(B, Hq, Hkv, N, d, s, seed, plant)
    return t["Q"].astype(np.float64), t["K"].astype(np.float64), t["V"].astype(np.float64)


# ---------------------------------------------------------------- pooling + scores

def test_block_score_is_mean_of_token_logits():
    """Bilinearity ("Practical Implementation of SSA": Mean(qK^T) = q Mean(K)^T):
    the pooled score equals the mean over t in block i, u in block j of the
    token logits scale*q_t.k_u, summed here by brute force."""
    Q, K, _ = tiny(Hq=4, Hkv=2, N=24, d=3, s=4)
    s, scale = 4, 0.37
    S = O.block_scores(Q, K, s, scale)
    B, Hq, N, d = Q.shape
    n = N // s
    for h in range(Hq):
        for i in range(n):
            for j in range(n):
                if j >= i:
                    assert S[0, h, i, j] == -np.inf
                    continue
                acc = 0.0
                for t in range(i * s, (i + 1) * s):
                    for u in range(j * s, (j + 1) * s):
                        acc += scale * sum(Q[0, h, t, c] * K[0, h // 2, u, c] for c in range(d))
                assert S[0, h, i, j] == pytest.approx(acc / (s * s), rel=1e-12, abs=1e-12)


# ---------------------------------------------------------------- top-k selection

@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_selection_brute_force(k):
    """Sel(i) \\ {i} is the (k-1)-subset of {0..i-1} with the largest total score
    (continuous random scores: the maximiser is unique); the diagonal is always
    in; rows with i+1 <= k keep every causal block."""
    n = 8
    S = make_scores(2, 3, n, seed=11 + k).astype(np.float64)
    idx = O.select_blocks(S, k)
    assert idx.shape == (2, 3, n, min(k, n))
    for b, h, i in itertools.product(range(2), range(3), range(n)):
        row = [int(j) for j in idx[b, h, i] if j >= 0]
        assert row == sorted(row)
        assert all(j == -1 for j in idx[b, h, i, len(row):])
        if i + 1 <= k:
            assert row == list(range(i + 1))
            continue
        best, best_set = -np.inf, None
        for sub in itertools.combinations(range(i), k - 1):
            tot = sum(S[b, h, i, j] for j in sub)
            if tot > best:
                best, best_set = tot, sub
        assert row == sorted(list(best_set) + [i])


def test_selection_tie_rule_and_stable_argsort():
    """Exact ties go to the smaller block index: equal scores pick 0..k-2,
    and on tie-heavy random rows the choice equals a stable argsort of -score."""
    n, k = 12, 5
    S = np.zeros((1, 1, n, n))
    S[..., np.triu_indices(n)[0], np.triu_indices(n)[1]] = -np.inf
    idx = O.select_blocks(S, k)
    for i in range(k, n):
        assert list(idx[0, 0, i]) == list(range(k - 1)) + [i]
    S = make_scores(2, 2, 40, seed=5, tie_frac=0.5).astype(np.float64)
    idx = O.select_blocks(S, 9)
    for b, h, i in itertools.product(range(2), range(2), range(9, 40)):
        order = np.argsort(-S[b, h, i, :i], kind="stable")[:8]
        assert list(idx[b, h, i]) == sorted(list(order) + [i])


def test_topk_larger_than_blocks_is_clamped():
    S = make_scores(1, 1, 6, seed=3).astype(np.float64)
    idx = O.select_blocks(S, 100)
    assert idx.shape[-1] == 6
    for i in range(6):
        assert list(idx[0, 0, i, : i + 1]) == list(range(i + 1))


# ---------------------------------------------------------------- streams

def _direct_causal(Q, K, V, scale):
    """Textbook causal softmax attention by explicit loops (one head)."""
    N, d = Q.shape
    out = np.zeros((N, d))
    for t in range(N):
        logits = [scale * float(Q[t] @ K[u]) for u in range(t + 1)]
        m = max(logits)
        w = [math.exp(x - m) for x in logits]
        z = sum(w)
        out[t] = sum(wi * V[u] for u, wi in enumerate(w)) / z
    return out


def test_full_budget_reduces_to_causal_attention():
    """With k >= n every causal block is kept: h_sparse = h_full, delta = 0, and
    h_full is textbook causal attention (torch fp64 SDPA and an explicit loop)."""
    Q, K, V = tiny(Hq=4, Hkv=2, N=32, d=8, s=8)
    s, scale = 8, 1 / math.sqrt(8)
    idx = O.select_blocks(O.block_scores(Q, K, s, scale), 4)
    f = O.forward_dual(Q, K, V, idx, s, scale)
    np.testing.assert_array_equal(f["delta"], 0.0)
    np.testing.assert_allclose(f["h_sparse"], f["h_full"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(f["lse_sel"], f["lse_full"], rtol=0, atol=1e-14)
    q = torch.from_numpy(Q)
    k = torch.from_numpy(np.repeat(K, 2, axis=1))
    v = torch.from_numpy(np.repeat(V, 2, axis=1))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)
    np.testing.assert_allclose(f["h_full"], ref.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(f["h_full"][0, 3], _direct_causal(Q[0, 3], K[0, 1], V[0, 1], scale),
                               rtol=0, atol=1e-12)
    # lse_full is log sum_{u<=t} exp(x_tu)
    x = scale * Q[0, 1] @ K[0, 0].T
    for t in (0, 5, 31):
        assert f["lse_full"][0, 1, t] == pytest.approx(math.log(sum(math.exp(v) for v in x[t, : t + 1])), abs=1e-12)


def test_softmax_rows_sum_to_one_and_respect_masks():
    Q, K, V = tiny(N=32, d=4, s=8)
    s, scale = 8, 0.5
    idx = O.select_blocks(O.block_scores(Q, K, s, scale), 2)
    P_full, P_sel = O.attention_weights(Q, K, idx, s, scale, 0, 1)
    np.testing.assert_allclose(P_full.sum(-1), 1.0, atol=1e-12)
    np.testing.assert_allclose(P_sel.sum(-1), 1.0, atol=1e-12)
    assert np.all(np.triu(P_full, 1) == 0) and np.all(np.triu(P_sel, 1) == 0)
    mask = O.selection_mask(idx, 4)[0, 1]
    tok = np.repeat(np.repeat(mask, s, 0), s, 1)
    assert np.all(P_sel[~tok] == 0)


def test_uniform_logits_closed_form():
    """Q = 0 makes every logit 0: all block scores tie, so Sel(i) = {0..k-2, i};
    both softmaxes are uniform, so h_full is the running mean of v, h_sparse the
    mean over A_t, delta_t = |D_t| / (t+1), lse_full = log(t+1), lse_sel = log|A_t|."""
    N, d, s, k = 48, 3, 8, 3
    _, K, V = tiny(N=N, d=d, s=s, Hq=1)
    Q = np.zeros((1, 1, N, d))
    idx = O.select_blocks(O.block_scores(Q, K, s, 0.5), k)
    f = O.forward_dual(Q, K, V, idx, s, 0.5)
    for t in range(N):
        i = t // s
        sel = set(range(i + 1)) if i + 1 <= k else set(range(k - 1)) | {i}
        assert set(int(j) for j in idx[0, 0, i] if j >= 0) == sel
        A = [u for u in range(t + 1) if u // s in sel]
        np.testing.assert_allclose(f["h_full"][0, 0, t], V[0, 0, : t + 1].mean(0), atol=1e-14)
        np.testing.assert_allclose(f["h_sparse"][0, 0, t], V[0, 0, A].mean(0), atol=1e-14)
        assert f["delta"][0, 0, t] == pytest.approx((t + 1 - len(A)) / (t + 1), abs=1e-15)
        assert f["lse_full"][0, 0, t] == pytest.approx(math.log(t + 1), abs=1e-14)
        assert f["lse_sel"][0, 0, t] == pytest.approx(math.log(len(A)), abs=1e-14)


def test_dropped_mass_decomposition_and_linear_bound():
    """h_full = (1 - delta) h_sparse + delta h_D, h_D the softmax average over the
    dropped set D_t (brute force per row); hence |h_full - h_sparse| <= 2 delta max|v|,
    the linear error bound in the dropped mass (record abstract; summary
    "3. Belangrijkste Bijdragen")."""
    Q, K, V = tiny(Hq=2, Hkv=1, N=64, d=4, s=8, seed=9)
    s, k, scale = 8, 3, 0.5
    idx = O.select_blocks(O.block_scores(Q, K, s, scale), k)
    f = O.forward_dual(Q, K, V, idx, s, scale)
    vmax = np.linalg.norm(V, axis=-1).max()
    for h in range(2):
        for t in range(64):
            i = t // s
            sel = set(int(j) for j in idx[0, h, i] if j >= 0)
            x = [scale * float(Q[0, h, t] @ K[0, 0, u]) for u in range(t + 1)]
            D = [u for u in range(t + 1) if u // s not in sel]
            dlt = f["delta"][0, h, t]
            gap = np.linalg.norm(f["h_full"][0, h, t] - f["h_sparse"][0, h, t])
            assert gap <= 2 * dlt * vmax + 1e-12
            if not D:
                assert dlt == 0.0
                continue
            m = max(x[u] for u in D)
            w = np.array([math.exp(x[u] - m) for u in D])
            hD = (w[:, None] * V[0, 0, D]).sum(0) / w.sum()
            recon = (1 - dlt) * f["h_sparse"][0, h, t] + dlt * hD
            np.testing.assert_allclose(f["h_full"][0, h, t], recon, atol=1e-12)
            assert 0.0 < dlt < 1.0


def test_two_partial_softmaxes_recombine_to_full():
    """One pass with two disjoint softmaxes (over A_t and over D_t, each with its
    own max) recombines to the full softmax: this is the merge rule the fused
    kernel relies on, checked against the oracle's direct full-row softmax."""
    Q, K, V = tiny(Hq=1, N=64, d=4, s=8, seed=13)
    s, k, scale = 8, 2, 0.8
    idx = O.select_blocks(O.block_scores(Q, K, s, scale), k)
    f = O.forward_dual(Q, K, V, idx, s, scale)
    for t in range(64):
        i = t // s
        sel = set(int(j) for j in idx[0, 0, i] if j >= 0)
        x = np.array([scale * float(Q[0, 0, t] @ K[0, 0, u]) for u in range(t + 1)])
        inA = np.array([u // s in sel for u in range(t + 1)])
        mA = x[inA].max()
        lA = np.exp(x[inA] - mA).sum()
        oA = (np.exp(x[inA] - mA)[:, None] * V[0, 0, : t + 1][inA]).sum(0)
        if (~inA).any():
            mD = x[~inA].max()
            lD = np.exp(x[~inA] - mD).sum()
            oD = (np.exp(x[~inA] - mD)[:, None] * V[0, 0, : t + 1][~inA]).sum(0)
        else:
            mD, lD, oD = -np.inf, 0.0, np.zeros(4)
        M = max(mA, mD)
        a, dd = math.exp(mA - M), (math.exp(mD - M) if lD > 0 else 0.0)
        np.testing.assert_allclose((a * oA + dd * oD) / (a * lA + dd * lD), f["h_full"][0, 0, t], atol=1e-12)
        np.testing.assert_allclose(oA / lA, f["h_sparse"][0, 0, t], atol=1e-12)
        lse_drop = mD + math.log(lD) if lD > 0 else -np.inf
        lse_full = np.logaddexp(mA + math.log(lA), lse_drop)
        assert f["lse_full"][0, 0, t] == pytest.approx(lse_full, abs=1e-12)
        assert f["delta"][0, 0, t] == pytest.approx(math.exp(lse_drop - lse_full) if lD > 0 else 0.0, abs=1e-12)


def test_dropped_mass_standalone_matches_definition():
    Q, K, V = tiny(Hq=2, N=32, d=4, s=8, seed=21)
    s, k, scale = 8, 2, 0.5
    idx = O.select_blocks(O.block_scores(Q, K, s, scale), k)
    dm = O.dropped_mass(Q, K, idx, s, scale)
    for h in range(2):
        P_full, _ = O.attention_weights(Q, K, idx, s, scale, 0, h)
        mask = np.repeat(np.repeat(O.selection_mask(idx, 4)[0, h], s, 0), s, 1)
        np.testing.assert_allclose(dm[0, h], 1.0 - (P_full * mask).sum(-1), atol=1e-14)


def test_gqa_equals_duplicated_kv_heads():
    """Query head h reads kv head h // g: the GQA result equals running with the
    kv heads repeated g times, and dK / dV are the per-copy sums."""
    Q, K, V = tiny(Hq=4, Hkv=2, N=32, d=4, s=8, seed=17)
    s, k, scale = 8, 2, 0.5
    Kd, Vd = np.repeat(K, 2, axis=1), np.repeat(V, 2, axis=1)
    S1, S2 = O.block_scores(Q, K, s, scale), O.block_scores(Q, Kd, s, scale)
    np.testing.assert_array_equal(S1, S2)
    idx = O.select_blocks(S1, k)
    f1, f2 = O.forward_dual(Q, K, V, idx, s, scale), O.forward_dual(Q, Kd, Vd, idx, s, scale)
    for key in f1:
        np.testing.assert_allclose(f1[key], f2[key], atol=1e-14)
    gf = make_upstream(Q.shape, 1).astype(np.float64)
    g1 = O.ssa_backward(Q, K, V, idx, s, scale, gf, None, 10.0)
    g2 = O.ssa_backward(Q, Kd, Vd, idx, s, scale, gf, None, 10.0)
    np.testing.assert_allclose(g1[0], g2[0], atol=1e-13)
    np.testing.assert_allclose(g1[1], g2[1].reshape(1, 2, 2, 32, 4).sum(2), atol=1e-13)
    np.testing.assert_allclose(g1[2], g2[2].reshape(1, 2, 2, 32, 4).sum(2), atol=1e-13)


# ---------------------------------------------------------------- backward

FD_CFG = dict(B=1, Hq=2, Hkv=1, N=32, d=4, s=8)


def _fd_grad(fun, arrays, eps=1e-6):
    grads = []
    for a in arrays:
        g = np.zeros_like(a)
        it = np.nditer(a, flags=["multi_index"])
        for _ in it:
            ix = it.multi_index
            old = a[ix]
            a[ix] = old + eps
            fp = fun()
            a[ix] = old - eps
            fm = fun()
            a[ix] = old
            g[ix] = (fp - fm) / (2 * eps)
        grads.append(g)
    return grads


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


@pytest.mark.parametrize("primary", ["sparse", "full"])
def test_backward_matches_finite_differences(primary):
    """Central differences of L = <g, h_primary> + alpha * mean((h_full - h_sparse)^2)
    with the selection held fixed.  With the stop-gradients, the gradient of
    L_sparsity + L_commitment equals the plain gradient of one mean squared
    difference (each stream gets 2(h_self - h_other)/M), which is what the
    finite differences see."""
    Q, K, V = tiny(**FD_CFG, seed=3)
    s, k, scale, alpha = 8, 2, 0.5, 10.0
    idx = O.select_blocks(O.block_scores(Q, K, s, scale), k)
    g = make_upstream(Q.shape, 5).astype(np.float64)
    gf, gs = (g, None) if primary == "full" else (None, g)

    def loss():
        f = O.forward_dual(Q, K, V, idx, s, scale)
        hp = f["h_full"] if primary == "full" else f["h_sparse"]
        return float((g * hp).sum() + alpha * np.mean((f["h_full"] - f["h_sparse"]) ** 2))

    dQ, dK, dV, l_align, fwd = O.ssa_backward(Q, K, V, idx, s, scale, gf, gs, alpha)
    fQ, fK, fV = _fd_grad(loss, [Q, K, V])
    assert _rel(dQ, fQ) < 1e-6 and _rel(dK, fK) < 1e-6 and _rel(dV, fV) < 1e-6
    assert l_align == pytest.approx(2 * np.mean((fwd["h_full"] - fwd["h_sparse"]) ** 2), rel=1e-14)
    assert l_align > 0


def test_stop_gradient_semantics():
    """L_sparsity moves only the full stream (h_sparse frozen), L_commitment only
    the sparse stream (h_full frozen) ("Bidirectional Attention Alignment")."""
    Q, K, V = tiny(**FD_CFG, seed=4)
    s, k, scale = 8, 2, 0.5
    idx = O.select_blocks(O.block_scores(Q, K, s, scale), k)
    f0 = O.forward_dual(Q, K, V, idx, s, scale)
    hf0, hs0 = f0["h_full"].copy(), f0["h_sparse"].copy()
    gr = O.align_grads(hf0, hs0)
    assert np.all(gr["sp_sparse"] == 0) and np.all(gr["cm_full"] == 0)

    def l_sp():
        return float(np.mean((O.forward_dual(Q, K, V, idx, s, scale)["h_full"] - hs0) ** 2))

    def l_cm():
        return float(np.mean((O.forward_dual(Q, K, V, idx, s, scale)["h_sparse"] - hf0) ** 2))

    for fun, dhf, dhs in ((l_sp, gr["sp_full"], None), (l_cm, None, gr["cm_sparse"])):
        got = O.backward_streams(Q, K, V, idx, s, scale, dhf, dhs)
        fd = _fd_grad(fun, [Q, K, V])
        for a, b in zip(got, fd):
            assert _rel(a, b) < 1e-5


def test_dropped_pairs_get_no_sparse_gradient():
    """A key whose block is dropped by every query block gets gradient only from
    the full stream: with dh_full = 0 its dK and dV are exactly zero."""
    Q, K, V = tiny(Hq=1, N=48, d=4, s=8, seed=8)
    s, k, scale = 8, 2, 0.5
    idx = O.select_blocks(O.block_scores(Q, K, s, scale), k)
    used = set(int(j) for j in idx[0, 0].ravel() if j >= 0)
    unused = [j for j in range(6) if j not in used]
    dQ, dK, dV = O.backward_streams(Q, K, V, idx, s, scale, None, make_upstream(Q.shape, 2))
    for j in unused:
        assert np.all(dK[0, 0, j * s:(j + 1) * s] == 0) and np.all(dV[0, 0, j * s:(j + 1) * s] == 0)
    _, dKf, dVf = O.backward_streams(Q, K, V, idx, s, scale, make_upstream(Q.shape, 2), None)
    for j in unused:
        assert np.abs(dVf[0, 0, j * s:(j + 1) * s]).sum() > 0


# ---------------------------------------------------------------- sparse stream alone

def _random_selection(B, H, n, k, seed):
    """Diagonal plus k-1 random earlier blocks per row; some rows drop their
    diagonal, repeat an entry or pad with -1."""
    rng = np.random.Generator(np.random.PCG64(seed))
    idx = np.full((B, H, n, k), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(n):
                row = list(range(i + 1)) if i + 1 <= k else sorted(
                    rng.choice(i, size=k - 1, replace=False).tolist() + [i])
                u = rng.random()
                if u < 0.25 and len(row) > 1:
                    row = row[:-1]
                elif u < 0.4 and len(row) > 1:
                    row = row[:-1] + [row[0]]
                idx[b, h, i, :len(row)] = row
    return idx


def test_sparse_alone_equals_masked_sparse_stream():
    """Gathering the selected blocks into a reduced K/V set ("Practical
    Implementation of SSA") gives the same h_sparse and lse_sel as masking the
    unselected blocks out of the whole causal row (forward_dual), for any
    selection, including rows without their diagonal block."""
    Q, K, V = tiny(Hq=4, Hkv=2, N=48, d=5, s=8, seed=21)
    s, scale = 8, 0.45
    idx = _random_selection(1, 4, 6, 3, seed=5)
    idx[0, 1, 3] = -1  # a query block that attends nothing
    a = O.forward_sparse(Q, K, V, idx, s, scale)
    f = O.forward_dual(Q, K, V, idx, s, scale)
    np.testing.assert_allclose(a["h_sparse"], f["h_sparse"], rtol=0, atol=1e-13)
    fin = np.isfinite(f["lse_sel"])
    assert np.array_equal(np.isfinite(a["lse_sel"]), fin) and not fin.all()
    np.testing.assert_allclose(a["lse_sel"][fin], f["lse_sel"][fin], rtol=0, atol=1e-13)


def test_sparse_alone_full_budget_is_causal_attention():
    """With every causal block selected the sparse stream is textbook causal
    attention (torch fp64 SDPA)."""
    Q, K, V = tiny(Hq=2, Hkv=1, N=40, d=6, s=8, seed=22)
    s, scale = 8, 1 / math.sqrt(6)
    idx = O.select_blocks(O.block_scores(Q, K, s, scale), 5)
    a = O.forward_sparse(Q, K, V, idx, s, scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q), torch.from_numpy(np.repeat(K, 2, axis=1)), torch.from_numpy(np.repeat(V, 2, axis=1)),
        is_causal=True, scale=scale)
    np.testing.assert_allclose(a["h_sparse"], ref.numpy(), rtol=0, atol=1e-12)


def test_sparse_alone_reads_only_selected_blocks():
    """K and V rows of a block that no query block selects may hold anything
    (NaN here): the sparse stream never reads them."""
    Q, K, V = tiny(Hq=2, Hkv=1, N=48, d=4, s=8, seed=23)
    s, scale = 8, 0.5
    idx = _random_selection(1, 2, 6, 2, seed=9)
    idx[idx == 2] = -1  # nobody selects block 2, not even query block 2
    ref = O.forward_sparse(Q, K, V, idx, s, scale)
    K2, V2 = K.copy(), V.copy()
    K2[:, :, 16:24] = np.nan
    V2[:, :, 16:24] = np.nan
    got = O.forward_sparse(Q, K2, V2, idx, s, scale)
    np.testing.assert_array_equal(got["h_sparse"], ref["h_sparse"])
    np.testing.assert_array_equal(got["lse_sel"], ref["lse_sel"])


def test_sparse_backward_matches_finite_differences():
    """Central differences of <g, h_sparse> for the sparse stream alone, the
    selection held fixed."""
    Q, K, V = tiny(**FD_CFG, seed=24)
    s, scale = 8, 0.5
    idx = _random_selection(1, FD_CFG["Hq"], FD_CFG["N"] // s, 2, seed=13)
    g = make_upstream(Q.shape, 25).astype(np.float64)

    def loss():
        return float((g * O.forward_sparse(Q, K, V, idx, s, scale)["h_sparse"]).sum())

    dQ, dK, dV = O.backward_sparse(Q, K, V, idx, s, scale, g)
    fQ, fK, fV = _fd_grad(loss, [Q, K, V])
    assert _rel(dQ, fQ) < 1e-6 and _rel(dK, fK) < 1e-6 and _rel(dV, fV) < 1e-6


# ---------------------------------------------------------------- decode

def test_decode_at_block_end_equals_forward_rule():
    """At the last token of a block the prefix of the block is the whole block,
    so the decode selection is the forward's selection of that query block and
    the decode output is the forward's sparse-stream row."""
    Q, K, V = tiny(Hq=4, Hkv=2, N=48, d=5, s=8, seed=31)
    s, k, scale = 8, 3, 0.4
    n = 6
    ref_idx = O.select_blocks(O.block_scores(Q, K, s, scale), k)
    ref = O.forward_sparse(Q, K, V, ref_idx, s, scale)
    for i in range(n):
        t = i * s + s - 1
        idx = O.decode_select(Q[:, :, i * s:t + 1], K, t, s, k, scale, n_cache=n)
        np.testing.assert_array_equal(idx, ref_idx[:, :, i])
        h, lse = O.decode_attend(Q[:, :, t], K, V, t, s, idx, scale)
        np.testing.assert_allclose(h, ref["h_sparse"][:, :, t], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse, ref["lse_sel"][:, :, t], rtol=0, atol=1e-13)


def test_decode_partial_block_uses_prefix_mean():
    """Mid-block, the query side is the mean of the block's queries so far;
    the kept set is the best-scoring (k-1)-subset of earlier blocks, found by
    enumeration from scores summed by explicit loops."""
    Q, K, _ = tiny(Hq=2, Hkv=1, N=48, d=3, s=8, seed=32)
    s, k, scale = 8, 3, 0.7
    for t in (19, 27, 41, 44):
        i = t // s
        idx = O.decode_select(Q[:, :, i * s:t + 1], K, t, s, k, scale, n_cache=6)
        for h in range(2):
            qbar = [sum(Q[0, h, u, c] for u in range(i * s, t + 1)) / (t - i * s + 1) for c in range(3)]
            sc = []
            for j in range(i):
                kbar = [sum(K[0, 0, u, c] for u in range(j * s, j * s + s)) / s for c in range(3)]
                sc.append(scale * sum(qbar[c] * kbar[c] for c in range(3)))
            best = max(itertools.combinations(range(i), k - 1), key=lambda c: sum(sc[j] for j in c))
            assert sorted(best) + [i] == [int(j) for j in idx[0, h] if j >= 0]


def test_decode_uniform_scores_tie_rule():
    """Q = 0: every score ties, so the smallest indices win: Sel = {0..k-2, i};
    the weights are uniform, so h is the mean of V over the kept keys <= t."""
    _, K, V = tiny(Hq=1, N=64, d=3, s=8, seed=33)
    s, k = 8, 3
    q = np.zeros((1, 1, 3))
    for t in (20, 35, 63):
        i = t // s
        idx = O.decode_select(np.zeros((1, 1, t - i * s + 1, 3)), K, t, s, k, 0.5, n_cache=8)
        assert [int(j) for j in idx[0, 0]] == [0, 1, i]
        h, lse = O.decode_attend(q, K, V, t, s, idx, 0.5)
        A = [u for u in range(t + 1) if u // s in (0, 1, i)]
        np.testing.assert_allclose(h[0, 0], V[0, 0, A].mean(0), atol=1e-14)
        assert lse[0, 0] == pytest.approx(math.log(len(A)), abs=1e-14)


def test_decode_full_budget_is_causal_attention():
    """With every block kept the decode output is the last row of textbook
    causal attention over the prefix (torch fp64 SDPA)."""
    Q, K, V = tiny(Hq=4, Hkv=2, N=40, d=6, s=8, seed=34)
    s, scale = 8, 1 / math.sqrt(6)
    for t in (0, 9, 23, 39):
        i = t // s
        idx = O.decode_select(Q[:, :, i * s:t + 1], K, t, s, 5, scale, n_cache=5)
        h, _ = O.decode_attend(Q[:, :, t], K, V, t, s, idx, scale)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q[:, :, :t + 1]), torch.from_numpy(np.repeat(K[:, :, :t + 1], 2, axis=1)),
            torch.from_numpy(np.repeat(V[:, :, :t + 1], 2, axis=1)), is_causal=True, scale=scale)
        np.testing.assert_allclose(h, ref.numpy()[:, :, t], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- per-token selection

def test_token_selection_brute_force():
    """Per token, the kept set is the best (k-1)-subset of the earlier blocks,
    found by enumeration from scores summed by explicit loops over q_t and the
    block's keys; the token's own block is always kept."""
    Q, K, _ = tiny(Hq=2, Hkv=1, N=40, d=3, s=8, seed=41)
    s, k, scale = 8, 3, 0.6
    idx = O.select_tokens(O.token_scores(Q, K, s, scale), k, s)
    for h in range(2):
        for t in range(40):
            i = t // s
            got = [int(j) for j in idx[0, h, t] if j >= 0]
            if i + 1 <= k:
                assert got == list(range(i + 1))
                continue
            sc = [scale * sum(Q[0, h, t, c] * sum(K[0, 0, u, c] for u in range(j * s, j * s + s)) / s
                              for c in range(3)) for j in range(i)]
            best = max(itertools.combinations(range(i), k - 1), key=lambda c: sum(sc[j] for j in c))
            assert got == sorted(best) + [i]


def test_token_mode_equals_block_mode_for_block_constant_queries():
    """When every query of a block is the same vector, each token's score row
    is its block's score row, so per-token selection equals per-block
    selection and every output and gradient agrees."""
    Q, K, V = tiny(Hq=4, Hkv=2, N=48, d=4, s=8, seed=42)
    s, k, scale = 8, 2, 0.5
    Qc = np.repeat(Q.reshape(1, 4, 6, 8, 4).mean(axis=3), 8, axis=2)     # block-constant queries
    ib = O.select_blocks(O.block_scores(Qc, K, s, scale), k)
    it = O.select_tokens(O.token_scores(Qc, K, s, scale), k, s)
    np.testing.assert_array_equal(it, np.repeat(ib, 8, axis=2))
    fb = O.forward_dual(Qc, K, V, ib, s, scale)
    ft = O.forward_dual(Qc, K, V, it, s, scale, per_token=True)
    for key in fb:
        np.testing.assert_allclose(ft[key], fb[key], rtol=0, atol=1e-13)
    g = make_upstream(Q.shape, 43).astype(np.float64)
    gb = O.ssa_backward(Qc, K, V, ib, s, scale, None, g, 5.0)
    gt = O.ssa_backward(Qc, K, V, it, s, scale, None, g, 5.0, per_token=True)
    for a, b in zip(gt[:3], gb[:3]):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_token_mode_rows_by_explicit_loops():
    """Rows of one block keep different sets; every row's sparse and full
    softmax, dropped mass and the gathered sparse stream match loops over
    that row's own kept keys."""
    Q, K, V = tiny(Hq=2, Hkv=1, N=48, d=3, s=8, seed=44)
    s, k, scale = 8, 2, 0.8
    idx = O.select_tokens(O.token_scores(Q, K, s, scale), k, s)
    assert any(len({tuple(idx[0, 0, t]) for t in range(i * s, i * s + s)}) > 1 for i in range(2, 6))
    f = O.forward_dual(Q, K, V, idx, s, scale, per_token=True)
    fs = O.forward_sparse(Q, K, V, idx, s, scale, per_token=True)
    dm = O.dropped_mass(Q, K, idx, s, scale, per_token=True)
    for h in range(2):
        for t in range(48):
            keep = {int(j) for j in idx[0, h, t] if j >= 0}
            x = [scale * sum(Q[0, h, t, c] * K[0, 0, u, c] for c in range(3)) for u in range(t + 1)]
            m = max(x)
            w = [math.exp(v - m) for v in x]
            A = [u for u in range(t + 1) if u // s in keep]
            zA, z = sum(w[u] for u in A), sum(w)
            hs = [sum(w[u] * V[0, 0, u, c] for u in A) / zA for c in range(3)]
            hf = [sum(w[u] * V[0, 0, u, c] for u in range(t + 1)) / z for c in range(3)]
            np.testing.assert_allclose(f["h_sparse"][0, h, t], hs, atol=1e-12)
            np.testing.assert_allclose(fs["h_sparse"][0, h, t], hs, atol=1e-12)
            np.testing.assert_allclose(f["h_full"][0, h, t], hf, atol=1e-12)
            assert f["delta"][0, h, t] == pytest.approx(1 - zA / z, abs=1e-12)
            assert dm[0, h, t] == pytest.approx(1 - zA / z, abs=1e-12)


def test_token_mode_backward_matches_finite_differences():
    """Central differences of <g, h_sparse> + alpha * mean((h_f - h_s)^2) with
    per-token selections held fixed."""
    Q, K, V = tiny(**FD_CFG, seed=45)
    s, k, scale, alpha = 8, 2, 0.5, 10.0
    idx = O.select_tokens(O.token_scores(Q, K, s, scale), k, s)
    g = make_upstream(Q.shape, 46).astype(np.float64)

    def loss():
        f = O.forward_dual(Q, K, V, idx, s, scale, per_token=True)
        return float((g * f["h_sparse"]).sum() + alpha * np.mean((f["h_full"] - f["h_sparse"]) ** 2))

    dQ, dK, dV, _, _ = O.ssa_backward(Q, K, V, idx, s, scale, None, g, alpha, per_token=True)
    fQ, fK, fV = _fd_grad(loss, [Q, K, V])
    assert _rel(dQ, fQ) < 1e-6 and _rel(dK, fK) < 1e-6 and _rel(dV, fV) < 1e-6


# ---------------------------------------------------------------- frozen regression fixture

def test_golden_fixture_is_reproduced():
    """tests/golden/oracle_tiny.json was written by tests/golden/make_golden.py,
    which calls only the oracle; any change to the oracle's arithmetic shows here."""
    with open(os.path.join(GOLDEN, "oracle_tiny.json")) as fh:
        gold = json.load(fh)
    from tests.golden.make_golden import compute
    now = compute()
    assert now["idx"] == gold["idx"]
    for key in ("delta", "lse_full", "lse_sel", "h_full_row0", "h_sparse_row0", "dQ_sum", "dK_sum", "dV_sum", "l_align"):
        np.testing.assert_allclose(np.array(now[key]), np.array(gold[key]), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- sampled query blocks

def test_query_block_sampling_matches_the_whole_problem():
    """The full-size GPU checks compare sampled query blocks against the oracle
    run on a prefix with qblocks=[i].  Causality fixes what that must give: rows
    of block i see only keys u <= t, so the prefix of rows 0 .. (i+1)s - 1 with
    only block i computed yields exactly the whole problem's rows of block i
    (outputs, log-sum-exps, dropped mass, dQ, with the alignment term scaled by
    the whole problem's element count M); and key block n-1 is reachable only
    from query block n-1, so its dK, dV from qblocks=[n-1] alone are the whole
    problem's."""
    Q, K, V = tiny(Hq=4, Hkv=2, N=48, d=4, s=8, seed=11)
    s, scale, k, alpha = 8, 0.41, 3, 10.0
    N = Q.shape[2]
    n = N // s
    idx = O.select_blocks(O.block_scores(Q, K, s, scale), k)
    g = make_upstream(Q.shape, 5)
    M = Q.size
    fs = O.forward_sparse(Q, K, V, idx, s, scale)
    fd = O.forward_dual(Q, K, V, idx, s, scale)
    dQs, dKs, dVs = O.backward_sparse(Q, K, V, idx, s, scale, g)
    dQd, dKd, dVd, _, _ = O.ssa_backward(Q, K, V, idx, s, scale, None, g, alpha)
    close = dict(rtol=1e-10, atol=1e-12)
    for i in range(n):
        N1, rows = (i + 1) * s, slice(i * s, (i + 1) * s)
        pre = (Q[:, :, :N1], K[:, :, :N1], V[:, :, :N1], idx[:, :, :i + 1])
        f = O.forward_sparse(*pre, s, scale, qblocks=[i])
        np.testing.assert_allclose(f["h_sparse"][:, :, rows], fs["h_sparse"][:, :, rows], **close)
        np.testing.assert_allclose(f["lse_sel"][:, :, rows], fs["lse_sel"][:, :, rows], **close)
        f = O.forward_dual(*pre, s, scale, qblocks=[i])
        for key in ("h_full", "h_sparse", "delta", "lse_full", "lse_sel"):
            np.testing.assert_allclose(f[key][:, :, rows], fd[key][:, :, rows], **close, err_msg=key)
        dq, _, _ = O.backward_sparse(*pre, s, scale, g[:, :, :N1], qblocks=[i])
        np.testing.assert_allclose(dq[:, :, rows], dQs[:, :, rows], **close)
        dq, _, _, _, _ = O.ssa_backward(*pre, s, scale, None, g[:, :, :N1], alpha, qblocks=[i], M=M)
        np.testing.assert_allclose(dq[:, :, rows], dQd[:, :, rows], **close)
    last = slice((n - 1) * s, N)
    _, dk, dv = O.backward_sparse(Q, K, V, idx, s, scale, g, qblocks=[n - 1])
    np.testing.assert_allclose(dk[:, :, last], dKs[:, :, last], **close)
    np.testing.assert_allclose(dv[:, :, last], dVs[:, :, last], **close)
    # the sample restricts: key block 0 takes gradient from query blocks other
    # than the sampled one, so there the sample and the whole problem differ
    assert not np.allclose(dk[:, :, :s], dKs[:, :, :s], rtol=1e-3, atol=1e-6)
    _, dk, dv, _, _ = O.ssa_backward(Q, K, V, idx, s, scale, None, g, alpha, qblocks=[n - 1], M=M)
    np.testing.assert_allclose(dk[:, :, last], dKd[:, :, last], **close)
    np.testing.assert_allclose(dv[:, :, last], dVd[:, :, last], **close)
    assert not np.allclose(dk[:, :, :s], dKd[:, :, :s], rtol=1e-3, atol=1e-6)
