"""Plain fp64 CPU oracle of the SSA hot path.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA path and imports nothing from it.

Sources (page title, then section):
  [digest]  "SSA: Achieving Sparser Attention by Aligning Full and Sparse
            Attention Outputs in Feature Space" (blog digest of the paper).
  [summary] "Technische Samenvatting: SSA (Sparse Sparse Attention)".
  [record]  "SSA: Sparse Sparse Attention by Aligning Full and Sparse Attention
            Outputs in Feature Space" (arXiv 2511.20102 library record, abstract).

Everything is computed from the definitions, in float64, one query block at a
time with numpy matmuls inside the block.  No online softmax, no tiling, no
fusion: every softmax is taken over its whole row at once.

Notation: B batch, Hq / Hkv query / key-value heads, g = Hq / Hkv, N tokens,
d head dim, s block size, n = N / s blocks, k budget in blocks (diagonal block
included).  Query head h reads kv head h // g.  Query token t lies in block
i = t // s.  Sel(i) is the selected block set of query block i;
A_t = {u <= t : block(u) in Sel(i)}, D_t = {u <= t : block(u) not in Sel(i)}.

Readings where the pages leave a step open (each also listed in the design
notes):
  * the query side of the block score is the mean of the block's queries
    (per query block selection);
  * scores carry the attention scale 1/sqrt(d) (ranking unchanged);
  * the diagonal block is always kept, counts toward k and is not scored;
  * query blocks with i + 1 <= k keep every causal block;
  * exact score ties go to the smaller block index;
  * the alignment norm is the mean squared error over all B*Hq*N*d elements,
    L_align = L_sparsity + L_commitment with unit weights;
  * no gradient flows through the selection or through delta.
Parity status: every function here is pinned by the CPU tests in
tests/test_oracle_pins.py (closed forms, brute force, torch's fp64 causal
attention, finite differences, and the decode functions against the
forward's rule at the end of each block).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "pool_blocks",
    "block_scores",
    "select_blocks",
    "selection_mask",
    "attention_weights",
    "forward_dual",
    "align_losses",
    "align_grads",
    "backward_streams",
    "ssa_backward",
    "dropped_mass",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def pool_blocks(X: np.ndarray, s: int) -> np.ndarray:
    """Mean of each run of s consecutive tokens: [..., N, d] -> [..., N/s, d].

    [digest] "Practical Implementation of SSA": split the sequence into blocks
    and take each block's representation by mean pooling.
    """
    X = _f64(X)
    N, d = X.shape[-2], X.shape[-1]
    if N % s:
        raise ValueError("N must be a multiple of the block size")
    return X.reshape(*X.shape[:-2], N // s, s, d).mean(axis=-2)


def block_scores(Q: np.ndarray, K: np.ndarray, s: int, scale: float) -> np.ndarray:
    """Block scores S[b, h, i, j] = scale * qbar_i . kbar_j for j < i, -inf elsewhere.

    [digest] "Practical Implementation of SSA": the query is scored against
    every earlier block representation; pooling keeps the ranking because the
    mean of q K^T over a block equals q times the mean of the block's keys.
    qbar_i is the mean of query block i (per query block selection).
    """
    Q, K = _f64(Q), _f64(K)
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    g = Hq // Hkv
    qbar = pool_blocks(Q, s)                       # [B,Hq,n,d]
    kbar = pool_blocks(K, s)                       # [B,Hkv,n,d]
    kbar_h = kbar[:, np.arange(Hq) // g]           # [B,Hq,n,d]
    S = scale * np.einsum("bhid,bhjd->bhij", qbar, kbar_h)
    n = N // s
    S[..., np.tril(np.ones((n, n), dtype=bool)) == 0] = -np.inf  # j > i
    S[..., np.arange(n), np.arange(n)] = -np.inf                  # j == i (forced, not scored)
    return S


def select_blocks(scores: np.ndarray, k: int) -> np.ndarray:
    """Selected block indices [B, H, n, min(k, n)] int32, ascending, -1 padded.

    [digest] "Practical Implementation of SSA": keep the top-k most relevant
    blocks.  Sel(i) = {i} plus the k-1 highest-scoring blocks j < i; ties go to
    the smaller j; when i + 1 <= k every block 0..i is kept.
    """
    S = _f64(scores)
    B, H, n, _ = S.shape
    kk = min(int(k), n)
    if kk < 1:
        raise ValueError("k must be >= 1")
    idx = np.full((B, H, n, kk), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(n):
                if i + 1 <= kk:
                    chosen = np.arange(i + 1)
                else:
                    cand = S[b, h, i, :i]
                    # primary key: score descending; secondary: index ascending
                    order = np.lexsort((np.arange(i), -cand))
                    chosen = np.sort(np.append(order[: kk - 1], i))
                idx[b, h, i, : chosen.size] = chosen
    return idx


def selection_mask(idx: np.ndarray, n: int) -> np.ndarray:
    """Boolean [B, H, n, n]: mask[b, h, i, j] is True when block j is in Sel(i)."""
    B, H, nn, kk = idx.shape
    mask = np.zeros((B, H, n, n), dtype=bool)
    for b in range(B):
        for h in range(H):
            for i in range(n):
                for j in idx[b, h, i]:
                    if j >= 0:
                        mask[b, h, i, j] = True
    return mask


def _row_logits(Qb, Kc, scale):
    return scale * (Qb @ Kc.T)


def attention_weights(Q, K, idx, s: int, scale: float, b: int, h: int):
    """Dense weights of one head: (P_full [N,N], P_sel [N,N]).

    P_full is the causal softmax of x_tu = scale q_t . k_u over u <= t.
    P_sel is the softmax over A_t only ([summary] "1. Probleemstelling":
    a sparse stream normalises over the selected subset, not the full set).
    Meant for tiny inputs (pins and brute force).
    """
    Q, K = _f64(Q), _f64(K)
    N = Q.shape[2]
    n = N // s
    g = Q.shape[1] // K.shape[1]
    X = scale * (Q[b, h] @ K[b, h // g].T)
    causal = np.tril(np.ones((N, N), dtype=bool))
    blk_sel = selection_mask(idx[b : b + 1, h : h + 1], n)[0, 0]      # [n,n]
    tok_sel = np.repeat(np.repeat(blk_sel, s, axis=0), s, axis=1)    # [N,N]
    A = causal & tok_sel
    P_full = _masked_softmax(X, causal)
    P_sel = _masked_softmax(X, A)
    return P_full, P_sel


def _masked_softmax(X: np.ndarray, mask: np.ndarray) -> np.ndarray:
    Xm = np.where(mask, X, -np.inf)
    m = Xm.max(axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    E = np.where(mask, np.exp(Xm - m), 0.0)
    Z = E.sum(axis=-1, keepdims=True)
    return np.where(Z > 0, E / np.where(Z > 0, Z, 1.0), 0.0)


def _logsumexp(X: np.ndarray, mask: np.ndarray) -> np.ndarray:
    Xm = np.where(mask, X, -np.inf)
    m = Xm.max(axis=-1)
    safe = np.where(np.isfinite(m), m, 0.0)
    Z = np.where(mask, np.exp(Xm - safe[..., None]), 0.0).sum(axis=-1)
    with np.errstate(divide="ignore"):
        return np.where(Z > 0, safe + np.log(Z), -np.inf)


def _block_masks(idx_row: np.ndarray, i: int, s: int):
    """For query block i: token-level (causal, selected) masks of shape [s, (i+1)s].

    idx_row is the block's selection [k], or (per-token selection) one
    selection per row of the block [s, k].
    """
    cols = (i + 1) * s
    t = i * s + np.arange(s)[:, None]
    u = np.arange(cols)[None, :]
    causal = u <= t
    rows = np.asarray(idx_row).reshape(-1, np.asarray(idx_row).shape[-1])
    sel = np.zeros((rows.shape[0], cols), dtype=bool)
    for r, row in enumerate(rows):
        for j in row:
            if 0 <= j <= i:
                sel[r, j * s:(j + 1) * s] = True
    return causal, causal & sel


def _sel(idx, b: int, h: int, i: int, s: int, per_token: bool):
    """Selection of query block i: idx[b, h, i] ([k]), or per token the
    block's s rows idx[b, h, i*s:(i+1)*s] ([s, k])."""
    return idx[b, h, i * s:(i + 1) * s] if per_token else idx[b, h, i]


def token_scores(Q: np.ndarray, K: np.ndarray, s: int, scale: float) -> np.ndarray:
    """Per-token block scores S[b, h, t, j] = scale * q_t . kbar_j for j < t // s.

    The literal reading of [digest] "Practical Implementation of SSA": the
    query (token t) is scored against every earlier block representation
    (the mean of the block's keys); -inf for the current and later blocks.
    """
    Q, K = _f64(Q), _f64(K)
    B, Hq, N, d = Q.shape
    g = Hq // K.shape[1]
    n = N // s
    kbar = pool_blocks(K, s)[:, np.arange(Hq) // g]          # [B,Hq,n,d]
    S = scale * np.einsum("bhtd,bhjd->bhtj", Q, kbar)
    tb = (np.arange(N) // s)[:, None]
    S[..., np.arange(n)[None, :] >= tb] = -np.inf
    return S


def select_tokens(scores: np.ndarray, k: int, s: int) -> np.ndarray:
    """Per-token selection [B, H, N, min(k, n)] int32, ascending, -1 padded:
    Sel(t) = {i} plus the k-1 highest-scoring blocks j < i = t // s, ties to
    the smaller j; every block 0..i when i + 1 <= k (the block rule of
    select_blocks applied to each token's own scores)."""
    S = _f64(scores)
    B, H, N, n = S.shape
    kk = min(int(k), n)
    idx = np.full((B, H, N, kk), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for t in range(N):
                i = t // s
                if i + 1 <= kk:
                    chosen = np.arange(i + 1)
                else:
                    cand = S[b, h, t, :i]
                    order = np.lexsort((np.arange(i), -cand))
                    chosen = np.sort(np.append(order[: kk - 1], i))
                idx[b, h, t, : chosen.size] = chosen
    return idx


def forward_dual(Q, K, V, idx, s: int, scale: float, qblocks=None, per_token: bool = False) -> dict[str, np.ndarray]:
    """Both attention streams, the dropped mass and the log-sum-exps.

    Returns float64 arrays:
      h_full   [B,Hq,N,d]  causal softmax attention over u <= t
               ([summary] "Kernmechanisme": the full stream sees every token);
      h_sparse [B,Hq,N,d]  softmax attention over A_t only ([digest]
               "Practical Implementation of SSA": attention over the reduced
               key/value set formed by the selected blocks);
      delta    [B,Hq,N]    full-attention weight that falls on D_t, the
               dropped attention mass ([summary] "1. Probleemstelling" and
               "Bidirectionele Uitlijning"; [record] abstract);
      lse_full, lse_sel [B,Hq,N]  natural-log normalisers of the two softmaxes.
    qblocks: optional iterable of query-block indices to compute (rows of other
    blocks are left at zero); used to sample large problems.
    per_token: idx holds one selection per token ([B, Hq, N, k]).
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, Hq, N, d = Q.shape
    g = Hq // K.shape[1]
    n = N // s
    h_full = np.zeros((B, Hq, N, d))
    h_sparse = np.zeros((B, Hq, N, d))
    delta = np.zeros((B, Hq, N))
    lse_full = np.zeros((B, Hq, N))
    lse_sel = np.zeros((B, Hq, N))
    blocks = range(n) if qblocks is None else sorted(set(int(i) for i in qblocks))
    for b in range(B):
        for h in range(Hq):
            kv = h // g
            for i in blocks:
                rows = slice(i * s, (i + 1) * s)
                cols = (i + 1) * s
                X = _row_logits(Q[b, h, rows], K[b, kv, :cols], scale)
                causal, A = _block_masks(_sel(idx, b, h, i, s, per_token), i, s)
                P_full = _masked_softmax(X, causal)
                P_sel = _masked_softmax(X, A)
                Vc = V[b, kv, :cols]
                h_full[b, h, rows] = P_full @ Vc
                h_sparse[b, h, rows] = P_sel @ Vc
                delta[b, h, rows] = np.where(causal & ~A, P_full, 0.0).sum(axis=-1)
                lse_full[b, h, rows] = _logsumexp(X, causal)
                lse_sel[b, h, rows] = _logsumexp(X, A)
    return {"h_full": h_full, "h_sparse": h_sparse, "delta": delta,
            "lse_full": lse_full, "lse_sel": lse_sel}


def align_losses(h_full, h_sparse) -> tuple[float, float]:
    """(L_sparsity, L_commitment), each the mean squared difference.

    [digest] "Bidirectional Attention Alignment": L_sparsity compares h_full
    with the stop-gradiented h_sparse, L_commitment compares h_sparse with the
    stop-gradiented h_full; L_alignment is their sum.  The norm is read as the
    mean squared error over all elements.  Their values coincide.
    """
    diff = _f64(h_full) - _f64(h_sparse)
    mse = float(np.mean(diff * diff))
    return mse, mse


def align_grads(h_full, h_sparse, M: int | None = None) -> dict[str, np.ndarray]:
    """Gradients of each alignment term w.r.t. each stream, stop-gradient applied.

    d L_sparsity / d h_full  = 2 (h_full - h_sparse) / M,  d L_sparsity / d h_sparse = 0;
    d L_commitment / d h_sparse = 2 (h_sparse - h_full) / M, d L_commitment / d h_full = 0;
    M = number of elements ([digest] "Bidirectional Attention Alignment":
    sg[.] blocks the gradient through the auxiliary operand).  M defaults to
    the size of the arrays given; pass the full problem's count when the arrays
    are a sample of it.
    """
    hf, hs = _f64(h_full), _f64(h_sparse)
    M = hf.size if M is None else int(M)
    zero = np.zeros_like(hf)
    return {"sp_full": 2.0 * (hf - hs) / M, "sp_sparse": zero,
            "cm_full": zero, "cm_sparse": 2.0 * (hs - hf) / M}


def backward_streams(Q, K, V, idx, s: int, scale: float, dh_full, dh_sparse, qblocks=None,
                     per_token: bool = False):
    """Backpropagate upstream gradients of h_full and h_sparse to Q, K, V.

    The two streams are differentiated separately, each through its own
    softmax Jacobian, and summed:
      dX_full   = P_full * (dP_full - rowsum(P_full * dP_full)),  dP_full = dh_full V^T
      dX_sparse = P_sel  * (dP_sel  - rowsum(P_sel  * dP_sel )),  dP_sel  = dh_sparse V^T
      dQ = scale (dX_full + dX_sparse) K,   dK = scale (dX_full + dX_sparse)^T Q,
      dV = P_full^T dh_full + P_sel^T dh_sparse,
    with dK and dV summed over the query heads that share a kv head.  The
    selection is held fixed ([digest] "The Root Cause Behind the Paradox" and
    "SSA's Dual-Stream Training Mechanism": dropped pairs get gradient only
    through the full stream).  dh_full / dh_sparse may be None (zero).
    qblocks: optional query blocks whose contributions are summed (all if None);
    dQ is then exact on those blocks, dK / dV hold only their contributions.
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    g = Hq // Hkv
    n = N // s
    dhf = np.zeros((B, Hq, N, d)) if dh_full is None else _f64(dh_full)
    dhs = np.zeros((B, Hq, N, d)) if dh_sparse is None else _f64(dh_sparse)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    blocks = range(n) if qblocks is None else sorted(set(int(i) for i in qblocks))
    for b in range(B):
        for h in range(Hq):
            kv = h // g
            for i in blocks:
                rows = slice(i * s, (i + 1) * s)
                cols = (i + 1) * s
                Kc, Vc = K[b, kv, :cols], V[b, kv, :cols]
                X = _row_logits(Q[b, h, rows], Kc, scale)
                causal, A = _block_masks(_sel(idx, b, h, i, s, per_token), i, s)
                P_full = _masked_softmax(X, causal)
                P_sel = _masked_softmax(X, A)
                dP_full = dhf[b, h, rows] @ Vc.T
                dP_sel = dhs[b, h, rows] @ Vc.T
                dX_full = P_full * (dP_full - (P_full * dP_full).sum(-1, keepdims=True))
                dX_sel = P_sel * (dP_sel - (P_sel * dP_sel).sum(-1, keepdims=True))
                dX = dX_full + dX_sel
                dQ[b, h, rows] += scale * dX @ Kc
                dK[b, kv, :cols] += scale * dX.T @ Q[b, h, rows]
                dV[b, kv, :cols] += P_full.T @ dhf[b, h, rows] + P_sel.T @ dhs[b, h, rows]
    return dQ, dK, dV


def ssa_backward(Q, K, V, idx, s: int, scale: float, g_full, g_sparse, alpha: float,
                 fwd: dict | None = None, qblocks=None, M: int | None = None, per_token: bool = False):
    """Gradients of L = <g_full, h_full> + <g_sparse, h_sparse> + alpha * L_align.

    [summary] "Bidirectionele Uitlijning": the objective adds alpha times the
    alignment loss to the stream losses; the stream losses reach this layer
    as the upstream gradients g_full / g_sparse (either may be None).
    qblocks / M sample a large problem: only those query blocks are computed,
    M is the full problem's element count (L_align is then that sample's share).
    Returns (dQ, dK, dV, L_align, fwd).
    """
    if fwd is None:
        fwd = forward_dual(Q, K, V, idx, s, scale, qblocks=qblocks, per_token=per_token)
    hf, hs = fwd["h_full"], fwd["h_sparse"]
    gr = align_grads(hf, hs, M)
    dh_full = alpha * (gr["sp_full"] + gr["cm_full"])
    dh_sparse = alpha * (gr["sp_sparse"] + gr["cm_sparse"])
    if g_full is not None:
        dh_full = dh_full + _f64(g_full)
    if g_sparse is not None:
        dh_sparse = dh_sparse + _f64(g_sparse)
    dQ, dK, dV = backward_streams(Q, K, V, idx, s, scale, dh_full, dh_sparse, qblocks=qblocks,
                                  per_token=per_token)
    l_sp, l_cm = align_losses(hf, hs)
    return dQ, dK, dV, l_sp + l_cm, fwd


def dropped_mass(Q, K, idx, s: int, scale: float, per_token: bool = False) -> np.ndarray:
    """delta(t): the full causal softmax weight of row t summed over D_t.

    [summary] "1. Probleemstelling": the dropped attention mass is the
    attention weight given to the tokens the sparse mechanism did not select.
    Computed here without V, straight from the causal softmax of each row.
    """
    Q, K = _f64(Q), _f64(K)
    B, Hq, N, d = Q.shape
    g = Hq // K.shape[1]
    n = N // s
    delta = np.zeros((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            for i in range(n):
                rows = slice(i * s, (i + 1) * s)
                cols = (i + 1) * s
                X = _row_logits(Q[b, h, rows], K[b, h // g, :cols], scale)
                causal, A = _block_masks(_sel(idx, b, h, i, s, per_token), i, s)
                P_full = _masked_softmax(X, causal)
                delta[b, h, rows] = np.where(causal & ~A, P_full, 0.0).sum(-1)
    return delta


def forward_sparse(Q, K, V, idx, s: int, scale: float, qblocks=None, per_token: bool = False) -> dict[str, np.ndarray]:
    """The sparse stream alone: h_sparse and lse_sel, reading only selected blocks.

    [digest] "Practical Implementation of SSA": the selected blocks are
    concatenated into a reduced key/value set and the query attends over it;
    [digest] "Training Efficiency Considerations": in sparse inference this
    is the whole of SSA's attention (the same operation as MoBA's).  Written
    the way the passage describes it -- gather the K/V rows of Sel(i) in
    ascending block order, then one softmax per row with the causal mask on
    the query's own block -- so that it checks forward_dual's masked
    formulation independently.  Returns float64 {"h_sparse", "lse_sel"};
    a row whose A_t is empty gets h_sparse = 0 and lse_sel = -inf.
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, Hq, N, d = Q.shape
    g = Hq // K.shape[1]
    n = N // s
    h_sparse = np.zeros((B, Hq, N, d))
    lse_sel = np.zeros((B, Hq, N))
    blocks = range(n) if qblocks is None else sorted(set(int(i) for i in qblocks))
    for b in range(B):
        for h in range(Hq):
            kv = h // g
            for i in blocks:
                for r in range(s):
                    t = i * s + r
                    row = idx[b, h, t] if per_token else idx[b, h, i]
                    sel = sorted(set(int(j) for j in row if 0 <= j <= i))
                    keys = np.concatenate([np.arange(j * s, (j + 1) * s) for j in sel]) if sel else np.zeros(0, int)
                    cols = keys[keys <= t]
                    if cols.size == 0:
                        lse_sel[b, h, t] = -np.inf
                        continue
                    x = scale * (K[b, kv, cols] @ Q[b, h, t])
                    m = x.max()
                    w = np.exp(x - m)
                    z = w.sum()
                    h_sparse[b, h, t] = (w / z) @ V[b, kv, cols]
                    lse_sel[b, h, t] = m + np.log(z)
    return {"h_sparse": h_sparse, "lse_sel": lse_sel}


def backward_sparse(Q, K, V, idx, s: int, scale: float, g_sparse, qblocks=None, per_token: bool = False):
    """Gradients (dQ, dK, dV) of <g_sparse, h_sparse> for the sparse stream alone.

    The sparse stream's own softmax Jacobian over A_t, the selection held
    fixed; dropped pairs get no gradient ([digest] "The Root Cause Behind the
    Paradox": a purely sparse stream gives no gradient to the tokens it does
    not select).  It is backward_streams with no full-stream gradient.
    """
    return backward_streams(Q, K, V, idx, s, scale, None, g_sparse, qblocks=qblocks, per_token=per_token)


def decode_select(q_prefix, K, t: int, s: int, k: int, scale: float, n_cache: int | None = None) -> np.ndarray:
    """Blocks kept for the generated token at position t: [B, Hq, k_eff] int32.

    The forward's rule ([digest] "Practical Implementation of SSA": score the
    query against every earlier block representation, keep the top-k; the
    current block always kept) applied to the tokens that exist at decode
    time: the query side is the mean of the current block's queries seen so
    far (q_prefix holds rows i*s .. t of block i = t // s), the key side the
    means of the complete blocks j < i.  k_eff = min(k, n_cache), n_cache the
    number of blocks of the cache (default (t+1) rounded up to blocks).
    """
    Qp, K = _f64(q_prefix), _f64(K)
    B, Hq, _, d = Qp.shape
    g = Hq // K.shape[1]
    i = t // s
    n = n_cache if n_cache is not None else i + 1
    kk = min(int(k), n)
    qbar = Qp.mean(axis=2)                                   # [B,Hq,d]
    idx = np.full((B, Hq, kk), -1, dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            if i + 1 <= kk:
                chosen = np.arange(i + 1)
            else:
                kbar = K[b, h // g, : i * s].reshape(i, s, d).mean(axis=1)   # complete blocks
                sc = scale * (kbar @ qbar[b, h])
                order = np.lexsort((np.arange(i), -sc))
                chosen = np.sort(np.append(order[: kk - 1], i))
            idx[b, h, : chosen.size] = chosen
    return idx


def decode_attend(q_t, K, V, t: int, s: int, idx, scale: float):
    """(h [B,Hq,d], lse [B,Hq]) of the token at position t over its kept blocks.

    Softmax of scale * q_t . k_u over A_t = {u <= t : u // s in Sel}, applied
    to V; Sel is idx[b, h] (entries outside [0, t // s] ignored).
    """
    q, K, V = _f64(q_t), _f64(K), _f64(V)
    B, Hq, d = q.shape
    g = Hq // K.shape[1]
    i = t // s
    h_out = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            sel = sorted(set(int(j) for j in idx[b, h] if 0 <= j <= i))
            cols = np.array([u for j in sel for u in range(j * s, j * s + s) if u <= t], dtype=int)
            if cols.size == 0:
                continue
            x = scale * (K[b, h // g, cols] @ q[b, h])
            m = x.max()
            w = np.exp(x - m)
            h_out[b, h] = (w / w.sum()) @ V[b, h // g, cols]
            lse[b, h] = m + np.log(w.sum())
    return h_out, lse
