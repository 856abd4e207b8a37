"""Helpers shared by the GPU parity tests: upload seeded inputs with exactly
the values the oracle sees, run the C-ABI path, and compare selections under
the near-tie rule (a mismatch is accepted only where the oracle's fp64 scores
of the two candidates differ by less than 1e-4 relative)."""
from __future__ import annotations

import numpy as np
import torch

from block_sparse_attention_ssa_b200 import api
from block_sparse_attention_ssa_b200.inputs import make_qkv, round_to_bf16

TOL = {"f32": dict(out=1e-4, lse=1e-4, grad=1e-4), "bf16": dict(out=2e-2, lse=2e-3, grad=5e-2)}
NEAR_TIE_REL = 1e-4


def ensure_library():
    from block_sparse_attention_ssa_b200 import build
    build.build()
    return api.load_library()


def upload(x: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """fp32 numpy -> device tensor holding exactly the values given to the oracle."""
    if dtype == "bf16":
        _, bits = round_to_bf16(x)
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def oracle_view(x: np.ndarray, dtype: str) -> np.ndarray:
    return round_to_bf16(x)[0] if dtype == "bf16" else np.asarray(x, dtype=np.float32)


def case_inputs(B, Hq, Hkv, N, d, s, seed, dtype, plant="exp1"):
    t = make_qkv(B, Hq, Hkv, N, d, s, seed, plant)
    host = {k: oracle_view(t[k], dtype) for k in ("Q", "K", "V")}
    dev = {k: upload(t[k], dtype) for k in ("Q", "K", "V")}
    return host, dev


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def compare_selection(gpu_idx: np.ndarray, ora_idx: np.ndarray, ora_scores: np.ndarray):
    """Rows where the selections differ.  Every such row must be a near tie:
    each block chosen by one side only has a score within NEAR_TIE_REL of the
    oracle's k-th (last kept) candidate score.  Returns the list of near-tie
    rows (b, h, i) so a caller can re-run downstream steps under the oracle's
    indices."""
    assert gpu_idx.shape == ora_idx.shape
    diff = np.any(gpu_idx != ora_idx, axis=-1)
    rows = list(zip(*np.nonzero(diff)))
    for (b, h, i) in rows:
        g = set(int(j) for j in gpu_idx[b, h, i] if j >= 0)
        o = set(int(j) for j in ora_idx[b, h, i] if j >= 0)
        assert len(g) == len(o), (b, h, i, g, o)
        assert i in g and i in o
        kept = [ora_scores[b, h, i, j] for j in o if j != i]
        thr = min(kept)
        for j in g ^ o:
            a = ora_scores[b, h, i, j]
            gap = abs(a - thr)
            assert gap <= NEAR_TIE_REL * max(abs(a), abs(thr)), (b, h, i, j, a, thr)
    return rows


def custom_idx(B, H, n, k, seed, drop_diag_frac=0.0, pad_frac=0.0):
    """Random selections: the diagonal plus k-1 random earlier blocks, with an
    optional share of rows that omit the diagonal, pad with -1 or repeat an
    entry.  Adjacent query blocks disagree often, which at block 64 makes many
    key tiles selected for one half of a 128-row query tile and dropped for
    the other."""
    rng = np.random.Generator(np.random.PCG64(seed))
    idx = np.full((B, H, n, k), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(n):
                if i + 1 <= k:
                    row = list(range(i + 1))
                else:
                    row = sorted(rng.choice(i, size=k - 1, replace=False).tolist() + [i])
                if rng.random() < drop_diag_frac and len(row) > 1:
                    row = row[:-1]
                if rng.random() < pad_frac and len(row) > 1:
                    row = row[:-1] + [row[0]]
                idx[b, h, i, :len(row)] = row
    return idx
