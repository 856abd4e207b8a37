"""Host-side pieces of bench.py that decide reported numbers, checked on the
CPU against brute force."""
import numpy as np
import pytest

import bench


def _brute_pairs(idx, s, per_token):
    B, H, rows, k = idx.shape
    N = rows if per_token else rows * s
    total = 0
    for b in range(B):
        for h in range(H):
            for t in range(N):
                i = t // s
                row = idx[b, h, t if per_token else i]
                kept = {int(j) for j in row if 0 <= j <= i}
                total += sum(1 for u in range(t + 1) if u // s in kept)
    return total


@pytest.mark.parametrize("per_token", [False, True])
@pytest.mark.parametrize("s", [4, 16])
def test_selected_pairs_matches_brute_force(per_token, s):
    """Random selections with duplicates, -1 padding, entries after the row's
    own block and rows that omit their diagonal."""
    rng = np.random.Generator(np.random.PCG64(3 + s + per_token))
    B, H, n, k = 2, 3, 9, 4
    rows = n * s if per_token else n
    idx = rng.integers(-2, n + 2, size=(B, H, rows, k)).astype(np.int32)
    idx[..., 1] = idx[..., 0]  # a duplicate in every row
    assert bench.selected_pairs(idx, s, per_token) == _brute_pairs(idx, s, per_token)


def test_selected_pairs_full_budget_is_every_causal_pair():
    """Every causal block selected: sum |A_t| = N (N + 1) / 2 per (batch, head)."""
    B, H, n, s = 1, 2, 6, 8
    idx = np.tile(np.arange(n, dtype=np.int32), (B, H, n, 1))
    N = n * s
    assert bench.selected_pairs(idx, s, False) == B * H * N * (N + 1) // 2
