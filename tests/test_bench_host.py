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


def test_measured_traffic_only_while_sources_match(tmp_path, monkeypatch):
    """A recorded DRAM-traffic figure is reported only while every kernel source
    it was taken from still has the recorded hash; a changed or missing source,
    or an unknown key, gives None."""
    import hashlib
    import json

    src = tmp_path / "k.cu"
    src.write_text("// kernel v1\n")
    (tmp_path / "profiles").mkdir()
    rec = {"fwd_dual@w": {"dram_bytes_per_launch": 1234,
                          "source_sha256": {"k.cu": hashlib.sha256(src.read_bytes()).hexdigest()}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("fwd_dual", "w") == 1234
    assert bench.measured_traffic("bwd_dual", "w") is None
    src.write_text("// kernel v2\n")
    assert bench.measured_traffic("fwd_dual", "w") is None
    src.unlink()
    assert bench.measured_traffic("fwd_dual", "w") is None
