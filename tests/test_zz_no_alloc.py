"""GPU test of ssa_block_scores_noalloc, the block-scoring entry point for
callers that cannot allocate device memory (it keeps its scratch in a fixed
array inside the library instead of a caller workspace).

Checked through the C ABI against ssa_block_scores, the workspace entry point,
on two calls in a row with different inputs, so a call cannot pass by reading
what the previous one left in the shared scratch.  This file sorts last so a
run that stops at the first failure has already run every other test; it
also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

from block_sparse_attention_ssa_b200 import api
from tests.gpu_util import case_inputs, ensure_library, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    return ensure_library()


def _close(got: torch.Tensor, ref: torch.Tensor):
    a, b = f64(got), f64(ref)
    fin = np.isfinite(b)
    assert np.array_equal(np.isfinite(a), fin)
    assert np.all(a[~fin] == b[~fin])
    scale = max(1.0, np.abs(b[fin]).max())
    np.testing.assert_allclose(a[fin], b[fin], rtol=1e-5, atol=1e-5 * scale)


@pytest.mark.parametrize("cfg", [(1, 8, 2, 2048, 128, 64, 16, "bf16"), (2, 4, 4, 1024, 64, 128, 4, "f32")])
def test_noalloc_matches_workspace_entry_point(cfg):
    B, Hq, Hkv, N, d, s, k, dt = cfg
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, dt)
    n = N // s
    ws = api.alloc_workspace(dims)
    for seed in (11, 12):  # two calls in a row, different inputs
        _, dev = case_inputs(B, Hq, Hkv, N, d, s, seed, dt)
        ref = torch.empty((B, Hq, n, n), dtype=torch.float32, device="cuda")
        got = torch.full((B, Hq, n, n), float("nan"), dtype=torch.float32, device="cuda")
        api.ssa_block_scores(dims, dev["Q"], dev["K"], ref, ws)
        api.ssa_block_scores_noalloc(dims, dev["Q"], dev["K"], got)
        torch.cuda.synchronize()
        _close(got, ref)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # B * (Hq + Hkv) * n * d = 8 * 40 * 256 * 128 floats > 4 Mi floats
    dims = api.make_dims(8, 32, 8, 16384, 128, 64, 16, "bf16")
    x = torch.zeros((1, 1, 64, 128), dtype=torch.bfloat16, device="cuda")
    scores = torch.zeros(1, dtype=torch.float32, device="cuda")
    with pytest.raises(api.SsaError) as ei:
        api.ssa_block_scores_noalloc(dims, x, x, scores)
    assert ei.value.code == api.SSA_ERR_WORKSPACE
