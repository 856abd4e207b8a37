"""Failure detection on the GPU without a fault.

A self-test kernel waits on a barrier that nothing completes; its bounded
wait runs out and it records SSA_ERR_TIMEOUT in the device status word, as a
stuck tensor-core kernel would.  The host reads the word; while it holds the
error the tensor-core kernels skip their work; clearing it restores them."""
import numpy as np
import pytest
import torch

from block_sparse_attention_ssa_b200 import api
from tests.gpu_util import case_inputs, ensure_library

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    return ensure_library()


def _forward(dims, dev):
    out = api.alloc_forward(dims)
    for key in ("h_full", "h_sparse", "lse_full", "delta"):
        out[key].fill_(float("nan"))
    ws = api.alloc_workspace(dims)
    api.forward(dims, dev["Q"], dev["K"], dev["V"], out, ws)
    torch.cuda.synchronize()
    return out


def test_timeout_is_reported_and_cleared():
    assert api.ssa_device_status(clear=True) == api.SSA_OK
    B, Hq, Hkv, N, d, s, k = 1, 2, 1, 512, 128, 64, 3
    _, dev = case_inputs(B, Hq, Hkv, N, d, s, 909, "bf16")
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, "bf16")
    good = _forward(dims, dev)
    assert torch.isfinite(good["h_full"].float()).all()

    api.ssa_selftest_timeout()
    assert api.ssa_device_status(clear=False) == api.SSA_ERR_TIMEOUT
    # the context is intact and the tensor-core forward skips its work
    skipped = _forward(dims, dev)
    assert torch.isnan(skipped["h_full"].float()).all()
    assert api.ssa_device_status(clear=True) == api.SSA_ERR_TIMEOUT
    assert api.ssa_device_status(clear=False) == api.SSA_OK

    again = _forward(dims, dev)
    for key in ("h_full", "h_sparse", "lse_full", "delta"):
        assert torch.equal(again[key], good[key]), key
