"""Failure detection on the GPU without a fault.

A self-test kernel waits on a barrier that nothing completes; its bounded
wait runs out and it records SSA_ERR_TIMEOUT in the per-device status report,
as a stuck tensor-core kernel would.  The host reads and clears the report.
The report is only a report: a timed-out call on one stream leaves the calls
on another stream (with their own workspace) correct, bit for bit, and calls
made while the report holds the error do their full work."""
import pytest
import torch

from block_sparse_attention_ssa_b200 import api
from tests.gpu_util import case_inputs, ensure_library

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    return ensure_library()


def _step(dims, dev, stream):
    """Selection, dual forward and dual backward on `stream`, every output
    NaN-filled first so that skipped work would show."""
    with torch.cuda.stream(stream):
        out = api.alloc_forward(dims)
        for key in ("h_full", "h_sparse", "lse_full", "lse_sel", "delta"):
            out[key].fill_(float("nan"))
        grads = api.alloc_backward(dims)
        for key in ("dQ", "dK", "dV"):
            grads[key].fill_(float("nan"))
        ws = api.alloc_workspace(dims)
        g = torch.ones_like(dev["Q"])
        api.forward(dims, dev["Q"], dev["K"], dev["V"], out, ws, stream)
        api.backward(dims, dev["Q"], dev["K"], dev["V"], out, None, g, 10.0, grads, ws, stream)
    return out, grads


def test_timeout_is_reported_and_leaves_other_streams_correct():
    assert api.ssa_device_status(clear=True) == api.SSA_OK
    B, Hq, Hkv, N, d, s, k = 1, 4, 2, 512, 128, 64, 3
    _, dev = case_inputs(B, Hq, Hkv, N, d, s, 909, "bf16")
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, "bf16")
    main = torch.cuda.current_stream()
    good_out, good_grads = _step(dims, dev, main)
    torch.cuda.synchronize()
    assert torch.isfinite(good_out["h_full"].float()).all()
    assert torch.isfinite(good_grads["dK"].float()).all()

    # A timed-out wait on stream A while stream B runs a whole step.
    stream_a, stream_b = torch.cuda.Stream(), torch.cuda.Stream()
    stream_a.wait_stream(main)
    stream_b.wait_stream(main)
    api.ssa_selftest_timeout(stream_a)
    out_b, grads_b = _step(dims, dev, stream_b)
    torch.cuda.synchronize()
    assert api.ssa_device_status(clear=False) == api.SSA_ERR_TIMEOUT

    # A step issued while the report holds the error, after the timeout ended.
    out_c, grads_c = _step(dims, dev, main)
    torch.cuda.synchronize()
    assert api.ssa_device_status(clear=True) == api.SSA_ERR_TIMEOUT
    assert api.ssa_device_status(clear=False) == api.SSA_OK

    for o, gr in ((out_b, grads_b), (out_c, grads_c)):
        for key in ("h_full", "h_sparse", "lse_full", "lse_sel", "delta"):
            assert torch.equal(o[key], good_out[key]), key
        for key in ("dQ", "dK", "dV", "align_loss"):
            assert torch.equal(gr[key], good_grads[key]), key
