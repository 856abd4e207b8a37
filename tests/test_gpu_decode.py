"""GPU parity of the decode step (ssa_decode_prefill, ssa_decode_step) against
the fp64 oracle (decode_select / decode_attend), through the C ABI.

Each case prefills the state from a prompt that ends mid-block, then decodes
token after token across block boundaries (the pooled-key cache grows and the
query-block sum restarts), checking every step's selection (bit-exact, near
ties logged and the output compared under the kernel's selection), output and
log-sum-exp, and at the end the state buffers.  A full-size case decodes the
last token of the gqa_16k cache.  Tolerances as for the forward."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_ssa_b200 import api
from block_sparse_attention_ssa_b200.inputs import WORKLOADS, make_workload_inputs
from oracle import ssa_oracle as O
from tests.gpu_util import NEAR_TIE_REL, TOL, case_inputs, ensure_library, f64

pytestmark = pytest.mark.gpu

# name: B, Hq, Hkv, N (cache), d, s, k, dtype, prompt length, decoded tokens
CASES = {
    "bf16_gqa4_s64": (1, 8, 2, 1024, 128, 64, 4, "bf16", 3 * 64 + 21, 150),
    "bf16_s128_b2": (2, 4, 1, 1024, 128, 128, 3, "bf16", 2 * 128 + 100, 170),
    "f32_d64": (1, 4, 4, 512, 64, 64, 3, "f32", 64 + 40, 100),
    "bf16_full_budget": (1, 4, 2, 512, 128, 64, 16, "bf16", 30, 60),
    "f32_from_empty_prompt": (1, 2, 1, 256, 128, 64, 2, "f32", 0, 140),
    # 16 heads per kv head and k = 40: each CTA's slice keeps 39 candidates
    # per head, merged from eight lists in shared memory (k > 16)
    "bf16_g16_k40_s16": (1, 16, 1, 4096, 64, 16, 40, "bf16", 2600, 120),
    # 32 heads per kv head: more than one 16-row fragment, so the attention
    # phase runs on CUDA cores with bf16 inputs
    "bf16_g32_cuda_cores": (1, 32, 1, 1024, 64, 64, 6, "bf16", 500, 60),
}


@pytest.fixture(scope="module", autouse=True)
def lib():
    return ensure_library()


def _near_tie_ok(gpu_sel, ora_sel, q_prefix, K, t, s, scale):
    """Every block chosen by one side only scores within NEAR_TIE_REL of the
    oracle's weakest kept block (fp64 scores)."""
    i = t // s
    d = K.shape[-1]
    qbar = q_prefix.mean(axis=0)
    kbar = K[: i * s].reshape(i, s, d).mean(axis=1)
    sc = scale * (kbar @ qbar)
    kept = [sc[j] for j in ora_sel if j != i]
    thr = min(kept)
    for j in set(gpu_sel) ^ set(ora_sel):
        assert abs(sc[j] - thr) <= NEAR_TIE_REL * max(abs(sc[j]), abs(thr)), (t, j, sc[j], thr)


@pytest.mark.parametrize("name", list(CASES))
def test_decode_sequence(name):
    B, Hq, Hkv, N, d, s, k, dt, t0, L = CASES[name]
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 919, dt)
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, dt)
    scale = 1 / math.sqrt(d)
    st = api.alloc_decode(dims)
    ws = api.alloc_workspace(dims)
    st["qsum"].fill_(float("nan"))  # prefill must define every entry it owns
    api.ssa_decode_prefill(dims, dev["Q"], dev["K"], t0, st["qsum"], st["kbar"])
    g = Hq // Hkv
    n_cache = N // s
    near = 0
    for t in range(t0, t0 + L):
        i = t // s
        api.ssa_decode_step(dims, dev["Q"][:, :, t:t + 1], dev["K"], dev["V"], t, st["qsum"], st["kbar"],
                            st["h"], st["lse"], st["idx"], ws)
        torch.cuda.synchronize()
        gidx = st["idx"].cpu().numpy()
        qp = host["Q"][:, :, i * s:t + 1].astype(np.float64)
        oidx = O.decode_select(qp, host["K"], t, s, k, scale, n_cache=n_cache)
        use = oidx
        if not np.array_equal(gidx, oidx):
            for b in range(B):
                for h in range(Hq):
                    gs = [int(j) for j in gidx[b, h] if j >= 0]
                    os_ = [int(j) for j in oidx[b, h] if j >= 0]
                    if gs != os_:
                        assert len(gs) == len(os_) and i in gs
                        _near_tie_ok(gs, os_, qp[b, h], host["K"][b, h // g].astype(np.float64), t, s, scale)
                        near += 1
            use = gidx
        h_ref, lse_ref = O.decode_attend(host["Q"][:, :, t], host["K"], host["V"], t, s, use, scale)
        err = np.abs(f64(st["h"])[:, :, 0] - h_ref).max()
        assert err <= TOL[dt]["out"], (t, err)
        assert np.abs(f64(st["lse"]) - lse_ref).max() <= TOL[dt]["lse"], t
    assert api.ssa_device_status() == api.SSA_OK
    if near:
        print(f"{name}: {near} near-tie rows compared under the kernel's selection")
    # state after the last token
    t_last = t0 + L - 1
    full = (t_last + 1) // s
    kb_ref = host["K"][:, :, : full * s].astype(np.float64).reshape(B, Hkv, full, s, d).mean(axis=3)
    np.testing.assert_allclose(f64(st["kbar"])[:, :, :full], kb_ref, rtol=1e-5, atol=1e-5)
    i = t_last // s
    if (t_last + 1) % s:
        qs_ref = host["Q"][:, :, i * s:t_last + 1].astype(np.float64).sum(axis=2)
        np.testing.assert_allclose(f64(st["qsum"]), qs_ref, rtol=1e-4, atol=1e-4)


def test_decode_rejects_bad_positions():
    B, Hq, Hkv, N, d, s, k = 1, 2, 1, 256, 64, 64, 2
    host, dev = case_inputs(B, Hq, Hkv, N, d, s, 3, "f32")
    dims = api.make_dims(B, Hq, Hkv, N, d, s, k, "f32")
    st = api.alloc_decode(dims)
    ws = api.alloc_workspace(dims)
    for t in (-1, N):
        with pytest.raises(api.SsaError) as ei:
            api.ssa_decode_step(dims, dev["Q"][:, :, 0:1], dev["K"], dev["V"], t, st["qsum"], st["kbar"],
                                st["h"], st["lse"], st["idx"], ws)
        assert ei.value.code == api.SSA_ERR_INVALID_ARG
    with pytest.raises(api.SsaError):
        api.ssa_decode_prefill(dims, dev["Q"], dev["K"], N + 1, st["qsum"], st["kbar"])


@pytest.mark.parametrize("wname", ["gqa_16k", "long_64k", "paper_b16_8k"])
def test_decode_last_token_full_size(wname):
    """Prefill N-1 tokens of a full-size workload and decode the last token
    (it closes the last block, so the selection is the forward's)."""
    w = WORKLOADS[wname]
    host = make_workload_inputs(w)
    dev = {x: torch.from_numpy(host[x + "_bits"].view(np.int16)).view(torch.bfloat16).cuda() for x in "QKV"}
    dims = api.make_dims(w.B, w.Hq, w.Hkv, w.N, w.d, w.block, w.topk, w.dtype)
    st = api.alloc_decode(dims)
    ws = api.alloc_workspace(dims)
    t = w.N - 1
    api.ssa_decode_prefill(dims, dev["Q"], dev["K"], t, st["qsum"], st["kbar"])
    api.ssa_decode_step(dims, dev["Q"][:, :, t:t + 1], dev["K"], dev["V"], t, st["qsum"], st["kbar"], st["h"],
                        st["lse"], st["idx"], ws)
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    s, scale = w.block, w.scale
    i = t // s
    rng = np.random.Generator(np.random.PCG64(77))
    heads = sorted({0, w.Hq - 1, int(rng.integers(w.Hq))})
    g = w.Hq // w.Hkv
    for b in range(w.B):
        for h in heads:
            Kh = host["K"][b:b + 1, h // g:h // g + 1].astype(np.float64)
            Vh = host["V"][b:b + 1, h // g:h // g + 1].astype(np.float64)
            qp = host["Q"][b:b + 1, h:h + 1, i * s:t + 1].astype(np.float64)
            oidx = O.decode_select(qp, Kh, t, s, w.topk, scale, n_cache=w.n_blocks)
            gsel = st["idx"][b:b + 1, h:h + 1].cpu().numpy()
            if not np.array_equal(gsel, oidx):
                _near_tie_ok([int(j) for j in gsel[0, 0] if j >= 0], [int(j) for j in oidx[0, 0] if j >= 0],
                             qp[0, 0], Kh[0, 0], t, s, scale)
            href, lref = O.decode_attend(host["Q"][b:b + 1, h:h + 1, t].astype(np.float64), Kh, Vh, t, s, gsel, scale)
            assert np.abs(f64(st["h"][b, h, 0]) - href[0, 0]).max() <= TOL["bf16"]["out"]
            assert abs(float(st["lse"][b, h]) - lref[0, 0]) <= TOL["bf16"]["lse"]
