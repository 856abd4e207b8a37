"""GPU parity at the full sizes of the five benchmark workloads, in the launch
configuration bench.py times (same entry points, same buffers, one stream).

* tiny_f32 is small enough for the whole oracle.
* For the other workloads the block selection is checked on every row (the
  oracle's pooled scores and top-k are cheap) under the near-tie rule, and
  the outputs are checked on sampled (batch, query head, query block) units
  that the oracle computes one by one from the prefix they depend on:
  forward rows, dropped mass, dQ rows of the sampled query blocks, and dK / dV
  of the last key block of a kv head (which only its own query block reaches).
* dK / dV of one whole (batch, kv head) group are checked at full size on
  gqa_16k and on sweep_32k with k = 64, with the oracle's backward over every
  query block of the group (the early key blocks collect from all of them).
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_ssa_b200 import api
from block_sparse_attention_ssa_b200.inputs import SWEEP_TOPK, WORKLOADS, make_workload_inputs
from oracle import ssa_oracle as O
from tests.gpu_util import TOL, compare_selection, ensure_library, f64, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    return ensure_library()


def _device(w, host):
    out = {}
    for name in ("Q", "K", "V"):
        if w.dtype == "bf16":
            out[name] = torch.from_numpy(host[name + "_bits"].view(np.int16)).view(torch.bfloat16).cuda()
        else:
            out[name] = torch.from_numpy(host[name]).cuda()
    return out


def _samples(w, rng):
    n = w.n_blocks
    blocks = sorted({0, min(w.topk - 1, n - 1), min(w.topk, n - 1), n // 2, n - 1, int(rng.integers(n))})
    heads = sorted({0, w.Hq - 1, int(rng.integers(w.Hq))})
    return [(int(rng.integers(w.B)), h, i) for h in heads for i in blocks]


def _run(w, with_bwd):
    host = make_workload_inputs(w)
    dev = _device(w, host)
    dims = api.make_dims(w.B, w.Hq, w.Hkv, w.N, w.d, w.block, w.topk, w.dtype)
    ws = api.alloc_workspace(dims)
    out = api.alloc_forward(dims)
    api.forward(dims, dev["Q"], dev["K"], dev["V"], out, ws)
    torch.cuda.synchronize()
    scale = 1.0 / math.sqrt(w.d)
    ora_scores = O.block_scores(host["Q"], host["K"], w.block, scale)
    ora_idx = O.select_blocks(ora_scores, w.topk)
    near = compare_selection(out["idx"].cpu().numpy(), ora_idx, ora_scores)
    if near:
        print(f"{w.name}: {len(near)} near-tie rows; downstream compared under the oracle's indices")
        out["idx"].copy_(torch.from_numpy(ora_idx))
        api.ssa_fwd_dual(dims, dev["Q"], dev["K"], dev["V"], out["idx"], out["h_full"], out["h_sparse"],
                         out["lse_full"], out["lse_sel"], out["delta"])
    grads = None
    if with_bwd:
        grads = api.alloc_backward(dims)
        ones = torch.ones((w.B, w.Hq, w.N, w.d), dtype=dims.torch_dtype, device="cuda")
        api.backward(dims, dev["Q"], dev["K"], dev["V"], out, None, ones, 10.0, grads, ws)
    delta2 = torch.empty_like(out["delta"])
    api.ssa_dropped_mass(dims, dev["Q"], dev["K"], out["idx"], out["lse_full"], delta2, ws)
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    return host, out, grads, delta2, ora_idx, scale


def _check_forward_samples(w, host, out, delta2, ora_idx, scale, rng):
    tol = TOL[w.dtype]
    s = w.block
    for (b, h, i) in _samples(w, rng):
        kv = h // w.group
        N1 = (i + 1) * s
        f = O.forward_dual(host["Q"][b:b + 1, h:h + 1, :N1], host["K"][b:b + 1, kv:kv + 1, :N1],
                           host["V"][b:b + 1, kv:kv + 1, :N1], ora_idx[b:b + 1, h:h + 1, :i + 1], s, scale,
                           qblocks=[i])
        rows = slice(i * s, N1)
        for key in ("h_full", "h_sparse", "delta"):
            got = f64(out[key][b, h, rows])
            err = np.abs(got - f[key][0, 0, rows]).max()
            assert err <= tol["out"], (w.name, b, h, i, key, err)
        assert np.abs(f64(out["lse_full"][b, h, rows]) - f["lse_full"][0, 0, rows]).max() <= tol["lse"]
        assert np.abs(f64(delta2[b, h, rows]) - f["delta"][0, 0, rows]).max() <= tol["out"]


def _check_backward_samples(w, host, grads, ora_idx, scale, rng):
    tol = TOL[w.dtype]["grad"]
    s, n = w.block, w.n_blocks
    M = w.B * w.Hq * w.N * w.d
    for (b, h, i) in _samples(w, rng)[:6]:
        kv = h // w.group
        N1 = (i + 1) * s
        g = np.ones((1, 1, N1, w.d))
        dQ, _, _, _, _ = O.ssa_backward(host["Q"][b:b + 1, h:h + 1, :N1], host["K"][b:b + 1, kv:kv + 1, :N1],
                                        host["V"][b:b + 1, kv:kv + 1, :N1], ora_idx[b:b + 1, h:h + 1, :i + 1], s,
                                        scale, None, g, 10.0, qblocks=[i], M=M)
        rows = slice(i * s, N1)
        err = rel_l2(f64(grads["dQ"][b, h, rows]), dQ[0, 0, rows])
        assert err < tol, (w.name, "dQ", b, h, i, err)
    # dK, dV of the last key block: only query block n-1 of the group's heads reaches it.
    b, kv = 0, int(rng.integers(w.Hkv))
    heads = slice(kv * w.group, (kv + 1) * w.group)
    g = np.ones((1, w.group, w.N, w.d))
    _, dK, dV, _, _ = O.ssa_backward(host["Q"][b:b + 1, heads], host["K"][b:b + 1, kv:kv + 1],
                                     host["V"][b:b + 1, kv:kv + 1], ora_idx[b:b + 1, heads], s, scale, None, g,
                                     10.0, qblocks=[n - 1], M=M)
    rows = slice((n - 1) * s, w.N)
    assert rel_l2(f64(grads["dK"][b, kv, rows]), dK[0, 0, rows]) < tol
    assert rel_l2(f64(grads["dV"][b, kv, rows]), dV[0, 0, rows]) < tol


def _compare_group(w, got_k, got_v, dK, dV, rng, what):
    tol = TOL[w.dtype]["grad"]
    s, n = w.block, w.n_blocks
    assert rel_l2(got_k, dK) < tol, (w.name, what, "dK")
    assert rel_l2(got_v, dV) < tol, (w.name, what, "dV")
    for j in sorted({0, n // 2, int(rng.integers(n))}):
        rows = slice(j * s, (j + 1) * s)
        ek, ev = rel_l2(got_k[rows], dK[rows]), rel_l2(got_v[rows], dV[rows])
        assert ek < tol and ev < tol, (w.name, what, "key block", j, ek, ev)


def test_full_size_group_backward_gqa16k():
    """dK, dV of one whole (batch, kv head) group of gqa_16k in the bench's
    configuration (sum(h_sparse), alpha = 10): the oracle runs the backward
    over every query block of the group's g heads, so every key block
    receives all its contributions -- key block 0 from all n query blocks of
    each head, the longest walks of the dK/dV kernel.  Compared on the whole
    group and on key blocks 0, n/2 and a random one."""
    w = WORKLOADS["gqa_16k"]
    rng = np.random.Generator(np.random.PCG64(4242))
    host, _, grads, _, ora_idx, scale = _run(w, with_bwd=True)
    M = w.B * w.Hq * w.N * w.d
    b, kv = int(rng.integers(w.B)), int(rng.integers(w.Hkv))
    heads = slice(kv * w.group, (kv + 1) * w.group)
    g = np.ones((1, w.group, w.N, w.d))
    _, dK, dV, _, _ = O.ssa_backward(host["Q"][b:b + 1, heads], host["K"][b:b + 1, kv:kv + 1],
                                     host["V"][b:b + 1, kv:kv + 1], ora_idx[b:b + 1, heads], w.block, scale, None, g,
                                     10.0, M=M)
    _compare_group(w, f64(grads["dK"][b, kv]), f64(grads["dV"][b, kv]), dK[0, 0], dV[0, 0], rng, (b, kv))


def test_full_size_group_backward_sweep32k_k64():
    """The same at sweep_32k with k = 64 (n = 512 key blocks, 64 selected per
    query block), with the upstream gradient on the full stream of one query
    head of the group (zero elsewhere, alpha = 0) so that the oracle needs one
    head: the kernel still walks all g heads and every causal query tile for
    each key tile, 512 of them for key block 0, adding the other heads' exact
    zeros."""
    w = WORKLOADS["sweep_32k"].with_topk(64)
    rng = np.random.Generator(np.random.PCG64(4343))
    host = make_workload_inputs(w)
    dev = _device(w, host)
    dims = api.make_dims(w.B, w.Hq, w.Hkv, w.N, w.d, w.block, w.topk, w.dtype)
    ws = api.alloc_workspace(dims)
    out = api.alloc_forward(dims)
    api.forward(dims, dev["Q"], dev["K"], dev["V"], out, ws)
    torch.cuda.synchronize()
    scale = 1.0 / math.sqrt(w.d)
    ora_scores = O.block_scores(host["Q"], host["K"], w.block, scale)
    ora_idx = O.select_blocks(ora_scores, w.topk)
    if compare_selection(out["idx"].cpu().numpy(), ora_idx, ora_scores):
        out["idx"].copy_(torch.from_numpy(ora_idx))
        api.ssa_fwd_dual(dims, dev["Q"], dev["K"], dev["V"], out["idx"], out["h_full"], out["h_sparse"],
                         out["lse_full"], out["lse_sel"], out["delta"])
    b, kv = 0, int(rng.integers(w.Hkv))
    h = kv * w.group + int(rng.integers(w.group))
    g_full = torch.zeros((w.B, w.Hq, w.N, w.d), dtype=dims.torch_dtype, device="cuda")
    g_full[b, h] = 1.0
    grads = api.alloc_backward(dims)
    api.backward(dims, dev["Q"], dev["K"], dev["V"], out, g_full, None, 0.0, grads, ws)
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    _, dK, dV = O.backward_streams(host["Q"][b:b + 1, h:h + 1], host["K"][b:b + 1, kv:kv + 1],
                                   host["V"][b:b + 1, kv:kv + 1], ora_idx[b:b + 1, h:h + 1], w.block, scale,
                                   np.ones((1, 1, w.N, w.d)), None)
    _compare_group(w, f64(grads["dK"][b, kv]), f64(grads["dV"][b, kv]), dK[0, 0], dV[0, 0], rng, (b, h))


def test_tiny_f32_whole_problem():
    w = WORKLOADS["tiny_f32"]
    host, out, _, delta2, ora_idx, scale = _run(w, with_bwd=False)
    f = O.forward_dual(host["Q"], host["K"], host["V"], ora_idx, w.block, scale)
    for key in ("h_full", "h_sparse", "delta", "lse_full", "lse_sel"):
        assert np.abs(f64(out[key]) - f[key]).max() <= 1e-4, key
    assert np.abs(f64(delta2) - f["delta"]).max() <= 1e-4


@pytest.mark.parametrize("name", ["mha_8k", "gqa_16k", "long_64k", "paper_b16_8k", "paper_b16_8k_d128"])
def test_full_size_sampled(name):
    w = WORKLOADS[name]
    rng = np.random.Generator(np.random.PCG64(77))
    host, out, grads, delta2, ora_idx, scale = _run(w, with_bwd=w.backward)
    _check_forward_samples(w, host, out, delta2, ora_idx, scale, rng)
    if w.backward:
        _check_backward_samples(w, host, grads, ora_idx, scale, rng)


@pytest.mark.parametrize("k", SWEEP_TOPK)
def test_budget_sweep(k):
    w = WORKLOADS["sweep_32k"].with_topk(k)
    rng = np.random.Generator(np.random.PCG64(100 + k))
    host, out, grads, delta2, ora_idx, scale = _run(w, with_bwd=True)
    _check_forward_samples(w, host, out, delta2, ora_idx, scale, rng)
    _check_backward_samples(w, host, grads, ora_idx, scale, rng)
    print(f"sweep_32k k={k}: mean delta {float(out['delta'].mean()):.4f}")


def test_maximum_block_count():
    """The largest supported selection: n = 2048 blocks (N = 131072 at block
    64) with k = 64, through block scores, top-k (2047 candidates per row),
    the dual forward, the dropped mass, the backward and the sparse stream
    alone; checked on sampled query blocks, including the last one, and on
    the last key block's gradients."""
    from block_sparse_attention_ssa_b200.inputs import Workload
    w = Workload("max_blocks", 1, 2, 1, 131072, 128, 64, 64, "bf16", 1007)
    rng = np.random.Generator(np.random.PCG64(5))
    host, out, grads, delta2, ora_idx, scale = _run(w, with_bwd=True)
    _check_forward_samples(w, host, out, delta2, ora_idx, scale, rng)
    _check_backward_samples(w, host, grads, ora_idx, scale, rng)
    dims = api.make_dims(w.B, w.Hq, w.Hkv, w.N, w.d, w.block, w.topk, w.dtype)
    dev = _device(w, host)
    hs = torch.empty_like(out["h_sparse"])
    lse = torch.empty_like(out["lse_sel"])
    api.ssa_fwd_sparse(dims, dev["Q"], dev["K"], dev["V"], out["idx"], hs, lse)
    torch.cuda.synchronize()
    assert api.ssa_device_status() == api.SSA_OK
    for (b, h, i) in _samples(w, rng):
        N1 = (i + 1) * w.block
        f = O.forward_sparse(host["Q"][b:b + 1, h:h + 1, :N1], host["K"][b:b + 1, :, :N1],
                             host["V"][b:b + 1, :, :N1], ora_idx[b:b + 1, h:h + 1, :i + 1], w.block, scale,
                             qblocks=[i])
        rows = slice(i * w.block, N1)
        assert np.abs(f64(hs[b, h, rows]) - f["h_sparse"][0, 0, rows]).max() <= TOL["bf16"]["out"], (b, h, i)
