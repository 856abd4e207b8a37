"""Thin Python binding of libssa (include/ssa.h).

Argument marshalling only: every function here has the name of the C entry
point it calls, turns torch tensors into raw device pointers and strides,
calls the C function on the current (or given) CUDA stream and raises
SsaError when it returns a non-OK status.  No arithmetic of the method runs
in Python; torch provides device memory and streams.

The library is loaded from this package directory.  If it is missing the
import of this module still succeeds (so host-only tools work), but the
first call raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import math
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libssa.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "ssa.h")

SSA_OK, SSA_ERR_INVALID_ARG, SSA_ERR_UNSUPPORTED, SSA_ERR_CUDA, SSA_ERR_TIMEOUT, SSA_ERR_WORKSPACE = range(6)
SSA_F32, SSA_BF16 = 0, 1
_DTYPES = {"f32": SSA_F32, "bf16": SSA_BF16}
_TORCH_DTYPES = {SSA_F32: torch.float32, SSA_BF16: torch.bfloat16}


class SsaError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: {msg} ({code})")
        self.code = code


class ssa_dims_t(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("N", ctypes.c_int32), ("d", ctypes.c_int32), ("block", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("scale", ctypes.c_float), ("dtype", ctypes.c_int32),
                ("per_token", ctypes.c_int32)]

    @property
    def n_blocks(self) -> int:
        return self.N // self.block

    @property
    def k_eff(self) -> int:
        return min(self.topk, self.N // self.block)

    @property
    def torch_dtype(self) -> torch.dtype:
        return _TORCH_DTYPES[self.dtype]

    @property
    def sel_rows(self) -> int:
        """Rows of a selection per head: N (per-token selection) or n."""
        return self.N if self.per_token else self.N // self.block


class ssa_tensor_t(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("stride_b", ctypes.c_int64),
                ("stride_h", ctypes.c_int64), ("stride_n", ctypes.c_int64)]


_P = ctypes.POINTER
_SIGS = {
    "ssa_version": (ctypes.c_int, []),
    "ssa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "ssa_workspace_bytes": (ctypes.c_size_t, [_P(ssa_dims_t)]),
    "ssa_block_scores": (ctypes.c_int, [_P(ssa_dims_t), _P(ssa_tensor_t), _P(ssa_tensor_t),
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "ssa_select_topk": (ctypes.c_int, [_P(ssa_dims_t), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "ssa_select_tokens": (ctypes.c_int, [_P(ssa_dims_t), _P(ssa_tensor_t), _P(ssa_tensor_t), ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "ssa_fwd_dual": (ctypes.c_int, [_P(ssa_dims_t), _P(ssa_tensor_t), _P(ssa_tensor_t), _P(ssa_tensor_t),
                                     ctypes.c_void_p, _P(ssa_tensor_t), _P(ssa_tensor_t), ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "ssa_bwd_dual": (ctypes.c_int, [_P(ssa_dims_t), _P(ssa_tensor_t), _P(ssa_tensor_t), _P(ssa_tensor_t),
                                     ctypes.c_void_p, _P(ssa_tensor_t), _P(ssa_tensor_t), ctypes.c_void_p,
                                     ctypes.c_void_p, _P(ssa_tensor_t), _P(ssa_tensor_t), ctypes.c_float,
                                     ctypes.c_void_p, _P(ssa_tensor_t), _P(ssa_tensor_t), _P(ssa_tensor_t),
                                     ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "ssa_fwd_sparse": (ctypes.c_int, [_P(ssa_dims_t), _P(ssa_tensor_t), _P(ssa_tensor_t), _P(ssa_tensor_t),
                                       ctypes.c_void_p, _P(ssa_tensor_t), ctypes.c_void_p, ctypes.c_void_p]),
    "ssa_bwd_sparse": (ctypes.c_int, [_P(ssa_dims_t), _P(ssa_tensor_t), _P(ssa_tensor_t), _P(ssa_tensor_t),
                                       ctypes.c_void_p, _P(ssa_tensor_t), ctypes.c_void_p, _P(ssa_tensor_t),
                                       _P(ssa_tensor_t), _P(ssa_tensor_t), _P(ssa_tensor_t), ctypes.c_void_p,
                                       ctypes.c_size_t, ctypes.c_void_p]),
    "ssa_decode_prefill": (ctypes.c_int, [_P(ssa_dims_t), _P(ssa_tensor_t), _P(ssa_tensor_t), ctypes.c_int32,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "ssa_decode_step": (ctypes.c_int, [_P(ssa_dims_t), _P(ssa_tensor_t), _P(ssa_tensor_t), _P(ssa_tensor_t),
                                        ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, _P(ssa_tensor_t),
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                        ctypes.c_void_p]),
    "ssa_dropped_mass": (ctypes.c_int, [_P(ssa_dims_t), _P(ssa_tensor_t), _P(ssa_tensor_t), ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                         ctypes.c_void_p]),
    "ssa_align_mse": (ctypes.c_int, [_P(ssa_dims_t), _P(ssa_tensor_t), _P(ssa_tensor_t), ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "ssa_device_status": (ctypes.c_int, [_P(ctypes.c_int32), ctypes.c_int, ctypes.c_void_p]),
    "ssa_launch_count": (ctypes.c_uint64, []),
    "ssa_selftest_timeout": (ctypes.c_int, [ctypes.c_void_p]),
    "ssa_block_scores_noalloc": (ctypes.c_int, [_P(ssa_dims_t), _P(ssa_tensor_t), _P(ssa_tensor_t),
                                                 ctypes.c_void_p, ctypes.c_void_p]),
}

_lib = None


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libssa.so (built by `python -m block_sparse_attention_ssa_b200.build`)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"libssa.so not found at {p}; build it with "
                          "`python -m block_sparse_attention_ssa_b200.build`")
    lib = ctypes.CDLL(p)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def header_symbols(path: str = HEADER_PATH) -> list[str]:
    """Names of the entry points declared in include/ssa.h."""
    with open(path) as fh:
        text = fh.read()
    return re.findall(r"SSA_API\s+[\w\s\*]+?\b(ssa_\w+)\s*\(", text)


def status_string(code: int) -> str:
    return load_library().ssa_status_string(code).decode()


def _check(fn: str, code: int) -> None:
    if code != SSA_OK:
        raise SsaError(fn, code, status_string(code))


def make_dims(B: int, Hq: int, Hkv: int, N: int, d: int, block: int, topk: int,
              dtype: str = "bf16", scale: float | None = None, per_token: bool = False) -> ssa_dims_t:
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    return ssa_dims_t(B, Hq, Hkv, N, d, block, topk, float(scale), _DTYPES[dtype], int(per_token))


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _t(x: torch.Tensor | None) -> ctypes._Pointer | None:
    """ssa_tensor_t for a [B, H, N, d] tensor with unit d stride (None -> NULL)."""
    if x is None:
        return None
    if x.dim() != 4 or x.stride(3) != 1:
        raise ValueError("expected a [B, H, N, d] tensor with a contiguous last dimension")
    return ctypes.pointer(ssa_tensor_t(x.data_ptr(), x.stride(0), x.stride(1), x.stride(2)))


def _p(x: torch.Tensor | None) -> ctypes.c_void_p | None:
    return None if x is None else ctypes.c_void_p(x.data_ptr())


def ssa_workspace_bytes(dims: ssa_dims_t) -> int:
    return int(load_library().ssa_workspace_bytes(ctypes.byref(dims)))


def ssa_block_scores(dims, Q, K, scores, ws, stream=None) -> None:
    _check("ssa_block_scores", load_library().ssa_block_scores(
        ctypes.byref(dims), _t(Q), _t(K), _p(scores), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def ssa_block_scores_noalloc(dims, Q, K, scores, stream=None) -> None:
    """ssa_block_scores with the library's fixed device scratch instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    _check("ssa_block_scores_noalloc", load_library().ssa_block_scores_noalloc(
        ctypes.byref(dims), _t(Q), _t(K), _p(scores), _stream(stream)))


def ssa_select_topk(dims, scores, idx, stream=None) -> None:
    _check("ssa_select_topk", load_library().ssa_select_topk(
        ctypes.byref(dims), _p(scores), _p(idx), _stream(stream)))


def ssa_select_tokens(dims, Q, K, idx, ws, stream=None) -> None:
    _check("ssa_select_tokens", load_library().ssa_select_tokens(
        ctypes.byref(dims), _t(Q), _t(K), _p(idx), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def ssa_fwd_dual(dims, Q, K, V, idx, h_full, h_sparse, lse_full, lse_sel, delta, stream=None) -> None:
    _check("ssa_fwd_dual", load_library().ssa_fwd_dual(
        ctypes.byref(dims), _t(Q), _t(K), _t(V), _p(idx), _t(h_full), _t(h_sparse),
        _p(lse_full), _p(lse_sel), _p(delta), _stream(stream)))


def ssa_bwd_dual(dims, Q, K, V, idx, h_full, h_sparse, lse_full, lse_sel, g_full, g_sparse,
                 alpha, align_loss, dQ, dK, dV, ws, stream=None) -> None:
    _check("ssa_bwd_dual", load_library().ssa_bwd_dual(
        ctypes.byref(dims), _t(Q), _t(K), _t(V), _p(idx), _t(h_full), _t(h_sparse), _p(lse_full),
        _p(lse_sel), _t(g_full), _t(g_sparse), float(alpha), _p(align_loss), _t(dQ), _t(dK), _t(dV),
        _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def ssa_fwd_sparse(dims, Q, K, V, idx, h_sparse, lse_sel, stream=None) -> None:
    _check("ssa_fwd_sparse", load_library().ssa_fwd_sparse(
        ctypes.byref(dims), _t(Q), _t(K), _t(V), _p(idx), _t(h_sparse), _p(lse_sel), _stream(stream)))


def ssa_bwd_sparse(dims, Q, K, V, idx, h_sparse, lse_sel, g_sparse, dQ, dK, dV, ws, stream=None) -> None:
    _check("ssa_bwd_sparse", load_library().ssa_bwd_sparse(
        ctypes.byref(dims), _t(Q), _t(K), _t(V), _p(idx), _t(h_sparse), _p(lse_sel), _t(g_sparse),
        _t(dQ), _t(dK), _t(dV), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def ssa_decode_prefill(dims, Q, K, t0, qsum, kbar, stream=None) -> None:
    _check("ssa_decode_prefill", load_library().ssa_decode_prefill(
        ctypes.byref(dims), _t(Q), _t(K), int(t0), _p(qsum), _p(kbar), _stream(stream)))


def ssa_decode_step(dims, q, K, V, t, qsum, kbar, h, lse, idx, ws, stream=None) -> None:
    _check("ssa_decode_step", load_library().ssa_decode_step(
        ctypes.byref(dims), _t(q), _t(K), _t(V), int(t), _p(qsum), _p(kbar), _t(h), _p(lse), _p(idx),
        _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def ssa_dropped_mass(dims, Q, K, idx, lse_full, delta, ws, stream=None) -> None:
    _check("ssa_dropped_mass", load_library().ssa_dropped_mass(
        ctypes.byref(dims), _t(Q), _t(K), _p(idx), _p(lse_full), _p(delta), _p(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def ssa_align_mse(dims, h_full, h_sparse, loss, ws, stream=None) -> None:
    _check("ssa_align_mse", load_library().ssa_align_mse(
        ctypes.byref(dims), _t(h_full), _t(h_sparse), _p(loss), _p(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def ssa_launch_count() -> int:
    return int(load_library().ssa_launch_count())


def ssa_selftest_timeout(stream=None) -> None:
    _check("ssa_selftest_timeout", load_library().ssa_selftest_timeout(_stream(stream)))


def ssa_device_status(clear: bool = True, stream=None) -> int:
    out = ctypes.c_int32(0)
    _check("ssa_device_status", load_library().ssa_device_status(ctypes.byref(out), int(clear), _stream(stream)))
    return int(out.value)


# ---------------------------------------------------------------- buffers
# Allocation helpers (torch device memory) for callers that do not manage
# their own buffers.  They allocate; the C library never does.

def alloc_workspace(dims: ssa_dims_t, device="cuda") -> torch.Tensor:
    nbytes = max(ssa_workspace_bytes(dims), 256)
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def alloc_forward(dims: ssa_dims_t, device="cuda") -> dict[str, torch.Tensor]:
    B, Hq, N, d, n, k = dims.B, dims.Hq, dims.N, dims.d, dims.n_blocks, dims.k_eff
    dt = dims.torch_dtype
    return {
        "scores": torch.empty((B, Hq, n, n), dtype=torch.float32, device=device),
        "idx": torch.empty((B, Hq, dims.sel_rows, k), dtype=torch.int32, device=device),
        "h_full": torch.empty((B, Hq, N, d), dtype=dt, device=device),
        "h_sparse": torch.empty((B, Hq, N, d), dtype=dt, device=device),
        "lse_full": torch.empty((B, Hq, N), dtype=torch.float32, device=device),
        "lse_sel": torch.empty((B, Hq, N), dtype=torch.float32, device=device),
        "delta": torch.empty((B, Hq, N), dtype=torch.float32, device=device),
    }


def alloc_backward(dims: ssa_dims_t, device="cuda") -> dict[str, torch.Tensor]:
    dt = dims.torch_dtype
    return {
        "dQ": torch.empty((dims.B, dims.Hq, dims.N, dims.d), dtype=dt, device=device),
        "dK": torch.empty((dims.B, dims.Hkv, dims.N, dims.d), dtype=dt, device=device),
        "dV": torch.empty((dims.B, dims.Hkv, dims.N, dims.d), dtype=dt, device=device),
        "align_loss": torch.empty((1,), dtype=torch.float32, device=device),
    }


def alloc_decode(dims: ssa_dims_t, device="cuda") -> dict[str, torch.Tensor]:
    """Decode state (qsum, kbar) and per-step outputs (h, lse, idx)."""
    B, Hq, Hkv, d, n, k = dims.B, dims.Hq, dims.Hkv, dims.d, dims.n_blocks, dims.k_eff
    return {
        "qsum": torch.zeros((B, Hq, d), dtype=torch.float32, device=device),
        "kbar": torch.zeros((B, Hkv, n, d), dtype=torch.float32, device=device),
        "h": torch.empty((B, Hq, 1, d), dtype=dims.torch_dtype, device=device),
        "lse": torch.empty((B, Hq), dtype=torch.float32, device=device),
        "idx": torch.empty((B, Hq, k), dtype=torch.int32, device=device),
    }


def forward(dims, Q, K, V, out, ws, stream=None) -> dict[str, torch.Tensor]:
    """The forward steps in order: selection (block scores + top-k, or the
    per-token selection), then the fused dual forward."""
    if dims.per_token:
        ssa_select_tokens(dims, Q, K, out["idx"], ws, stream)
    else:
        ssa_block_scores(dims, Q, K, out["scores"], ws, stream)
        ssa_select_topk(dims, out["scores"], out["idx"], stream)
    ssa_fwd_dual(dims, Q, K, V, out["idx"], out["h_full"], out["h_sparse"], out["lse_full"],
                 out["lse_sel"], out["delta"], stream)
    return out


def backward(dims, Q, K, V, fwd, g_full, g_sparse, alpha, grads, ws, stream=None):
    ssa_bwd_dual(dims, Q, K, V, fwd["idx"], fwd["h_full"], fwd["h_sparse"], fwd["lse_full"],
                 fwd["lse_sel"], g_full, g_sparse, alpha, grads["align_loss"], grads["dQ"], grads["dK"],
                 grads["dV"], ws, stream)
    return grads
