"""SSA (Sparse Sparse Attention) hot path for B200 (sm_100a).

Block scoring, top-k block selection, the fused dual-stream forward
(h_sparse, h_full, dropped mass delta) and the backward with the alignment
loss, as hand-written CUDA kernels behind the C ABI in include/ssa.h.
`api` is the thin Python binding; `inputs` draws the seeded synthetic
workloads.
"""
from . import api, inputs  # noqa: F401
from .api import (  # noqa: F401
    SsaError,
    alloc_backward,
    alloc_forward,
    alloc_workspace,
    backward,
    forward,
    load_library,
    make_dims,
    ssa_align_mse,
    ssa_block_scores,
    ssa_bwd_dual,
    ssa_device_status,
    ssa_dropped_mass,
    ssa_fwd_dual,
    ssa_select_topk,
    ssa_workspace_bytes,
)
