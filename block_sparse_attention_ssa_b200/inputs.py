"""Seeded synthetic inputs for the SSA hot path.

This module only draws random tensors. It holds none of the method's
arithmetic, so both the CUDA path and the fp64 oracle may take their inputs
from it.

Distribution (the "planted direction" workload):
  * Q, K, V are i.i.d. N(0, 1), drawn in fp32 with numpy PCG64.
  * One direction u per (batch, kv head): u = g / |g| * d**0.25, g ~ N(0, I_d).
    With the attention scale 1/sqrt(d) a key shifted by s*u raises the logit
    of a query shifted by u by s*|u|^2/sqrt(d) = s.
  * Every query of the kv head's query group gets +u.
  * Every key in key block b gets +s_b * u, s_b ~ Exp(mean 1) per
    (batch, kv head, block).  The long-context workload instead plants
    s_b = 4 on round(5 %) of the blocks (drawn without replacement) and
    s_b ~ Exp(mean 0.5) on the others.
  * V carries no plant.
bf16 workloads round the fp32 draws to bf16 with round-to-nearest-even; the
rounded values are what both sides see.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and budget of one synthetic SSA workload."""

    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    block: int
    topk: int
    dtype: str  # "f32" or "bf16"
    seed: int
    plant: str = "exp1"  # "exp1" | "sparse5"
    backward: bool = True

    @property
    def n_blocks(self) -> int:
        return self.N // self.block

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_topk(self, k: int) -> "Workload":
        return dataclasses.replace(self, topk=k, name=f"{self.name.split('@')[0]}@k{k}")

    def causal_pairs(self) -> int:
        """Number of (query, key) pairs with key <= query, over all heads."""
        return self.B * self.Hq * self.N * (self.N + 1) // 2


# The benchmark workloads (the five synthetic suites and the pages' own model
# shape).  Seeds are 1000 + the workload's
# ordinal; the budget sweep reuses one tensor set for every budget.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 1, 1, 1024, 64, 64, 4, "f32", 1001, backward=False),
    "mha_8k": Workload("mha_8k", 1, 16, 16, 8192, 128, 64, 16, "bf16", 1002, backward=False),
    "gqa_16k": Workload("gqa_16k", 2, 32, 8, 16384, 128, 64, 16, "bf16", 1003),
    "long_64k": Workload("long_64k", 1, 32, 8, 65536, 128, 128, 16, "bf16", 1004, plant="sparse5"),
    "sweep_32k": Workload("sweep_32k", 1, 32, 8, 32768, 128, 64, 16, "bf16", 1005),
    # The attention layer of the pages' 1B model (32 query heads, 2 kv heads,
    # hidden 2048 -> d = 64) with their 16 x 16 receptive field at the 8K
    # training context.
    "paper_b16_8k": Workload("paper_b16_8k", 1, 32, 2, 8192, 64, 16, 16, "bf16", 1006),
    # The same selection (block 16, 16 blocks) at head dimension 128, the
    # head size of the five suites above.
    "paper_b16_8k_d128": Workload("paper_b16_8k_d128", 1, 32, 2, 8192, 128, 16, 16, "bf16", 1008),
}
SWEEP_TOPK = (4, 8, 16, 32, 64)


def round_to_bf16(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Round fp32 values to bf16 (nearest, ties to even).

    Returns (values as fp32 holding the bf16-exact numbers, raw bf16 bits as
    uint16).  Inputs are finite draws, so NaN handling is not needed.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16).astype(np.uint16)
    back = (rounded.astype(np.uint32) << 16).view(np.float32)
    return back, rounded


def make_qkv(B: int, Hq: int, Hkv: int, N: int, d: int, block: int, seed: int,
             plant: str = "exp1") -> dict[str, np.ndarray]:
    """Draw fp32 Q [B,Hq,N,d], K/V [B,Hkv,N,d] with the planted direction."""
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    if N % block:
        raise ValueError("N must be a multiple of the block size")
    rng = np.random.Generator(np.random.PCG64(seed))
    g = Hq // Hkv
    n = N // block
    Q = rng.standard_normal((B, Hq, N, d), dtype=np.float32)
    K = rng.standard_normal((B, Hkv, N, d), dtype=np.float32)
    V = rng.standard_normal((B, Hkv, N, d), dtype=np.float32)
    u = rng.standard_normal((B, Hkv, d)).astype(np.float64)
    u = u / np.linalg.norm(u, axis=-1, keepdims=True) * d ** 0.25
    if plant == "exp1":
        s_b = rng.exponential(1.0, size=(B, Hkv, n))
    elif plant == "sparse5":
        s_b = rng.exponential(0.5, size=(B, Hkv, n))
        n_hot = int(round(0.05 * n))
        for b in range(B):
            for h in range(Hkv):
                hot = rng.choice(n, size=n_hot, replace=False)
                s_b[b, h, hot] = 4.0
    elif plant == "none":
        s_b = np.zeros((B, Hkv, n))
        u[:] = 0.0
    else:
        raise ValueError(f"unknown plant {plant!r}")
    u32 = u.astype(np.float32)
    Q += np.repeat(u32, g, axis=1)[:, :, None, :]
    shift = (s_b[..., None] * u[:, :, None, :]).astype(np.float32)  # [B,Hkv,n,d]
    K += np.repeat(shift, block, axis=2)
    return {"Q": Q, "K": K, "V": V, "s_b": s_b, "u": u}


def make_workload_inputs(w: Workload) -> dict[str, np.ndarray]:
    """Inputs of one workload.  For bf16 workloads the returned fp32 arrays hold
    the bf16-rounded values and '<name>_bits' holds the raw uint16 bits."""
    t = make_qkv(w.B, w.Hq, w.Hkv, w.N, w.d, w.block, w.seed, w.plant)
    out = {"s_b": t["s_b"], "u": t["u"]}
    for name in ("Q", "K", "V"):
        if w.dtype == "bf16":
            vals, bits = round_to_bf16(t[name])
            out[name] = vals
            out[name + "_bits"] = bits
        else:
            out[name] = t[name]
    return out


def make_upstream(shape: tuple[int, ...], seed: int) -> np.ndarray:
    """A seeded random upstream gradient (fp32) for backward tests."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.standard_normal(shape, dtype=np.float32)


def make_scores(B: int, H: int, n: int, seed: int, tie_frac: float = 0.0) -> np.ndarray:
    """Random fp32 block scores [B,H,n,n] with an optional share of exact ties.

    Entries on and above the diagonal are set to -inf (they are never
    candidates).  With tie_frac > 0 that share of each row's candidates is
    overwritten with copies of other candidates of the same row, so the
    lower-index tie rule is exercised.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    S = rng.standard_normal((B, H, n, n), dtype=np.float32)
    if tie_frac > 0:
        for b in range(B):
            for h in range(H):
                for i in range(2, n):
                    m = int(tie_frac * i)
                    if m == 0:
                        continue
                    dst = rng.choice(i, size=m, replace=False)
                    src = rng.integers(0, i, size=m)
                    S[b, h, i, dst] = S[b, h, i, src]
    S[:, :, np.triu_indices(n)[0], np.triu_indices(n)[1]] = -np.inf
    return S
