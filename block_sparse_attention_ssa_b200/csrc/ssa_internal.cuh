// Internal declarations shared by the libssa translation units.
// Nothing here is part of the C ABI (see include/ssa.h).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssa.h"

namespace ssa {

// Validated problem shape.
struct Dims {
  int B, Hq, Hkv, N, d, s, topk, k, n, g;  // k = min(topk, n), g = Hq / Hkv
  float scale;
  int dtype;
  int per_token;  // selection per query token (1) or per query block (0)
  int rows_sel;   // rows of the selection per head: N (per token) or n
};

// A [B, H, N, d] tensor with a contiguous d dimension; strides in elements.
struct TensorRef {
  const void* p;
  int64_t sb, sh, sn;
};

template <typename T>
__device__ __forceinline__ const T* row_ptr(const TensorRef& t, int b, int h, int64_t r) {
  return static_cast<const T*>(t.p) + b * t.sb + h * t.sh + r * t.sn;
}
template <typename T>
__device__ __forceinline__ T* row_ptr_w(const TensorRef& t, int b, int h, int64_t r) {
  return const_cast<T*>(static_cast<const T*>(t.p)) + b * t.sb + h * t.sh + r * t.sn;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Loads 16 bytes of T (4 floats or 8 bf16) starting at a 16-byte aligned
// address and widens them to float.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
  static constexpr int kN = 4;
  __device__ __forceinline__ static void load(const float* p, float* out) {
    float4 v = *reinterpret_cast<const float4*>(p);
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
  }
};
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int kN = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float* out) {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      out[2 * i] = f.x;
      out[2 * i + 1] = f.y;
    }
  }
};

constexpr float kNegInf = -__builtin_huge_valf();

// 64-key tiles at key u0 (CUDA-core kernels): bit c is set when key u0 + c
// lies in a block whose bit is set in `blocks` (the selected-block set of a
// row's query block); s is the block size.  Blocks of 64 or more keys cover
// the whole tile; smaller blocks give one run of s bits per block.
__device__ __forceinline__ unsigned long long tile_keep_mask(const uint32_t* blocks, int u0, int s) {
  if (s >= 64) {
    const int j = u0 / s;
    return ((blocks[j >> 5] >> (j & 31)) & 1u) ? ~0ull : 0ull;
  }
  unsigned long long m = 0ull;
  const unsigned long long run = (1ull << s) - 1ull;
  for (int c0 = 0; c0 < 64; c0 += s) {
    const int j = (u0 + c0) / s;
    if ((blocks[j >> 5] >> (j & 31)) & 1u) m |= run << c0;
  }
  return m;
}

// The same mask for s = 1 << ls, s >= 16 (the supported block sizes are
// powers of two): the tile's 64 / s blocks sit in one aligned 32-bit word.
__device__ __forceinline__ unsigned long long tile_keep_mask_p2(const uint32_t* blocks, int u0, int ls) {
  const int jb = u0 >> ls;
  const uint32_t word = blocks[jb >> 5] >> (jb & 31);
  if (ls >= 6) return (word & 1u) ? ~0ull : 0ull;
  const int nb = 64 >> ls;
  const unsigned long long run = (1ull << (1 << ls)) - 1ull;
  unsigned long long m = 0ull;
  for (int b = 0; b < nb; ++b)
    if ((word >> b) & 1u) m |= run << (b << ls);
  return m;
}

// Bit c is set when key u0 + c <= t (a causal pair of query t).
__device__ __forceinline__ unsigned long long causal_mask(int t, int u0) {
  const int lim = t - u0;
  return lim >= 63 ? ~0ull : (lim < 0 ? 0ull : ((2ull << lim) - 1ull));
}

// Host-side count of kernels enqueued by this library (ssa_launch_count).
void count_launches(int n);

// ---------------------------------------------------------------- launchers
// Each returns the launch status; none synchronises.

// Mean of each block of s rows: X [B,H,N,d] -> out [B,H,n,d] fp32 (dense).
cudaError_t launch_pool(const Dims& D, const TensorRef& X, int H, float* out, cudaStream_t st);

// scores[b,h,i,j] = scale * qbar[b,h,i] . kbar[b,h/g,j] for j < i, else -inf.
cudaError_t launch_scores(const Dims& D, const float* qbar, const float* kbar, float* scores,
                          cudaStream_t st);

// Top-k block selection with the forced diagonal.
cudaError_t launch_select(const Dims& D, const float* scores, int32_t* idx, cudaStream_t st);

// Bit mask [B, Hq, rows_sel, words] of each selection row built from idx
// (entries outside [0, i] ignored, i the row's query block).
cudaError_t launch_build_mask(const Dims& D, const int32_t* idx, uint32_t* mask, int words,
                              cudaStream_t st);

// Per-token selection: kbar [B,Hkv,n,d] fp32 (pooled keys) -> idx [B,Hq,N,k].
cudaError_t launch_select_tokens(const Dims& D, const TensorRef& Q, const float* kbar, int32_t* idx,
                                 cudaStream_t st);

struct FwdArgs {
  TensorRef q, k, v, hf, hs;
  const int32_t* idx;
  float* lse_full;
  float* lse_sel;
  float* delta;
  const float* lse_in;  // dropped-mass mode only: given lse_full, or nullptr
  bool sparse_only;     // sparse stream alone: only selected blocks are read;
                        // hf, lse_full and delta are not written (may be null)
};

// CUDA-core dual-stream forward (fp32 math; any supported dtype / d).
cudaError_t launch_fwd_simt(const Dims& D, const FwdArgs& a, cudaStream_t st);
// CUDA-core dropped mass (no V).
cudaError_t launch_dropped_simt(const Dims& D, const FwdArgs& a, cudaStream_t st);
// Tensor-core dropped mass (bf16, d = 128; same envelope as the forward).
cudaError_t launch_dropped_tc(const Dims& D, const FwdArgs& a, int32_t* dev_status, cudaStream_t st);

// Warp-level tensor-core (mma.sync) dual-stream forward and dropped mass:
// bf16, d = 64 or 128, any block size and either selection mode.
bool fwd_mma_supported(const Dims& D);
cudaError_t launch_fwd_mma(const Dims& D, const FwdArgs& a, cudaStream_t st);
// Sparse stream alone, blocks of 16 or 32, per-block selection (bf16, mma.sync):
// each query block walks its own selected key blocks.
bool fwd_walk_supported(const Dims& D);
cudaError_t launch_fwd_walk(const Dims& D, const FwdArgs& a, int32_t* dev_status, cudaStream_t st);
cudaError_t launch_dropped_mma(const Dims& D, const FwdArgs& a, cudaStream_t st);

// Envelope of the first tensor-core kernels: bf16, d = 128, blocks of 64 or
// 128, per-block selection (n <= 2048).
bool fwd_tc_supported(const Dims& D);
// Tensor-core (tcgen05 / TMEM / TMA) dual-stream forward and sparse stream
// alone in that envelope, selected blocks first: one softmax and one
// accumulator per query tile, h_sparse read off after the selected blocks, two
// CTAs per SM.  Returns cudaErrorNotSupported outside the envelope.
cudaError_t launch_fwd_ord(const Dims& D, const FwdArgs& a, int32_t* dev_status, cudaStream_t st);

// 4-D TMA map over a [B, H, N, d] bf16 tensor (d = 64 or 128): dims
// (d, N, H, B), box (64 columns, `rows` rows), 128-byte swizzle, zero fill
// out of bounds.
bool make_tma_map_bf16(CUtensorMap* map, const TensorRef& t, int B, int H, int N, int rows, int d = 128);

// Tensor-core dual-stream forward with per-row selection masks (bf16, d = 64
// or 128, any block size, per-block or per-token selection; dual mode only).
bool fwd_tcm_supported(const Dims& D);
cudaError_t launch_fwd_tcm(const Dims& D, const FwdArgs& a, int32_t* dev_status, cudaStream_t st);
// Its dropped-mass mode (QK^T only; delta from a.lse_in when given).
cudaError_t launch_dropped_tcm(const Dims& D, const FwdArgs& a, int32_t* dev_status, cudaStream_t st);

struct BwdArgs {
  TensorRef q, k, v, hf, hs, gf, gs, dq, dk, dv;  // gf / gs .p may be null
  const int32_t* idx;
  const float* lse_full;
  const float* lse_sel;
  float alpha;
  float* align_loss;  // may be null
  // workspace pieces
  float* dhf;          // [B,Hq,N,d] fp32: dL/dh_full
  float* doc;          // [B,Hq,N,d] fp32: dh_full + r * dh_sparse
  float* Df;           // [B,Hq,N]
  float* Dc;           // [B,Hq,N]
  uint32_t* mask;      // [B,Hq,n,words]
  int words;
  float* partials;     // per-block partial sums of (h_full - h_sparse)^2
  int n_partials;
  // Sparse stream alone: the caller passes hf = hs, lse_full = lse_sel,
  // gf = null and alpha = 0, so dh_f = 0 and r = 1; the kernels then skip
  // every (query block, key block) pair that is not selected.
  bool sparse_only;
  float* kvpart;       // warp-level tensor-core backward: fp32 dK / dV partials (or null)
  uint32_t* maskT;     // sparse stream alone at blocks of 16 / 32: [B,Hq,n,words], bit i of row j set
                       // when query block i selected key block j (or null)
};

cudaError_t launch_bwd_pre(const Dims& D, const BwdArgs& a, cudaStream_t st);
// Tensor-core backward (bf16, d = 128): preprocess + dK/dV + dQ launches.
bool bwd_tc_supported(const Dims& D);
cudaError_t launch_bwd_tc(const Dims& D, const BwdArgs& a, int32_t* dev_status, cudaStream_t st);
cudaError_t launch_bwd_simt(const Dims& D, const BwdArgs& a, cudaStream_t st);
// Warp-level tensor-core (mma.sync) backward: bf16, d = 64 or 128, any block
// size and either selection mode (runs its own preprocess).
bool bwd_mma_supported(const Dims& D);
int bwd_mma_heads_per_cta(const Dims& D);
size_t bwd_mma_partial_bytes(const Dims& D);  // workspace for a.kvpart (0: none needed)
cudaError_t launch_bwd_mma(const Dims& D, const BwdArgs& a, int32_t* status, cudaStream_t st);
// Ordered sum of fp32 dK / dV partials (chunks of a kv group) into a.dk, a.dv.
cudaError_t launch_kvsum(const Dims& D, const BwdArgs& a, const float* part, int chunks, cudaStream_t st);
// Sparse stream alone at blocks of 16 or 32, backward: dQ walk (also writes D_t to a.Dc), dK / dV per (query head,
// key slice) into fp32 partials in the a.dhf / a.doc regions, then kvsum.
bool bwd_walk_supported(const Dims& D);
cudaError_t launch_bwd_walk(const Dims& D, const BwdArgs& a, int32_t* dev_status, cudaStream_t st);
// Tensor-core (tcgen05) dual backward with per-row selection masks, bf16,
// d = 64; takes the bf16 dh_f / dO_c written by the warp-level preprocess.
bool bwd_tcm_supported(const Dims& D);
cudaError_t launch_bwd_tcm(const Dims& D, const BwdArgs& a, const void* dhf_bf16, const void* doc_bf16, int hpc,
                           int32_t* status, cudaStream_t st);

struct DecodeArgs {
  TensorRef q, k, v, h;  // q, h: [B,Hq,1,d] (prefill: q = the prompt's Q [B,Hq,N,d]); k, v: caches [B,Hkv,N,d]
  float* lse;            // [B,Hq]
  int32_t* idx;          // [B,Hq,k_eff]
  float* qsum;           // [B,Hq,d] running sum of the current block's queries
  float* kbar;           // [B,Hkv,n,d] means of the complete key blocks
  int t;                 // position of the new token (prefill: prompt length)
  void* ws;              // decode step: caller workspace (unused: scratch lives in shared memory)
};

// Sparse-stream decode of the token at position a.t (one cluster launch; the
// bf16 attention products on mma.sync).
cudaError_t launch_decode(const Dims& D, const DecodeArgs& a, int32_t* dev_status, cudaStream_t st);
// Decode state from a prompt of a.t tokens: kbar of its complete blocks, qsum of the partial block.
cudaError_t launch_decode_prefill(const Dims& D, const DecodeArgs& a, cudaStream_t st);
// Dynamic shared memory the decode kernels need for these dims.
size_t decode_smem_bytes(const Dims& D);
// The decode step's envelope: k_eff <= 64 and its shared memory fits a CTA.
bool decode_supported(const Dims& D);
// Workspace bytes of one decode step.
size_t decode_ws_bytes(const Dims& D);

// One-CTA kernel whose bounded barrier wait runs out: records SSA_ERR_TIMEOUT.
cudaError_t launch_selftest_timeout(int32_t* status, long long limit_cycles, cudaStream_t st);

// Sum of squared differences of two [B,Hq,N,d] tensors into per-block
// partials, then a fixed-order final reduction: out[0..n_out) = sum / count.
cudaError_t launch_sqdiff_partials(const Dims& D, const TensorRef& a, const TensorRef& b,
                                   float* partials, int n_partials, cudaStream_t st);
cudaError_t launch_finish_mean(const float* partials, int n_partials, double count, float mult,
                               float* out, int n_out, cudaStream_t st);
int sqdiff_partial_count(const Dims& D);

}  // namespace ssa
