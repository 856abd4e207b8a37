// Block pooling, block scoring and top-k block selection.
//
// "SSA: Achieving Sparser Attention by Aligning Full and Sparse Attention
// Outputs in Feature Space", section "Practical Implementation of SSA": the
// sequence is cut into blocks, each block is represented by the mean of its
// keys, the query is scored against every earlier block representation and
// the top-k blocks are kept.  Selection is per query block (the query side is
// the mean of the block's queries) and per query head; the diagonal block is
// always kept and counts toward k.
//
// The kernels are HBM-, latency- or (per-token scoring) FMA-bound and run on
// CUDA cores.
#include <climits>

#include "ssa_internal.cuh"

namespace ssa {
namespace {

// ------------------------------------------------------------------ pooling
// grid (n, H, B), 128 threads.  Each thread owns 16 bytes of a row; RPI rows
// are summed in parallel and folded through shared memory.  Reads are 16-byte
// vectors, a warp covers 2 (bf16, d=128) to 8 rows of 256 / 512 bytes.
template <typename T, int D>
__global__ void __launch_bounds__(128) pool_kernel(TensorRef X, int H, int s, int n, float* out) {
  constexpr int VEC = Vec16<T>::kN;
  constexpr int TPR = D / VEC;     // threads per row
  constexpr int RPI = 128 / TPR;   // rows per iteration
  __shared__ float part[RPI][D];
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int r = threadIdx.x / TPR, c0 = (threadIdx.x % TPR) * VEC;
  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
  for (int rr = r; rr < s; rr += RPI) {
    float v[VEC];
    Vec16<T>::load(row_ptr<T>(X, b, h, (int64_t)blk * s + rr) + c0, v);
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] += v[e];
  }
#pragma unroll
  for (int e = 0; e < VEC; ++e) part[r][c0 + e] = acc[e];
  __syncthreads();
  const float inv = 1.0f / (float)s;
  for (int c = threadIdx.x; c < D; c += 128) {
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < RPI; ++q) sum += part[q][c];
    out[(((int64_t)b * H + h) * n + blk) * D + c] = sum * inv;
  }
}

// ------------------------------------------------------------------ scores
// grid (ceil(n/32) j-tiles, ceil(n/32) i-tiles, B*Hq), 256 threads.
template <int D>
__global__ void __launch_bounds__(256) score_kernel(const float* __restrict__ qbar,
                                                    const float* __restrict__ kbar,
                                                    float* __restrict__ scores, int Hq, int g,
                                                    int n, float scale) {
  __shared__ float qs[32][D + 1];
  __shared__ float ks[32][D + 1];
  const int j0 = blockIdx.x * 32, i0 = blockIdx.y * 32;
  const int bh = blockIdx.z, b = bh / Hq, h = bh % Hq, kvh = h / g;
  const int Hkv = Hq / g;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  float* out = scores + (int64_t)bh * n * n;
  if (j0 >= i0 + 31) {  // every (i, j) of the tile has j >= i
    for (int r = ty; r < 32; r += 8) {
      int i = i0 + r, j = j0 + tx;
      if (i < n && j < n) out[(int64_t)i * n + j] = kNegInf;
    }
    return;
  }
  const float* qsrc = qbar + (int64_t)bh * n * D;
  const float* ksrc = kbar + ((int64_t)b * Hkv + kvh) * n * D;
  for (int e = threadIdx.x; e < 32 * D; e += 256) {
    int r = e / D, c = e % D;
    qs[r][c] = (i0 + r < n) ? qsrc[(int64_t)(i0 + r) * D + c] : 0.f;
    ks[r][c] = (j0 + r < n) ? ksrc[(int64_t)(j0 + r) * D + c] : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int r = ty + 8 * q, i = i0 + r, j = j0 + tx;
    float acc = 0.f;
#pragma unroll 16
    for (int c = 0; c < D; ++c) acc = fmaf(qs[r][c], ks[tx][c], acc);
    if (i < n && j < n) out[(int64_t)i * n + j] = (j < i) ? scale * acc : kNegInf;
  }
}

// ------------------------------------------------------------------ top-k
// One warp per (b, h, i) row.  Candidate j lives in lane j % 32, slot j / 32.
// k-1 rounds of a warp arg-max with the order (score desc, index asc) pick the
// blocks; the chosen set is then written in ascending order by a ballot scan.
__device__ __forceinline__ bool better(float a, int ja, float b, int jb) {
  return a > b || (a == b && ja < jb);
}

// Warp-wide top-k of one selection row whose query block is i: v[m] holds the
// score of candidate j = lane + 32 m (j < i).  Writes Sel ascending to orow,
// -1 padded.
template <int CPL>
__device__ __forceinline__ void select_row(float (&v)[CPL], int i, int n, int k, int lane, int32_t* orow) {
  uint64_t taken = 0;
  if (i + 1 <= k) {
#pragma unroll
    for (int m = 0; m < CPL; ++m)
      if (lane + 32 * m <= i) taken |= 1ull << m;
  } else {
    // Candidates that cannot be chosen (j >= i, or already taken) hold NaN,
    // which compares false with everything, so a round's lane-local scan is
    // one ordered compare per slot (slots ascend in j: the first of equal
    // scores is the smaller j; the first -inf counts when nothing better is
    // left).
    const float kOut = __int_as_float(0x7fffffff);
#pragma unroll
    for (int m = 0; m < CPL; ++m)
      if (lane + 32 * m >= i) v[m] = kOut;
    for (int round = 0; round < k - 1; ++round) {
      float bv = kNegInf;
      int bj = INT_MAX;
#pragma unroll
      for (int m = 0; m < CPL; ++m) {
        if (v[m] > bv || (v[m] == bv && bj == INT_MAX)) {
          bv = v[m];
          bj = lane + 32 * m;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oj = __shfl_xor_sync(0xffffffffu, bj, off);
        if (better(ov, oj, bv, bj)) {
          bv = ov;
          bj = oj;
        }
      }
      if (bj != INT_MAX && (bj & 31) == lane) {
        taken |= 1ull << (bj >> 5);
#pragma unroll
        for (int m = 0; m < CPL; ++m)
          if (m == (bj >> 5)) v[m] = kOut;
      }
    }
    if ((i & 31) == lane) taken |= 1ull << (i >> 5);
  }
  int base = 0;
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int m = 0; m < CPL; ++m) {
    if (32 * m >= n) break;
    const bool mine = (taken >> m) & 1ull;
    const unsigned bal = __ballot_sync(0xffffffffu, mine);
    if (mine) orow[base + __popc(bal & lt)] = lane + 32 * m;
    base += __popc(bal);
  }
  for (int p = base + lane; p < k; p += 32) orow[p] = -1;
}

template <int CPL>
__global__ void __launch_bounds__(256) select_kernel(const float* __restrict__ scores,
                                                     int32_t* __restrict__ idx, int64_t rows,
                                                     int n, int k) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int i = (int)(row % n);
  const float* srow = scores + row * n;
  float v[CPL];
#pragma unroll
  for (int m = 0; m < CPL; ++m) {
    const int j = lane + 32 * m;
    float x = (j < i) ? srow[j] : kNegInf;
    v[m] = (x != x) ? kNegInf : x;  // NaN ranks as -inf
  }
  select_row<CPL>(v, i, n, k, lane, idx + row * k);
}

// ------------------------------------------------------------------ per-token selection
// One warp per (b, h, t) row: the token's own query scores the pooled keys of
// the complete earlier blocks (score_j = scale q_t . kbar_j, j < i = t / s;
// lanes split d, RPW pooled keys in flight), then the same top-k as above.
template <typename T, int D, int CPL>
__global__ void __launch_bounds__(256) token_select_kernel(TensorRef Q, const float* __restrict__ kbar,
                                                           int32_t* __restrict__ idx, int64_t rows, int Hq, int g,
                                                           int N, int s, int n, int k, float scale) {
  constexpr int PER = D / 32, RPW = 4;
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int t = (int)(row % N);
  const int bh = (int)(row / N), b = bh / Hq, h = bh % Hq;
  const int i = t / s;
  float qv[PER];
  const T* qrow = row_ptr<T>(Q, b, h, t);
#pragma unroll
  for (int c = 0; c < PER; ++c) qv[c] = to_f32(qrow[lane * PER + c]);
  const float* kb = kbar + ((int64_t)b * (Hq / g) + h / g) * n * D;
  float v[CPL];
#pragma unroll
  for (int m = 0; m < CPL; ++m) v[m] = kNegInf;
  for (int j0 = 0; j0 < i; j0 += RPW) {
    float kv[RPW][PER];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
#pragma unroll
      for (int c = 0; c < PER; ++c) kv[r][c] = (j0 + r < i) ? kb[(int64_t)(j0 + r) * D + lane * PER + c] : 0.f;
    }
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      float p = 0.f;
#pragma unroll
      for (int c = 0; c < PER; ++c) p = fmaf(qv[c], kv[r][c], p);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
      const int j = j0 + r;
      if (j < i && (j & 31) == lane) {
        float x = scale * p;
#pragma unroll
        for (int m = 0; m < CPL; ++m)
          if (m == (j >> 5)) v[m] = (x != x) ? kNegInf : x;
      }
    }
  }
  select_row<CPL>(v, i, n, k, lane, idx + row * k);
}

// Shared-memory form, used when the pooled keys of one kv head fit: a CTA of
// TOK_WARPS warps takes TOK_PER_CTA consecutive tokens of one (b, h) and stages the
// pooled keys its tokens can rank (blocks j < jmax) transposed, kT[c][j]
// with a row pitch of n + 1 floats (the transposing stores fall in distinct
// banks).  Lane l then forms whole dot products for its blocks j = l + 32 m
// (the query broadcast from shared memory): no cross-lane reduction per
// block, and each pooled key is read from global memory once per CTA
// instead of once per token.
constexpr int TOK_PER_CTA = 256;
constexpr int TOK_WARPS = 16;  // 512 threads share one staged copy of the pooled keys

template <typename T, int D, int CPL>
__global__ void __launch_bounds__(TOK_WARPS * 32) token_select_smem_kernel(TensorRef Q, const float* __restrict__ kbar,
                                                                int32_t* __restrict__ idx, int Hq, int g, int N,
                                                                int s, int n, int k, float scale) {
  extern __shared__ float kT[];  // [D][n + 1] (+ 32 floats of slack: lanes past i read, and discard, the tail)
  __shared__ float qs[TOK_WARPS][D];  // each warp's current query row
  const int t0 = blockIdx.x * TOK_PER_CTA, h = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tend = min(t0 + TOK_PER_CTA, N);
  const int jmax = (tend - 1) / s;
  const int pitch = n + 1;
  const float* kb = kbar + ((int64_t)b * (Hq / g) + h / g) * n * D;
  for (int e = threadIdx.x; e < jmax * D; e += TOK_WARPS * 32) {
    const int j = e / D, c = e % D;
    kT[c * pitch + j] = kb[(int64_t)j * D + c];
  }
  __syncthreads();
  for (int t = t0 + warp; t < tend; t += TOK_WARPS) {
    const int i = t / s;
    const T* qrow = row_ptr<T>(Q, b, h, t);
    for (int c = lane; c < D; c += 32) qs[warp][c] = to_f32(qrow[c]);
    __syncwarp();
    // One group of 32 blocks at a time; groups past the token's causal
    // range are skipped as a whole (the guard is warp-uniform).
    float acc[CPL];
#pragma unroll
    for (int m = 0; m < CPL; ++m) {
      acc[m] = 0.f;
      if (32 * m < i) {
        const float* col = kT + lane + 32 * m;
        float a0 = 0.f, a1 = 0.f;
#pragma unroll 16
        for (int c = 0; c < D; c += 2) {
          a0 = fmaf(qs[warp][c], col[c * pitch], a0);
          a1 = fmaf(qs[warp][c + 1], col[(c + 1) * pitch], a1);
        }
        acc[m] = a0 + a1;
      }
    }
    __syncwarp();
    float v[CPL];
#pragma unroll
    for (int m = 0; m < CPL; ++m) {
      const float x = scale * acc[m];
      v[m] = (lane + 32 * m < i && x == x) ? x : kNegInf;  // NaN ranks as -inf
    }
    select_row<CPL>(v, i, n, k, lane, idx + (((int64_t)b * Hq + h) * N + t) * k);
  }
}

size_t token_select_smem_bytes(int n, int d) { return ((size_t)d * (n + 1) + 32) * sizeof(float); }
constexpr size_t kTokenSelectSmemMax = 200 * 1024;

// ------------------------------------------------------------------ mask
// grid = rows, 32 threads: words of the selected-block bit set of one
// selection row (a query block, or a token when div = s: i = (row % rph) / div).
__global__ void mask_kernel(const int32_t* __restrict__ idx, uint32_t* __restrict__ mask, int rph, int div,
                            int k, int words) {
  __shared__ uint32_t w[64];
  const int64_t row = blockIdx.x;
  const int i = (int)(row % rph) / div;
  for (int q = threadIdx.x; q < words; q += 32) w[q] = 0u;
  __syncwarp();
  for (int e = threadIdx.x; e < k; e += 32) {
    const int j = idx[row * k + e];
    if (j >= 0 && j <= i) atomicOr(&w[j >> 5], 1u << (j & 31));
  }
  __syncwarp();
  for (int q = threadIdx.x; q < words; q += 32) mask[row * words + q] = w[q];
}

}  // namespace

cudaError_t launch_pool(const Dims& D, const TensorRef& X, int H, float* out, cudaStream_t st) {
  dim3 grid(D.n, H, D.B);
  if (D.dtype == SSA_BF16) {
    if (D.d == 128) pool_kernel<__nv_bfloat16, 128><<<grid, 128, 0, st>>>(X, H, D.s, D.n, out);
    else pool_kernel<__nv_bfloat16, 64><<<grid, 128, 0, st>>>(X, H, D.s, D.n, out);
  } else {
    if (D.d == 128) pool_kernel<float, 128><<<grid, 128, 0, st>>>(X, H, D.s, D.n, out);
    else pool_kernel<float, 64><<<grid, 128, 0, st>>>(X, H, D.s, D.n, out);
  }
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_scores(const Dims& D, const float* qbar, const float* kbar, float* scores,
                          cudaStream_t st) {
  const int t = (D.n + 31) / 32;
  dim3 grid(t, t, D.B * D.Hq);
  if (D.d == 128) score_kernel<128><<<grid, 256, 0, st>>>(qbar, kbar, scores, D.Hq, D.g, D.n, D.scale);
  else score_kernel<64><<<grid, 256, 0, st>>>(qbar, kbar, scores, D.Hq, D.g, D.n, D.scale);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_select(const Dims& D, const float* scores, int32_t* idx, cudaStream_t st) {
  const int64_t rows = (int64_t)D.B * D.Hq * D.n;
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  const int cpl = (D.n + 31) / 32;
  if (cpl <= 1) select_kernel<1><<<blocks, 256, 0, st>>>(scores, idx, rows, D.n, D.k);
  else if (cpl <= 2) select_kernel<2><<<blocks, 256, 0, st>>>(scores, idx, rows, D.n, D.k);
  else if (cpl <= 4) select_kernel<4><<<blocks, 256, 0, st>>>(scores, idx, rows, D.n, D.k);
  else if (cpl <= 8) select_kernel<8><<<blocks, 256, 0, st>>>(scores, idx, rows, D.n, D.k);
  else if (cpl <= 16) select_kernel<16><<<blocks, 256, 0, st>>>(scores, idx, rows, D.n, D.k);
  else if (cpl <= 32) select_kernel<32><<<blocks, 256, 0, st>>>(scores, idx, rows, D.n, D.k);
  else select_kernel<64><<<blocks, 256, 0, st>>>(scores, idx, rows, D.n, D.k);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_build_mask(const Dims& D, const int32_t* idx, uint32_t* mask, int words,
                              cudaStream_t st) {
  const int64_t rows = (int64_t)D.B * D.Hq * D.rows_sel;
  mask_kernel<<<(unsigned)rows, 32, 0, st>>>(idx, mask, D.rows_sel, D.per_token ? D.s : 1, D.k, words);
  count_launches(1);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t token_select_t(const Dims& Dm, const TensorRef& Q, const float* kbar, int32_t* idx, cudaStream_t st) {
  const int cpl = (Dm.n + 31) / 32;
  const size_t smem = token_select_smem_bytes(Dm.n, D);
  if (smem <= kTokenSelectSmemMax) {
    const dim3 grid((unsigned)((Dm.N + TOK_PER_CTA - 1) / TOK_PER_CTA), (unsigned)Dm.Hq, (unsigned)Dm.B);
    cudaError_t e = cudaSuccess;
#define SSA_TOKSEL_SMEM(C)                                                                                \
  do {                                                                                                    \
    auto kern = token_select_smem_kernel<T, D, C>;                                                        \
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);               \
    if (e == cudaSuccess)                                                                                 \
      kern<<<grid, TOK_WARPS * 32, smem, st>>>(Q, kbar, idx, Dm.Hq, Dm.g, Dm.N, Dm.s, Dm.n, Dm.k, Dm.scale); \
  } while (0)
    if (cpl <= 1) SSA_TOKSEL_SMEM(1);
    else if (cpl <= 2) SSA_TOKSEL_SMEM(2);
    else if (cpl <= 4) SSA_TOKSEL_SMEM(4);
    else if (cpl <= 8) SSA_TOKSEL_SMEM(8);
    else if (cpl <= 16) SSA_TOKSEL_SMEM(16);
    else {
      if constexpr (D == 64) SSA_TOKSEL_SMEM(32);
      else return cudaErrorInvalidConfiguration;  // unreachable: d = 128 fits at most 399 pooled keys
    }
#undef SSA_TOKSEL_SMEM
    if (e != cudaSuccess) return e;
    count_launches(1);
    return cudaGetLastError();
  }
  const int64_t rows = (int64_t)Dm.B * Dm.Hq * Dm.N;
  const unsigned grid = (unsigned)((rows + 7) / 8);
#define SSA_TOKSEL(C) token_select_kernel<T, D, C><<<grid, 256, 0, st>>>(Q, kbar, idx, rows, Dm.Hq, Dm.g, Dm.N, Dm.s, Dm.n, Dm.k, Dm.scale)
  if (cpl <= 1) SSA_TOKSEL(1);
  else if (cpl <= 2) SSA_TOKSEL(2);
  else if (cpl <= 4) SSA_TOKSEL(4);
  else if (cpl <= 8) SSA_TOKSEL(8);
  else if (cpl <= 16) SSA_TOKSEL(16);
  else if (cpl <= 32) SSA_TOKSEL(32);
  else SSA_TOKSEL(64);
#undef SSA_TOKSEL
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_select_tokens(const Dims& D, const TensorRef& Q, const float* kbar, int32_t* idx,
                                 cudaStream_t st) {
  if (D.dtype == SSA_BF16)
    return D.d == 128 ? token_select_t<__nv_bfloat16, 128>(D, Q, kbar, idx, st)
                      : token_select_t<__nv_bfloat16, 64>(D, Q, kbar, idx, st);
  return D.d == 128 ? token_select_t<float, 128>(D, Q, kbar, idx, st) : token_select_t<float, 64>(D, Q, kbar, idx, st);
}

}  // namespace ssa
