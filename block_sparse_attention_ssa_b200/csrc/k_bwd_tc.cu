// Tensor-core backward of both attention streams (sm_100a, bf16, d = 128).
//
// Objective ("Technische Samenvatting: SSA", "Bidirectionele Uitlijning";
// "SSA: Achieving Sparser Attention ...", "Bidirectional Attention
// Alignment"): L = <g_f, h_full> + <g_s, h_sparse> + alpha (L_sp + L_cm), with
// dh_f = g_f + 2 alpha (h_f - h_s)/M and dh_s = g_s + 2 alpha (h_s - h_f)/M.
//
// The two streams are independent softmax attentions over the same Q, K, V
// and their gradients add.  Each is differentiated on its own:
//   stream f (full):   every causal pair,        P = exp(x - lse_full), dh_f, D_f = dh_f . h_f
//   stream s (sparse): pairs with u in A_t only, P = exp(x - lse_sel),  dh_s, D_s = dh_s . h_s
//   dS = P (dh . v_u - D),  dQ_t += scale sum_u dS K_u,  dK_u += scale sum_t dS Q_t,
//   dV_u += sum_t P dh_t.
// A kernel walks 128 x 128 (key, query) tiles: first every causal tile of
// stream f, then the tiles of stream s that hold at least one selected
// (query block, key block) pair; inside such a tile the unselected blocks are
// masked like the causal triangle.  Every tile is therefore the same uniform
// step, and all tensor-core products are 128 x 128 x 16.
//
// Three launches:
//   pre  (CUDA cores, HBM-bound): dh_f, dh_s in bf16, D_f, D_s, lse in base 2,
//        and the partial sums of (h_f - h_s)^2 for the alignment loss;
//   dkv  one 128-key tile per CTA, walking the g query heads of its kv head:
//        S^T = K Q^T, dP^T = V dh^T (SS MMAs into TMEM); P^T and dS^T go back
//        to TMEM as bf16; dV += P^T dh, dK += dS^T Q (TS MMAs);
//   dq   one 128-row query tile per CTA, with Q and dh held in TMEM as the A
//        operands: S = Q K^T, dP = dh V^T (TS MMAs), dS -> TMEM over dP
//        (bf16), dQ += dS K (TS MMA); K and V stream through a 3-deep ring.
// No atomics: every output element is written by exactly one CTA, in a fixed
// order of steps, so results are bit-reproducible.
#include "ssa_internal.cuh"
#include "sm100_ptx.cuh"

namespace ssa {
namespace {

using namespace sm100;

constexpr int HD = 128;
// Gradient kernels: warps 0-7 compute P / dS (warp w reads TMEM lanes
// 32(w%4).. and columns 64(w/4)..; no two warps touch the same columns),
// warp 8 loads by TMA, warp 9 owns TMEM and issues the MMAs.
constexpr int NTHREADS = 320;
constexpr int WARP_TMA = 8, WARP_MMA = 9;
constexpr float kLog2e = 1.4426950408889634f;

constexpr int TILE = 128;                // keys and queries per step
constexpr int HALF = TILE * 128;         // 16 KB: 128 rows x 64 bf16 (one 128-byte swizzle span)
constexpr int TILE_B = 2 * HALF;         // 32 KB: one 128 x 128 bf16 tile
constexpr int kMaxSmem = 232448;         // 227 KB per CTA
constexpr uint32_t IDESC_S = idesc_bf16_f32(TILE, TILE, false, false);  // both operands K-major
constexpr uint32_t IDESC_ACC = idesc_bf16_f32(TILE, HD, false, true);   // B (rows = reduction) MN-major

// ================================================================ preprocess
// One warp per row (b, h, t); lane l holds columns 4l .. 4l+3.
__global__ void __launch_bounds__(256) bwd_pre_tc_kernel(TensorRef hf_t, TensorRef hs_t, TensorRef gf_t,
                                                        TensorRef gs_t, int Hq, int N, float c2,
                                                        __nv_bfloat16* dhf, __nv_bfloat16* dhs, float* Df,
                                                        float* Ds, float* partials, const float* lse_full,
                                                        const float* lse_sel, float* lse2f, float* lse2s) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t row = (int64_t)blockIdx.x * 8 + w;
  const int t = (int)(row % N), bh = (int)(row / N), b = bh / Hq, h = bh % Hq;
  const int c = 4 * lane;
  auto load4 = [](const __nv_bfloat16* p, float (&x)[4]) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    x[0] = __uint_as_float(v.x << 16);
    x[1] = __uint_as_float(v.x & 0xffff0000u);
    x[2] = __uint_as_float(v.y << 16);
    x[3] = __uint_as_float(v.y & 0xffff0000u);
  };
  float xf[4], xs[4], gf[4] = {0.f, 0.f, 0.f, 0.f}, gs[4] = {0.f, 0.f, 0.f, 0.f};
  load4(row_ptr<__nv_bfloat16>(hf_t, b, h, t) + c, xf);
  load4(row_ptr<__nv_bfloat16>(hs_t, b, h, t) + c, xs);
  if (gf_t.p) load4(row_ptr<__nv_bfloat16>(gf_t, b, h, t) + c, gf);
  if (gs_t.p) load4(row_ptr<__nv_bfloat16>(gs_t, b, h, t) + c, gs);
  float sq = 0.f, df = 0.f, ds = 0.f;
  uint32_t of[2], os[2];
#pragma unroll
  for (int e = 0; e < 4; e += 2) {
    float bf[2], bs[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float diff = xf[e + k] - xs[e + k];
      sq = fmaf(diff, diff, sq);
      bf[k] = gf[e + k] + c2 * diff;
      bs[k] = gs[e + k] - c2 * diff;
    }
    of[e / 2] = pack_bf16(bf[0], bf[1]);
    os[e / 2] = pack_bf16(bs[0], bs[1]);
    // D is formed from the rounded values the MMAs will see.
    df = fmaf(__uint_as_float(of[e / 2] << 16), xf[e], df);
    df = fmaf(__uint_as_float(of[e / 2] & 0xffff0000u), xf[e + 1], df);
    ds = fmaf(__uint_as_float(os[e / 2] << 16), xs[e], ds);
    ds = fmaf(__uint_as_float(os[e / 2] & 0xffff0000u), xs[e + 1], ds);
  }
  *reinterpret_cast<uint2*>(dhf + row * HD + c) = make_uint2(of[0], of[1]);
  *reinterpret_cast<uint2*>(dhs + row * HD + c) = make_uint2(os[0], os[1]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    sq += __shfl_xor_sync(0xffffffffu, sq, off);
    df += __shfl_xor_sync(0xffffffffu, df, off);
    ds += __shfl_xor_sync(0xffffffffu, ds, off);
  }
  __shared__ float part[8];
  if (lane == 0) {
    Df[row] = df;
    Ds[row] = ds;
    part[w] = sq;
    // lse in base 2; an empty selected set maps to +inf, so 2^(x - lse) is 0.
    const float ls = lse_sel[row];
    lse2f[row] = lse_full[row] * kLog2e;
    lse2s[row] = ls == kNegInf ? __builtin_huge_valf() : ls * kLog2e;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) s += part[q];
    partials[blockIdx.x] = s;
  }
}

struct BwdTcParams {
  TensorRef dq, dk, dv;     // outputs (bf16, strided)
  const float* lse2[2];     // [B,Hq,N] per stream (0 = full, 1 = sparse), base 2
  const float* D[2];        // [B,Hq,N] per stream
  const uint32_t* mask;     // [B,Hq,rows,words]: a row per query block (or per token)
  int words, rows;
  int32_t* status;
  int Hq, g, N, n, s, ls, NT;  // ls = log2(s); NT = number of 128-row tiles
  int full;                 // 0: sparse stream alone (no stream-f steps)
  // Element masks for the sparse stream: blocks of 16 / 32, or a selection
  // per token, make the selected set vary inside a 64 x 64 quarter of a step.
  int fine, per_token;
  // dK / dV kernel: a CTA walks hpc of the g query heads of its kv head; with
  // more than one chunk per group it writes fp32 partials [chunk][2][B][Hkv][N][d]
  // (dK unscaled, dV) that a second kernel adds in chunk order.
  int hpc;
  float* part;
  float c;                  // scale * log2(e)
  float scale;
};

// Word j / 32 of selection row i (a query block, or a token when per_token).
__device__ __forceinline__ uint32_t mask_word(const BwdTcParams& p, int b, int h, int i, int j) {
  return __ldg(p.mask + (((int64_t)b * p.Hq + h) * p.rows + i) * p.words + (j >> 5));
}

// Selection bits of key blocks kb0 .. kb0 + nb - 1 (nb | 32, kb0 a multiple of
// nb, so they share a word) for selection row i, in the low nb bits.
__device__ __forceinline__ uint32_t row_key_bits(const BwdTcParams& p, int b, int h, int i, int kb0, int nb) {
  const uint32_t w = mask_word(p, b, h, i, kb0) >> (kb0 & 31);
  return nb >= 32 ? w : (w & ((1u << nb) - 1u));
}

// Fine selections: bit c of the result is set when query t0 + c (c < 64,
// queries past N excluded) selected the key block of key u (lane-cooperative:
// every lane of the warp passes the same t0; u may differ per lane).
__device__ __forceinline__ unsigned long long query_sel_mask64(const BwdTcParams& p, int b, int h, int t0, int u,
                                                               int lane) {
  const int kb = u >> p.ls, sh = kb & 31;
  if (!p.per_token) {
    // the 64 queries span 64 / s query blocks (or lie inside one block)
    unsigned long long m = 0ull;
    const int qb0 = t0 >> p.ls, nq = p.s >= 64 ? 1 : 64 >> p.ls;
    for (int e = 0; e < nq; ++e) {
      const int qb = qb0 + e;
      if (qb >= p.n) break;
      if ((mask_word(p, b, h, qb, kb) >> sh) & 1u)
        m |= (p.s >= 64 ? ~0ull : ((1ull << p.s) - 1ull) << (e * p.s));
    }
    return m;
  }
  const int ta = t0 + lane, tb = t0 + 32 + lane;
  const uint32_t wa = ta < p.N ? mask_word(p, b, h, ta, kb) : 0u;  // word index is lane-uniform per key tile
  const uint32_t wb = tb < p.N ? mask_word(p, b, h, tb, kb) : 0u;
  unsigned long long m = 0ull;
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const uint32_t xa = __shfl_sync(0xffffffffu, wa, c), xb = __shfl_sync(0xffffffffu, wb, c);
    m |= (unsigned long long)((xa >> sh) & 1u) << c;
    m |= (unsigned long long)((xb >> sh) & 1u) << (32 + c);
  }
  return m;
}

// Fine selections: bit c set when key u0 + c (c < 64) lies in a block that
// selection row i selected.
__device__ __forceinline__ unsigned long long key_sel_mask64(const BwdTcParams& p, int b, int h, int i, int u0) {
  if (p.s >= 64) return ((mask_word(p, b, h, i, u0 >> p.ls) >> ((u0 >> p.ls) & 31)) & 1u) ? ~0ull : 0ull;
  const int nb = 64 >> p.ls;
  const uint32_t bits = row_key_bits(p, b, h, i, u0 >> p.ls, nb);
  unsigned long long m = 0ull;
  const unsigned long long run = (1ull << p.s) - 1ull;
  for (int e = 0; e < nb; ++e)
    if ((bits >> e) & 1u) m |= run << (e * p.s);
  return m;
}

// Which (query block, key block) pairs of the 128 x 128 tile (qt, kt) of query
// head h the sparse stream holds: bit 2*qh + kh for the 64-row halves (block
// 64), all four bits for block 128.  Blocks past the end and key blocks after
// the query block are never set.
__device__ __forceinline__ uint32_t tile_bits(const BwdTcParams& p, int b, int h, int qt, int kt) {
  if (p.fine) {
    // any selected (query, key) pair in the step: the 128 keys are 128 / s
    // blocks of one word; element masks then pick the pairs
    if (kt > qt) return 0u;
    const int nb = 128 >> p.ls, kb0 = (kt * TILE) >> p.ls;
    uint32_t any = 0u;
    if (p.per_token) {
      const int t1 = min(qt * TILE + TILE, p.N);
      for (int t = qt * TILE; t < t1 && !any; ++t) any |= row_key_bits(p, b, h, t, kb0, nb);
    } else {
      const int i1 = min(((qt + 1) * TILE) >> p.ls, p.n);
      for (int i = (qt * TILE) >> p.ls; i < i1 && !any; ++i) any |= row_key_bits(p, b, h, i, kb0, nb);
    }
    return any ? 0xFu : 0u;
  }
  if (p.s == 128) {
    if (kt > qt || qt >= p.n) return 0u;
    return ((mask_word(p, b, h, qt, kt) >> (kt & 31)) & 1u) ? 0xFu : 0u;
  }
  uint32_t bits = 0;
#pragma unroll
  for (int qh = 0; qh < 2; ++qh) {
    const int i = 2 * qt + qh;
    if (i >= p.n) continue;
    const uint32_t wd = mask_word(p, b, h, i, 2 * kt);
#pragma unroll
    for (int kh = 0; kh < 2; ++kh) {
      const int j = 2 * kt + kh;
      if (j <= i && ((wd >> (j & 31)) & 1u)) bits |= 1u << (2 * qh + kh);
    }
  }
  return bits;
}

// Block-wide compaction: every thread offers one candidate (`keep`, `entry`);
// kept entries are appended to list[] in candidate order.  `total` is the
// running count (same value in every thread); wsum is 10 ints of scratch.
template <typename E>
__device__ __forceinline__ void compact_append(bool keep, uint32_t entry, E* list, int cap, int* wsum,
                                               int& total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bal = __ballot_sync(0xffffffffu, keep);
  if (lane == 0) wsum[warp] = __popc(bal);
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < NTHREADS / 32; ++w) {
    const int c = wsum[w];
    before += (w < warp) ? c : 0;
    all += c;
  }
  const int pos = total + before + __popc(bal & ((1u << lane) - 1u));
  if (keep && pos < cap) list[pos] = (E)entry;
  __syncthreads();
  total += all;
}

// P = 2^(x c - lse2[col]) for 32 columns of one row, packed to bf16 pairs.
// MASKED: columns with keep(col) false are 0.
template <bool MASKED, typename Keep>
__device__ __forceinline__ void p_block(const uint32_t (&x)[32], const float* lse2, float c, Keep keep,
                                        uint32_t* pk) {
#pragma unroll
  for (int k = 0; k < 32; k += 4) {
    const float4 l = *reinterpret_cast<const float4*>(lse2 + k);
    float v[4];
    v[0] = ex2(fmaf(__uint_as_float(x[k]), c, -l.x));
    v[1] = ex2(fmaf(__uint_as_float(x[k + 1]), c, -l.y));
    v[2] = ex2(fmaf(__uint_as_float(x[k + 2]), c, -l.z));
    v[3] = ex2(fmaf(__uint_as_float(x[k + 3]), c, -l.w));
    if (MASKED) {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (!keep(k + e)) v[e] = 0.f;
    }
    pk[k / 2] = pack_bf16(v[0], v[1]);
    pk[k / 2 + 1] = pack_bf16(v[2], v[3]);
  }
}

// dS = P (dP - D[col]) for 32 columns, P given as packed bf16 pairs.
__device__ __forceinline__ void ds_block(const uint32_t (&y)[32], const float* D, const uint32_t* pk,
                                         uint32_t* out) {
#pragma unroll
  for (int k = 0; k < 32; k += 4) {
    const float4 dd = *reinterpret_cast<const float4*>(D + k);
    const float p0 = __uint_as_float(pk[k / 2] << 16), p1 = __uint_as_float(pk[k / 2] & 0xffff0000u);
    const float p2 = __uint_as_float(pk[k / 2 + 1] << 16), p3 = __uint_as_float(pk[k / 2 + 1] & 0xffff0000u);
    out[k / 2] = pack_bf16(p0 * (__uint_as_float(y[k]) - dd.x), p1 * (__uint_as_float(y[k + 1]) - dd.y));
    out[k / 2 + 1] = pack_bf16(p2 * (__uint_as_float(y[k + 2]) - dd.z), p3 * (__uint_as_float(y[k + 3]) - dd.w));
  }
}

// Same with one D for the whole row (dQ kernel).
__device__ __forceinline__ void ds_block_row(const uint32_t (&y)[32], float D, const uint32_t* pk,
                                             uint32_t* out) {
#pragma unroll
  for (int k = 0; k < 32; k += 2) {
    const float p0 = __uint_as_float(pk[k / 2] << 16), p1 = __uint_as_float(pk[k / 2] & 0xffff0000u);
    out[k / 2] = pack_bf16(p0 * (__uint_as_float(y[k]) - D), p1 * (__uint_as_float(y[k + 1]) - D));
  }
}

// P for 32 columns of one row with one lse for the row (dQ kernel).
template <bool MASKED, typename Keep>
__device__ __forceinline__ void p_block_row(const uint32_t (&x)[32], float l2, float c, Keep keep,
                                            uint32_t* pk) {
#pragma unroll
  for (int k = 0; k < 32; k += 2) {
    float v0 = ex2(fmaf(__uint_as_float(x[k]), c, -l2));
    float v1 = ex2(fmaf(__uint_as_float(x[k + 1]), c, -l2));
    if (MASKED) {
      if (!keep(k)) v0 = 0.f;
      if (!keep(k + 1)) v1 = 0.f;
    }
    pk[k / 2] = pack_bf16(v0, v1);
  }
}

// SS product of two 128 x 128 K-major tiles (reduction over d = 128).
__device__ __forceinline__ void mma_tile_ss(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk) {
    const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
    mma_ss(d_tmem, smem_desc_sw128(a_smem + off, 16, 1024), smem_desc_sw128(b_smem + off, 16, 1024), IDESC_S,
           kk > 0 ? 1u : 0u);
  }
}

// TS product over d = 128: A = 128 rows x 128 bf16 in TMEM (d columns 16kk..
// packed at column 8kk), B = a 128 x 128 K-major smem tile.
__device__ __forceinline__ void mma_tile_ts_k(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem) {
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk) {
    const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
    mma_ts(d_tmem, a_tmem + 8 * kk, smem_desc_sw128(b_smem + off, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
  }
}

// TS product: D (+)= A[TMEM, 128 x 128 bf16 as written by the P / dS warps]
// x B[smem tile, rows = reduction index, MN-major].  The warp with column
// range 64h.. leaves its 64 packed values in columns 64h .. 64h+31.
__device__ __forceinline__ void mma_tile_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < TILE / 16; ++kk) {
    const uint32_t a = a_tmem + 64 * (kk >> 2) + 8 * (kk & 3);
    mma_ts(d_tmem, a, smem_desc_sw128(b_smem + kk * 2048, HALF, 1024), IDESC_ACC,
           (accumulate || kk > 0) ? 1u : 0u);
  }
}

__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, const uint32_t (&r)[32], float mult) {
  uint32_t o[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) o[c] = pack_bf16(__uint_as_float(r[2 * c]) * mult, __uint_as_float(r[2 * c + 1]) * mult);
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) d4[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
}

// ================================================================ dK / dV kernel
namespace dkv {
constexpr int NS = 2;
constexpr int OFF_K = 0, OFF_V = TILE_B;
constexpr int SCAL = TILE * 4;                 // 128 floats
// A stage holds one step's Q tile with its lse2 and D (released after dK) and
// its dh tile (released after dV, earlier), each with its own barriers.
constexpr int STAGE = 2 * TILE_B + 2 * SCAL;
constexpr int OFF_STAGE = 2 * TILE_B;
constexpr int OFF_MISC = OFF_STAGE + NS * STAGE;
constexpr int MAX_SPARSE = 4096;               // g * NT
// TMEM columns: dK, dV accumulators, S^T (P^T over it), dP^T (dS^T over it).
constexpr uint32_t COL_DK = 0, COL_DV = 128, COL_S = 256, COL_DP = 384;

struct Misc {
  uint64_t kv_full;
  uint64_t q_full[NS], q_empty[NS], dh_full[NS], dh_empty[NS];
  uint64_t s_full, dp_full, p_full, ds_full, done, drain;
  uint32_t tmem_base;
  int abort;
  int wsum[NTHREADS / 32];
  // sparse steps: (head * query tiles + query tile offset) << 4 | pair bits
  uint16_t list[MAX_SPARSE];
};
constexpr int SMEM = OFF_MISC + (int)sizeof(Misc);
static_assert(SMEM <= kMaxSmem, "dkv shared-memory budget");
static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte alignment of swizzled tiles");
}  // namespace dkv

template <bool FINE>
__global__ void __launch_bounds__(NTHREADS, 1)
    bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDhf,
                      const __grid_constant__ CUtensorMap tmDhs, BwdTcParams p) {
  using namespace dkv;
  // Used directly (no pointer arithmetic on the address) so that accesses
  // through it stay shared-memory loads; TMA tiles with 128-byte swizzle need
  // the 1024-byte alignment, which is checked rather than assumed.
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(p.status, 0, (int)SSA_ERR_UNSUPPORTED);
    return;
  }
  dkv::Misc& M = *reinterpret_cast<dkv::Misc*>(smem + OFF_MISC);
  volatile int* abort = &M.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = (int)blockIdx.x;  // low key tiles have the most query tiles and launch first
  const int chunks = p.g / p.hpc;
  const int kvh = blockIdx.y / chunks, chunk = blockIdx.y % chunks, b = blockIdx.z;
  const int h0 = kvh * p.g + chunk * p.hpc;  // first query head of this CTA
  const int u0 = kt * TILE;
  const int nqt = p.NT - kt;       // causal query tiles per head
  const int n_cand = p.hpc * nqt;  // (head, query tile) pairs of the causal range
  const int n_full = p.full ? n_cand : 0;
  auto stage_ptr = [&](int st) { return smem + OFF_STAGE + st * STAGE; };

  if (threadIdx.x == 0) {
    mbar_init(&M.kv_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&M.q_full[s], 1);
      mbar_init(&M.q_empty[s], 1);
      mbar_init(&M.dh_full[s], 1);
      mbar_init(&M.dh_empty[s], 1);
    }
    mbar_init(&M.s_full, 1);
    mbar_init(&M.dp_full, 1);
    mbar_init(&M.p_full, 8);
    mbar_init(&M.ds_full, 8);
    mbar_init(&M.done, 1);
    mbar_init(&M.drain, 1);
    M.abort = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(&M.tmem_base, 512);
    tmem_relinquish();
  }
  // A ragged last query tile copies only its valid scalars; the rest of the
  // scalar slots must hold finite values (their columns are masked).
  for (int i = threadIdx.x; i < NS * 2 * TILE; i += NTHREADS)
    reinterpret_cast<float*>(stage_ptr(i / (2 * TILE)) + 2 * TILE_B)[i % (2 * TILE)] = 0.f;
  // Sparse-stream steps: (head, query tile) pairs holding a selected pair.
  int n_sparse = 0;
  for (int base = 0; base < n_cand; base += NTHREADS) {
    const int it = base + (int)threadIdx.x;
    uint32_t bits = 0;
    if (it < n_cand) bits = tile_bits(p, b, h0 + it / nqt, kt + it % nqt, kt);
    compact_append(bits != 0, ((uint32_t)it << 4) | bits, M.list, MAX_SPARSE, M.wsum, n_sparse);
  }
  n_sparse = min(n_sparse, MAX_SPARSE);
  const int T = n_full + n_sparse;
  // The scalar slots are also written by the async proxy (bulk copies).
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = M.tmem_base;
  uint8_t* sK = smem + OFF_K;
  uint8_t* sV = smem + OFF_V;
  // step j -> (head within the group, query tile, stream, pair bits)
  auto decode = [&](int j, int& hh, int& qt, int& sp, uint32_t& bits) {
    int it;
    if (j < n_full) {
      it = j;
      sp = 0;
      bits = 0xFu;
    } else {
      const uint32_t e = M.list[j - n_full];
      it = (int)(e >> 4);
      sp = 1;
      bits = e & 0xFu;
    }
    hh = it / nqt;
    qt = kt + it % nqt;
  };

  if (warp == WARP_TMA) {
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmDhf);
      prefetch_tensormap(&tmDhs);
      mbar_expect_tx(&M.kv_full, 2 * TILE_B);
      tma_load_4d(sK, &tmK, &M.kv_full, 0, u0, kvh, b);
      tma_load_4d(sK + HALF, &tmK, &M.kv_full, 64, u0, kvh, b);
      tma_load_4d(sV, &tmV, &M.kv_full, 0, u0, kvh, b);
      tma_load_4d(sV + HALF, &tmV, &M.kv_full, 64, u0, kvh, b);
      int issued = 0;
      for (int j = 0; j < T; ++j) {
        const int st = j % NS;
        const uint32_t ph = (uint32_t)(j / NS - 1) & 1u;
        int hh, qt, sp;
        uint32_t bits;
        decode(j, hh, qt, sp, bits);
        const int h = h0 + hh, t0 = qt * TILE;
        uint8_t* sp_ = stage_ptr(st);
        // dh first: its slot frees after dV, before the Q slot frees after dK
        if (j >= NS && !mbar_wait(&M.dh_empty[st], ph, abort)) break;
        const CUtensorMap* md = sp ? &tmDhs : &tmDhf;
        mbar_expect_tx(&M.dh_full[st], TILE_B);
        tma_load_4d(sp_ + TILE_B, md, &M.dh_full[st], 0, t0, h, b);
        tma_load_4d(sp_ + TILE_B + HALF, md, &M.dh_full[st], 64, t0, h, b);
        if (j >= NS && !mbar_wait(&M.q_empty[st], ph, abort)) {
          issued = -(j + 1);  // dh of step j issued, Q not
          break;
        }
        const int valid = min(TILE, p.N - t0);  // a multiple of 64
        mbar_expect_tx(&M.q_full[st], TILE_B + 2 * valid * 4);
        tma_load_4d(sp_, &tmQ, &M.q_full[st], 0, t0, h, b);
        tma_load_4d(sp_ + HALF, &tmQ, &M.q_full[st], 64, t0, h, b);
        const int64_t ro = ((int64_t)b * p.Hq + h) * p.N + t0;
        bulk_load(sp_ + 2 * TILE_B, p.lse2[sp] + ro, (uint32_t)valid * 4, &M.q_full[st]);
        bulk_load(sp_ + 2 * TILE_B + SCAL, p.D[sp] + ro, (uint32_t)valid * 4, &M.q_full[st]);
        issued = j + 1;
      }
      // no copy may still be in flight when the CTA exits
      int dummy = 0;
      mbar_wait(&M.kv_full, 0, &dummy);
      const int nq = issued < 0 ? -issued - 1 : issued, nd = issued < 0 ? -issued : issued;
      for (int j = (nq > NS ? nq - NS : 0); j < nq; ++j) {
        dummy = 0;
        mbar_wait(&M.q_full[j % NS], (uint32_t)(j / NS) & 1u, &dummy);
      }
      for (int j = (nd > NS ? nd - NS : 0); j < nd; ++j) {
        dummy = 0;
        mbar_wait(&M.dh_full[j % NS], (uint32_t)(j / NS) & 1u, &dummy);
      }
    }
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      const uint32_t ak = smem_u32(sK), av = smem_u32(sV);
      bool ok = T > 0 && mbar_wait(&M.kv_full, 0, abort) && mbar_wait(&M.q_full[0], 0, abort) &&
                mbar_wait(&M.dh_full[0], 0, abort);
      if (ok) {
        tc_fence_after();
        const uint32_t s0 = smem_u32(stage_ptr(0));
        mma_tile_ss(tmem + COL_S, ak, s0);
        tc_commit(&M.s_full);
        mma_tile_ss(tmem + COL_DP, av, s0 + TILE_B);
        tc_commit(&M.dp_full);
      }
      for (int j = 0; ok && j < T; ++j) {
        const int st = j % NS, st1 = (j + 1) % NS;
        const uint32_t ph1 = (uint32_t)((j + 1) / NS) & 1u;
        const uint32_t sq = smem_u32(stage_ptr(st)), sq1 = smem_u32(stage_ptr(st1));
        const bool more = j + 1 < T;
        // dV += P^T dh once the P warps have written P^T over S^T.
        if (!mbar_wait(&M.p_full, (uint32_t)j & 1u, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        mma_tile_ts(tmem + COL_DV, tmem + COL_S, sq + TILE_B, j > 0);
        tc_commit(&M.dh_empty[st]);
        // S^T of the next step reuses the S columns (ordered after dV).
        if (more) {
          if (!mbar_wait(&M.q_full[st1], ph1, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_tile_ss(tmem + COL_S, ak, sq1);
          tc_commit(&M.s_full);
        }
        // dK += dS^T Q once dS^T is over dP^T.
        if (!mbar_wait(&M.ds_full, (uint32_t)j & 1u, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        mma_tile_ts(tmem + COL_DK, tmem + COL_DP, sq, j > 0);
        tc_commit(&M.q_empty[st]);
        if (more) {
          if (!mbar_wait(&M.dh_full[st1], ph1, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_tile_ss(tmem + COL_DP, av, sq1 + TILE_B);
          tc_commit(&M.dp_full);
        }
      }
      tc_commit(&M.done);
      tc_commit(&M.drain);
      int dummy = 0;
      mbar_wait(&M.drain, 0, &dummy);
    }
  } else {
    const int quarter = warp & 3, ch = warp >> 2;  // lanes 32*quarter.., query columns 64*ch..
    const int r = quarter * 32 + lane;             // key row within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t cS = lane_base + COL_S + 64 * ch, cP = lane_base + COL_DP + 64 * ch;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int st = j % NS;
      int hh, qt, sp;
      uint32_t bits;
      decode(j, hh, qt, sp, bits);
      // the per-query scalars arrived with the Q copy of the stage
      if (!mbar_wait(&M.q_full[st], (uint32_t)(j / NS) & 1u, abort) ||
          !mbar_wait(&M.s_full, (uint32_t)j & 1u, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* L2 = reinterpret_cast<const float*>(stage_ptr(st) + 2 * TILE_B) + 64 * ch;
      const float* Dq = reinterpret_cast<const float*>(stage_ptr(st) + 2 * TILE_B + SCAL) + 64 * ch;
      bool sel = (bits >> (2 * ch + (r >> 6))) & 1u;
      const int tq = qt * TILE + 64 * ch;  // first query of this warp's columns
      const bool diag = qt == kt;
      const bool ragged = tq + 64 > p.N;
      // Sparse-stream step with fine selections: the pairs this key row holds
      // among the warp's 64 queries (the warp skips the step when none does).
      unsigned long long fm = ~0ull;
      if (FINE && sp) {
        fm = query_sel_mask64(p, b, h0 + hh, tq, u0 + r, lane);
        sel = __any_sync(0xffffffffu, fm != 0ull);
      }
      uint32_t pk[32];
      if (sel) {
        uint32_t x0[32], x1[32];
        tmem_ld32(cS, x0);
        tmem_ld32(cS + 32, x1);
        tmem_wait_ld();
        if (FINE && sp) {
          const int lim = p.N - tq;
          auto keep0 = [&](int col) { return ((fm >> col) & 1ull) && (!diag || r <= 64 * ch + col) && col < lim; };
          auto keep1 = [&](int col) {
            return ((fm >> (32 + col)) & 1ull) && (!diag || r <= 64 * ch + 32 + col) && 32 + col < lim;
          };
          p_block<true>(x0, L2, p.c, keep0, pk);
          p_block<true>(x1, L2 + 32, p.c, keep1, pk + 16);
        } else if (diag || ragged) {
          // key u0 + r may attend query tq + col only if r <= 64 ch + col, and the query must exist
          const int lim = p.N - tq;
          auto keep0 = [&](int col) { return (!diag || r <= 64 * ch + col) && col < lim; };
          auto keep1 = [&](int col) { return (!diag || r <= 64 * ch + 32 + col) && 32 + col < lim; };
          p_block<true>(x0, L2, p.c, keep0, pk);
          p_block<true>(x1, L2 + 32, p.c, keep1, pk + 16);
        } else {
          auto all = [](int) { return true; };
          p_block<false>(x0, L2, p.c, all, pk);
          p_block<false>(x1, L2 + 32, p.c, all, pk + 16);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      tmem_st32(cS, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&M.p_full);
      if (!mbar_wait(&M.dp_full, (uint32_t)j & 1u, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t dk[32];
      if (sel) {
        uint32_t y0[32], y1[32];
        tmem_ld32(cP, y0);
        tmem_ld32(cP + 32, y1);
        tmem_wait_ld();
        ds_block(y0, Dq, pk, dk);
        ds_block(y1, Dq + 32, pk + 16, dk + 16);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) dk[c] = 0u;
      }
      tmem_st32(cP, dk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&M.ds_full);
    }
    if (ok && mbar_wait(&M.done, 0, abort)) {
      tc_fence_after();
      const int u = u0 + r;
      const bool store = u < p.N;
      __nv_bfloat16* okp = store ? row_ptr_w<__nv_bfloat16>(p.dk, b, kvh, u) : nullptr;
      __nv_bfloat16* ovp = store ? row_ptr_w<__nv_bfloat16>(p.dv, b, kvh, u) : nullptr;
#pragma unroll 1
      for (int c0 = 64 * ch; c0 < 64 * ch + 64; c0 += 32) {
        uint32_t rk[32], rv[32];
        tmem_ld32(lane_base + COL_DK + c0, rk);
        tmem_ld32(lane_base + COL_DV + c0, rv);
        tmem_wait_ld();
        if (T == 0) {  // no step touched these keys (a selection without them)
#pragma unroll
          for (int c = 0; c < 32; ++c) rk[c] = rv[c] = 0u;
        }
        if (store && p.part == nullptr) {
          store_row_bf16(okp + c0, rk, p.scale);
          store_row_bf16(ovp + c0, rv, 1.f);
        } else if (store) {
          const int64_t plane = (int64_t)gridDim.z * (gridDim.y / chunks) * p.N * HD;
          float* pk = p.part + (int64_t)chunk * 2 * plane + (((int64_t)b * (gridDim.y / chunks) + kvh) * p.N + u) * HD + c0;
          float* pv = pk + plane;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            reinterpret_cast<float4*>(pk)[q] = make_float4(__uint_as_float(rk[4 * q]), __uint_as_float(rk[4 * q + 1]),
                                                           __uint_as_float(rk[4 * q + 2]), __uint_as_float(rk[4 * q + 3]));
            reinterpret_cast<float4*>(pv)[q] = make_float4(__uint_as_float(rv[4 * q]), __uint_as_float(rv[4 * q + 1]),
                                                           __uint_as_float(rv[4 * q + 2]), __uint_as_float(rv[4 * q + 3]));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (M.abort && threadIdx.x == 0) atomicCAS(p.status, 0, (int)SSA_ERR_TIMEOUT);
  if (warp == WARP_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ================================================================ dQ kernel
namespace dq {
constexpr int NS = 3;
constexpr int OFF_K = 0, OFF_V = NS * TILE_B;  // rings of K and V tiles
constexpr int OFF_MISC = 2 * NS * TILE_B;
constexpr int MAX_KT = 1024;                   // NT
// TMEM columns: dQ accumulator, S, dP (dS over it), then the A operands of
// S = Q K^T and dP = dh V^T as packed bf16 (64 columns each).
constexpr uint32_t COL_DQ = 0, COL_S = 128, COL_DP = 256, COL_Q = 384, COL_DH = 448;

struct Misc {
  uint64_t k_full[NS], k_empty[NS], v_full[NS], v_empty[NS];
  uint64_t a_ready, s_full, s_read, dp_full, ds_full, done, drain;
  uint32_t tmem_base;
  int abort;
  int wsum[NTHREADS / 32];
  uint32_t list[MAX_KT];  // sparse steps: key tile << 4 | pair bits
};
constexpr int SMEM = OFF_MISC + (int)sizeof(Misc);
static_assert(SMEM <= kMaxSmem, "dq shared-memory budget");
}  // namespace dq

// Row t (64 columns from c0) of a [B,H,N,128] bf16 tensor into this thread's
// TMEM lane as 32 packed columns; zeros past the end.
__device__ __forceinline__ void row_to_tmem(const TensorRef& X, int b, int h, int t, bool valid, int c0,
                                            uint32_t taddr) {
  uint32_t v[32];
  if (valid) {
    const uint4* src = reinterpret_cast<const uint4*>(row_ptr<__nv_bfloat16>(X, b, h, t) + c0);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint4 x = src[q];
      v[4 * q] = x.x;
      v[4 * q + 1] = x.y;
      v[4 * q + 2] = x.z;
      v[4 * q + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = 0u;
  }
  tmem_st32(taddr, v);
}

template <bool FINE>
__global__ void __launch_bounds__(NTHREADS, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     TensorRef Qr, TensorRef dhf_r, TensorRef dhs_r, BwdTcParams p) {
  using namespace dq;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(p.status, 0, (int)SSA_ERR_UNSUPPORTED);
    return;
  }
  dq::Misc& M = *reinterpret_cast<dq::Misc*>(smem + OFF_MISC);
  volatile int* abort = &M.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = (int)(gridDim.x - 1 - blockIdx.x);  // heaviest query tiles launch first
  const int h = blockIdx.y, b = blockIdx.z, kvh = h / p.g;
  const int q0 = qt * TILE;
  const int n_cand = qt + 1;  // causal key tiles
  const int n_full = p.full ? n_cand : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&M.k_full[s], 1);
      mbar_init(&M.k_empty[s], 1);
      mbar_init(&M.v_full[s], 1);
      mbar_init(&M.v_empty[s], 1);
    }
    mbar_init(&M.a_ready, 8);
    mbar_init(&M.s_full, 1);
    mbar_init(&M.s_read, 8);
    mbar_init(&M.dp_full, 1);
    mbar_init(&M.ds_full, 8);
    mbar_init(&M.done, 1);
    mbar_init(&M.drain, 1);
    M.abort = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(&M.tmem_base, 512);
    tmem_relinquish();
  }
  // Sparse-stream steps: key tiles holding a selected pair of this query tile.
  int n_sparse = 0;
  for (int base = 0; base < n_cand; base += NTHREADS) {
    const int kt = base + (int)threadIdx.x;
    const uint32_t bits = kt < n_cand ? tile_bits(p, b, h, qt, kt) : 0u;
    compact_append(bits != 0, ((uint32_t)kt << 4) | bits, M.list, MAX_KT, M.wsum, n_sparse);
  }
  n_sparse = min(n_sparse, MAX_KT);
  const int T = n_full + n_sparse;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = M.tmem_base;
  auto decode = [&](int j, int& kt, int& sp, uint32_t& bits) {
    if (j < n_full) {
      kt = j;
      sp = 0;
      bits = 0xFu;
    } else {
      const uint32_t e = M.list[j - n_full];
      kt = (int)(e >> 4);
      sp = 1;
      bits = e & 0xFu;
    }
  };

  if (warp == WARP_TMA) {
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      int kiss = 0, viss = 0;
      for (int j = 0; j < T; ++j) {
        const int st = j % NS;
        const uint32_t ph = (uint32_t)(j / NS - 1) & 1u;
        int kt, sp;
        uint32_t bits;
        decode(j, kt, sp, bits);
        if (j >= NS && !mbar_wait(&M.k_empty[st], ph, abort)) break;
        mbar_expect_tx(&M.k_full[st], TILE_B);
        tma_load_4d(smem + OFF_K + st * TILE_B, &tmK, &M.k_full[st], 0, kt * TILE, kvh, b);
        tma_load_4d(smem + OFF_K + st * TILE_B + HALF, &tmK, &M.k_full[st], 64, kt * TILE, kvh, b);
        kiss = j + 1;
        if (j >= NS && !mbar_wait(&M.v_empty[st], ph, abort)) break;
        mbar_expect_tx(&M.v_full[st], TILE_B);
        tma_load_4d(smem + OFF_V + st * TILE_B, &tmV, &M.v_full[st], 0, kt * TILE, kvh, b);
        tma_load_4d(smem + OFF_V + st * TILE_B + HALF, &tmV, &M.v_full[st], 64, kt * TILE, kvh, b);
        viss = j + 1;
      }
      int dummy = 0;
      for (int j = (kiss > NS ? kiss - NS : 0); j < kiss; ++j) {
        dummy = 0;
        mbar_wait(&M.k_full[j % NS], (uint32_t)(j / NS) & 1u, &dummy);
      }
      for (int j = (viss > NS ? viss - NS : 0); j < viss; ++j) {
        dummy = 0;
        mbar_wait(&M.v_full[j % NS], (uint32_t)(j / NS) & 1u, &dummy);
      }
    }
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      const uint32_t sk0 = smem_u32(smem + OFF_K), sv0 = smem_u32(smem + OFF_V);
      bool ok = T > 0 && mbar_wait(&M.a_ready, 0, abort) && mbar_wait(&M.k_full[0], 0, abort) &&
                mbar_wait(&M.v_full[0], 0, abort);
      if (ok) {
        tc_fence_after();
        mma_tile_ts_k(tmem + COL_S, tmem + COL_Q, sk0);
        tc_commit(&M.s_full);
        mma_tile_ts_k(tmem + COL_DP, tmem + COL_DH, sv0);
        tc_commit(&M.dp_full);
        tc_commit(&M.v_empty[0]);
      }
      for (int j = 0; ok && j < T; ++j) {
        const int st = j % NS, st1 = (j + 1) % NS;
        const uint32_t ph1 = (uint32_t)((j + 1) / NS) & 1u;
        const bool more = j + 1 < T;
        // S of the next step as soon as the dS warps hold S(j) in registers.
        if (!mbar_wait(&M.s_read, (uint32_t)j & 1u, abort)) {
          ok = false;
          break;
        }
        if (more) {
          if (!mbar_wait(&M.k_full[st1], ph1, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_tile_ts_k(tmem + COL_S, tmem + COL_Q, sk0 + st1 * TILE_B);
          tc_commit(&M.s_full);
        }
        // dQ += dS K once dS is over dP (for the first sparse step the dS
        // warps have also put dh_s in place of dh_f by then).
        if (!mbar_wait(&M.ds_full, (uint32_t)j & 1u, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        mma_tile_ts(tmem + COL_DQ, tmem + COL_DP, sk0 + st * TILE_B, j > 0);
        tc_commit(&M.k_empty[st]);
        if (more) {
          if (!mbar_wait(&M.v_full[st1], ph1, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_tile_ts_k(tmem + COL_DP, tmem + COL_DH, sv0 + st1 * TILE_B);
          tc_commit(&M.dp_full);
          tc_commit(&M.v_empty[st1]);
        }
      }
      tc_commit(&M.done);
      tc_commit(&M.drain);
      int dummy = 0;
      mbar_wait(&M.drain, 0, &dummy);
    }
  } else {
    const int quarter = warp & 3, ch = warp >> 2;  // lanes 32*quarter.., key columns 64*ch..
    const int r = quarter * 32 + lane;             // query row within the tile
    const int t = q0 + r;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const bool in_range = t < p.N;
    const int64_t ro = ((int64_t)b * p.Hq + h) * p.N + (in_range ? t : 0);
    const float l2[2] = {in_range ? p.lse2[0][ro] : 0.f, in_range ? p.lse2[1][ro] : 0.f};
    const float Dv[2] = {in_range ? p.D[0][ro] : 0.f, in_range ? p.D[1][ro] : 0.f};
    // A operands: Q and dh_f rows (dh_s when there are no stream-f steps),
    // d columns 64 ch .. 64 ch + 63.
    row_to_tmem(Qr, b, h, t, in_range, 64 * ch, lane_base + COL_Q + 32 * ch);
    row_to_tmem(n_full > 0 ? dhf_r : dhs_r, b, h, t, in_range, 64 * ch, lane_base + COL_DH + 32 * ch);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&M.a_ready);
    const uint32_t cS = lane_base + COL_S + 64 * ch, cP = lane_base + COL_DP + 64 * ch;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      int kt, sp;
      uint32_t bits;
      decode(j, kt, sp, bits);
      if (!mbar_wait(&M.s_full, (uint32_t)j & 1u, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      bool sel = (bits >> (2 * (r >> 6) + ch)) & 1u;
      // Sparse-stream step with fine selections: the keys of the warp's 64
      // columns this query row selected (the warp skips when no row does).
      unsigned long long fm = ~0ull;
      if (FINE && sp) {
        fm = in_range ? key_sel_mask64(p, b, h, p.per_token ? t : (t >> p.ls), kt * TILE + 64 * ch) : 0ull;
        sel = __any_sync(0xffffffffu, fm != 0ull);
      }
      uint32_t x0[32], x1[32];
      if (sel) {
        tmem_ld32(cS, x0);
        tmem_ld32(cS + 32, x1);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&M.s_read);
      uint32_t pk[32];
      if (sel) {
        const float lv = sp ? l2[1] : l2[0];
        if (FINE && sp) {
          const bool dg = kt == qt;
          auto keep0 = [&](int col) { return ((fm >> col) & 1ull) && (!dg || 64 * ch + col <= r); };
          auto keep1 = [&](int col) { return ((fm >> (32 + col)) & 1ull) && (!dg || 64 * ch + 32 + col <= r); };
          p_block_row<true>(x0, lv, p.c, keep0, pk);
          p_block_row<true>(x1, lv, p.c, keep1, pk + 16);
        } else if (kt == qt) {
          // query q0 + r attends key 128 kt + 64 ch + col only if 64 ch + col <= r
          auto keep0 = [&](int col) { return 64 * ch + col <= r; };
          auto keep1 = [&](int col) { return 64 * ch + 32 + col <= r; };
          p_block_row<true>(x0, lv, p.c, keep0, pk);
          p_block_row<true>(x1, lv, p.c, keep1, pk + 16);
        } else {
          auto all = [](int) { return true; };
          p_block_row<false>(x0, lv, p.c, all, pk);
          p_block_row<false>(x1, lv, p.c, all, pk + 16);
        }
      }
      if (!mbar_wait(&M.dp_full, (uint32_t)j & 1u, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t dsk[32];
      if (sel) {
        uint32_t y0[32], y1[32];
        tmem_ld32(cP, y0);
        tmem_ld32(cP + 32, y1);
        tmem_wait_ld();
        const float dv = sp ? Dv[1] : Dv[0];
        ds_block_row(y0, dv, pk, dsk);
        ds_block_row(y1, dv, pk + 16, dsk + 16);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) dsk[c] = 0u;
      }
      tmem_st32(cP, dsk);
      // dP of this step was the last product to read dh_f: the sparse steps
      // that follow use dh_s in the same columns.
      if (j + 1 == n_full && n_sparse > 0)
        row_to_tmem(dhs_r, b, h, t, in_range, 64 * ch, lane_base + COL_DH + 32 * ch);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&M.ds_full);
    }
    if (ok && mbar_wait(&M.done, 0, abort)) {
      tc_fence_after();
      __nv_bfloat16* out = in_range ? row_ptr_w<__nv_bfloat16>(p.dq, b, h, t) : nullptr;
#pragma unroll 1
      for (int c0 = 64 * ch; c0 < 64 * ch + 64; c0 += 32) {
        uint32_t rq[32];
        tmem_ld32(lane_base + COL_DQ + c0, rq);
        tmem_wait_ld();
        if (T == 0) {  // this query tile attends no listed block
#pragma unroll
          for (int c = 0; c < 32; ++c) rq[c] = 0u;
        }
        if (in_range) store_row_bf16(out + c0, rq, p.scale);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (M.abort && threadIdx.x == 0) atomicCAS(p.status, 0, (int)SSA_ERR_TIMEOUT);
  if (warp == WARP_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool bwd_tc_supported(const Dims& D) {
  const int NT = (D.N + TILE - 1) / TILE;
  return D.dtype == SSA_BF16 && D.d == 128 && (D.s == 16 || D.s == 32 || D.s == 64 || D.s == 128) && D.n <= 2048 &&
         (int64_t)bwd_mma_heads_per_cta(D) * NT <= dkv::MAX_SPARSE && NT <= dq::MAX_KT && D.g <= 255;
}

cudaError_t launch_bwd_tc(const Dims& D, const BwdArgs& a, int32_t* status, cudaStream_t st) {
  if (!bwd_tc_supported(D)) return cudaErrorNotSupported;
  // Workspace reuse: the fp32 dh_f / dO_c regions hold bf16 dh_f / dh_s in
  // their lower halves, Df / Dc hold D_f / D_s, and the upper half of the dh_f
  // region holds lse_full and lse_sel in base 2.
  __nv_bfloat16* dhf = reinterpret_cast<__nv_bfloat16*>(a.dhf);
  __nv_bfloat16* dhs = reinterpret_cast<__nv_bfloat16*>(a.doc);
  const double Mtot = (double)D.B * D.Hq * D.N * D.d;
  const float c2 = (float)(2.0 * (double)a.alpha / Mtot);
  const unsigned pre_blocks = (unsigned)sqdiff_partial_count(D);
  const int64_t rows = (int64_t)D.B * D.Hq * D.N;
  float* lse2f = reinterpret_cast<float*>(reinterpret_cast<char*>(a.dhf) + rows * D.d * 2);
  float* lse2s = lse2f + rows;
  bwd_pre_tc_kernel<<<pre_blocks, 256, 0, st>>>(a.hf, a.hs, a.gf, a.gs, D.Hq, D.N, c2, dhf, dhs, a.Df, a.Dc,
                                                a.partials, a.lse_full, a.lse_sel, lse2f, lse2s);
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.align_loss != nullptr) {
    e = launch_finish_mean(a.partials, a.n_partials, Mtot, 2.0f, a.align_loss, 1, st);
    if (e != cudaSuccess) return e;
  }
  const int64_t rowstride = (int64_t)D.N * D.d;
  TensorRef rdhf{dhf, (int64_t)D.Hq * rowstride, rowstride, D.d};
  TensorRef rdhs{dhs, (int64_t)D.Hq * rowstride, rowstride, D.d};
  CUtensorMap mq, mk, mv, mf, ms;
  if (!make_tma_map_bf16(&mq, a.q, D.B, D.Hq, D.N, TILE) || !make_tma_map_bf16(&mk, a.k, D.B, D.Hkv, D.N, TILE) ||
      !make_tma_map_bf16(&mv, a.v, D.B, D.Hkv, D.N, TILE) || !make_tma_map_bf16(&mf, rdhf, D.B, D.Hq, D.N, TILE) ||
      !make_tma_map_bf16(&ms, rdhs, D.B, D.Hq, D.N, TILE))
    return cudaErrorInvalidValue;
  BwdTcParams p;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.lse2[0] = lse2f;
  p.lse2[1] = lse2s;
  p.D[0] = a.Df;
  p.D[1] = a.Dc;
  p.mask = a.mask;
  p.words = a.words;
  p.rows = D.rows_sel;
  p.ls = D.s == 16 ? 4 : D.s == 32 ? 5 : D.s == 64 ? 6 : 7;
  p.per_token = D.per_token;
  p.fine = (D.s < 64 || D.per_token) ? 1 : 0;
  p.hpc = bwd_mma_heads_per_cta(D);
  const int chunks = D.g / p.hpc;
  p.part = chunks > 1 ? a.kvpart : nullptr;
  p.status = status;
  p.Hq = D.Hq;
  p.g = D.g;
  p.N = D.N;
  p.n = D.n;
  p.s = D.s;
  p.NT = (D.N + TILE - 1) / TILE;
  p.c = D.scale * kLog2e;
  p.scale = D.scale;
  p.full = a.sparse_only ? 0 : 1;
  auto kdq = p.fine ? bwd_dq_tc_kernel<true> : bwd_dq_tc_kernel<false>;
  auto kdkv = p.fine ? bwd_dkv_tc_kernel<true> : bwd_dkv_tc_kernel<false>;
  e = cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize, dq::SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kdkv, cudaFuncAttributeMaxDynamicSharedMemorySize, dkv::SMEM);
  if (e != cudaSuccess) return e;
  kdkv<<<dim3(p.NT, D.Hkv * chunks, D.B), NTHREADS, dkv::SMEM, st>>>(mq, mk, mv, mf, ms, p);
  count_launches(1);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (chunks > 1 && (e = launch_kvsum(D, a, a.kvpart, chunks, st)) != cudaSuccess) return e;
  kdq<<<dim3(p.NT, D.Hq, D.B), NTHREADS, dq::SMEM, st>>>(mk, mv, a.q, rdhf, rdhs, p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace ssa
