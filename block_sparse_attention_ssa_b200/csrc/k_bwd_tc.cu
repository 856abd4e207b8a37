// Tensor-core backward of both attention streams (sm_100a, bf16, d = 128).
//
// Objective ("Technische Samenvatting: SSA", "Bidirectionele Uitlijning";
// "SSA: Achieving Sparser Attention ...", "Bidirectional Attention
// Alignment"): L = <g_f, h_full> + <g_s, h_sparse> + alpha (L_sp + L_cm), with
// dh_f = g_f + 2 alpha (h_f - h_s)/M and dh_s = g_s + 2 alpha (h_s - h_f)/M.
//
// The two streams are kept apart.  For a causal pair (t, u):
//   P_f = exp(x - lse_full)                      (every causal pair)
//   P_s = exp(x - lse_sel)  if u is in A_t, else 0
//   dX  = P_f (dh_f . v_u - D_f) + P_s (dh_s . v_u - D_s),
//   D_f = dh_f . h_f,  D_s = dh_s . h_s,
//   dQ_t = scale sum_u dX K_u,  dK_u = scale sum_t dX Q_t,
//   dV_u = sum_t P_f dh_f,t + sum_t P_s dh_s,t.
// The sparse-stream products run only for tiles that contain a selected pair,
// and a tile never needs a per-row choice of operand.
//
// Three launches:
//   pre  (CUDA cores, HBM-bound): dh_f, dh_s in bf16, D_f, D_s, and the
//        partial sums of (h_f - h_s)^2 for the alignment loss;
//   dq   one 128-row query tile per CTA, walking 64-key tiles:
//        S = Q K^T, dP_f = dh_f V^T, dP_s = dh_s V^T (SS MMAs into TMEM),
//        dS -> TMEM (bf16), dQ += dS K (TS MMA);
//   dkv  one 128-key tile per CTA, walking the g query heads of its kv head and
//        every causal 64-row query tile:
//        S^T = K Q^T, dP_f^T = V dh_f^T, dP_s^T = V dh_s^T (SS MMAs),
//        P^T, P_s^T, dS^T -> TMEM (bf16), dV += P^T dh_f + P_s^T dh_s,
//        dK += dS^T Q (TS MMAs).
// No atomics: every output element is written by exactly one CTA.
#include "ssa_internal.cuh"
#include "sm100_ptx.cuh"

namespace ssa {
namespace {

using namespace sm100;

constexpr int HD = 128;
// Gradient kernels: warps 0-7 compute P / dS (warps w and w+4 share TMEM lanes
// 32(w%4).. and split a tile's columns), warp 8 loads by TMA, warp 9 owns
// TMEM and issues the MMAs.
constexpr int NTHREADS = 320;
constexpr int WARP_TMA = 8, WARP_MMA = 9;
constexpr float kLog2e = 1.4426950408889634f;

// ================================================================ preprocess
template <typename T>
__global__ void __launch_bounds__(256) bwd_pre_tc_kernel(TensorRef hf_t, TensorRef hs_t, TensorRef gf_t,
                                                        TensorRef gs_t, int Hq, int N, float c2,
                                                        __nv_bfloat16* dhf, __nv_bfloat16* dhs, float* Df,
                                                        float* Ds, float* partials, const float* lse_full,
                                                        const float* lse_sel, float4* scal) {
  constexpr int PER = HD / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t row = (int64_t)blockIdx.x * 8 + w;
  const int t = (int)(row % N), bh = (int)(row / N), b = bh / Hq, h = bh % Hq;
  const T* hf = row_ptr<T>(hf_t, b, h, t);
  const T* hs = row_ptr<T>(hs_t, b, h, t);
  const T* gf = gf_t.p ? row_ptr<T>(gf_t, b, h, t) : nullptr;
  const T* gs = gs_t.p ? row_ptr<T>(gs_t, b, h, t) : nullptr;
  float sq = 0.f, df = 0.f, ds = 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const int c = lane + 32 * e;
    const float xf = to_f32(hf[c]), xs = to_f32(hs[c]);
    const float diff = xf - xs;
    sq = fmaf(diff, diff, sq);
    const float vf = (gf ? to_f32(gf[c]) : 0.f) + c2 * diff;
    const float vs = (gs ? to_f32(gs[c]) : 0.f) - c2 * diff;
    const __nv_bfloat16 bf = __float2bfloat16_rn(vf), bs = __float2bfloat16_rn(vs);
    // D is formed from the rounded values the MMAs will see.
    df = fmaf(__bfloat162float(bf), xf, df);
    ds = fmaf(__bfloat162float(bs), xs, ds);
    dhf[row * HD + c] = bf;
    dhs[row * HD + c] = bs;
  }
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
    // {lse_full, lse_sel} in base 2 (an empty selected set maps to +inf, so
    // 2^(x - lse) is 0 there), then D_f, D_s: one 16-byte load per query.
    const float ls = lse_sel[row];
    scal[row] = make_float4(lse_full[row] * kLog2e, ls == kNegInf ? __builtin_huge_valf() : ls * kLog2e, df, ds);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) s += part[q];
    partials[blockIdx.x] = s;
  }
}

// Both warps of a lane quarter (w, w+4) reach this point before either
// continues; bounded like every other wait.  `uses` counts this warp's
// passes, which the partner matches one for one.
__device__ __forceinline__ bool pair_sync(uint64_t* bar, uint32_t& uses, int lane, volatile int* abort) {
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
  const bool ok = mbar_wait(bar, uses & 1u, abort);
  ++uses;
  tc_fence_after();
  return ok;
}

struct BwdTcParams {
  TensorRef dq, dk, dv;     // outputs (bf16, strided)
  const float* lse_full;    // [B,Hq,N]
  const float* lse_sel;
  const float* Df;          // [B,Hq,N]
  const float* Ds;
  const uint32_t* mask;     // [B,Hq,n,words]
  const float4* scal;       // [B,Hq,N]: {lse2_full, lse2_sel, D_f, D_s}
  int words;
  int32_t* status;
  int Hq, g, N, n, s;
  float c;                  // scale * log2(e)
  float scale;
};

__device__ __forceinline__ bool sel_bit(const BwdTcParams& p, int b, int h, int i, int j) {
  const uint32_t w = __ldg(p.mask + (((int64_t)b * p.Hq + h) * p.n + i) * p.words + (j >> 5));
  return (w >> (j & 31)) & 1u;
}

// State of a (query block i, key block j) pair: 0 no causal key, 1 selected, 2 dropped.
__device__ __forceinline__ int pair_state(const BwdTcParams& p, int b, int h, int i, bool qvalid, int j) {
  if (!qvalid || j > i) return 0;
  return sel_bit(p, b, h, i, j) ? 1 : 2;
}

// P / dS of one 32-column slice of a dK/dV step (keys in lanes, queries in
// columns).  SEL: the slice's key block is selected for the query block, so
// the sparse stream contributes; DIAG: the slice touches the causal diagonal.
template <bool SEL, bool DIAG>
__device__ __forceinline__ void dkv_slice(const uint32_t (&rs)[32], const uint32_t (&rf)[32],
                                          const uint32_t (&rp)[32], const float4* sc, int u, int tq0, float c,
                                          uint32_t (&pf_pk)[16], uint32_t (&ps_pk)[16], uint32_t (&ds_pk)[16]) {
#pragma unroll
  for (int k = 0; k < 32; k += 2) {
    float pf[2], ps[2], dsv[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float4 v4 = sc[k + e];  // lse2_f, lse2_s, D_f, D_s of query tq0 + k + e
      const float x = __uint_as_float(rs[k + e]);
      pf[e] = ex2(fmaf(x, c, -v4.x));
      if (DIAG && u > tq0 + k + e) pf[e] = 0.f;
      dsv[e] = pf[e] * (__uint_as_float(rf[k + e]) - v4.z);
      ps[e] = 0.f;
      if (SEL) {
        ps[e] = ex2(fmaf(x, c, -v4.y));
        if (DIAG && u > tq0 + k + e) ps[e] = 0.f;
        dsv[e] = fmaf(ps[e], __uint_as_float(rp[k + e]) - v4.w, dsv[e]);
      }
    }
    pf_pk[k / 2] = pack_bf16(pf[0], pf[1]);
    if (SEL) ps_pk[k / 2] = pack_bf16(ps[0], ps[1]);
    ds_pk[k / 2] = pack_bf16(dsv[0], dsv[1]);
  }
}

// dS of one 32-key slice of a dQ tile (queries in lanes, keys in columns).
template <bool SEL, bool DIAG>
__device__ __forceinline__ void dq_slice(const uint32_t (&rs)[32], const uint32_t (&rf)[32],
                                         const uint32_t (&rp)[32], float l2f, float l2s, float Dfv, float Dsv,
                                         int u0, int t, float c, uint32_t (&pk)[16]) {
#pragma unroll
  for (int k = 0; k < 32; k += 2) {
    float ds[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float x = __uint_as_float(rs[k + e]);
      float pf = ex2(fmaf(x, c, -l2f));
      if (DIAG && u0 + k + e > t) pf = 0.f;
      ds[e] = pf * (__uint_as_float(rf[k + e]) - Dfv);
      if (SEL) {
        float ps = ex2(fmaf(x, c, -l2s));
        if (DIAG && u0 + k + e > t) ps = 0.f;
        ds[e] = fmaf(ps, __uint_as_float(rp[k + e]) - Dsv, ds[e]);
      }
    }
    pk[k / 2] = pack_bf16(ds[0], ds[1]);
  }
}

// ================================================================ dQ kernel
namespace dq {
constexpr int BM = 128;  // query rows
constexpr int BK = 64;   // keys per tile
constexpr int NS = 3;
constexpr int TILE_A = BM * HD * 2;  // 32 KB: Q, dh_f, dh_s tiles
constexpr int TILE_K = BK * HD * 2;  // 16 KB: K or V tile
constexpr int OFF_Q = 0, OFF_DHF = TILE_A, OFF_DHS = 2 * TILE_A;
constexpr int OFF_K = 3 * TILE_A;
constexpr int OFF_V = OFF_K + NS * TILE_K;
constexpr int OFF_MISC = OFF_V + NS * TILE_K;
constexpr int SMEM = OFF_MISC + 1024 + 4096 + 1024;
constexpr uint32_t COL_DQ = 0, COL_S = 128, COL_DPF = 256, COL_DPS = 384;
constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BK, false, false);
constexpr uint32_t IDESC_DQ = idesc_bf16_f32(BM, HD, false, true);

constexpr int MAX_TILES = 4096;  // N / 64 for n <= 2048 and block <= 128
struct Misc {
  uint64_t a_full;
  uint64_t k_full[NS], k_empty[NS], v_full[NS], v_empty[NS];
  uint64_t s_full[2], ds_full[2];
  uint64_t pair[4];  // warps w and w+4: both hold their inputs before either writes
  uint64_t done, drain;
  uint32_t tmem_base;
  int abort;
  uint8_t state[MAX_TILES];  // per key tile: half-0 state | half-1 state << 2
};
static_assert(sizeof(Misc) <= SMEM - OFF_MISC - 1024, "dq shared-memory budget");
}  // namespace dq

__global__ void __launch_bounds__(NTHREADS, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDhf,
                     const __grid_constant__ CUtensorMap tmDhs, BwdTcParams p) {
  using namespace dq;
  if (*reinterpret_cast<volatile int32_t*>(p.status) != 0) return;
  // Used directly (no pointer arithmetic on the address) so that accesses
  // through it stay shared-memory loads; TMA tiles with 128-byte swizzle need
  // the 1024-byte alignment, which is checked rather than assumed.
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(p.status, 0, (int)SSA_ERR_UNSUPPORTED);
    return;
  }
  dq::Misc& M = *reinterpret_cast<dq::Misc*>(smem + OFF_MISC);
  volatile int* abort = &M.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = (int)(gridDim.x - 1 - blockIdx.x);
  const int h = blockIdx.y, b = blockIdx.z, kvh = h / p.g;
  const int q0 = qt * BM;
  const int q_end = min(q0 + BM, p.N);
  const int T = (q_end + BK - 1) / BK;
  // query blocks of the two 64-row halves
  const int ib0 = q0 / p.s, ib1 = (q0 + 64) / p.s;
  const bool valid1 = q0 + 64 < p.N;

  if (threadIdx.x == 0) {
    mbar_init(&M.a_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&M.k_full[s], 1);
      mbar_init(&M.k_empty[s], 1);
      mbar_init(&M.v_full[s], 1);
      mbar_init(&M.v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&M.s_full[s], 1);
      mbar_init(&M.ds_full[s], 8);
    }
    for (int q = 0; q < 4; ++q) mbar_init(&M.pair[q], 2);
    mbar_init(&M.done, 1);
    mbar_init(&M.drain, 1);
    M.abort = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(&M.tmem_base, 512);
    tmem_relinquish();
  }
  // (half, key block) states of every key tile, read once from the mask
  for (int j = threadIdx.x; j < T; j += NTHREADS) {
    const int jb = (j * BK) / p.s;
    M.state[j] = (uint8_t)(pair_state(p, b, h, ib0, true, jb) | (pair_state(p, b, h, ib1, valid1, jb) << 2));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = M.tmem_base;
  uint8_t* sQ = smem + OFF_Q;
  uint8_t* sDhf = smem + OFF_DHF;
  uint8_t* sDhs = smem + OFF_DHS;
  uint8_t* sK = smem + OFF_K;
  uint8_t* sV = smem + OFF_V;

  if (warp == WARP_TMA) {
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      mbar_expect_tx(&M.a_full, 3 * TILE_A);
      tma_load_4d(sQ, &tmQ, &M.a_full, 0, q0, h, b);
      tma_load_4d(sQ + TILE_A / 2, &tmQ, &M.a_full, 64, q0, h, b);
      tma_load_4d(sDhf, &tmDhf, &M.a_full, 0, q0, h, b);
      tma_load_4d(sDhf + TILE_A / 2, &tmDhf, &M.a_full, 64, q0, h, b);
      tma_load_4d(sDhs, &tmDhs, &M.a_full, 0, q0, h, b);
      tma_load_4d(sDhs + TILE_A / 2, &tmDhs, &M.a_full, 64, q0, h, b);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < T; ++j) {
        const int st = j % NS;
        const uint32_t use = (uint32_t)(j / NS);
        if (j >= NS && !mbar_wait(&M.k_empty[st], (use - 1) & 1u, abort)) break;
        mbar_expect_tx(&M.k_full[st], TILE_K);
        tma_load_4d(sK + st * TILE_K, &tmK, &M.k_full[st], 0, j * BK, kvh, b);
        tma_load_4d(sK + st * TILE_K + TILE_K / 2, &tmK, &M.k_full[st], 64, j * BK, kvh, b);
        k_issued = j + 1;
        if (j >= NS && !mbar_wait(&M.v_empty[st], (use - 1) & 1u, abort)) break;
        mbar_expect_tx(&M.v_full[st], TILE_K);
        tma_load_4d(sV + st * TILE_K, &tmV, &M.v_full[st], 0, j * BK, kvh, b);
        tma_load_4d(sV + st * TILE_K + TILE_K / 2, &tmV, &M.v_full[st], 64, j * BK, kvh, b);
        v_issued = j + 1;
      }
      int dummy = 0;
      mbar_wait(&M.a_full, 0, &dummy);
      for (int j = (k_issued > NS ? k_issued - NS : 0); j < k_issued; ++j) {
        dummy = 0;
        mbar_wait(&M.k_full[j % NS], (uint32_t)(j / NS) & 1u, &dummy);
      }
      for (int j = (v_issued > NS ? v_issued - NS : 0); j < v_issued; ++j) {
        dummy = 0;
        mbar_wait(&M.v_full[j % NS], (uint32_t)(j / NS) & 1u, &dummy);
      }
    }
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      const uint32_t aq = smem_u32(sQ), af = smem_u32(sDhf), as = smem_u32(sDhs);
      bool ok = mbar_wait(&M.a_full, 0, abort);
      bool started = false;
      auto issue_dq = [&](int jj) -> bool {
        const int sb = jj & 1;
        if (!mbar_wait(&M.ds_full[sb], (uint32_t)(jj >> 1) & 1u, abort)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + (jj % NS) * TILE_K);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t bdesc = smem_desc_sw128(k_addr + kk * 16 * 128, TILE_K / 2, 1024);
          mma_ts(tmem + COL_DQ, tmem + COL_S + sb * 64 + kk * 8, bdesc, IDESC_DQ, (started || kk > 0) ? 1u : 0u);
        }
        started = true;
        tc_commit(&M.k_empty[jj % NS]);
        return true;
      };
      for (int j = 0; ok && j < T; ++j) {
        const int st = j % NS, sb = j & 1;
        const uint32_t ph = (uint32_t)(j / NS) & 1u;
        if (!mbar_wait(&M.k_full[st], ph, abort) || !mbar_wait(&M.v_full[st], ph, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int stj = M.state[j];
        const bool any_sel = (stj & 3) == 1 || (stj >> 2) == 1;
        const uint32_t k_addr = smem_u32(sK + st * TILE_K), v_addr = smem_u32(sV + st * TILE_K);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t offa = (kk >> 2) * (TILE_A / 2) + (kk & 3) * 32;
          const uint32_t offb = (kk >> 2) * (TILE_K / 2) + (kk & 3) * 32;
          const uint64_t kdesc = smem_desc_sw128(k_addr + offb, 16, 1024);
          const uint64_t vdesc = smem_desc_sw128(v_addr + offb, 16, 1024);
          mma_ss(tmem + COL_S + sb * 64, smem_desc_sw128(aq + offa, 16, 1024), kdesc, IDESC_S, kk > 0);
          mma_ss(tmem + COL_DPF + sb * 64, smem_desc_sw128(af + offa, 16, 1024), vdesc, IDESC_S, kk > 0);
          if (any_sel) mma_ss(tmem + COL_DPS + sb * 64, smem_desc_sw128(as + offa, 16, 1024), vdesc, IDESC_S, kk > 0);
        }
        tc_commit(&M.s_full[sb]);
        tc_commit(&M.v_empty[st]);
        if (j >= 1 && !issue_dq(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && T >= 1) issue_dq(T - 1);
      tc_commit(&M.done);
      tc_commit(&M.drain);
      int dummy = 0;
      mbar_wait(&M.drain, 0, &dummy);
    }
  } else {
    const int quarter = warp & 3, ch = warp >> 2;  // lanes 32*quarter.., key columns 32*ch..
    const int row = quarter * 32 + lane;
    const int t = q0 + row;
    const int half = quarter >> 1;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const bool in_range = t < p.N;
    const int64_t ro = ((int64_t)b * p.Hq + h) * p.N + (in_range ? t : 0);
    const float4 sc = p.scal[ro];
    const float l2f = sc.x, l2s = sc.y, Dfv = sc.z, Dsv = sc.w;
    uint32_t pair_uses = 0;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int sb = j & 1;
      if (!mbar_wait(&M.s_full[sb], (uint32_t)(j >> 1) & 1u, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int mine = half ? (M.state[j] >> 2) : (M.state[j] & 3);
      const uint32_t c0 = 32 * ch;
      uint32_t pk[16];
      if (mine == 0) {
#pragma unroll
        for (int c = 0; c < 16; ++c) pk[c] = 0u;
      } else {
        uint32_t rs[32], rf[32], rp[32];
        tmem_ld32(lane_base + COL_S + sb * 64 + c0, rs);
        tmem_ld32(lane_base + COL_DPF + sb * 64 + c0, rf);
        if (mine == 1) tmem_ld32(lane_base + COL_DPS + sb * 64 + c0, rp);
        tmem_wait_ld();
        // dS overwrites the S columns this pair reads: both warps must hold
        // their inputs before either writes.
        if (!pair_sync(&M.pair[quarter], pair_uses, lane, abort)) {
          ok = false;
          break;
        }
        const int u0 = j * BK + (int)c0;
        const bool diag = u0 + 31 > q0 + quarter * 32;  // some key of the slice is after some row
        if (mine == 1) {
          if (diag) dq_slice<true, true>(rs, rf, rp, l2f, l2s, Dfv, Dsv, u0, t, p.c, pk);
          else dq_slice<true, false>(rs, rf, rp, l2f, l2s, Dfv, Dsv, u0, t, p.c, pk);
        } else {
          if (diag) dq_slice<false, true>(rs, rf, rp, l2f, l2s, Dfv, Dsv, u0, t, p.c, pk);
          else dq_slice<false, false>(rs, rf, rp, l2f, l2s, Dfv, Dsv, u0, t, p.c, pk);
        }
      }
      tmem_st16(lane_base + COL_S + sb * 64 + 16 * ch, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&M.ds_full[sb]);
    }
    if (ok && mbar_wait(&M.done, 0, abort)) {
      tc_fence_after();
      __nv_bfloat16* out = in_range ? row_ptr_w<__nv_bfloat16>(p.dq, b, h, t) : nullptr;
#pragma unroll 1
      for (int c0 = 64 * ch; c0 < 64 * ch + 64; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lane_base + COL_DQ + c0, r);
        tmem_wait_ld();
        if (in_range) {
          uint32_t o[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            o[c] = pack_bf16(__uint_as_float(r[2 * c]) * p.scale, __uint_as_float(r[2 * c + 1]) * p.scale);
          uint4* dst = reinterpret_cast<uint4*>(out + c0);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
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

// ================================================================ dK / dV kernel
namespace dkv {
constexpr int BKEY = 128;  // keys per CTA
constexpr int BQ = 64;     // queries per step
constexpr int NS = 3;
constexpr int TILE_KV = BKEY * HD * 2;  // 32 KB: K or V
constexpr int TILE_Q = BQ * HD * 2;     // 16 KB: Q, dh_f or dh_s step tile
constexpr int SCAL = BQ * 16;           // {lse2_f, lse2_s, D_f, D_s} of one step (1 KB)
constexpr int MAX_STEPS = 8192;         // g * N / 64
constexpr int STAGE = 3 * TILE_Q + SCAL;
constexpr int OFF_K = 0, OFF_V = TILE_KV;
constexpr int OFF_STAGE = 2 * TILE_KV;
constexpr int OFF_MISC = OFF_STAGE + NS * STAGE;
constexpr int SMEM = OFF_MISC + 1024 + MAX_STEPS + 1024;
// TMEM: dK, dV, then two step buffers of [S^T 64 | dP_f^T 64] columns.  A step
// with a selected pair puts dP_s^T in the other buffer's dP_f^T columns.
constexpr uint32_t COL_DK = 0, COL_DV = 128, COL_BUF = 256, BUF_COLS = 128, OFF_DP = 64;
constexpr uint32_t IDESC_S = idesc_bf16_f32(BKEY, BQ, false, false);
constexpr uint32_t IDESC_ACC = idesc_bf16_f32(BKEY, HD, false, true);

struct Misc {
  uint64_t kv_full;
  uint64_t full[NS], empty[NS];
  uint64_t s_full[2], p_full[2], done, drain;
  uint64_t pair[4];  // warps w and w+4: both hold their inputs before either writes
  uint32_t tmem_base;
  int abort;
  // per step: key-half-0 state | key-half-1 state << 2 | any selected << 4
  uint8_t state[MAX_STEPS];
};
static_assert(sizeof(Misc) <= SMEM - OFF_MISC - 1024, "dkv shared-memory budget");
}  // namespace dkv

__global__ void __launch_bounds__(NTHREADS, 1)
    bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDhf,
                      const __grid_constant__ CUtensorMap tmDhs, BwdTcParams p) {
  using namespace dkv;
  if (*reinterpret_cast<volatile int32_t*>(p.status) != 0) return;
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
  const int kt = (int)blockIdx.x;  // lightest-last order: low key tiles have the most query tiles
  const int kvh = blockIdx.y, b = blockIdx.z;
  const int u0 = kt * BKEY;
  // key blocks of the two 64-key halves
  const int kb0 = u0 / p.s, kb1 = (u0 + 64) / p.s;
  const bool kvalid1 = u0 + 64 < p.N;
  const int nq = p.N / BQ;
  const int qt0 = u0 / BQ;               // first query tile with a causal pair
  const int steps_per_head = nq - qt0;
  const int steps = p.g * steps_per_head;

  if (threadIdx.x == 0) {
    mbar_init(&M.kv_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&M.full[s], 1);
      mbar_init(&M.empty[s], 1);
    }
    for (int s2 = 0; s2 < 2; ++s2) {
      mbar_init(&M.s_full[s2], 1);
      mbar_init(&M.p_full[s2], 8);
    }
    for (int q = 0; q < 4; ++q) mbar_init(&M.pair[q], 2);
    mbar_init(&M.done, 1);
    mbar_init(&M.drain, 1);
    M.abort = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(&M.tmem_base, 512);
    tmem_relinquish();
  }
  // Steps walk (head hh, query tile qt) with qt fastest.  Their states are
  // read once from the mask into shared memory.
  for (int it = threadIdx.x; it < steps; it += NTHREADS) {
    const int h = kvh * p.g + it / steps_per_head;
    const int i = ((qt0 + it % steps_per_head) * BQ) / p.s;
    const int s0 = pair_state(p, b, h, i, true, kb0);
    const int s1 = kvalid1 ? pair_state(p, b, h, i, true, kb1) : 0;
    M.state[it] = (uint8_t)(s0 | (s1 << 2) | ((s0 == 1 || s1 == 1) ? 16 : 0));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = M.tmem_base;
  uint8_t* sK = smem + OFF_K;
  uint8_t* sV = smem + OFF_V;
  auto stage_ptr = [&](int st) { return smem + OFF_STAGE + st * STAGE; };

  if (warp == WARP_TMA) {
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmDhf);
      prefetch_tensormap(&tmDhs);
      mbar_expect_tx(&M.kv_full, 2 * TILE_KV);
      tma_load_4d(sK, &tmK, &M.kv_full, 0, u0, kvh, b);
      tma_load_4d(sK + TILE_KV / 2, &tmK, &M.kv_full, 64, u0, kvh, b);
      tma_load_4d(sV, &tmV, &M.kv_full, 0, u0, kvh, b);
      tma_load_4d(sV + TILE_KV / 2, &tmV, &M.kv_full, 64, u0, kvh, b);
      int issued = 0;
      int h = kvh * p.g, qt = qt0;
      for (int it = 0; it < steps; ++it) {
        const int st = it % NS;
        const uint32_t use = (uint32_t)(it / NS);
        if (it >= NS && !mbar_wait(&M.empty[st], (use - 1) & 1u, abort)) break;
        const int t0 = qt * BQ;
        const bool any = (M.state[it] & 16) != 0;
        uint8_t* sp = stage_ptr(st);
        mbar_expect_tx(&M.full[st], (any ? 3 : 2) * TILE_Q + SCAL);
        tma_load_4d(sp, &tmQ, &M.full[st], 0, t0, h, b);
        tma_load_4d(sp + TILE_Q / 2, &tmQ, &M.full[st], 64, t0, h, b);
        tma_load_4d(sp + TILE_Q, &tmDhf, &M.full[st], 0, t0, h, b);
        tma_load_4d(sp + TILE_Q + TILE_Q / 2, &tmDhf, &M.full[st], 64, t0, h, b);
        if (any) {
          tma_load_4d(sp + 2 * TILE_Q, &tmDhs, &M.full[st], 0, t0, h, b);
          tma_load_4d(sp + 2 * TILE_Q + TILE_Q / 2, &tmDhs, &M.full[st], 64, t0, h, b);
        }
        const int64_t ro = ((int64_t)b * p.Hq + h) * p.N + t0;
        bulk_load(sp + 3 * TILE_Q, p.scal + ro, SCAL, &M.full[st]);
        issued = it + 1;
        if (++qt == qt0 + steps_per_head) {
          qt = qt0;
          ++h;
        }
      }
      int dummy = 0;
      mbar_wait(&M.kv_full, 0, &dummy);
      for (int it = (issued > NS ? issued - NS : 0); it < issued; ++it) {
        dummy = 0;
        mbar_wait(&M.full[it % NS], (uint32_t)(it / NS) & 1u, &dummy);
      }
    }
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      const uint32_t ak = smem_u32(sK), av = smem_u32(sV);
      bool ok = mbar_wait(&M.kv_full, 0, abort);
      bool started = false;
      // dV += P^T dh_f (+ P_s^T dh_s), dK += dS^T Q for step jt (buffer jt & 1).
      auto accumulate = [&](int jt) -> bool {
        if (!mbar_wait(&M.p_full[jt & 1], (uint32_t)(jt >> 1) & 1u, abort)) return false;
        tc_fence_after();
        const int st = jt % NS;
        const uint32_t sq = smem_u32(stage_ptr(st));
        const uint32_t sf = sq + TILE_Q, ss = sq + 2 * TILE_Q;
        const uint32_t buf = COL_BUF + (uint32_t)(jt & 1) * BUF_COLS;
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk) {
          const uint32_t off = kk * 16 * 128;
          const uint32_t acc = (started || kk > 0) ? 1u : 0u;
          mma_ts(tmem + COL_DV, tmem + buf + kk * 8, smem_desc_sw128(sf + off, TILE_Q / 2, 1024), IDESC_ACC, acc);
          mma_ts(tmem + COL_DK, tmem + buf + OFF_DP + kk * 8, smem_desc_sw128(sq + off, TILE_Q / 2, 1024), IDESC_ACC,
                 acc);
        }
        started = true;
        if (M.state[jt] & 16) {
#pragma unroll
          for (int kk = 0; kk < BQ / 16; ++kk)
            mma_ts(tmem + COL_DV, tmem + buf + 32 + kk * 8, smem_desc_sw128(ss + kk * 16 * 128, TILE_Q / 2, 1024),
                   IDESC_ACC, 1u);
        }
        tc_commit(&M.empty[st]);
        return true;
      };
      for (int it = 0; ok && it < steps; ++it) {
        const int st = it % NS, b2 = it & 1;
        if (!mbar_wait(&M.full[st], (uint32_t)(it / NS) & 1u, abort)) {
          ok = false;
          break;
        }
        // A selected previous step left its dP_s^T in this step's buffer:
        // its softmax must be done with it first.
        if (it >= 1 && (M.state[it - 1] & 16) &&
            !mbar_wait(&M.p_full[(it - 1) & 1], (uint32_t)((it - 1) >> 1) & 1u, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const bool sel = (M.state[it] & 16) != 0;
        const uint32_t sq = smem_u32(stage_ptr(st));
        const uint32_t sf = sq + TILE_Q, ss = sq + 2 * TILE_Q;
        const uint32_t buf = COL_BUF + (uint32_t)b2 * BUF_COLS;
        const uint32_t other = COL_BUF + (uint32_t)(b2 ^ 1) * BUF_COLS;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t offa = (kk >> 2) * (TILE_KV / 2) + (kk & 3) * 32;
          const uint32_t offb = (kk >> 2) * (TILE_Q / 2) + (kk & 3) * 32;
          mma_ss(tmem + buf, smem_desc_sw128(ak + offa, 16, 1024), smem_desc_sw128(sq + offb, 16, 1024), IDESC_S,
                 kk > 0);
          mma_ss(tmem + buf + OFF_DP, smem_desc_sw128(av + offa, 16, 1024), smem_desc_sw128(sf + offb, 16, 1024),
                 IDESC_S, kk > 0);
        }
        if (!sel) tc_commit(&M.s_full[b2]);
        if (it >= 1 && !accumulate(it - 1)) {
          ok = false;
          break;
        }
        if (sel) {
          // after dK of the previous step has read its dS^T from `other`
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t offa = (kk >> 2) * (TILE_KV / 2) + (kk & 3) * 32;
            const uint32_t offb = (kk >> 2) * (TILE_Q / 2) + (kk & 3) * 32;
            mma_ss(tmem + other + OFF_DP, smem_desc_sw128(av + offa, 16, 1024), smem_desc_sw128(ss + offb, 16, 1024),
                   IDESC_S, kk > 0);
          }
          tc_commit(&M.s_full[b2]);
        }
      }
      if (ok && steps >= 1) accumulate(steps - 1);
      tc_commit(&M.done);
      tc_commit(&M.drain);
      int dummy = 0;
      mbar_wait(&M.drain, 0, &dummy);
    }
  } else {
    const int quarter = warp & 3, ch = warp >> 2;  // lanes 32*quarter.., query columns 32*ch..
    const int row = quarter * 32 + lane;           // key within the tile
    const int u = u0 + row;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    int qt = qt0;
    uint32_t pair_uses = 0;
    bool ok = true;
    for (int it = 0; it < steps; ++it) {
      const int b2 = it & 1;
      if (!mbar_wait(&M.s_full[b2], (uint32_t)(it >> 1) & 1u, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int st = it % NS;
      const uint32_t COL_S = COL_BUF + (uint32_t)b2 * BUF_COLS;
      const uint32_t COL_DPF = COL_S + OFF_DP;
      const uint32_t COL_DPS = COL_BUF + (uint32_t)(b2 ^ 1) * BUF_COLS + OFF_DP;
      // the per-query scalars of this stage arrived with the stage's copies
      if (!mbar_wait(&M.full[st], (uint32_t)(it / NS) & 1u, abort)) {
        ok = false;
        break;
      }
      const int t0 = qt * BQ;
      const int stt = M.state[it];
      const int mine = (quarter >> 1) ? ((stt >> 2) & 3) : (stt & 3);
      const bool any = (stt & 16) != 0;
      if (++qt == qt0 + steps_per_head) qt = qt0;
      const float4* sc = reinterpret_cast<const float4*>(stage_ptr(st) + 3 * TILE_Q);
      const uint32_t c0 = 32 * ch;
      // P^T -> S cols [16ch, 16ch+16); P_s^T -> S cols [32+16ch, ...); dS^T -> dP_f cols [16ch, ...).
      uint32_t pf_pk[16], ps_pk[16], ds_pk[16];
      if (mine == 0) {
#pragma unroll
        for (int c = 0; c < 16; ++c) pf_pk[c] = ps_pk[c] = ds_pk[c] = 0u;
      } else {
        uint32_t rs[32], rf[32], rp[32];
        tmem_ld32(lane_base + COL_S + c0, rs);
        tmem_ld32(lane_base + COL_DPF + c0, rf);
        if (mine == 1) tmem_ld32(lane_base + COL_DPS + c0, rp);
        tmem_wait_ld();
        // the outputs overwrite columns the partner warp reads
        if (!pair_sync(&M.pair[quarter], pair_uses, lane, abort)) {
          ok = false;
          break;
        }
        const int tq0 = t0 + (int)c0;                   // first query of the slice
        const bool diag = u0 + quarter * 32 + 31 > tq0;  // some key of the warp after some query
        if (mine == 1) {
          if (diag) dkv_slice<true, true>(rs, rf, rp, sc + c0, u, tq0, p.c, pf_pk, ps_pk, ds_pk);
          else dkv_slice<true, false>(rs, rf, rp, sc + c0, u, tq0, p.c, pf_pk, ps_pk, ds_pk);
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) ps_pk[c] = 0u;
          if (diag) dkv_slice<false, true>(rs, rf, rp, sc + c0, u, tq0, p.c, pf_pk, ps_pk, ds_pk);
          else dkv_slice<false, false>(rs, rf, rp, sc + c0, u, tq0, p.c, pf_pk, ps_pk, ds_pk);
        }
      }
      tmem_st16(lane_base + COL_S + 16 * ch, pf_pk);
      if (any) tmem_st16(lane_base + COL_S + 32 + 16 * ch, ps_pk);
      tmem_st16(lane_base + COL_DPF + 16 * ch, ds_pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&M.p_full[b2]);
    }
    if (ok && mbar_wait(&M.done, 0, abort)) {
      tc_fence_after();
      const bool store = u < p.N;
      __nv_bfloat16* ok_ = store ? row_ptr_w<__nv_bfloat16>(p.dk, b, kvh, u) : nullptr;
      __nv_bfloat16* ov_ = store ? row_ptr_w<__nv_bfloat16>(p.dv, b, kvh, u) : nullptr;
#pragma unroll 1
      for (int c0 = 64 * ch; c0 < 64 * ch + 64; c0 += 32) {
        uint32_t rk[32], rv[32];
        tmem_ld32(lane_base + COL_DK + c0, rk);
        tmem_ld32(lane_base + COL_DV + c0, rv);
        tmem_wait_ld();
        if (store) {
          uint32_t okp[16], ovp[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            okp[c] = pack_bf16(__uint_as_float(rk[2 * c]) * p.scale, __uint_as_float(rk[2 * c + 1]) * p.scale);
            ovp[c] = pack_bf16(__uint_as_float(rv[2 * c]), __uint_as_float(rv[2 * c + 1]));
          }
          uint4* dk4 = reinterpret_cast<uint4*>(ok_ + c0);
          uint4* dv4 = reinterpret_cast<uint4*>(ov_ + c0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            dk4[q] = make_uint4(okp[4 * q], okp[4 * q + 1], okp[4 * q + 2], okp[4 * q + 3]);
            dv4[q] = make_uint4(ovp[4 * q], ovp[4 * q + 1], ovp[4 * q + 2], ovp[4 * q + 3]);
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

}  // namespace

bool bwd_tc_supported(const Dims& D) {
  return D.dtype == SSA_BF16 && D.d == 128 && (D.s == 64 || D.s == 128) && D.n <= 2048 &&
         (int64_t)D.g * (D.N / dkv::BQ) <= dkv::MAX_STEPS && D.N / dq::BK <= dq::MAX_TILES;
}

cudaError_t launch_bwd_tc(const Dims& D, const BwdArgs& a, int32_t* status, cudaStream_t st) {
  if (!bwd_tc_supported(D)) return cudaErrorNotSupported;
  // Workspace reuse: the fp32 dh_f / dO_c regions hold bf16 dh_f / dh_s here,
  // Df / Dc hold D_f / D_s.
  __nv_bfloat16* dhf = reinterpret_cast<__nv_bfloat16*>(a.dhf);
  __nv_bfloat16* dhs = reinterpret_cast<__nv_bfloat16*>(a.doc);
  const double Mtot = (double)D.B * D.Hq * D.N * D.d;
  const float c2 = (float)(2.0 * (double)a.alpha / Mtot);
  const unsigned pre_blocks = (unsigned)sqdiff_partial_count(D);
  // The packed per-query scalars go in the upper half of the fp32 dh_f
  // region (the bf16 dh_f uses only the lower half).
  const int64_t rows = (int64_t)D.B * D.Hq * D.N;
  float4* scal = reinterpret_cast<float4*>(reinterpret_cast<char*>(a.dhf) + rows * D.d * 2);
  bwd_pre_tc_kernel<__nv_bfloat16><<<pre_blocks, 256, 0, st>>>(a.hf, a.hs, a.gf, a.gs, D.Hq, D.N, c2, dhf, dhs,
                                                                a.Df, a.Dc, a.partials, a.lse_full, a.lse_sel, scal);
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
  CUtensorMap mq128, mk64, mv64, mf128, ms128, mq64, mk128, mv128, mf64, ms64;
  if (!make_tma_map_bf16(&mq128, a.q, D.B, D.Hq, D.N, 128) || !make_tma_map_bf16(&mk64, a.k, D.B, D.Hkv, D.N, 64) ||
      !make_tma_map_bf16(&mv64, a.v, D.B, D.Hkv, D.N, 64) || !make_tma_map_bf16(&mf128, rdhf, D.B, D.Hq, D.N, 128) ||
      !make_tma_map_bf16(&ms128, rdhs, D.B, D.Hq, D.N, 128) || !make_tma_map_bf16(&mq64, a.q, D.B, D.Hq, D.N, 64) ||
      !make_tma_map_bf16(&mk128, a.k, D.B, D.Hkv, D.N, 128) || !make_tma_map_bf16(&mv128, a.v, D.B, D.Hkv, D.N, 128) ||
      !make_tma_map_bf16(&mf64, rdhf, D.B, D.Hq, D.N, 64) || !make_tma_map_bf16(&ms64, rdhs, D.B, D.Hq, D.N, 64))
    return cudaErrorInvalidValue;
  BwdTcParams p;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.lse_full = a.lse_full;
  p.lse_sel = a.lse_sel;
  p.Df = a.Df;
  p.Ds = a.Dc;
  p.mask = a.mask;
  p.scal = scal;
  p.words = a.words;
  p.status = status;
  p.Hq = D.Hq;
  p.g = D.g;
  p.N = D.N;
  p.n = D.n;
  p.s = D.s;
  p.c = D.scale * kLog2e;
  p.scale = D.scale;
  e = cudaFuncSetAttribute(bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dq::SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dkv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dkv::SMEM);
  if (e != cudaSuccess) return e;
  bwd_dkv_tc_kernel<<<dim3((D.N + dkv::BKEY - 1) / dkv::BKEY, D.Hkv, D.B), NTHREADS, dkv::SMEM, st>>>(
      mq64, mk128, mv128, mf64, ms64, p);
  count_launches(1);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dq_tc_kernel<<<dim3((D.N + dq::BM - 1) / dq::BM, D.Hq, D.B), NTHREADS, dq::SMEM, st>>>(mq128, mk64, mv64,
                                                                                            mf128, ms128, p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace ssa
