// Tensor-core dual-stream forward with per-row selection masks (sm_100a,
// bf16 in, fp32 accumulate, d = 64 or 128, blocks of 16 to 128 keys,
// selection per query block or per query token).
//
// What it computes ("SSA: Achieving Sparser Attention ...", "Practical
// Implementation of SSA"; "Technische Samenvatting: SSA", "1. Probleemstelling"
// and "Bidirectionele Uitlijning"): per query t two disjoint online
// softmaxes, over A_t (causal keys in selected blocks) and D_t (the other
// causal keys), merged at the end into h_sparse, h_full, lse_sel, lse_full and
// the dropped mass delta.
//
// The layout of the roles follows the tcgen05 forward for d = 128 and blocks
// of 64 / 128 (which classifies whole 64-row x 64-key sub-tiles), but here a
// 64-key sub-block can hold selected and dropped keys in one row and in
// different rows (blocks of 16 / 32, or every row its own selection), so each
// row routes its logits element by element with a 64-bit kept-key mask.
//
// CTA = one 128-row query tile of one (batch, query head), 320 threads:
//   warps 0-7  softmax / rescale / epilogue: warps w and w+4 share TMEM lanes
//              32(w%4).., i.e. query rows 32(w%4).., one row per thread; warp
//              w takes the 64-key sub-block w/4 of each 128-key tile;
//   warp 8     TMA producer (Q once, then K and V tiles through an NS-deep ring);
//   warp 9     TMEM allocator and single-thread tcgen05.mma issuer.
// TMEM: O_A [0, d), O_D [d, 2d), two S buffers of 128 columns after them.
// After both warps of a row have read a buffer's S, it holds bf16 P: the
// selected weights of sub-block q at columns [32q, 32q+32), the dropped
// weights at [64+32q, 64+32q+32).  The MMA warp multiplies a region into O_A
// (O_D) only when some row of the tile can hold a selected (dropped) key in
// that sub-block; it decides this from the OR / AND of the tile's selection
// rows, the same test the softmax warps use to decide which regions to write
// (zeros where a row has no key of the set).
//
// Softmax in base 2 with the scale folded in: p = 2^(S*c - m), c = scale*log2(e).
// The two warps of a row trade their sub-block maxima per set through shared
// memory; a set's running max is raised only when a tile's max exceeds it by
// more than 8 (p stays below 2^8), and O and l are then rescaled in place
// after the earlier PV products have completed.
#include "ssa_internal.cuh"
#include "sm100_ptx.cuh"

namespace ssa {
namespace {

using namespace sm100;

constexpr int BM = 128;  // query rows per CTA
constexpr int BN = 128;  // keys per tile
constexpr int SUB = 64;  // keys per sub-block
constexpr int NTHREADS = 320;
constexpr int WARP_TMA = 8, WARP_MMA = 9;
constexpr float kRescaleThreshold = 8.0f;

template <int HD>
struct Cfg {
  static constexpr int NS = HD == 64 ? 3 : 2;  // K/V stages
  static constexpr int Q_BYTES = BM * HD * 2;
  static constexpr int KV_BYTES = BN * HD * 2;
  static constexpr int HALF_Q = BM * 128;  // one 64-column (128-byte swizzle) span of the Q tile
  static constexpr int HALF_KV = BN * 128;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_MISC = OFF_V + NS * KV_BYTES;
  static constexpr uint32_t COL_OA = 0, COL_OD = HD, COL_S = 2 * HD;
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, false, true);
};

template <int NS>
struct Misc {
  uint64_t q_full;
  uint64_t k_full[NS], k_empty[NS], v_full[NS], v_empty[NS];
  uint64_t s_full[2], p_full[2];
  uint64_t o_done, o_final, drain;
  uint64_t pair[4];  // warps w and w+4 (one per lane quarter)
  uint32_t tmem_base;
  int abort;
  uint32_t uni[64];    // OR of the tile's selection rows
  uint32_t inter[64];  // AND of the tile's selection rows
  float xmax[2][2][2][128];  // [S buffer][sub-block][set][row]: scaled tile max
  float lsum[2][2][128];     // epilogue: [sub-block warp][set][row]
  // followed by the selection rows, 64 words each: one per query block of the
  // tile, or one per query row (per-token selection)
};

struct TcmParams {
  TensorRef hf, hs;
  const int32_t* idx;
  float* lse_full;
  float* lse_sel;
  float* delta;
  const float* lse_in;  // dropped-mass mode: the given lse_full, or null
  int32_t* status;
  int Hq, g, N, n, k, ls, per_token;
  float c;  // scale * log2(e)
};

__host__ __device__ inline int tcm_sel_rows(int per_token, int ls) {
  return per_token ? BM : (ls >= 7 ? 1 : (BM >> ls));
}

__device__ __forceinline__ bool pair_sync(uint64_t* bar, uint32_t& uses, int lane, volatile int* abort) {
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
  const bool ok = mbar_wait(bar, uses & 1u, abort);
  ++uses;
  tc_fence_after();
  return ok;
}

// WITH_V = false is the dropped-mass probe: no V, no PV products, only the
// two sets' running sums, and delta written (from lse_in when it is given).
template <int HD, bool WITH_V>
__global__ void __launch_bounds__(NTHREADS, 1)
    fwd_tcm_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, TcmParams p) {
  using C = Cfg<HD>;
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Misc<NS>& M = *reinterpret_cast<Misc<NS>*>(smem + C::OFF_MISC);
  uint32_t (*sel)[64] = reinterpret_cast<uint32_t (*)[64]>(smem + C::OFF_MISC + sizeof(Misc<NS>));
  volatile int* abort = &M.abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = (int)(gridDim.x - 1 - blockIdx.x);  // heaviest tiles first
  const int h = blockIdx.y, b = blockIdx.z, kvh = h / p.g;
  const int q0 = qt * BM;
  const int ib0 = q0 >> p.ls;
  const int nsel = tcm_sel_rows(p.per_token, p.ls);
  const int rph = p.per_token ? p.N : p.n;  // selection rows per head

  // ---- set-up
  if (threadIdx.x == 0) {
    mbar_init(&M.q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&M.k_full[s], 1);
      mbar_init(&M.k_empty[s], 1);
      mbar_init(&M.v_full[s], 1);
      mbar_init(&M.v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&M.s_full[s], 1);
      mbar_init(&M.p_full[s], 8);
    }
    mbar_init(&M.o_done, 1);
    mbar_init(&M.o_final, 1);
    mbar_init(&M.drain, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&M.pair[q], 2);
    M.abort = 0;
    fence_mbar_init();
  }
  for (int w = threadIdx.x; w < nsel * 64; w += NTHREADS) (&sel[0][0])[w] = 0u;
  if (warp == WARP_MMA) {
    tmem_alloc(&M.tmem_base, 512);
    tmem_relinquish();
  }
  __syncthreads();
  // Selection rows (entries outside 0..i are ignored), then their OR and AND
  // over the rows that exist.
  int nvalid = 0;  // selection rows of the tile inside the sequence
  if (p.per_token) nvalid = min(BM, p.N - q0);
  else nvalid = min(nsel, p.n - ib0);
  for (int e = threadIdx.x; e < nvalid * p.k; e += NTHREADS) {
    const int r = e / p.k;
    const int64_t srow = p.per_token ? (int64_t)q0 + r : (int64_t)ib0 + r;
    const int iblk = p.per_token ? (q0 + r) >> p.ls : ib0 + r;
    const int j = p.idx[(((int64_t)b * p.Hq + h) * rph + srow) * p.k + e % p.k];
    if (j >= 0 && j <= iblk) atomicOr(&sel[r][j >> 5], 1u << (j & 31));
  }
  __syncthreads();
  if (threadIdx.x < 64) {
    uint32_t o = 0u, a = ~0u;
    for (int r = 0; r < nvalid; ++r) {
      o |= sel[r][threadIdx.x];
      a &= sel[r][threadIdx.x];
    }
    M.uni[threadIdx.x] = o;
    M.inter[threadIdx.x] = a;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // Which P regions of the sub-block starting at key u some row can use.
  auto regions = [&](int u, bool& anyA, bool& anyD) {
    const int jb = u >> p.ls;
    const int nb = p.ls >= 6 ? 1 : (SUB >> p.ls);
    const uint32_t m = (nb >= 32 ? ~0u : ((1u << nb) - 1u)) << (jb & 31);
    anyA = (M.uni[jb >> 5] & m) != 0u;
    anyD = (M.inter[jb >> 5] & m) != m;
  };

  const int T = (min(q0 + BM, p.N) + BN - 1) / BN;  // causal key tiles
  const uint32_t tmem = M.tmem_base;
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;

  if (warp == WARP_TMA) {
    // ================================================================ producer
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      if (WITH_V) prefetch_tensormap(&tmV);
      mbar_expect_tx(&M.q_full, C::Q_BYTES);
#pragma unroll
      for (int hh = 0; hh < HD / 64; ++hh) tma_load_4d(sQ + hh * C::HALF_Q, &tmQ, &M.q_full, 64 * hh, q0, h, b);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < T; ++j) {
        const int st = j % NS;
        const uint32_t use = (uint32_t)(j / NS);
        auto load_tile = [&](uint8_t* dst, const CUtensorMap* map, uint64_t* bar) {
          mbar_expect_tx(bar, C::KV_BYTES);
#pragma unroll
          for (int hh = 0; hh < HD / 64; ++hh) tma_load_4d(dst + hh * C::HALF_KV, map, bar, 64 * hh, j * BN, kvh, b);
        };
        if (j >= NS && !mbar_wait(&M.k_empty[st], (use - 1) & 1u, abort)) break;
        load_tile(sK + st * C::KV_BYTES, &tmK, &M.k_full[st]);
        k_issued = j + 1;
        if (!WITH_V) continue;
        if (j >= NS && !mbar_wait(&M.v_empty[st], (use - 1) & 1u, abort)) break;
        load_tile(sV + st * C::KV_BYTES, &tmV, &M.v_full[st]);
        v_issued = j + 1;
      }
      // Drain: every copy this thread issued must have landed before the CTA exits.
      int dummy = 0;
      mbar_wait(&M.q_full, 0, &dummy);
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
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(sQ);
      bool started_a = false, started_d = false;
      bool ok = mbar_wait(&M.q_full, 0, abort);
      auto issue_pv = [&](int jj) -> bool {
        const int sb = jj & 1;
        if (!mbar_wait(&M.p_full[sb], (uint32_t)(jj >> 1) & 1u, abort)) return false;
        if (!WITH_V) return true;  // the S buffer is free again; nothing to multiply
        const int st = jj % NS;
        if (!mbar_wait(&M.v_full[st], (uint32_t)(jj / NS) & 1u, abort)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sV + st * C::KV_BYTES);
        const uint32_t s_col = C::COL_S + (uint32_t)sb * BN;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          bool anyA, anyD;
          regions(jj * BN + q * SUB, anyA, anyD);
          auto pv = [&](uint32_t o_col, uint32_t pcol, bool& started) {
#pragma unroll
            for (int kk = 0; kk < SUB / 16; ++kk) {
              const uint64_t bdesc = smem_desc_sw128(v_addr + (q * SUB + kk * 16) * 128, C::HALF_KV, 1024);
              mma_ts(tmem + o_col, tmem + pcol + kk * 8, bdesc, C::IDESC_PV, (started || kk > 0) ? 1u : 0u);
            }
            started = true;
          };
          if (anyA) pv(C::COL_OA, s_col + 32 * q, started_a);
          if (anyD) pv(C::COL_OD, s_col + 64 + 32 * q, started_d);
        }
        tc_commit(&M.v_empty[st]);
        tc_commit(&M.o_done);
        return true;
      };
      for (int j = 0; ok && j < T; ++j) {
        const int st = j % NS;
        if (!mbar_wait(&M.k_full[st], (uint32_t)(j / NS) & 1u, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + st * C::KV_BYTES);
        const uint32_t s_col = C::COL_S + (uint32_t)(j & 1) * BN;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off_q = (kk >> 2) * C::HALF_Q + (kk & 3) * 32;
          const uint32_t off_k = (kk >> 2) * C::HALF_KV + (kk & 3) * 32;
          mma_ss(tmem + s_col, smem_desc_sw128(q_addr + off_q, 16, 1024), smem_desc_sw128(k_addr + off_k, 16, 1024),
                 C::IDESC_QK, kk > 0 ? 1u : 0u);
        }
        tc_commit(&M.s_full[j & 1]);
        tc_commit(&M.k_empty[st]);
        if (j >= 1 && !issue_pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && T >= 1) ok = issue_pv(T - 1);
      tc_commit(&M.o_final);
      tc_commit(&M.drain);
      int dummy = 0;
      mbar_wait(&M.drain, 0, &dummy);
    }
  } else {
    // ================================================================ softmax
    const int quarter = warp & 3, q = warp >> 2;  // lane quarter, key sub-block
    const int row = quarter * 32 + lane;           // row within the tile == TMEM lane
    const int t = q0 + row;                        // query token
    const bool valid = t < p.N;
    const uint32_t* selw = sel[p.per_token ? row : min((t >> p.ls) - ib0, nsel - 1)];
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    float m2[2] = {kNegInf, kNegInf};  // running max (scaled, base 2), [0]=A [1]=D
    float l[2] = {0.f, 0.f};           // this warp's partial sums
    const bool direct = !WITH_V && p.lse_in != nullptr;  // uniform over the CTA
    const float lse2_in = (direct && valid) ? p.lse_in[((int64_t)b * p.Hq + h) * p.N + t] * 1.4426950408889634f : 0.f;
    uint32_t pair_uses = 0;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int sb = j & 1;
      if (!mbar_wait(&M.s_full[sb], (uint32_t)(j >> 1) & 1u, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int u0 = j * BN + q * SUB;  // first key of this warp's sub-block
      bool anyA, anyD;
      regions(u0, anyA, anyD);
      // Blocks have 16 keys or more, so a row's selection is constant over
      // each 16-key group of the sub-block: bit 16g of the row's kept-block
      // mask says whether group g is selected.  Causality only cuts the
      // diagonal sub-blocks; there the keys after t are set to -inf.
      const unsigned long long km = tile_keep_mask_p2(selw, u0, p.ls);
      bool gA[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) gA[g] = (km >> (16 * g)) & 1ull;
      const int lim = valid ? t - u0 : -1;  // keys c <= lim are causal
      const uint32_t s_addr = lane_base + C::COL_S + (uint32_t)sb * BN;
      if (direct) {
        // Dropped mass with lse_full given: sum 2^(S*c - lse2) over the
        // dropped keys directly; no running max, nothing traded.
        if (__any_sync(0xffffffffu, lim >= 0)) {
#pragma unroll
          for (int c0 = 0; c0 < SUB; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(s_addr + q * SUB + c0, r);
            tmem_wait_ld();
            float sD = 0.f;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const bool use = !gA[(c0 + c) >> 4] && (c0 + c <= lim);
              sD += use ? ex2(fmaf(__uint_as_float(r[c]), p.c, -lse2_in)) : 0.f;
            }
            l[1] += sD;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&M.p_full[sb]);
        continue;
      }
      float x[SUB];  // raw S of this warp's sub-block; the scale is folded into the exponent
      float mxA = kNegInf, mxD = kNegInf;
      if (__any_sync(0xffffffffu, lim >= 0)) {
#pragma unroll
        for (int c0 = 0; c0 < SUB; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(s_addr + q * SUB + c0, r);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c0 + c] = __uint_as_float(r[c]);
        }
        if (lim < SUB - 1) {
#pragma unroll
          for (int c = 0; c < SUB; ++c) x[c] = (c <= lim) ? x[c] : kNegInf;
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float a0 = x[16 * g], a1 = x[16 * g + 1], a2 = x[16 * g + 2], a3 = x[16 * g + 3];
#pragma unroll
          for (int c = 16 * g + 4; c < 16 * g + 16; c += 4) {
            a0 = fmaxf(a0, x[c]);
            a1 = fmaxf(a1, x[c + 1]);
            a2 = fmaxf(a2, x[c + 2]);
            a3 = fmaxf(a3, x[c + 3]);
          }
          const float gm = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
          mxA = gA[g] ? fmaxf(mxA, gm) : mxA;
          mxD = gA[g] ? mxD : fmaxf(mxD, gm);
        }
        mxA *= p.c;  // scale > 0
        mxD *= p.c;
      } else {
#pragma unroll
        for (int c = 0; c < SUB; ++c) x[c] = kNegInf;
      }
      // Trade sub-block maxima with the partner warp; after this point both
      // warps have read their S columns, so P may overwrite them.
      M.xmax[sb][q][0][row] = mxA;
      M.xmax[sb][q][1][row] = mxD;
      if (!pair_sync(&M.pair[quarter], pair_uses, lane, abort)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int X = 0; X < 2; ++X) {
        const float mxs = fmaxf(X == 0 ? mxA : mxD, M.xmax[sb][q ^ 1][X][row]);
        const float m_old = m2[X];
        const bool need = (m_old != kNegInf) && (mxs > m_old + kRescaleThreshold);
        if (!WITH_V) {
          if (need) {
            l[X] *= ex2(m_old - mxs);
            m2[X] = mxs;
          }
        } else if (__any_sync(0xffffffffu, need)) {
          // O_X must hold every earlier PV before it is rescaled; this warp
          // rescales its half of the columns.
          if (j >= 1 && !mbar_wait(&M.o_done, (uint32_t)(j - 1) & 1u, abort)) ok = false;
          if (__any_sync(0xffffffffu, !ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float f = need ? ex2(m_old - mxs) : 1.0f;
          const uint32_t o_addr = lane_base + (X == 0 ? C::COL_OA : C::COL_OD) + q * (HD / 2);
#pragma unroll 1
          for (int c0 = 0; c0 < HD / 2; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(o_addr + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * f);
            tmem_st32(o_addr + c0, r);
          }
          tmem_wait_st();
          if (need) {
            l[X] *= f;
            m2[X] = mxs;
          }
        }
        if (m2[X] == kNegInf) m2[X] = mxs;
      }
      if (!ok) break;
      // Weights: one exponential per key against its group's set max; each
      // group's packed weights go to its set's region, zeros to the other.
      {
        const float nA = m2[0] == kNegInf ? 0.f : -m2[0];
        const float nD = m2[1] == kNegInf ? 0.f : -m2[1];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t pa[16], pd[16];
#pragma unroll
          for (int gg = 0; gg < 2; ++gg) {
            const int g = 2 * hh + gg;
            const float ng = gA[g] ? nA : nD;
            float sg0 = 0.f, sg1 = 0.f;
#pragma unroll
            for (int c = 0; c < 16; c += 2) {
              const float e0 = ex2(fmaf(x[16 * g + c], p.c, ng));
              const float e1 = ex2(fmaf(x[16 * g + c + 1], p.c, ng));
              sg0 += e0;
              sg1 += e1;
              const uint32_t pk = pack_bf16(e0, e1);
              pa[8 * gg + c / 2] = gA[g] ? pk : 0u;
              pd[8 * gg + c / 2] = gA[g] ? 0u : pk;
            }
            const float sg = sg0 + sg1;
            l[0] += gA[g] ? sg : 0.f;
            l[1] += gA[g] ? 0.f : sg;
          }
          if (WITH_V && anyA) tmem_st16(s_addr + 32 * q + 16 * hh, pa);
          if (WITH_V && anyD) tmem_st16(s_addr + 64 + 32 * q + 16 * hh, pd);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&M.p_full[sb]);
    }

    // ================================================================ epilogue
    // Add the partner's partial sums (same running maxima in both warps).
    M.lsum[q][0][row] = l[0];
    M.lsum[q][1][row] = l[1];
    if (ok && !pair_sync(&M.pair[quarter], pair_uses, lane, abort)) ok = false;
    if (ok && !WITH_V && q == 0 && valid) {
      const float lA = l[0] + M.lsum[1][0][row], lD = l[1] + M.lsum[1][1][row];
      const int64_t o = ((int64_t)b * p.Hq + h) * p.N + t;
      if (direct) {
        p.delta[o] = lD;
      } else {
        const float lse2_a = (lA > 0.f) ? m2[0] + log2f(lA) : kNegInf;
        const float lse2_d = (lD > 0.f) ? m2[1] + log2f(lD) : kNegInf;
        const float hi = fmaxf(lse2_a, lse2_d), lo = fminf(lse2_a, lse2_d);
        const float lse2_f = (lo == kNegInf) ? hi : hi + log2f(1.0f + ex2(lo - hi));
        p.delta[o] = (lD > 0.f) ? ex2(lse2_d - lse2_f) : 0.f;
      }
    }
    if (WITH_V && ok && mbar_wait(&M.o_final, 0, abort)) {
      tc_fence_after();
      const float lA = l[0] + M.lsum[q ^ 1][0][row], lD = l[1] + M.lsum[q ^ 1][1][row];
      const float mA = m2[0], mD = m2[1];
      const float Mx = fmaxf(mA, mD);
      const float wa = (lA > 0.f) ? ex2(mA - Mx) : 0.f;
      const float wd = (lD > 0.f) ? ex2(mD - Mx) : 0.f;
      const float inv_full = 1.0f / (wa * lA + wd * lD);
      const float inv_sel = (lA > 0.f) ? 1.0f / lA : 0.f;
      __nv_bfloat16* hf = valid ? row_ptr_w<__nv_bfloat16>(p.hf, b, h, t) : nullptr;
      __nv_bfloat16* hs = valid ? row_ptr_w<__nv_bfloat16>(p.hs, b, h, t) : nullptr;
#pragma unroll 1
      for (int c0 = q * (HD / 2); c0 < (q + 1) * (HD / 2); c0 += 32) {
        uint32_t ra[32], rd[32];
        tmem_ld32(lane_base + C::COL_OA + c0, ra);
        tmem_ld32(lane_base + C::COL_OD + c0, rd);
        tmem_wait_ld();
        if (valid) {
          uint32_t of[16], os[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float a0 = (lA > 0.f) ? __uint_as_float(ra[c]) : 0.f;
            const float a1 = (lA > 0.f) ? __uint_as_float(ra[c + 1]) : 0.f;
            const float d0 = (lD > 0.f) ? __uint_as_float(rd[c]) : 0.f;
            const float d1 = (lD > 0.f) ? __uint_as_float(rd[c + 1]) : 0.f;
            os[c / 2] = pack_bf16(a0 * inv_sel, a1 * inv_sel);
            of[c / 2] = pack_bf16((wa * a0 + wd * d0) * inv_full, (wa * a1 + wd * d1) * inv_full);
          }
          uint4* dst_s = reinterpret_cast<uint4*>(hs + c0);
          uint4* dst_f = reinterpret_cast<uint4*>(hf + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            dst_s[v] = make_uint4(os[4 * v], os[4 * v + 1], os[4 * v + 2], os[4 * v + 3]);
            dst_f[v] = make_uint4(of[4 * v], of[4 * v + 1], of[4 * v + 2], of[4 * v + 3]);
          }
        }
      }
      if (valid && q == 0) {
        constexpr float kLn2 = 0.6931471805599453f;
        const float lse2_a = (lA > 0.f) ? mA + log2f(lA) : kNegInf;
        const float lse2_d = (lD > 0.f) ? mD + log2f(lD) : kNegInf;
        const float hi = fmaxf(lse2_a, lse2_d), lo = fminf(lse2_a, lse2_d);
        const float lse2_f = (lo == kNegInf) ? hi : hi + log2f(1.0f + ex2(lo - hi));
        const int64_t o = ((int64_t)b * p.Hq + h) * p.N + t;
        p.lse_sel[o] = (lA > 0.f) ? lse2_a * kLn2 : kNegInf;
        p.lse_full[o] = lse2_f * kLn2;
        p.delta[o] = (lD > 0.f) ? ex2(lse2_d - lse2_f) : 0.f;
      }
    }
  }

  // ---- tear-down
  tc_fence_before();
  __syncthreads();
  if (M.abort && threadIdx.x == 0) atomicCAS(p.status, 0, (int)SSA_ERR_TIMEOUT);
  if (warp == WARP_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int HD, bool WITH_V>
cudaError_t launch_hd(const Dims& D, const FwdArgs& a, int32_t* status, cudaStream_t st) {
  using C = Cfg<HD>;
  CUtensorMap mq, mk, mv;
  if (!make_tma_map_bf16(&mq, a.q, D.B, D.Hq, D.N, BM, HD) || !make_tma_map_bf16(&mk, a.k, D.B, D.Hkv, D.N, BN, HD) ||
      !make_tma_map_bf16(&mv, a.v, D.B, D.Hkv, D.N, BN, HD))
    return cudaErrorInvalidValue;
  TcmParams p;
  p.hf = a.hf;
  p.hs = a.hs;
  p.idx = a.idx;
  p.lse_full = a.lse_full;
  p.lse_sel = a.lse_sel;
  p.delta = a.delta;
  p.lse_in = WITH_V ? nullptr : a.lse_in;
  p.status = status;
  p.Hq = D.Hq;
  p.g = D.g;
  p.N = D.N;
  p.n = D.n;
  p.k = D.k;
  p.ls = __builtin_ctz((unsigned)D.s);
  p.per_token = D.per_token;
  p.c = D.scale * 1.4426950408889634f;
  const int smem = C::OFF_MISC + (int)sizeof(Misc<C::NS>) + tcm_sel_rows(D.per_token, p.ls) * 64 * 4 + 1024;
  auto kern = fwd_tcm_kernel<HD, WITH_V>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((D.N + BM - 1) / BM, D.Hq, D.B);
  kern<<<grid, NTHREADS, smem, st>>>(mq, mk, mv, p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

bool fwd_tcm_supported(const Dims& D) {
  return D.dtype == SSA_BF16 && (D.d == 64 || D.d == 128) && D.n <= 2048;
}

cudaError_t launch_fwd_tcm(const Dims& D, const FwdArgs& a, int32_t* dev_status, cudaStream_t st) {
  if (!fwd_tcm_supported(D) || a.sparse_only) return cudaErrorNotSupported;
  return D.d == 128 ? launch_hd<128, true>(D, a, dev_status, st) : launch_hd<64, true>(D, a, dev_status, st);
}

cudaError_t launch_dropped_tcm(const Dims& D, const FwdArgs& a, int32_t* dev_status, cudaStream_t st) {
  if (!fwd_tcm_supported(D)) return cudaErrorNotSupported;
  return D.d == 128 ? launch_hd<128, false>(D, a, dev_status, st) : launch_hd<64, false>(D, a, dev_status, st);
}

}  // namespace ssa
