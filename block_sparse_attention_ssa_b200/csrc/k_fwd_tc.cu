// Tensor-core dual-stream forward for sm_100a (bf16 in, fp32 accumulate, d = 128).
//
// What it computes is the same as the CUDA-core kernel ("SSA: Achieving
// Sparser Attention ...", "Practical Implementation of SSA"; "Technische
// Samenvatting: SSA", "1. Probleemstelling" and "Bidirectionele Uitlijning"):
// per query t two disjoint online softmaxes, over A_t (keys in selected
// blocks) and D_t (the other causal keys), merged at the end into h_sparse,
// h_full, lse_sel, lse_full and the dropped mass delta.  Every causal K/V tile
// is read once and multiplied once: each key's P goes into exactly one of the
// two output accumulators per row, so the dual stream costs the MMAs of one
// causal attention.
//
// CTA = one 128-row query tile of one (batch, query head), 320 threads:
//   warps 0-7  softmax / rescale / epilogue; warps w and w+4 share TMEM lanes
//              32(w%4)..+31, i.e. query rows 32(w%4).. of the tile, one row per
//              thread; warp w takes the tile's 64-key sub-block w/4;
//   warp 8     TMA producer (Q once, then 128-key K and V tiles, 2-stage ring);
//   warp 9     TMEM allocator and single-thread tcgen05.mma issuer.
// TMEM (512 columns): O_A [0,128), O_D [128,256), S ping-pong [256,384), [384,512).
// P (bf16, two per column) overwrites its S buffer and feeds the PV MMA from TMEM.
//
// A 128-key tile is two 64-key sub-blocks.  With block 64 each sub-block is a
// key block of its own, and each 64-row half of the query tile is a query
// block of its own, so a sub-block can be selected for one half and dropped
// for the other ("mixed"): that sub-block then gets a second P region in which
// only the dropped half's rows are non-zero, and the MMA warp issues one PV
// per accumulator for it.  Every (half, sub-block) pair is in one of three
// states: no causal key, selected (A) or dropped (D).
//
// Softmax in base 2 with the scale folded in: p = 2^(S*c - m), c = scale*log2(e).
// The two warps of a row trade their sub-block maxima through shared memory,
// so both hold the same running max per set; each keeps its own partial row
// sum, and the partials are added at the end.  A row's running max m of each
// set is raised only when a tile's max for that set exceeds it by more than 8
// (p stays below 2^8); O and l are then rescaled in place (each warp of the
// pair rescales half of the columns) after the previous PV has completed.
#include "ssa_internal.cuh"
#include "sm100_ptx.cuh"

#include <cudaTypedefs.h>

namespace ssa {
namespace {

using namespace sm100;

constexpr int BM = 128;    // query rows per CTA
constexpr int BN = 128;    // keys per tile
constexpr int SUB = 64;    // keys per sub-block
constexpr int HD = 128;
constexpr int NTHREADS = 320;
constexpr int WARP_TMA = 8, WARP_MMA = 9;
constexpr int NS = 2;      // K/V stages
constexpr float kRescaleThreshold = 8.0f;

constexpr int Q_BYTES = BM * HD * 2;
constexpr int KV_BYTES = BN * HD * 2;  // one K or V tile
constexpr int OFF_Q = 0;
constexpr int OFF_K = Q_BYTES;
constexpr int OFF_V = OFF_K + NS * KV_BYTES;
constexpr int OFF_MISC = OFF_V + NS * KV_BYTES;
constexpr uint32_t COL_OA = 0, COL_OD = 128, COL_S = 256;
constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, false, true);

struct Misc {
  uint64_t q_full;
  uint64_t k_full[NS], k_empty[NS], v_full[NS], v_empty[NS];
  uint64_t s_full[2], p_full[2];
  uint64_t o_done, o_final, drain;
  uint64_t pair[4];     // warps w and w+4 (one per lane quarter)
  uint32_t tmem_base;
  int abort;
  uint32_t sel[2][64];  // selected-block bits of the tile's two query blocks
  int nlist;            // sparse-only mode: selected key blocks of either half,
  uint16_t list[2048];  // ascending
  float xmax[2][2][128];  // [tile parity][sub-block][row]: scaled tile max of its set
  float lsum[2][2][128];  // epilogue: per sub-block warp, per set, per row
};
constexpr int SMEM_BYTES = OFF_MISC + (int)sizeof(Misc) + 1024;  // + alignment slack

struct TcParams {
  TensorRef hf, hs;
  const int32_t* idx;
  float* lse_full;
  float* lse_sel;
  float* delta;
  int32_t* status;
  int Hq, g, N, n, k;
  float c;  // scale * log2(e)
};

// State of (query block ib, key block kb): 0 no causal key, 1 selected, 2 dropped.
__device__ __forceinline__ int pair_state(int kb, int ib, bool valid, const uint32_t* selw) {
  if (!valid || kb > ib) return 0;
  return ((selw[kb >> 5] >> (kb & 31)) & 1u) ? 1 : 2;
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

// SPARSE: the sparse stream alone (inference mode).  Only the key blocks
// that one of the tile's query blocks selected are loaded, by 64-row TMA
// boxes: with block 64 a step pairs two selected blocks (in ascending order,
// not necessarily adjacent) as its two sub-blocks, with block 128 a step is
// one selected block.  Dropped pairs count as "no key"; only O_A is used and
// only h_sparse and lse_sel are written.
template <int S_BLK, bool SPARSE>
__global__ void __launch_bounds__(NTHREADS, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Misc& M = *reinterpret_cast<Misc*>(smem + OFF_MISC);
  volatile int* abort = &M.abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = (int)(gridDim.x - 1 - blockIdx.x);  // heaviest tiles first
  const int h = blockIdx.y, b = blockIdx.z, kvh = h / p.g;
  const int q0 = qt * BM;
  const int ib0 = q0 / S_BLK, ib1 = (q0 + SUB) / S_BLK;  // query blocks of the two halves
  const bool valid1 = q0 + SUB < p.N;
  // First key of sub-block q of step j, or -1 when that sub-block is empty.
  auto sub_start = [&](int j, int q) -> int {
    if (!SPARSE) return j * BN + q * SUB;
    if (S_BLK == 128) return (int)M.list[j] * 128 + q * SUB;
    const int e = 2 * j + q;
    return e < M.nlist ? (int)M.list[e] * 64 : -1;
  };
  // State of the (query block ib, sub-block starting at u) pair.
  auto state_of = [&](int u, int ib, bool valid, const uint32_t* selw) -> int {
    if (u < 0) return 0;
    const int s = pair_state(u / S_BLK, ib, valid, selw);
    return (SPARSE && s == 2) ? 0 : s;
  };

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
  for (int w = threadIdx.x; w < 2 * 64; w += NTHREADS) (&M.sel[0][0])[w] = 0u;
  if (warp == WARP_MMA) {
    tmem_alloc(&M.tmem_base, 512);
    tmem_relinquish();
  }
  __syncthreads();
  {
    const int32_t* r0 = p.idx + (((int64_t)b * p.Hq + h) * p.n + ib0) * p.k;
    for (int e = threadIdx.x; e < p.k; e += NTHREADS) {
      const int j = r0[e];
      if (j >= 0 && j <= ib0) atomicOr(&M.sel[0][j >> 5], 1u << (j & 31));
    }
    if (ib1 != ib0 && valid1) {
      const int32_t* r1 = p.idx + (((int64_t)b * p.Hq + h) * p.n + ib1) * p.k;
      for (int e = threadIdx.x; e < p.k; e += NTHREADS) {
        const int j = r1[e];
        if (j >= 0 && j <= ib1) atomicOr(&M.sel[1][j >> 5], 1u << (j & 31));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (SPARSE) {
    // Ascending list of the blocks either half selected (bit sets of the
    // halves: M.sel[1] is zero when both halves are one query block).
    if (warp == 0) {
      const uint32_t w0 = M.sel[0][2 * lane] | M.sel[1][2 * lane];
      const uint32_t w1 = M.sel[0][2 * lane + 1] | M.sel[1][2 * lane + 1];
      const int c = __popc(w0) + __popc(w1);
      int incl = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      int pos = incl - c;
      for (uint32_t x = w0; x; x &= x - 1) M.list[pos++] = (uint16_t)(64 * lane + __ffs(x) - 1);
      for (uint32_t x = w1; x; x &= x - 1) M.list[pos++] = (uint16_t)(64 * lane + 32 + __ffs(x) - 1);
      if (lane == 31) M.nlist = incl;
    }
    __syncthreads();
  }
  const int T = !SPARSE ? (min(q0 + BM, p.N) + BN - 1) / BN                 // causal key tiles
                        : (S_BLK == 128 ? M.nlist : (M.nlist + 1) / 2);  // selected blocks
  const uint32_t tmem = M.tmem_base;
  const uint32_t* sel0 = M.sel[0];
  const uint32_t* sel1 = (ib1 != ib0) ? M.sel[1] : M.sel[0];

  uint8_t* sQ = smem + OFF_Q;
  uint8_t* sK = smem + OFF_K;
  uint8_t* sV = smem + OFF_V;

  if (warp == WARP_TMA) {
    // ================================================================ producer
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      mbar_expect_tx(&M.q_full, Q_BYTES);
      tma_load_4d(sQ, &tmQ, &M.q_full, 0, q0, h, b);
      tma_load_4d(sQ + Q_BYTES / 2, &tmQ, &M.q_full, 64, q0, h, b);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < T; ++j) {
        const int st = j % NS;
        const uint32_t use = (uint32_t)(j / NS);
        // Dual mode: one 128-row box per column half.  Sparse mode: one
        // 64-row box per non-empty sub-block and column half, placed at the
        // sub-block's rows (the 128-byte swizzle repeats every 8 rows, so
        // the layout equals that of a 128-row box).
        const int ua = sub_start(j, 0), ub = SPARSE ? sub_start(j, 1) : -1;
        const uint32_t bytes = !SPARSE ? KV_BYTES : (ub >= 0 ? KV_BYTES : KV_BYTES / 2);
        auto load_tile = [&](uint8_t* dst, const CUtensorMap* map, uint64_t* bar) {
          mbar_expect_tx(bar, bytes);
          tma_load_4d(dst, map, bar, 0, ua, kvh, b);
          tma_load_4d(dst + KV_BYTES / 2, map, bar, 64, ua, kvh, b);
          if (ub >= 0) {
            tma_load_4d(dst + SUB * 128, map, bar, 0, ub, kvh, b);
            tma_load_4d(dst + KV_BYTES / 2 + SUB * 128, map, bar, 64, ub, kvh, b);
          }
        };
        if (j >= NS && !mbar_wait(&M.k_empty[st], (use - 1) & 1u, abort)) break;
        load_tile(sK + st * KV_BYTES, &tmK, &M.k_full[st]);
        k_issued = j + 1;
        if (j >= NS && !mbar_wait(&M.v_empty[st], (use - 1) & 1u, abort)) break;
        load_tile(sV + st * KV_BYTES, &tmV, &M.v_full[st]);
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
        const int st = jj % NS;
        if (!mbar_wait(&M.v_full[st], (uint32_t)(jj / NS) & 1u, abort)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sV + st * KV_BYTES);
        const uint32_t s_col = COL_S + (uint32_t)sb * BN;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int u = sub_start(jj, q);
          const int s0 = state_of(u, ib0, true, sel0);
          const int s1 = state_of(u, ib1, valid1, sel1);
          if (s0 == 0 && s1 == 0) continue;
          const bool mixed = (s0 != 0 && s1 != 0 && s0 != s1);
          const int target = s0 != 0 ? s0 : s1;
          auto pv = [&](uint32_t o_col, uint32_t pcol, bool& started) {
#pragma unroll
            for (int kk = 0; kk < SUB / 16; ++kk) {
              const uint64_t bdesc = smem_desc_sw128(v_addr + (q * SUB + kk * 16) * 128, KV_BYTES / 2, 1024);
              mma_ts(tmem + o_col, tmem + pcol + kk * 8, bdesc, IDESC_PV, (started || kk > 0) ? 1u : 0u);
            }
            started = true;
          };
          const uint32_t p0 = s_col + 32 * q, p1 = s_col + 64 + 32 * q;
          if (mixed) {
            pv(COL_OA, p0, started_a);
            pv(COL_OD, p1, started_d);
          } else if (target == 1) {
            pv(COL_OA, p0, started_a);
          } else {
            pv(COL_OD, p0, started_d);
          }
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
        const uint32_t k_addr = smem_u32(sK + st * KV_BYTES);
        const uint32_t s_col = COL_S + (uint32_t)(j & 1) * BN;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off_q = (kk >> 2) * (Q_BYTES / 2) + (kk & 3) * 32;
          const uint32_t off_k = (kk >> 2) * (KV_BYTES / 2) + (kk & 3) * 32;
          mma_ss(tmem + s_col, smem_desc_sw128(q_addr + off_q, 16, 1024), smem_desc_sw128(k_addr + off_k, 16, 1024),
                 IDESC_QK, kk > 0 ? 1u : 0u);
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
    const int half = quarter >> 1;
    const int ib = half ? ib1 : ib0;
    const bool hvalid = half ? valid1 : true;
    const uint32_t* selw = half ? sel1 : sel0;
    const int row = quarter * 32 + lane;  // row within the tile == TMEM lane
    const int t = q0 + row;               // query token
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    float m2[2] = {kNegInf, kNegInf};  // running max (scaled, base 2), [0]=A [1]=D
    float l[2] = {0.f, 0.f};           // this warp's partial sums
    uint32_t pair_uses = 0;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int sb = j & 1;
      if (!mbar_wait(&M.s_full[sb], (uint32_t)(j >> 1) & 1u, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      int st[2];  // this row's state of sub-blocks 0 and 1
      bool mixed_q;
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) st[qq] = state_of(sub_start(j, qq), ib, hvalid, selw);
      const int u0 = sub_start(j, q);  // first key of this warp's sub-block
      {
        const int o0 = state_of(u0, ib0, true, sel0);
        const int o1 = state_of(u0, ib1, valid1, sel1);
        mixed_q = (o0 != 0 && o1 != 0 && o0 != o1);
      }
      const int mine = st[q];
      const uint32_t s_addr = lane_base + COL_S + (uint32_t)sb * BN;
      float x[SUB];  // raw S of this warp's sub-block; the scale is folded into the exponent
      float mx = kNegInf;
      if (mine != 0) {
#pragma unroll
        for (int c0 = 0; c0 < SUB; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(s_addr + q * SUB + c0, r);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c0 + c] = __uint_as_float(r[c]);
        }
        if (u0 + SUB - 1 > t) {  // causal mask inside the diagonal sub-block
#pragma unroll
          for (int c = 0; c < SUB; ++c)
            if (u0 + c > t) x[c] = kNegInf;
        }
        float a0 = kNegInf, a1 = kNegInf, a2 = kNegInf, a3 = kNegInf;
#pragma unroll
        for (int c = 0; c < SUB; c += 4) {
          a0 = fmaxf(a0, x[c]);
          a1 = fmaxf(a1, x[c + 1]);
          a2 = fmaxf(a2, x[c + 2]);
          a3 = fmaxf(a3, x[c + 3]);
        }
        mx = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)) * p.c;  // scale > 0
      }
      // Trade sub-block maxima with the partner warp; after this point both
      // warps have read their S columns, so P may overwrite them.
      M.xmax[sb][q][row] = mx;
      if (!pair_sync(&M.pair[quarter], pair_uses, lane, abort)) {
        ok = false;
        break;
      }
      const float mx_other = M.xmax[sb][q ^ 1][row];
      const int st_other = st[q ^ 1];
#pragma unroll
      for (int X = 0; X < 2; ++X) {
        float mxs = kNegInf;
        if (mine == X + 1) mxs = mx;
        if (st_other == X + 1) mxs = fmaxf(mxs, mx_other);
        const float m_old = m2[X];
        const bool need = (m_old != kNegInf) && (mxs > m_old + kRescaleThreshold);
        if (__any_sync(0xffffffffu, need)) {
          // O_X must hold every earlier PV before it is rescaled; this warp
          // rescales its half of the columns.
          if (j >= 1 && !mbar_wait(&M.o_done, (uint32_t)(j - 1) & 1u, abort)) ok = false;
          if (__any_sync(0xffffffffu, !ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float f = need ? ex2(m_old - mxs) : 1.0f;
          const uint32_t o_addr = lane_base + (X == 0 ? COL_OA : COL_OD) + q * (HD / 2);
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
      uint32_t pk[SUB / 2];
      if (mine == 0) {
#pragma unroll
        for (int c = 0; c < SUB / 2; ++c) pk[c] = 0u;
      } else {
        const float nm = -m2[mine - 1];
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int c = 0; c < SUB; c += 2) {
          const float e0 = ex2(fmaf(x[c], p.c, nm));
          const float e1 = ex2(fmaf(x[c + 1], p.c, nm));
          s0 += e0;
          s1 += e1;
          pk[c / 2] = pack_bf16(e0, e1);
        }
        l[mine - 1] += s0 + s1;
      }
      // Sub-block q's P at columns [32q, 32q+32) of the S buffer; for a mixed
      // sub-block the dropped half's rows use [64+32q, 64+32q+32) instead and
      // write zeros to the first.
      const uint32_t p0 = s_addr + 32 * q, p1 = s_addr + 64 + 32 * q;
      const uint32_t(&blk)[32] = *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]);
      if (mixed_q) {
        uint32_t z[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) z[c] = 0u;
        if (mine == 1) {
          tmem_st32(p0, blk);
          tmem_st32(p1, z);
        } else {
          tmem_st32(p0, z);
          tmem_st32(p1, blk);
        }
      } else {
        tmem_st32(p0, blk);
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
    if (ok && mbar_wait(&M.o_final, 0, abort)) {
      tc_fence_after();
      const float lA = l[0] + M.lsum[q ^ 1][0][row], lD = l[1] + M.lsum[q ^ 1][1][row];
      const bool store = t < p.N;
      const float mA = m2[0], mD = m2[1];
      const float Mx = fmaxf(mA, mD);
      const float wa = (lA > 0.f) ? ex2(mA - Mx) : 0.f;
      const float wd = (lD > 0.f) ? ex2(mD - Mx) : 0.f;
      const float inv_full = 1.0f / (wa * lA + wd * lD);
      const float inv_sel = (lA > 0.f) ? 1.0f / lA : 0.f;
      __nv_bfloat16* hf = (store && !SPARSE) ? row_ptr_w<__nv_bfloat16>(p.hf, b, h, t) : nullptr;
      __nv_bfloat16* hs = store ? row_ptr_w<__nv_bfloat16>(p.hs, b, h, t) : nullptr;
#pragma unroll 1
      for (int c0 = q * (HD / 2); c0 < (q + 1) * (HD / 2); c0 += 32) {
        uint32_t ra[32], rd[32];
        tmem_ld32(lane_base + COL_OA + c0, ra);
        if (!SPARSE) tmem_ld32(lane_base + COL_OD + c0, rd);
        tmem_wait_ld();
        if (store) {
          uint32_t of[16], os[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float a0 = (lA > 0.f) ? __uint_as_float(ra[c]) : 0.f;
            const float a1 = (lA > 0.f) ? __uint_as_float(ra[c + 1]) : 0.f;
            os[c / 2] = pack_bf16(a0 * inv_sel, a1 * inv_sel);
            if (!SPARSE) {
              const float d0 = (lD > 0.f) ? __uint_as_float(rd[c]) : 0.f;
              const float d1 = (lD > 0.f) ? __uint_as_float(rd[c + 1]) : 0.f;
              of[c / 2] = pack_bf16((wa * a0 + wd * d0) * inv_full, (wa * a1 + wd * d1) * inv_full);
            }
          }
          uint4* dst_s = reinterpret_cast<uint4*>(hs + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst_s[v] = make_uint4(os[4 * v], os[4 * v + 1], os[4 * v + 2], os[4 * v + 3]);
          if (!SPARSE) {
            uint4* dst_f = reinterpret_cast<uint4*>(hf + c0);
#pragma unroll
            for (int v = 0; v < 4; ++v) dst_f[v] = make_uint4(of[4 * v], of[4 * v + 1], of[4 * v + 2], of[4 * v + 3]);
          }
        }
      }
      if (store && q == 0) {
        constexpr float kLn2 = 0.6931471805599453f;
        const float lse2_a = (lA > 0.f) ? mA + log2f(lA) : kNegInf;
        const float lse2_d = (lD > 0.f) ? mD + log2f(lD) : kNegInf;
        const float hi = fmaxf(lse2_a, lse2_d), lo = fminf(lse2_a, lse2_d);
        const float lse2_f = (lo == kNegInf) ? hi : hi + log2f(1.0f + ex2(lo - hi));
        const int64_t o = ((int64_t)b * p.Hq + h) * p.N + t;
        p.lse_sel[o] = (lA > 0.f) ? lse2_a * kLn2 : kNegInf;
        if (!SPARSE) {
          p.lse_full[o] = lse2_f * kLn2;
          p.delta[o] = (lD > 0.f) ? ex2(lse2_d - lse2_f) : 0.f;
        }
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

template <int S_BLK, bool SPARSE>
cudaError_t launch_blk(const Dims& D, const FwdArgs& a, int32_t* status, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  const int kv_rows = SPARSE ? SUB : BN;  // sparse mode loads 64-key sub-blocks
  if (!make_tma_map_bf16(&mq, a.q, D.B, D.Hq, D.N, BM) || !make_tma_map_bf16(&mk, a.k, D.B, D.Hkv, D.N, kv_rows) ||
      !make_tma_map_bf16(&mv, a.v, D.B, D.Hkv, D.N, kv_rows))
    return cudaErrorInvalidValue;
  TcParams p;
  p.hf = a.hf;
  p.hs = a.hs;
  p.idx = a.idx;
  p.lse_full = a.lse_full;
  p.lse_sel = a.lse_sel;
  p.delta = a.delta;
  p.status = status;
  p.Hq = D.Hq;
  p.g = D.g;
  p.N = D.N;
  p.n = D.n;
  p.k = D.k;
  p.c = D.scale * 1.4426950408889634f;
  auto kern = fwd_tc_kernel<S_BLK, SPARSE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((D.N + BM - 1) / BM, D.Hq, D.B);
  kern<<<grid, NTHREADS, SMEM_BYTES, st>>>(mq, mk, mv, p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 4-D map over a [B, H, N, d] bf16 tensor: dims (d, N, H, B), box (64, rows, 1, 1).
bool make_tma_map_bf16(CUtensorMap* map, const TensorRef& t, int B, int H, int N, int rows, int d) {
  auto enc = get_encode();
  if (enc == nullptr || (d != 64 && d != 128)) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)t.sn * 2, (cuuint64_t)t.sh * 2, (cuuint64_t)t.sb * 2};
  // A zero stride (a broadcast dimension of size 1) is not accepted; any
  // positive multiple of 16 describes the same single slice.
  for (int i = 0; i < 3; ++i)
    if (strides[i] == 0) strides[i] = 16;
  cuuint32_t box[4] = {64, (cuuint32_t)rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(t.p), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool fwd_tc_supported(const Dims& D) {
  return D.dtype == SSA_BF16 && D.d == 128 && (D.s == 64 || D.s == 128) && D.n <= 2048 && !D.per_token;
}

cudaError_t launch_fwd_tc(const Dims& D, const FwdArgs& a, int32_t* dev_status, cudaStream_t st) {
  if (!fwd_tc_supported(D)) return cudaErrorNotSupported;
  if (a.sparse_only)
    return D.s == 64 ? launch_blk<64, true>(D, a, dev_status, st) : launch_blk<128, true>(D, a, dev_status, st);
  return D.s == 64 ? launch_blk<64, false>(D, a, dev_status, st) : launch_blk<128, false>(D, a, dev_status, st);
}

}  // namespace ssa
