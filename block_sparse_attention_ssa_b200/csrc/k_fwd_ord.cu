// Tensor-core dual-stream forward for sm_100a, selected blocks first
// (bf16 in, fp32 accumulate, d = 128, blocks of 64 or 128, per-block selection).
//
// What it computes ("SSA: Achieving Sparser Attention ...", "Practical
// Implementation of SSA"; "Technische Samenvatting: SSA", "1. Probleemstelling"
// and "Bidirectionele Uitlijning"): for each query t, h_sparse = softmax over
// A_t (keys in the selected blocks) applied to V, h_full = causal softmax over
// all keys u <= t applied to V, the dropped mass delta = full-softmax weight on
// D_t, and both log-sum-exps.
//
// Order of the key walk.  A query tile first visits the key blocks its query
// blocks selected (phase A), then the causal blocks they dropped (phase D),
// with ONE online softmax and ONE output accumulator.  After phase A the
// accumulator and the row statistics are exactly the sparse stream's, so
// h_sparse and lse_sel are read off at the phase boundary; phase D continues
// the same softmax over the rest of the causal keys, which ends as the full
// stream.  delta is the phase-D share of the final row sum (kept separately,
// so small masses keep their relative precision).  Every causal K/V tile is
// still multiplied once, as in one causal attention, and a query tile needs
// only 256 TMEM columns (O 128 + two 64-column S buffers), so two CTAs share
// an SM: while one CTA's softmax warps work, the tensor core runs its own next
// logits and the other CTA's products.
//
// With block 64 a 128-row query tile holds two query blocks whose selections
// differ: phase A walks the union of the two selections and phase D the blocks
// that either half dropped; a 64-key unit that belongs to the other phase for
// one half is masked for that half's rows (P = 0).  A step is one 64-key unit
// (a block of 64, or half of a block of 128), loaded by 64-row TMA boxes into
// two-slot K and V rings.
//
// CTA = one 128-row query tile of one (batch, query head), 192 threads:
//   warps 0-3  softmax, rescale, snapshot and epilogue: warp w owns TMEM lanes
//              32w..32w+31 = query rows 32w.. of the tile, one row per thread,
//              the 64 key columns of a step;
//   warp 4     TMA producer (Q once, then K and V of each step, two slots each);
//   warp 5     TMEM allocator and single-thread tcgen05.mma issuer.
// TMEM (256 columns): O [0,128), two S buffers [128,192) and [192,256); step
// j uses buffer j & 1.  P (bf16, two per column) overwrites the first 32
// columns of its S buffer and feeds the PV product from TMEM.  The products
// of step j + 2 are issued right after PV of step j, so the tensor core forms
// the next step's logits while the softmax warps work on this one's.  The
// tensor core runs one CTA's products in issue order: S of step j + 2 reuses
// the columns PV of step j read.  O is touched by the softmax warps only for a
// rescale or a snapshot, after the preceding PV has completed.
//
// Softmax in base 2 with the scale folded in: p = 2^(S*c - m), c = scale*log2(e).
// A row's running max m is raised only when a step's max exceeds it by more
// than 8 (p stays below 2^8); O and the row sums are then rescaled in place.
#include "ssa_internal.cuh"
#include "sm100_ptx.cuh"

namespace ssa {
namespace {

using namespace sm100;

constexpr int BM = 128;    // query rows per CTA
constexpr int UNIT = 64;   // keys per step (a TMA box of 64 rows)
constexpr int HD = 128;
constexpr int NTHREADS = 192;
constexpr int WARP_TMA = 4, WARP_MMA = 5;
constexpr float kRescaleThreshold = 8.0f;
constexpr int MAX_LIST = 4096;  // phase-A plus phase-D entries (<= 2 n, n <= 2048)

constexpr int Q_BYTES = BM * HD * 2;
constexpr int KV_BYTES = UNIT * HD * 2;  // one K or V tile of a step
constexpr int KV_HALF = UNIT * 128;      // its 64-column half (64 rows x 128 B)
constexpr int OFF_Q = 0;
constexpr int OFF_K = Q_BYTES;               // two K slots
constexpr int OFF_V = OFF_K + 2 * KV_BYTES;  // two V slots
constexpr int OFF_MISC = OFF_V + 2 * KV_BYTES;
constexpr uint32_t COL_O = 0, COL_S = 128;  // S buffers at COL_S and COL_S + 64
constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, UNIT, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, false, true);

struct Misc {
  // one barrier per S buffer where the waiter could otherwise fall two phases behind
  uint64_t q_full, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2], p_full[2], pv_done, o_final, drain;
  uint32_t tmem_base;
  int abort;
  int nA, nD;             // entries of the two phases in list[]
  uint32_t sel[2][64];    // selected-block bits of the tile's two query blocks
  uint16_t list[MAX_LIST];  // phase A entries (ascending), then phase D entries
};
constexpr int SMEM_BYTES = OFF_MISC + (int)sizeof(Misc) + 1024;  // + alignment slack
static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");

struct OrdParams {
  TensorRef hf, hs;
  const int32_t* idx;
  float* lse_full;
  float* lse_sel;
  float* delta;
  int32_t* status;
  int Hq, g, N, n, k;
  float c;  // scale * log2(e)
};

// SPARSE: the sparse stream alone (inference mode): phase A only; h_full,
// lse_full and delta are not written.
template <int S_BLK, bool SPARSE>
__global__ void __launch_bounds__(NTHREADS, 2)
    fwd_ord_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, OrdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Misc& M = *reinterpret_cast<Misc*>(smem + OFF_MISC);
  volatile int* abort = &M.abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = (int)(gridDim.x - 1 - blockIdx.x);  // heaviest tiles first
  const int h = blockIdx.y, b = blockIdx.z, kvh = h / p.g;
  const int q0 = qt * BM;
  const int ib0 = q0 / S_BLK, ib1 = (q0 + UNIT) / S_BLK;  // query blocks of the two 64-row halves
  const bool valid1 = q0 + UNIT < p.N;

  // ---- set-up
  if (threadIdx.x == 0) {
    mbar_init(&M.q_full, 1);
    for (int s2 = 0; s2 < 2; ++s2) {
      mbar_init(&M.k_full[s2], 1);
      mbar_init(&M.k_empty[s2], 1);
      mbar_init(&M.v_full[s2], 1);
      mbar_init(&M.v_empty[s2], 1);
      mbar_init(&M.s_full[s2], 1);
      mbar_init(&M.p_full[s2], 4);
    }
    mbar_init(&M.pv_done, 1);
    mbar_init(&M.o_final, 1);
    mbar_init(&M.drain, 1);
    M.abort = 0;
    fence_mbar_init();
  }
  for (int w = threadIdx.x; w < 2 * 64; w += NTHREADS) (&M.sel[0][0])[w] = 0u;
  if (warp == WARP_MMA) {
    tmem_alloc(&M.tmem_base, 256);
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
  __syncthreads();
  // Phase lists (warp 0): A = blocks some half selected, D = causal blocks
  // some half did not select, each ascending.  With one query block per tile
  // (block 128) sel[1] stays zero and half 1 uses sel[0].
  const bool two = (ib1 != ib0);
  if (warp == 0) {
    uint32_t a[2], dd[2];
    int c = 0;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int wd = 2 * lane + e;
      auto causal_word = [&](int ib) -> uint32_t {  // bits j <= ib of word wd
        const int lo = wd * 32;
        if (ib < lo) return 0u;
        if (ib >= lo + 31) return 0xffffffffu;
        return (2u << (ib - lo)) - 1u;
      };
      const uint32_t s0 = M.sel[0][wd], s1 = two ? M.sel[1][wd] : s0;
      const uint32_t c0 = causal_word(ib0), c1 = (two && valid1) ? causal_word(ib1) : 0u;
      a[e] = s0 | (two ? s1 : 0u);
      dd[e] = SPARSE ? 0u : ((c0 & ~s0) | (c1 & ~s1));
      c += __popc(a[e]);
    }
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    const int nA = __shfl_sync(0xffffffffu, incl, 31);
    int pos = incl - c;
#pragma unroll
    for (int e = 0; e < 2; ++e)
      for (uint32_t x = a[e]; x; x &= x - 1) M.list[pos++] = (uint16_t)(64 * lane + 32 * e + __ffs(x) - 1);
    const int cd = __popc(dd[0]) + __popc(dd[1]);
    int incd = cd;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incd, off);
      if (lane >= off) incd += y;
    }
    pos = nA + incd - cd;
#pragma unroll
    for (int e = 0; e < 2; ++e)
      for (uint32_t x = dd[e]; x; x &= x - 1) M.list[pos++] = (uint16_t)(64 * lane + 32 * e + __ffs(x) - 1);
    if (lane == 31) {
      M.nA = nA;
      M.nD = incd;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int nA = M.nA, nD = M.nD;
  // Steps: one 64-key unit each (a list entry at block 64, half of one at 128).
  constexpr int UPB = S_BLK / UNIT;  // units per block
  const int TA = UPB * nA, TD = UPB * nD;
  const int T = TA + TD;
  const uint32_t tmem = M.tmem_base;

  // The unit of step j: its first key and its block.
  auto unit_of = [&](int j, int& u0, int& blk) {
    const int jj = j < TA ? j : j - TA;
    blk = M.list[(j < TA ? 0 : nA) + jj / UPB];
    u0 = blk * S_BLK + (jj % UPB) * UNIT;
  };

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
        const int sl = j & 1;
        int u0, blk;
        unit_of(j, u0, blk);
        // the slot's previous tile (step j - 2) must have been consumed
        if (j >= 2 && !mbar_wait(&M.k_empty[sl], (uint32_t)((j - 2) >> 1) & 1u, abort)) break;
        mbar_expect_tx(&M.k_full[sl], KV_BYTES);
        tma_load_4d(sK + sl * KV_BYTES, &tmK, &M.k_full[sl], 0, u0, kvh, b);
        tma_load_4d(sK + sl * KV_BYTES + KV_HALF, &tmK, &M.k_full[sl], 64, u0, kvh, b);
        k_issued = j + 1;
        if (j >= 2 && !mbar_wait(&M.v_empty[sl], (uint32_t)((j - 2) >> 1) & 1u, abort)) break;
        mbar_expect_tx(&M.v_full[sl], KV_BYTES);
        tma_load_4d(sV + sl * KV_BYTES, &tmV, &M.v_full[sl], 0, u0, kvh, b);
        tma_load_4d(sV + sl * KV_BYTES + KV_HALF, &tmV, &M.v_full[sl], 64, u0, kvh, b);
        v_issued = j + 1;
      }
      // Drain: every copy this thread issued must have landed before the CTA exits.
      int dummy = 0;
      mbar_wait(&M.q_full, 0, &dummy);
      for (int j = k_issued > 2 ? k_issued - 2 : 0; j < k_issued; ++j) {
        dummy = 0;
        mbar_wait(&M.k_full[j & 1], (uint32_t)(j >> 1) & 1u, &dummy);
      }
      for (int j = v_issued > 2 ? v_issued - 2 : 0; j < v_issued; ++j) {
        dummy = 0;
        mbar_wait(&M.v_full[j & 1], (uint32_t)(j >> 1) & 1u, &dummy);
      }
    }
  } else if (warp == WARP_MMA) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      bool ok = mbar_wait(&M.q_full, 0, abort);
      // S of step j into buffer j & 1
      auto issue_s = [&](int j) {
        const int sl = j & 1;
        if (!mbar_wait(&M.k_full[sl], (uint32_t)(j >> 1) & 1u, abort)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off_q = (kk >> 2) * (Q_BYTES / 2) + (kk & 3) * 32;
          const uint32_t off_k = sl * KV_BYTES + (kk >> 2) * KV_HALF + (kk & 3) * 32;
          mma_ss(tmem + COL_S + 64 * sl, smem_desc_sw128(q_addr + off_q, 16, 1024),
                 smem_desc_sw128(k_addr + off_k, 16, 1024), IDESC_QK, kk > 0 ? 1u : 0u);
        }
        tc_commit(&M.s_full[sl]);
        tc_commit(&M.k_empty[sl]);
        return true;
      };
      if (ok && T > 0) ok = issue_s(0);
      if (ok && T > 1) ok = issue_s(1);
      for (int j = 0; ok && j < T; ++j) {
        const int sl = j & 1;
        if (!mbar_wait(&M.p_full[sl], (uint32_t)(j >> 1) & 1u, abort) ||
            !mbar_wait(&M.v_full[sl], (uint32_t)(j >> 1) & 1u, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < UNIT / 16; ++kk) {
          const uint64_t bdesc = smem_desc_sw128(v_addr + sl * KV_BYTES + kk * 16 * 128, KV_HALF, 1024);
          mma_ts(tmem + COL_O, tmem + COL_S + 64 * sl + 8 * kk, bdesc, IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&M.v_empty[sl]);
        tc_commit(&M.pv_done);
        // S of step j + 2 reuses the buffer this PV read (in issue order)
        if (j + 2 < T && !issue_s(j + 2)) {
          ok = false;
          break;
        }
      }
      tc_commit(&M.o_final);
      tc_commit(&M.drain);
      int dummy = 0;
      mbar_wait(&M.drain, 0, &dummy);
    }
  } else {
    // ================================================================ softmax
    const int row = warp * 32 + lane;     // row within the tile == TMEM lane
    const int t = q0 + row;               // query token
    const int half = row >> 6;
    const int ib = half ? ib1 : ib0;
    const bool hvalid = half ? valid1 : true;
    const uint32_t* selw = (half && two) ? M.sel[1] : M.sel[0];
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t s_base = lane_base + COL_S, o_addr = lane_base + COL_O;
    const bool store = t < p.N;
    constexpr float kLn2 = 0.6931471805599453f;
    float m = kNegInf;   // running max (scaled, base 2)
    float l = 0.f;       // row sum of every key visited so far (relative to m)
    float lD = 0.f;      // phase-D part of l
    bool ok = true;
    bool snapped = false;

    // h_sparse and lse_sel from the accumulator after phase A (O must hold
    // every phase-A product and nothing else).
    auto snapshot = [&]() {
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      __nv_bfloat16* hs = store ? row_ptr_w<__nv_bfloat16>(p.hs, b, h, t) : nullptr;
#pragma unroll 1
      for (int c0 = 0; c0 < HD; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(o_addr + c0, r);
        tmem_wait_ld();
        if (store) {
          uint32_t o[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2)
            o[c / 2] = pack_bf16(l > 0.f ? __uint_as_float(r[c]) * inv : 0.f,
                                 l > 0.f ? __uint_as_float(r[c + 1]) * inv : 0.f);
          uint4* dst = reinterpret_cast<uint4*>(hs + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
        }
      }
      if (store) {
        const int64_t o = ((int64_t)b * p.Hq + h) * p.N + t;
        p.lse_sel[o] = l > 0.f ? (m + log2f(l)) * kLn2 : kNegInf;
      }
      snapped = true;
    };

    // O is quiescent once PV of step j - 1 has completed (the only product
    // that may still be running while the softmax of step j starts).
    auto wait_prev_pv = [&](int j) {
      if (j >= 1 && !__all_sync(0xffffffffu, mbar_wait(&M.pv_done, (uint32_t)(j - 1) & 1u, abort))) ok = false;
      tc_fence_after();
    };
    for (int j = 0; j < T; ++j) {
      const bool phaseA = j < TA;
      const int sb = j & 1;
      const uint32_t s_addr = s_base + 64 * sb;
      // all lanes leave together (the TMEM accesses below are warp-wide)
      if (!__all_sync(0xffffffffu, mbar_wait(&M.s_full[sb], (uint32_t)(j >> 1) & 1u, abort))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // First phase-D step: O holds every phase-A product once the last
      // phase-A PV has completed.
      if (!phaseA && !snapped) {
        wait_prev_pv(j);
        snapshot();
      }
      // Whether this row keeps the step's unit: in phase A the blocks of its
      // own selection, in phase D the others; causal only.
      int u0, blk;
      unit_of(j, u0, blk);
      const bool causal = hvalid && blk <= ib;
      const bool insel = (selw[blk >> 5] >> (blk & 31)) & 1u;
      const bool keep = causal && (phaseA ? insel : !insel);
      // The unit's 64 raw logits stay in registers from the row max to the
      // exponentials (keys after t are masked only in a unit that reaches
      // past t).
      float xq[UNIT];
      float mx = kNegInf;
      if (keep) {
        tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&xq[0]));
        tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&xq[32]));
        tmem_wait_ld();
        const int lim = t - u0;  // keys u0 + c with c > lim are after t
        if (lim < UNIT - 1) {
#pragma unroll
          for (int c = 0; c < UNIT; ++c)
            if (c > lim) xq[c] = kNegInf;
        }
        float a0 = kNegInf, a1 = kNegInf, a2 = kNegInf, a3 = kNegInf;
#pragma unroll
        for (int c = 0; c < UNIT; c += 4) {
          a0 = fmaxf(a0, xq[c]);
          a1 = fmaxf(a1, xq[c + 1]);
          a2 = fmaxf(a2, xq[c + 2]);
          a3 = fmaxf(a3, xq[c + 3]);
        }
        mx = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
      }
      mx *= p.c;  // scale > 0
      // Raise the running max when the step's max exceeds it by more than the
      // threshold; O (after the previous PV) and the row sums are rescaled in
      // place.
      const bool need = (m != kNegInf) && (mx > m + kRescaleThreshold);
      if (__any_sync(0xffffffffu, need)) {
        wait_prev_pv(j);
        const float f = need ? ex2(m - mx) : 1.0f;
#pragma unroll 1
        for (int c0 = 0; c0 < HD; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(o_addr + c0, r);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * f);
          tmem_st32(o_addr + c0, r);
        }
        tmem_wait_st();
        if (need) {
          l *= f;
          lD *= f;
          m = mx;
        }
      }
      if (m == kNegInf) m = mx;
      const float nm = -m;
      // P (bf16 pairs) over the first 32 columns of the step's S buffer.
      uint32_t pk[32];
      float sum = 0.f;
      if (keep) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int c = 0; c < UNIT; c += 2) {
          const float e0 = ex2(fmaf(xq[c], p.c, nm));
          const float e1 = ex2(fmaf(xq[c + 1], p.c, nm));
          s0 += e0;
          s1 += e1;
          pk[c / 2] = pack_bf16(e0, e1);
        }
        sum = s0 + s1;
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      tmem_st32(s_addr, pk);
      l += sum;
      if (!phaseA) lD += sum;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&M.p_full[sb]);
    }

    // ================================================================ epilogue
    if (ok && __all_sync(0xffffffffu, mbar_wait(&M.o_final, 0, abort))) {
      tc_fence_after();
      if (!snapped) snapshot();  // no phase-D step: both streams coincide
      if (!SPARSE) {
        const float inv = l > 0.f ? 1.0f / l : 0.f;
        __nv_bfloat16* hf = store ? row_ptr_w<__nv_bfloat16>(p.hf, b, h, t) : nullptr;
#pragma unroll 1
        for (int c0 = 0; c0 < HD; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(o_addr + c0, r);
          tmem_wait_ld();
          if (store) {
            uint32_t o[16];
#pragma unroll
            for (int c = 0; c < 32; c += 2)
              o[c / 2] = pack_bf16(__uint_as_float(r[c]) * inv, __uint_as_float(r[c + 1]) * inv);
            uint4* dst = reinterpret_cast<uint4*>(hf + c0);
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
          }
        }
        if (store) {
          const int64_t o = ((int64_t)b * p.Hq + h) * p.N + t;
          p.lse_full[o] = (m + log2f(l)) * kLn2;
          p.delta[o] = lD > 0.f ? lD / l : 0.f;
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
    tmem_dealloc(tmem, 256);
  }
}

template <int S_BLK, bool SPARSE>
cudaError_t launch_ord(const Dims& D, const FwdArgs& a, int32_t* status, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_tma_map_bf16(&mq, a.q, D.B, D.Hq, D.N, BM) || !make_tma_map_bf16(&mk, a.k, D.B, D.Hkv, D.N, UNIT) ||
      !make_tma_map_bf16(&mv, a.v, D.B, D.Hkv, D.N, UNIT))
    return cudaErrorInvalidValue;
  OrdParams p;
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
  auto kern = fwd_ord_kernel<S_BLK, SPARSE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  // the largest shared-memory carve-out, so that two CTAs fit on an SM
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  dim3 grid((D.N + BM - 1) / BM, D.Hq, D.B);
  kern<<<grid, NTHREADS, SMEM_BYTES, st>>>(mq, mk, mv, p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_ord(const Dims& D, const FwdArgs& a, int32_t* dev_status, cudaStream_t st) {
  if (!fwd_tc_supported(D)) return cudaErrorNotSupported;
  if (a.sparse_only)
    return D.s == 64 ? launch_ord<64, true>(D, a, dev_status, st) : launch_ord<128, true>(D, a, dev_status, st);
  return D.s == 64 ? launch_ord<64, false>(D, a, dev_status, st) : launch_ord<128, false>(D, a, dev_status, st);
}

}  // namespace ssa
