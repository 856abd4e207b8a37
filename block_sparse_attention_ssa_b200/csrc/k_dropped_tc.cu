// Tensor-core dropped-mass probe (sm_100a, bf16, d = 128).
//
// delta(t) is the full causal softmax weight of query t that falls on the
// keys of unselected blocks ("Technische Samenvatting: SSA", section
// "1. Probleemstelling"; "SSA: Achieving Sparser Attention ...", section
// "Phenomenon 3").  Only S = Q K^T is needed, no V:
//   * with lse_full given:  delta = sum over D_t of 2^(S c - lse2_full); tiles
//     that hold no dropped pair for either half of the query tile are skipped
//     by every role (no load, no MMA, no exponentials);
//   * without it: two online log-sum-exps, over A_t and over D_t, and
//     delta = 2^(lse2_D - logaddexp2(lse2_A, lse2_D)).
// The sum runs over D_t itself, never as 1 - (sum over A_t), so small masses
// keep their relative precision.
//
// CTA = one 128-row query tile, 192 threads: warps 0-3 read S rows from TMEM
// (one row per thread), warp 4 streams 128-key K tiles by TMA, warp 5 issues
// the QK^T MMAs into a TMEM double buffer (256 columns).  A tile is two 64-key
// sub-blocks; each (64-row query half, sub-block) pair is "none", selected or
// dropped, as in the fused forward.
#include "ssa_internal.cuh"
#include "sm100_ptx.cuh"

namespace ssa {
namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int SUB = 64;
constexpr int HD = 128;
constexpr int NTHREADS = 192;

struct DCfg {
  static constexpr int NS = 2;
  static constexpr int Q_BYTES = BM * HD * 2;
  static constexpr int K_BYTES = BN * HD * 2;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_MISC = OFF_K + NS * K_BYTES;
  static constexpr int SMEM = OFF_MISC + 2048 + 1024;
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, false, false);
};

struct DMisc {
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4];
  uint64_t s_full[2], s_free[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  uint32_t sel[2][64];
};
static_assert(sizeof(DMisc) <= DCfg::SMEM - DCfg::OFF_MISC - 1024, "dropped shared-memory budget");

struct DParams {
  const int32_t* idx;
  const float* lse_in;  // may be null
  float* delta;
  int32_t* status;
  int Hq, g, N, n, k;
  float c;  // scale * log2(e)
};

__device__ __forceinline__ int dstate(int kb, int ib, bool valid, const uint32_t* selw) {
  if (!valid || kb > ib) return 0;
  return ((selw[kb >> 5] >> (kb & 31)) & 1u) ? 1 : 2;
}

template <int S_BLK, bool GIVEN>
__global__ void __launch_bounds__(NTHREADS, 1)
    dropped_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, DParams p) {
  using C = DCfg;
  // Used directly (no pointer arithmetic on the address) so that accesses
  // through it stay shared-memory loads; TMA tiles with 128-byte swizzle need
  // the 1024-byte alignment, which is checked rather than assumed.
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(p.status, 0, (int)SSA_ERR_UNSUPPORTED);
    return;
  }
  DMisc& M = *reinterpret_cast<DMisc*>(smem + C::OFF_MISC);
  volatile int* abort = &M.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = (int)(gridDim.x - 1 - blockIdx.x);
  const int h = blockIdx.y, b = blockIdx.z, kvh = h / p.g;
  const int q0 = qt * BM;
  const int ib0 = q0 / S_BLK, ib1 = (q0 + SUB) / S_BLK;
  const bool valid1 = q0 + SUB < p.N;
  const int T = (min(q0 + BM, p.N) + BN - 1) / BN;
  auto kblk = [](int j, int q) { return (j * BN + q * SUB) / S_BLK; };

  if (threadIdx.x == 0) {
    mbar_init(&M.q_full, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&M.k_full[s], 1);
      mbar_init(&M.k_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&M.s_full[s], 1);
      mbar_init(&M.s_free[s], 4);
    }
    mbar_init(&M.drain, 1);
    M.abort = 0;
    fence_mbar_init();
  }
  for (int w = threadIdx.x; w < 128; w += NTHREADS) (&M.sel[0][0])[w] = 0u;
  if (warp == 5) {
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = M.tmem_base;
  const uint32_t* sel0 = M.sel[0];
  const uint32_t* sel1 = (ib1 != ib0) ? M.sel[1] : M.sel[0];
  // With lse_full given only tiles holding a dropped pair do any work.
  auto useful = [&](int j) {
    if (!GIVEN) return true;
    bool any = false;
#pragma unroll
    for (int q = 0; q < 2; ++q)
      any |= dstate(kblk(j, q), ib0, true, sel0) == 2 || dstate(kblk(j, q), ib1, valid1, sel1) == 2;
    return any;
  };
  uint8_t* sQ = smem;
  uint8_t* sK = smem + C::OFF_K;

  if (warp == 4) {
    if (lane == 0) {
      mbar_expect_tx(&M.q_full, C::Q_BYTES);
      tma_load_4d(sQ, &tmQ, &M.q_full, 0, q0, h, b);
      tma_load_4d(sQ + C::Q_BYTES / 2, &tmQ, &M.q_full, 64, q0, h, b);
      int issued = 0;
      for (int j = 0; j < T; ++j) {
        if (!useful(j)) continue;
        const int st = issued % C::NS;
        const uint32_t use = (uint32_t)(issued / C::NS);
        if (issued >= C::NS && !mbar_wait(&M.k_empty[st], (use - 1) & 1u, abort)) break;
        mbar_expect_tx(&M.k_full[st], C::K_BYTES);
        tma_load_4d(sK + st * C::K_BYTES, &tmK, &M.k_full[st], 0, j * BN, kvh, b);
        tma_load_4d(sK + st * C::K_BYTES + C::K_BYTES / 2, &tmK, &M.k_full[st], 64, j * BN, kvh, b);
        ++issued;
      }
      int dummy = 0;
      mbar_wait(&M.q_full, 0, &dummy);
      for (int u = (issued > C::NS ? issued - C::NS : 0); u < issued; ++u) {
        dummy = 0;
        mbar_wait(&M.k_full[u % C::NS], (uint32_t)(u / C::NS) & 1u, &dummy);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(sQ);
      bool ok = mbar_wait(&M.q_full, 0, abort);
      int u = 0;
      for (int j = 0; ok && j < T; ++j) {
        if (!useful(j)) continue;
        const int st = u % C::NS, sb = u & 1;
        if (!mbar_wait(&M.k_full[st], (uint32_t)(u / C::NS) & 1u, abort)) break;
        if (u >= 2 && !mbar_wait(&M.s_free[sb], (uint32_t)((u - 2) >> 1) & 1u, abort)) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + st * C::K_BYTES);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off_q = (kk >> 2) * (C::Q_BYTES / 2) + (kk & 3) * 32;
          const uint32_t off_k = (kk >> 2) * (C::K_BYTES / 2) + (kk & 3) * 32;
          mma_ss(tmem + (uint32_t)sb * BN, smem_desc_sw128(q_addr + off_q, 16, 1024),
                 smem_desc_sw128(k_addr + off_k, 16, 1024), C::IDESC_QK, kk > 0 ? 1u : 0u);
        }
        tc_commit(&M.s_full[sb]);
        tc_commit(&M.k_empty[st]);
        ++u;
      }
      tc_commit(&M.drain);
      int dummy = 0;
      mbar_wait(&M.drain, 0, &dummy);
    }
  } else {
    const int half = warp >> 1;
    const int ib = half ? ib1 : ib0;
    const bool hvalid = half ? valid1 : true;
    const uint32_t* selw = half ? sel1 : sel0;
    const int t = q0 + warp * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const int64_t o = ((int64_t)b * p.Hq + h) * p.N + (t < p.N ? t : 0);
    const float lse2_in = GIVEN ? p.lse_in[o] * 1.4426950408889634f : 0.f;
    float m2[2] = {kNegInf, kNegInf}, l[2] = {0.f, 0.f};
    float dsum = 0.f;
    bool ok = true;
    int u = 0;
    for (int j = 0; j < T; ++j) {
      if (!useful(j)) continue;
      const int sb = u & 1;
      if (!mbar_wait(&M.s_full[sb], (uint32_t)(u >> 1) & 1u, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int mine = dstate(kblk(j, q), ib, hvalid, selw);
        if (mine == 0 || (GIVEN && mine != 2)) continue;
        const uint32_t sa = lane_base + (uint32_t)sb * BN + q * SUB;
        const int u0 = j * BN + q * SUB;
        const bool diag = u0 + SUB - 1 > t;
        uint32_t r[64];
        tmem_ld32(sa, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        tmem_ld32(sa + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        tmem_wait_ld();
        if (diag) {
#pragma unroll
          for (int c = 0; c < SUB; ++c)
            if (u0 + c > t) r[c] = __float_as_uint(kNegInf);
        }
        if (GIVEN) {
          float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
          for (int c = 0; c < SUB; c += 2) {
            acc0 += ex2(fmaf(__uint_as_float(r[c]), p.c, -lse2_in));
            acc1 += ex2(fmaf(__uint_as_float(r[c + 1]), p.c, -lse2_in));
          }
          dsum += acc0 + acc1;
        } else {
          const int X = mine - 1;
          float a0 = kNegInf, a1 = kNegInf, a2 = kNegInf, a3 = kNegInf;
#pragma unroll
          for (int c = 0; c < SUB; c += 4) {
            a0 = fmaxf(a0, __uint_as_float(r[c]));
            a1 = fmaxf(a1, __uint_as_float(r[c + 1]));
            a2 = fmaxf(a2, __uint_as_float(r[c + 2]));
            a3 = fmaxf(a3, __uint_as_float(r[c + 3]));
          }
          const float mnew = fmaxf(m2[X], fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)) * p.c);
          float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
          for (int c = 0; c < SUB; c += 2) {
            acc0 += ex2(fmaf(__uint_as_float(r[c]), p.c, -mnew));
            acc1 += ex2(fmaf(__uint_as_float(r[c + 1]), p.c, -mnew));
          }
          l[X] = (m2[X] == kNegInf ? 0.f : l[X] * ex2(m2[X] - mnew)) + acc0 + acc1;
          m2[X] = mnew;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&M.s_free[sb]);
      ++u;
    }
    if (ok && t < p.N) {
      if (GIVEN) {
        p.delta[o] = dsum;
      } else {
        const float la = (l[0] > 0.f) ? m2[0] + log2f(l[0]) : kNegInf;
        const float ld = (l[1] > 0.f) ? m2[1] + log2f(l[1]) : kNegInf;
        const float hi = fmaxf(la, ld), lo = fminf(la, ld);
        const float lf = (lo == kNegInf) ? hi : hi + log2f(1.0f + ex2(lo - hi));
        p.delta[o] = (l[1] > 0.f) ? ex2(ld - lf) : 0.f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (M.abort && threadIdx.x == 0) atomicCAS(p.status, 0, (int)SSA_ERR_TIMEOUT);
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int S_BLK, bool GIVEN>
cudaError_t launch_d(const Dims& D, const FwdArgs& a, int32_t* status, cudaStream_t st) {
  using C = DCfg;
  CUtensorMap mq, mk;
  if (!make_tma_map_bf16(&mq, a.q, D.B, D.Hq, D.N, BM) || !make_tma_map_bf16(&mk, a.k, D.B, D.Hkv, D.N, BN))
    return cudaErrorInvalidValue;
  DParams p;
  p.idx = a.idx;
  p.lse_in = a.lse_in;
  p.delta = a.delta;
  p.status = status;
  p.Hq = D.Hq;
  p.g = D.g;
  p.N = D.N;
  p.n = D.n;
  p.k = D.k;
  p.c = D.scale * 1.4426950408889634f;
  auto kern = dropped_tc_kernel<S_BLK, GIVEN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<dim3((D.N + BM - 1) / BM, D.Hq, D.B), NTHREADS, C::SMEM, st>>>(mq, mk, p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dropped_tc(const Dims& D, const FwdArgs& a, int32_t* status, cudaStream_t st) {
  if (!fwd_tc_supported(D)) return cudaErrorNotSupported;
  const bool given = a.lse_in != nullptr;
  if (D.s == 64) return given ? launch_d<64, true>(D, a, status, st) : launch_d<64, false>(D, a, status, st);
  return given ? launch_d<128, true>(D, a, status, st) : launch_d<128, false>(D, a, status, st);
}

}  // namespace ssa
