// Tensor-core backward with per-row selection masks (sm_100a, bf16, d = 64):
// blocks of 16 to 128 keys, selection per query block or per query token.
//
// Objective ("Technische Samenvatting: SSA", "Bidirectionele Uitlijning";
// "SSA: Achieving Sparser Attention ...", "Bidirectional Attention
// Alignment"): L = <g_f, h_full> + <g_s, h_sparse> + alpha (L_sp + L_cm).
// As in the warp-level kernels the two streams collapse into one softmax
// backward over the full stream's weights P = exp(x - lse_full):
//   selected pair (u in A_t): dX = P (dO_c . v_u - D_c),  dV_u += P dO_c,
//   dropped pair  (u in D_t): dX = P (dh_f . v_u - D_f),  dV_u += P dh_f,
// dQ_t = scale sum_u dX K_u, dK_u = scale sum_t dX Q_t (the preprocess of the
// warp-level backward supplies dO_c and dh_f in bf16, D_c and D_f).
//
// Two kernels, 320 threads each: warps 0-7 compute (warps w and w+4 share
// TMEM lanes 32(w%4).., warp w takes the 64 columns w/4), warp 8 loads by
// TMA, warp 9 owns TMEM and issues the MMAs.  All tiles are 128 x 64 bf16
// (one 128-byte swizzle span per row).
//
//   dq   one 128-row query tile per CTA, walking its causal key tiles 64 keys
//        (a half step) at a time.  TMEM: dQ [0,64), then two buffers of S,
//        dP_c, dP_f (64 columns each), so that the products of the next half
//        step run while this one is computed.  Per half step: S = Q K^T,
//        dP_c = dO_c V^T, dP_f = dh_f V^T (each only when a row of the tile
//        can use it), dS = P (dP_x - D_x) routed per 16-key group by the row's
//        selection, written as bf16 over the warp's own S columns, then
//        dQ += dS K.
//   dkv  one 128-key tile per CTA, walking a chunk of at most 4 query heads
//        of its kv group and their causal query tiles, 64 queries (a half
//        step) at a time.  TMEM: dK [0,64), dV [64,128), then two buffers of
//        S^T, dP_c^T, dP_f^T (64 columns each), so that the products of the
//        next half step run while this one is computed.  Per half step:
//        S^T = K Q^T, dP_c^T = V dO_c^T, dP_f^T = V dh_f^T, then P_A^T over
//        S^T, P_D^T over dP_f^T and dS^T over dP_c^T (each warp packs into
//        columns it has already read), dV += P_A^T dO_c + P_D^T dh_f and
//        dK += dS^T Q.  A query's selection word decides, per key block, the
//        set of each element.  With more than one chunk per group the chunks
//        write fp32 partials that the warp-level backward's sum adds in order.
// No atomics: every output element is written by one CTA in a fixed order.
#include "ssa_internal.cuh"
#include "sm100_ptx.cuh"

namespace ssa {
namespace {

using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int HD = 64;
constexpr int TILE = 128;
constexpr int TB = TILE * HD * 2;  // 16 KB: one 128 x 64 bf16 tile
constexpr int NTHREADS = 320;
constexpr int WARP_TMA = 8, WARP_MMA = 9;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t IDESC_ACC = idesc_bf16_f32(TILE, HD, false, true);   // B MN-major (rows = reduction)

struct TcmBwdParams {
  TensorRef dq, dk, dv;
  const float* lse;  // lse_full [B,Hq,N]
  const float* Dc;   // [B,Hq,N]
  const float* Df;
  const uint32_t* mask;  // [B,Hq,rows,words] selected-block bit sets
  int words;
  float* part;  // fp32 dK / dV partials, or null
  int32_t* status;
  int Hq, g, N, n, ls, per_token, hpc, NT;
  float c;  // scale * log2(e)
  float scale;
};

// Half steps of 64 along the MMA's N / reduction dimension.
constexpr uint32_t IDESC_S64 = idesc_bf16_f32(TILE, 64, false, false);  // both K-major, N = 64

// D (128 x 64) = A (128 x 64) B^T, B = 64 rows of a K-major smem tile.
__device__ __forceinline__ void mma_ss_n64(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk)
    mma_ss(d_tmem, smem_desc_sw128(a_smem + kk * 32, 16, 1024), smem_desc_sw128(b_smem + kk * 32, 16, 1024),
           IDESC_S64, kk > 0 ? 1u : 0u);
}

// D (128 x 64) (+)= A (TMEM, 128 rows x 64 reduction as bf16 pairs: indices
// 0-31 at columns a..a+15, 32-63 at a+32..a+47) x B (64 rows of a smem tile,
// rows = reduction index).
__device__ __forceinline__ void mma_ts_k64(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    mma_ts(d_tmem, a_tmem + 32 * (kk >> 1) + 8 * (kk & 1), smem_desc_sw128(b_smem + kk * 2048, TB, 1024), IDESC_ACC,
           (accumulate || kk > 0) ? 1u : 0u);
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__host__ __device__ inline int sel_rows_tile(int per_token, int ls) {
  return per_token ? TILE : (ls >= 7 ? 1 : (TILE >> ls));
}

// ================================================================ dQ
namespace dqm {
constexpr int NS = 3;
constexpr int OFF_Q = 0, OFF_OC = TB, OFF_F = 2 * TB, OFF_K = 3 * TB, OFF_V = OFF_K + NS * TB;
constexpr int OFF_MISC = OFF_V + NS * TB;
// TMEM: dQ, then two buffers of one 64-key half step each: S, dP_c, dP_f
// (64 columns apiece) at COL_BUF + 192 b.
constexpr uint32_t COL_DQ = 0, COL_BUF = 64;
struct Misc {
  uint64_t q_full;
  uint64_t k_full[NS], k_empty[NS], v_full[NS], v_empty[NS];
  uint64_t s_full[2], ds_full[2], done, drain;
  uint32_t tmem_base;
  int abort;
  uint32_t uni[64], inter[64];  // OR / AND of the tile's selection rows
  // followed by the selection rows (64 words each)
};
}  // namespace dqm

__global__ void __launch_bounds__(NTHREADS, 1)
    bwd_dq_tcm_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmOc,
                      const __grid_constant__ CUtensorMap tmF, TcmBwdParams p) {
  using namespace dqm;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  Misc& M = *reinterpret_cast<Misc*>(smem + OFF_MISC);
  uint32_t (*sel)[64] = reinterpret_cast<uint32_t (*)[64]>(smem + OFF_MISC + sizeof(Misc));
  volatile int* abort = &M.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = (int)(gridDim.x - 1 - blockIdx.x);  // the longest rows first
  const int h = blockIdx.y, b = blockIdx.z, kvh = h / p.g;
  const int q0 = qt * TILE;
  const int ib0 = q0 >> p.ls;
  const int nsel = sel_rows_tile(p.per_token, p.ls);
  const int rph = p.per_token ? p.N : p.n;

  if (threadIdx.x == 0) {
    mbar_init(&M.q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&M.k_full[s], 1);
      mbar_init(&M.k_empty[s], 1);
      mbar_init(&M.v_full[s], 1);
      mbar_init(&M.v_empty[s], 1);
    }
    for (int bb = 0; bb < 2; ++bb) {
      mbar_init(&M.s_full[bb], 1);
      mbar_init(&M.ds_full[bb], 8);
    }
    mbar_init(&M.done, 1);
    mbar_init(&M.drain, 1);
    M.abort = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(&M.tmem_base, 512);
    tmem_relinquish();
  }
  const int nvalid = p.per_token ? min(TILE, p.N - q0) : min(nsel, p.n - ib0);
  for (int e = threadIdx.x; e < nsel * 64; e += NTHREADS) {
    const int r = e >> 6, w = e & 63;
    uint32_t v = 0u;
    if (r < nvalid && w < p.words) {
      const int64_t mrow = p.per_token ? (int64_t)q0 + r : (int64_t)ib0 + r;
      v = p.mask[(((int64_t)b * p.Hq + h) * rph + mrow) * p.words + w];
    }
    sel[r][w] = v;
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

  // Whether some row of the tile can have a selected / dropped key in the
  // 64 keys starting at u.
  auto flags = [&](int u, bool& anyA, bool& anyD) {
    const int jb = u >> p.ls;
    const int nb = p.ls >= 6 ? 1 : (64 >> p.ls);
    const uint32_t m = ((1u << nb) - 1u) << (jb & 31);
    anyA = (M.uni[jb >> 5] & m) != 0u;
    anyD = (M.inter[jb >> 5] & m) != m;
  };

  const int T = qt + 1;  // causal key tiles
  const uint32_t tmem = M.tmem_base;
  uint8_t* sQ = smem + OFF_Q;
  uint8_t* sOc = smem + OFF_OC;
  uint8_t* sF = smem + OFF_F;
  uint8_t* sK = smem + OFF_K;
  uint8_t* sV = smem + OFF_V;

  if (warp == WARP_TMA) {
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      mbar_expect_tx(&M.q_full, 3 * TB);
      tma_load_4d(sQ, &tmQ, &M.q_full, 0, q0, h, b);
      tma_load_4d(sOc, &tmOc, &M.q_full, 0, q0, h, b);
      tma_load_4d(sF, &tmF, &M.q_full, 0, q0, h, b);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < T; ++j) {
        const int st = j % NS;
        const uint32_t use = (uint32_t)(j / NS);
        if (j >= NS && !mbar_wait(&M.k_empty[st], (use - 1) & 1u, abort)) break;
        mbar_expect_tx(&M.k_full[st], TB);
        tma_load_4d(sK + st * TB, &tmK, &M.k_full[st], 0, j * TILE, kvh, b);
        k_issued = j + 1;
        if (j >= NS && !mbar_wait(&M.v_empty[st], (use - 1) & 1u, abort)) break;
        mbar_expect_tx(&M.v_full[st], TB);
        tma_load_4d(sV + st * TB, &tmV, &M.v_full[st], 0, j * TILE, kvh, b);
        v_issued = j + 1;
      }
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
    // Half step hs = 2 j + y covers keys 64y.. of key tile j and uses TMEM
    // buffer hs & 1: its S / dP products are issued before the dQ product of
    // half step hs - 1, so they overlap that half step's compute.
    if (lane == 0) {
      const uint32_t aq = smem_u32(sQ), aoc = smem_u32(sOc), af = smem_u32(sF);
      bool ok = mbar_wait(&M.q_full, 0, abort);
      const int H = 2 * T;
      auto front = [&](int hs) -> bool {
        const int j = hs >> 1, y = hs & 1, st = j % NS, bsel = hs & 1;
        const uint32_t ph = (uint32_t)(j / NS) & 1u;
        bool anyA, anyD;
        flags(j * TILE + 64 * y, anyA, anyD);
        const uint32_t ak = smem_u32(sK + st * TB) + 8192u * y, av = smem_u32(sV + st * TB) + 8192u * y;
        const uint32_t base = tmem + COL_BUF + 192 * bsel;
        if (!mbar_wait(&M.k_full[st], ph, abort)) return false;
        tc_fence_after();
        mma_ss_n64(base, aq, ak);
        if (!mbar_wait(&M.v_full[st], ph, abort)) return false;
        tc_fence_after();
        if (anyA) mma_ss_n64(base + 64, aoc, av);
        if (anyD) mma_ss_n64(base + 128, af, av);
        tc_commit(&M.s_full[bsel]);
        if (y == 1) tc_commit(&M.v_empty[st]);
        return true;
      };
      auto back = [&](int hs) -> bool {
        const int j = hs >> 1, y = hs & 1, st = j % NS, bsel = hs & 1;
        if (!mbar_wait(&M.ds_full[bsel], (uint32_t)(hs >> 1) & 1u, abort)) return false;
        tc_fence_after();
        mma_ts_k64(tmem + COL_DQ, tmem + COL_BUF + 192 * bsel, smem_u32(sK + st * TB) + 8192u * y, hs > 0);
        if (y == 1) tc_commit(&M.k_empty[st]);
        return true;
      };
      if (ok && H > 0) ok = front(0);
      for (int hs = 0; ok && hs < H; ++hs) {
        if (hs + 1 < H && !front(hs + 1)) {
          ok = false;
          break;
        }
        if (!back(hs)) {
          ok = false;
          break;
        }
      }
      tc_commit(&M.done);
      tc_commit(&M.drain);
      int dummy = 0;
      mbar_wait(&M.drain, 0, &dummy);
    }
  } else {
    const int quarter = warp & 3, ch = warp >> 2;  // rows 32*quarter.., keys 32*ch.. of a half step
    const int row = quarter * 32 + lane;
    const int t = q0 + row;
    const bool valid = t < p.N;
    const uint32_t* selw = sel[p.per_token ? row : min((t >> p.ls) - ib0, nsel - 1)];
    const int64_t ro = ((int64_t)b * p.Hq + h) * p.N + t;
    const float lse2 = valid ? p.lse[ro] * kLog2e : 0.f;
    const float Dc = valid ? p.Dc[ro] : 0.f, Df = valid ? p.Df[ro] : 0.f;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    bool ok = true;
    for (int hs = 0; hs < 2 * T; ++hs) {
      const int j = hs >> 1, y = hs & 1, bsel = hs & 1;
      if (!mbar_wait(&M.s_full[bsel], (uint32_t)(hs >> 1) & 1u, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      bool anyA, anyD;
      const int uh = j * TILE + 64 * y;  // first key of the half step
      flags(uh, anyA, anyD);
      // bit 16g of km: key group g of this warp's 32 keys
      const unsigned long long km = tile_keep_mask_p2(selw, uh, p.ls) >> (32 * ch);
      const int lim = valid ? t - (uh + 32 * ch) : -1;  // keys c <= lim are causal
      const uint32_t base = lane_base + COL_BUF + 192 * bsel + 32 * ch;
      uint32_t s[32], pc[32], pf[32];
      tmem_ld32(base, s);
      if (anyA) tmem_ld32(base + 64, pc);
      if (anyD) tmem_ld32(base + 128, pf);
      tmem_wait_ld();
      uint32_t ds[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        float v[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int kc = c + e;  // key within the warp's 32
          const bool inA = (km >> (kc & ~15)) & 1ull;
          const bool live = kc <= lim;
          const float pv = ex2(fmaf(__uint_as_float(s[kc]), p.c, -lse2));
          const float dpx = inA ? __uint_as_float(pc[kc]) - Dc : __uint_as_float(pf[kc]) - Df;
          v[e] = live ? pv * dpx : 0.f;
        }
        ds[c / 2] = pack_bf16(v[0], v[1]);
      }
      tmem_st16(base, ds);  // packed into the first 16 of the warp's own 32 S columns
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&M.ds_full[bsel]);
    }
    if (ok && mbar_wait(&M.done, 0, abort)) {
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32(lane_base + COL_DQ + 32 * ch, r);
      tmem_wait_ld();
      if (valid) {
        uint32_t o[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          o[c] = pack_bf16(__uint_as_float(r[2 * c]) * p.scale, __uint_as_float(r[2 * c + 1]) * p.scale);
        uint4* d4 = reinterpret_cast<uint4*>(row_ptr_w<bf16>(p.dq, b, h, t) + 32 * ch);
#pragma unroll
        for (int q = 0; q < 4; ++q) d4[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
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

// ================================================================ dK, dV
namespace dkvm {
constexpr int NS = 2;
// A stage: the step's Q, dO_c and dh_f tiles, then lse, D_c, D_f (128 floats
// each) and the 128 query rows' selection words that cover this key tile.
constexpr int SC = TILE * 4;
constexpr int STAGE = 3 * TB + 4 * SC;
constexpr int OFF_K = 0, OFF_V = TB, OFF_STAGE = 2 * TB;
constexpr int OFF_MISC = OFF_STAGE + NS * STAGE;
// TMEM: dK, dV, then two buffers of one 64-query half step each: S^T, dP_c^T,
// dP_f^T (64 columns apiece) at COL_BUF + 192 b.
constexpr uint32_t COL_DK = 0, COL_DV = 64, COL_BUF = 128;
struct Misc {
  uint64_t kv_full;
  uint64_t q_full[NS], q_empty[NS];
  uint64_t s_full[2], p_full[2], done, drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte alignment of swizzled tiles");
}  // namespace dkvm

__global__ void __launch_bounds__(NTHREADS, 1)
    bwd_dkv_tcm_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmOc,
                       const __grid_constant__ CUtensorMap tmF, TcmBwdParams p) {
  using namespace dkvm;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  Misc& M = *reinterpret_cast<Misc*>(smem + OFF_MISC);
  volatile int* abort = &M.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = (int)blockIdx.x;  // the most query tiles first
  const int chunks = p.g / p.hpc;
  const int kvh = blockIdx.y / chunks, chunk = blockIdx.y % chunks;
  const int b = blockIdx.z;
  const int Hkv = p.Hq / p.g;
  const int u0 = kt * TILE;
  const int nq = p.NT - kt;  // causal query tiles per head
  const int T = p.hpc * nq;  // steps: hh * nq + (qt - kt)
  const int rph = p.per_token ? p.N : p.n;
  const int wi = (u0 >> p.ls) >> 5;  // the selection word holding this key tile's blocks
  const int nbt = p.ls >= 7 ? 1 : (TILE >> p.ls);
  const uint32_t tbm = ((nbt >= 32 ? 0u : (1u << nbt)) - 1u) << ((u0 >> p.ls) & 31);
  auto stage_ptr = [&](int st) { return smem + OFF_STAGE + st * STAGE; };

  if (threadIdx.x == 0) {
    mbar_init(&M.kv_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&M.q_full[s], 1);
      mbar_init(&M.q_empty[s], 1);
    }
    for (int bb = 0; bb < 2; ++bb) {
      mbar_init(&M.s_full[bb], 1);
      mbar_init(&M.p_full[bb], 8);
    }
    mbar_init(&M.done, 1);
    mbar_init(&M.drain, 1);
    M.abort = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(&M.tmem_base, 512);
    tmem_relinquish();
  }
  // Scalar slots of ragged query tiles stay finite (their columns are masked).
  for (int i = threadIdx.x; i < NS * 4 * TILE; i += NTHREADS)
    reinterpret_cast<float*>(stage_ptr(i / (4 * TILE)) + 3 * TB)[i % (4 * TILE)] = 0.f;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = M.tmem_base;
  uint8_t* sK = smem + OFF_K;
  uint8_t* sV = smem + OFF_V;
  auto decode = [&](int j, int& h, int& qt) {
    h = (kvh * chunks + chunk) * p.hpc + j / nq;
    qt = kt + j % nq;
  };
  // Whether some of the 64 queries of a half step selected / dropped some key
  // block of the tile (words: the half's 64 selection words).
  auto half_flags = [&](const uint32_t* words, bool& anyA, bool& anyD) {
    bool a = false, d = false;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint32_t w = words[lane + 32 * i] & tbm;
      a |= w != 0u;
      d |= w != tbm;
    }
    anyA = __any_sync(0xffffffffu, a);
    anyD = __any_sync(0xffffffffu, d);
  };

  if (warp == WARP_TMA) {
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmOc);
      prefetch_tensormap(&tmF);
      mbar_expect_tx(&M.kv_full, 2 * TB);
      tma_load_4d(sK, &tmK, &M.kv_full, 0, u0, kvh, b);
      tma_load_4d(sV, &tmV, &M.kv_full, 0, u0, kvh, b);
    }
    int issued = 0;
    for (int j = 0; j < T; ++j) {
      const int st = j % NS;
      bool okw = true;
      if (lane == 0 && j >= NS) okw = mbar_wait(&M.q_empty[st], (uint32_t)(j / NS - 1) & 1u, abort);
      if (!__shfl_sync(0xffffffffu, okw ? 1 : 0, 0)) break;
      int h, qt;
      decode(j, h, qt);
      const int t0 = qt * TILE;
      const int valid = min(TILE, p.N - t0);  // a multiple of 64
      uint8_t* sp_ = stage_ptr(st);
      // selection words of the step's query rows (0 past the end)
      uint32_t* words = reinterpret_cast<uint32_t*>(sp_ + 3 * TB + 3 * SC);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = lane + 32 * i;
        uint32_t w = 0u;
        if (r < valid) {
          const int64_t mrow = p.per_token ? (int64_t)t0 + r : (int64_t)((t0 + r) >> p.ls);
          w = p.mask[(((int64_t)b * p.Hq + h) * rph + mrow) * p.words + wi];
        }
        words[r] = w;
      }
      __syncwarp();
      if (lane == 0) {
        const int64_t ro = ((int64_t)b * p.Hq + h) * p.N + t0;
        mbar_expect_tx(&M.q_full[st], 3 * TB + 3 * (uint32_t)valid * 4);
        tma_load_4d(sp_, &tmQ, &M.q_full[st], 0, t0, h, b);
        tma_load_4d(sp_ + TB, &tmOc, &M.q_full[st], 0, t0, h, b);
        tma_load_4d(sp_ + 2 * TB, &tmF, &M.q_full[st], 0, t0, h, b);
        bulk_load(sp_ + 3 * TB, p.lse + ro, (uint32_t)valid * 4, &M.q_full[st]);
        bulk_load(sp_ + 3 * TB + SC, p.Dc + ro, (uint32_t)valid * 4, &M.q_full[st]);
        bulk_load(sp_ + 3 * TB + 2 * SC, p.Df + ro, (uint32_t)valid * 4, &M.q_full[st]);
      }
      issued = j + 1;
    }
    if (lane == 0) {
      int dummy = 0;
      mbar_wait(&M.kv_full, 0, &dummy);
      for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j) {
        dummy = 0;
        mbar_wait(&M.q_full[j % NS], (uint32_t)(j / NS) & 1u, &dummy);
      }
    }
  } else if (warp == WARP_MMA) {
    // Half step hs = 2 j + x covers queries 64x.. of step j and uses TMEM
    // buffer hs & 1: its S^T / dP^T products are issued before the dV / dK
    // products of half step hs - 1, so they overlap that half step's compute.
    const uint32_t ak = smem_u32(sK), av = smem_u32(sV);
    bool ok = true;
    if (lane == 0) ok = T == 0 || mbar_wait(&M.kv_full, 0, abort);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    bool started_dv = false, started_dk = false;
    bool fA0 = false, fD0 = false, fA1 = false, fD1 = false;  // flags of the half steps in buffers 0 / 1
    const int H = 2 * T;
    auto front = [&](int hs) -> bool {
      const int j = hs >> 1, x = hs & 1, st = j % NS, bsel = hs & 1;
      // every lane reads the step's selection words: every lane acquires the stage
      const bool okf = mbar_wait(&M.q_full[st], (uint32_t)(j / NS) & 1u, abort);
      if (!__all_sync(0xffffffffu, okf)) return false;
      tc_fence_after();
      uint8_t* sp_ = stage_ptr(st);
      bool anyA, anyD;
      half_flags(reinterpret_cast<const uint32_t*>(sp_ + 3 * TB + 3 * SC) + 64 * x, anyA, anyD);
      if (bsel) {
        fA1 = anyA;
        fD1 = anyD;
      } else {
        fA0 = anyA;
        fD0 = anyD;
      }
      if (lane == 0) {
        const uint32_t base = tmem + COL_BUF + 192 * bsel, off = 8192u * x;
        mma_ss_n64(base, ak, smem_u32(sp_) + off);
        if (anyA) mma_ss_n64(base + 64, av, smem_u32(sp_ + TB) + off);
        if (anyD) mma_ss_n64(base + 128, av, smem_u32(sp_ + 2 * TB) + off);
        tc_commit(&M.s_full[bsel]);
      }
      __syncwarp();
      return true;
    };
    auto back = [&](int hs) -> bool {
      const int j = hs >> 1, x = hs & 1, st = j % NS, bsel = hs & 1;
      const bool anyA = bsel ? fA1 : fA0, anyD = bsel ? fD1 : fD0;
      bool okb = true;
      if (lane == 0) {
        okb = mbar_wait(&M.p_full[bsel], (uint32_t)(hs >> 1) & 1u, abort);
        if (okb) {
          tc_fence_after();
          uint8_t* sp_ = stage_ptr(st);
          const uint32_t base = tmem + COL_BUF + 192 * bsel, off = 8192u * x;
          if (anyA) {
            mma_ts_k64(tmem + COL_DV, base, smem_u32(sp_ + TB) + off, started_dv);
            started_dv = true;
          }
          if (anyD) {
            mma_ts_k64(tmem + COL_DV, base + 128, smem_u32(sp_ + 2 * TB) + off, started_dv);
            started_dv = true;
          }
          mma_ts_k64(tmem + COL_DK, base + 64, smem_u32(sp_) + off, started_dk);
          started_dk = true;
          if (x == 1) tc_commit(&M.q_empty[st]);
        }
      }
      return __shfl_sync(0xffffffffu, okb ? 1 : 0, 0) != 0;
    };
    if (ok && H > 0) ok = front(0);
    for (int hs = 0; ok && hs < H; ++hs) {
      if (hs + 1 < H && !front(hs + 1)) {
        ok = false;
        break;
      }
      if (!back(hs)) {
        ok = false;
        break;
      }
    }
    if (lane == 0) {
      tc_commit(&M.done);
      tc_commit(&M.drain);
      int dummy = 0;
      mbar_wait(&M.drain, 0, &dummy);
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3, ch = warp >> 2;  // key lanes 32*quarter.., query columns 32*ch.. of a half
    const int r = quarter * 32 + lane;              // key row within the tile
    const int bp = ((u0 + r) >> p.ls) & 31;        // its block's bit in a selection word
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    bool ok = true;
    for (int hs = 0; hs < 2 * T; ++hs) {
      const int j = hs >> 1, x = hs & 1, st = j % NS, bsel = hs & 1;
      if (!mbar_wait(&M.q_full[st], (uint32_t)(j / NS) & 1u, abort) ||
          !mbar_wait(&M.s_full[bsel], (uint32_t)(hs >> 1) & 1u, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      int h, qt;
      decode(j, h, qt);
      const bool diag = qt == kt;
      const int lim = p.N - qt * TILE;  // columns c < lim are queries of the sequence
      const uint8_t* sp_ = stage_ptr(st);
      const float* L = reinterpret_cast<const float*>(sp_ + 3 * TB);
      const float* DcS = reinterpret_cast<const float*>(sp_ + 3 * TB + SC);
      const float* DfS = reinterpret_cast<const float*>(sp_ + 3 * TB + 2 * SC);
      const uint32_t* words = reinterpret_cast<const uint32_t*>(sp_ + 3 * TB + 3 * SC);
      bool anyA, anyD;
      half_flags(words + 64 * x, anyA, anyD);
      const uint32_t base = lane_base + COL_BUF + 192 * bsel;
      const int c0 = 64 * x + 32 * ch;  // first query column (within the tile) of this warp
      uint32_t s[32], pc[32], pf[32];
      tmem_ld32(base + 32 * ch, s);
      if (anyA) tmem_ld32(base + 64 + 32 * ch, pc);
      if (anyD) tmem_ld32(base + 128 + 32 * ch, pf);
      tmem_wait_ld();
      uint32_t pa[16], pd[16], ds[16];
#pragma unroll
      for (int k8 = 0; k8 < 32; k8 += 8) {
        // the eight columns' scalars and selection words as 16-byte loads
        float lv[8], dcv[8], dfv[8];
        uint32_t wv[8];
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          const float4 l4 = *reinterpret_cast<const float4*>(L + c0 + k8 + 4 * v);
          const float4 c4 = *reinterpret_cast<const float4*>(DcS + c0 + k8 + 4 * v);
          const float4 f4 = *reinterpret_cast<const float4*>(DfS + c0 + k8 + 4 * v);
          const uint4 w4 = *reinterpret_cast<const uint4*>(words + c0 + k8 + 4 * v);
          lv[4 * v] = l4.x; lv[4 * v + 1] = l4.y; lv[4 * v + 2] = l4.z; lv[4 * v + 3] = l4.w;
          dcv[4 * v] = c4.x; dcv[4 * v + 1] = c4.y; dcv[4 * v + 2] = c4.z; dcv[4 * v + 3] = c4.w;
          dfv[4 * v] = f4.x; dfv[4 * v + 1] = f4.y; dfv[4 * v + 2] = f4.z; dfv[4 * v + 3] = f4.w;
          wv[4 * v] = w4.x; wv[4 * v + 1] = w4.y; wv[4 * v + 2] = w4.z; wv[4 * v + 3] = w4.w;
        }
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
          float va[2], vd[2], vs[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int i = k8 + c + e;  // column within the warp's 32
            const int col = c0 + i;
            const bool live = col < lim && (!diag || r <= col);
            const bool inA = (wv[c + e] >> bp) & 1u;
            const float pv = ex2(fmaf(__uint_as_float(s[i]), p.c, -lv[c + e] * kLog2e));
            const float dpx = inA ? __uint_as_float(pc[i]) - dcv[c + e] : __uint_as_float(pf[i]) - dfv[c + e];
            va[e] = (live && inA) ? pv : 0.f;
            vd[e] = (live && !inA) ? pv : 0.f;
            vs[e] = live ? pv * dpx : 0.f;
          }
          pa[(k8 + c) / 2] = pack_bf16(va[0], va[1]);
          pd[(k8 + c) / 2] = pack_bf16(vd[0], vd[1]);
          ds[(k8 + c) / 2] = pack_bf16(vs[0], vs[1]);
        }
      }
      // packed into the first 16 of the warp's own 32 columns of each product
      tmem_st16(base + 32 * ch, pa);
      if (anyD) tmem_st16(base + 128 + 32 * ch, pd);
      tmem_st16(base + 64 + 32 * ch, ds);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&M.p_full[bsel]);
    }
    if (ok && (T == 0 || mbar_wait(&M.done, 0, abort))) {
      tc_fence_after();
      const int u = u0 + r;
      uint32_t rk[32], rv[32];
      tmem_ld32(lane_base + COL_DK + 32 * ch, rk);
      tmem_ld32(lane_base + COL_DV + 32 * ch, rv);
      tmem_wait_ld();
      if (T == 0) {
#pragma unroll
        for (int c = 0; c < 32; ++c) rk[c] = rv[c] = 0u;
      }
      if (u < p.N) {
        if (p.part == nullptr) {
          uint32_t ok_[16], ov_[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            ok_[c] = pack_bf16(__uint_as_float(rk[2 * c]) * p.scale, __uint_as_float(rk[2 * c + 1]) * p.scale);
            ov_[c] = pack_bf16(__uint_as_float(rv[2 * c]), __uint_as_float(rv[2 * c + 1]));
          }
          uint4* dk4 = reinterpret_cast<uint4*>(row_ptr_w<bf16>(p.dk, b, kvh, u) + 32 * ch);
          uint4* dv4 = reinterpret_cast<uint4*>(row_ptr_w<bf16>(p.dv, b, kvh, u) + 32 * ch);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            dk4[q] = make_uint4(ok_[4 * q], ok_[4 * q + 1], ok_[4 * q + 2], ok_[4 * q + 3]);
            dv4[q] = make_uint4(ov_[4 * q], ov_[4 * q + 1], ov_[4 * q + 2], ov_[4 * q + 3]);
          }
        } else {
          // fp32 partials [chunk][2][B][Hkv][N][64] (dK unscaled, dV)
          const int64_t plane = (int64_t)gridDim.z * Hkv * p.N * HD;
          float* pk = p.part + (int64_t)chunk * 2 * plane + (((int64_t)b * Hkv + kvh) * p.N + u) * HD + 32 * ch;
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

}  // namespace

bool bwd_tcm_supported(const Dims& D) { return D.dtype == SSA_BF16 && D.d == 64 && D.n <= 2048; }

cudaError_t launch_bwd_tcm(const Dims& D, const BwdArgs& a, const void* dhf_bf16, const void* doc_bf16, int hpc,
                           int32_t* status, cudaStream_t st) {
  if (!bwd_tcm_supported(D) || a.sparse_only) return cudaErrorNotSupported;
  const int64_t rs = (int64_t)D.N * HD;
  const TensorRef rdhf{dhf_bf16, (int64_t)D.Hq * rs, rs, HD};
  const TensorRef rdoc{doc_bf16, (int64_t)D.Hq * rs, rs, HD};
  CUtensorMap mq, mk, mv, moc, mf;
  if (!make_tma_map_bf16(&mq, a.q, D.B, D.Hq, D.N, TILE, HD) || !make_tma_map_bf16(&mk, a.k, D.B, D.Hkv, D.N, TILE, HD) ||
      !make_tma_map_bf16(&mv, a.v, D.B, D.Hkv, D.N, TILE, HD) || !make_tma_map_bf16(&moc, rdoc, D.B, D.Hq, D.N, TILE, HD) ||
      !make_tma_map_bf16(&mf, rdhf, D.B, D.Hq, D.N, TILE, HD))
    return cudaErrorInvalidValue;
  TcmBwdParams p;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.lse = a.lse_full;
  p.Dc = a.Dc;
  p.Df = a.Df;
  p.mask = a.mask;
  p.words = a.words;
  p.status = status;
  p.Hq = D.Hq;
  p.g = D.g;
  p.N = D.N;
  p.n = D.n;
  p.ls = __builtin_ctz((unsigned)D.s);
  p.per_token = D.per_token;
  p.hpc = hpc;
  p.NT = (D.N + TILE - 1) / TILE;
  p.c = D.scale * kLog2e;
  p.scale = D.scale;
  const int chunks = D.g / hpc;
  p.part = chunks > 1 ? a.kvpart : nullptr;
  const int smem_dkv = dkvm::OFF_MISC + (int)sizeof(dkvm::Misc) + 1024;
  cudaError_t e = cudaFuncSetAttribute(bwd_dkv_tcm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dkv);
  if (e != cudaSuccess) return e;
  bwd_dkv_tcm_kernel<<<dim3(p.NT, D.Hkv * chunks, D.B), NTHREADS, smem_dkv, st>>>(mq, mk, mv, moc, mf, p);
  count_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int smem_dq =
      dqm::OFF_MISC + (int)sizeof(dqm::Misc) + sel_rows_tile(D.per_token, p.ls) * 64 * (int)sizeof(uint32_t) + 1024;
  e = cudaFuncSetAttribute(bwd_dq_tcm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dq);
  if (e != cudaSuccess) return e;
  bwd_dq_tcm_kernel<<<dim3(p.NT, D.Hq, D.B), NTHREADS, smem_dq, st>>>(mq, mk, mv, moc, mf, p);
  count_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (chunks > 1) e = launch_kvsum(D, a, a.kvpart, chunks, st);
  return e;
}

}  // namespace ssa
