// Warp-level tensor-core backward of both attention streams (mma.sync
// m16n8k16, bf16 operands, fp32 accumulation), for the bf16 shapes the
// tcgen05 backward does not take: head dim 64, blocks of 16 or 32 keys,
// per-token selection.
//
// Objective ("Technische Samenvatting: SSA", "Bidirectionele Uitlijning";
// "SSA: Achieving Sparser Attention ...", "Bidirectional Attention
// Alignment"): L = <g_f, h_full> + <g_s, h_sparse> + alpha (L_sp + L_cm), so
// dh_f = g_f + 2 alpha (h_f - h_s)/M and dh_s = g_s + 2 alpha (h_s - h_f)/M
// (M = B*Hq*N*d).  As in the CUDA-core kernels the two streams collapse into
// one softmax backward over the full stream's weights P = exp(x - lse_full):
// on A_t the sparse weights are r_t P with r_t = exp(lse_full - lse_sel), so
//   selected pair (u in A_t): dX = P (dO_c . v_u - D_c),  dV_u += P dO_c,
//   dropped pair  (u in D_t): dX = P (dh_f . v_u - D_f),  dV_u += P dh_f,
// with dO_c = dh_f + r dh_s, dQ_t = scale sum_u dX K_u, dK_u = scale sum_t dX Q_t.
//
// Launches:
//   pre  one warp per row: dh_f and dO_c rounded to bf16 (the operands the
//        products see), D_f = dh_f' . h_f and D_c = D_f + (dO_c' - dh_f') . h_s
//        from the rounded values, so that every row's dX still sums to zero
//        over its causal keys; partial sums of (h_f - h_s)^2;
//   dq   one 64-row query tile per CTA (4 warps x 16 rows) walking its key
//        tiles: S = Q K^T, dP_c = dO_c V^T and dP_f = dh_f V^T (each only on
//        the 8-key column groups that hold pairs of its set), dS in
//        registers, dQ += dS K;
//   dkv  one 64-key tile per CTA (4 warps x 16 keys) walking a chunk of at
//        most 4 query heads of its kv group and their query tiles:
//        S^T = K Q^T, dP^T = V dO^T, then dV += P_A^T dO_c + P_D^T dh_f and
//        dK += dS^T Q straight from the registers; with more than one chunk
//        per group each chunk writes fp32 partials that
//   kvsum adds in a fixed order (no atomics anywhere: bit-reproducible).
// In the sparse-only mode (hf = hs, lse_full = lse_sel, no g_f, alpha = 0)
// only selected pairs carry gradient, and both walks visit only the tiles
// that hold one.
#include <type_traits>

#include "mma_sync.cuh"
#include "ssa_internal.cuh"

namespace ssa {
namespace {

using namespace warp_mma;
using bf16 = __nv_bfloat16;

constexpr int BM = 64;   // query rows per tile
constexpr int BN = 64;   // keys per tile
constexpr int NT = 128;  // 4 warps
constexpr int kMaxHeadsPerCta = 4;
constexpr float kLog2e = 1.4426950408889634f;

struct MmaShape {
  int Hq, g, N, s, n, k;
  float scale;
  int per_token;
  int ls;     // log2 of the block size
  int words;  // 32-bit words per selection row
  int hpc;    // query heads per dK/dV CTA
};

__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(saddr(dst)), "l"(src) : "memory");
}

// OR of v over the warp.
__device__ __forceinline__ uint32_t warp_or(uint32_t v) { return __reduce_or_sync(0xffffffffu, v); }

// ================================================================ preprocess
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_mma_kernel(BwdArgs a, int Hq, int N, float c2, bf16* dhf_out,
                                                          bf16* doc_out) {
  constexpr int PER = D / 32;  // consecutive columns per lane
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t row = (int64_t)blockIdx.x * 8 + w;
  const int t = (int)(row % N), bh = (int)(row / N), b = bh / Hq, h = bh % Hq;
  const int c0 = lane * PER;
  auto load = [&](const TensorRef& ref, float (&x)[PER]) {
    const bf16* p = row_ptr<bf16>(ref, b, h, t) + c0;
#pragma unroll
    for (int e = 0; e < PER; ++e) x[e] = __bfloat162float(p[e]);
  };
  float xf[PER], xs[PER], gf[PER], gs[PER];
  load(a.hf, xf);
  load(a.hs, xs);
#pragma unroll
  for (int e = 0; e < PER; ++e) gf[e] = gs[e] = 0.f;
  if (a.gf.p) load(a.gf, gf);
  if (a.gs.p) load(a.gs, gs);
  const float lf = a.lse_full[row], ls = a.lse_sel[row];
  const float r = (ls == kNegInf) ? 0.f : expf(lf - ls);
  float sq = 0.f, df = 0.f, dx = 0.f;
  uint32_t of[PER / 2], oc[PER / 2];
#pragma unroll
  for (int e = 0; e < PER; e += 2) {
    float vf[2], vc[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float diff = xf[e + k] - xs[e + k];
      sq = fmaf(diff, diff, sq);
      vf[k] = gf[e + k] + c2 * diff;
      vc[k] = fmaf(r, gs[e + k] - c2 * diff, vf[k]);
    }
    of[e / 2] = pack2(vf[0], vf[1]);
    oc[e / 2] = pack2(vc[0], vc[1]);
    const float rf0 = __uint_as_float(of[e / 2] << 16), rf1 = __uint_as_float(of[e / 2] & 0xffff0000u);
    const float rc0 = __uint_as_float(oc[e / 2] << 16), rc1 = __uint_as_float(oc[e / 2] & 0xffff0000u);
    df = fmaf(rf0, xf[e], fmaf(rf1, xf[e + 1], df));
    dx = fmaf(rc0 - rf0, xs[e], fmaf(rc1 - rf1, xs[e + 1], dx));
  }
  uint32_t* pf = reinterpret_cast<uint32_t*>(dhf_out + row * D + c0);
  uint32_t* pc = reinterpret_cast<uint32_t*>(doc_out + row * D + c0);
#pragma unroll
  for (int e = 0; e < PER / 2; ++e) {
    pf[e] = of[e];
    pc[e] = oc[e];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    sq += __shfl_xor_sync(0xffffffffu, sq, off);
    df += __shfl_xor_sync(0xffffffffu, df, off);
    dx += __shfl_xor_sync(0xffffffffu, dx, off);
  }
  __shared__ float part[8];
  if (lane == 0) {
    a.Df[row] = df;
    a.Dc[row] = df + dx;
    part[w] = sq;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) s += part[q];
    a.partials[blockIdx.x] = s;
  }
}

// ================================================================ dQ
template <int D, bool SPARSE>
struct DqSmem {
  static constexpr int LD = D + 8;  // 8 ldmatrix rows fall in 8 distinct 16-byte bank groups
  bf16 q[BM][LD];                   // Q tile; each warp's rows double as its output staging
  bf16 doc[BM][LD];
  bf16 dhf[SPARSE ? 1 : BM][LD];
  bf16 k[2][BN][LD];
  bf16 v[2][BN][LD];
  unsigned long long cm[BM];        // per row: selected causal keys of the current key tile
  uint32_t uni[64];
  uint32_t tiles[128];              // bit kt: key tile kt is visited
  // followed by the tile's selection rows, 64 words each (one per query
  // block of the tile, or per query row with per-token selection)
};

__host__ __device__ inline int sel_rows(int per_token, int s) { return per_token ? BM : (s >= BM ? 1 : BM / s); }

template <int D, bool SPARSE>
__global__ void __launch_bounds__(NT, D == 64 ? 3 : 1)
    bwd_dq_mma_kernel(BwdArgs a, MmaShape sh, const bf16* __restrict__ dhf, const bf16* __restrict__ doc) {
  constexpr int NK = 32;  // keys per register sub-tile
  constexpr int NN = NK / 8;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  DqSmem<D, SPARSE>& S = *reinterpret_cast<DqSmem<D, SPARSE>*>(smem_raw);
  uint32_t (*sel)[64] = reinterpret_cast<uint32_t (*)[64]>(smem_raw + sizeof(DqSmem<D, SPARSE>));
  const int qt = gridDim.x - 1 - blockIdx.x;  // the longest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / sh.g;
  const int t0 = qt * BM;
  const int ib0 = t0 / sh.s;
  const int nqb = sh.s >= BM ? 1 : BM / sh.s;
  const int nsel = sh.per_token ? BM : nqb;
  const int rph = sh.per_token ? sh.N : sh.n;
  const int64_t rbase = ((int64_t)b * sh.Hq + h) * sh.N + t0;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int e = tid; e < BM * D / 8; e += NT) {
    const int r = e / (D / 8), c = (e % (D / 8)) * 8;
    cp_async16(&S.q[r][c], row_ptr<bf16>(a.q, b, h, t0 + r) + c, 16);
    cp_async16(&S.doc[r][c], doc + (rbase + r) * D + c, 16);
    if (!SPARSE) cp_async16(&S.dhf[r][c], dhf + (rbase + r) * D + c, 16);
  }
  for (int w = tid; w < nsel * 64; w += NT) (&sel[0][0])[w] = 0u;
  if (tid < 64) S.uni[tid] = 0u;
  S.tiles[tid] = 0u;
  __syncthreads();
  for (int e = tid; e < nsel * sh.words; e += NT) {
    const int r = e / sh.words, wi = e % sh.words;
    const int64_t mrow = sh.per_token ? (int64_t)t0 + r : (int64_t)ib0 + r;
    const uint32_t v = a.mask[(((int64_t)b * sh.Hq + h) * rph + mrow) * sh.words + wi];
    sel[r][wi] = v;
    if (SPARSE && v) atomicOr(&S.uni[wi], v);
  }
  __syncthreads();
  for (int kt = tid; kt <= qt; kt += NT) {
    bool need = true;
    if (SPARSE) {
      need = false;
      for (int j = kt * BN / sh.s; j <= (kt * BN + BN - 1) / sh.s; ++j) need |= (S.uni[j >> 5] >> (j & 31)) & 1u;
    }
    if (need) atomicOr(&S.tiles[kt >> 5], 1u << (kt & 31));
  }
  __syncthreads();

  const int ntw = qt / 32 + 1;
  auto next_tile = [&](int from) -> int {
    for (int w = from >> 5; w < ntw; ++w) {
      uint32_t bits = S.tiles[w];
      if (w == (from >> 5)) bits &= ~0u << (from & 31);
      if (bits) return w * 32 + __ffs(bits) - 1;
    }
    return -1;
  };
  auto load_kv = [&](int kt, int buf) {
    const int u0 = kt * BN;
    for (int e = tid; e < BN * D / 8; e += NT) {
      const int r = e / (D / 8), c = (e % (D / 8)) * 8;
      int bytes = 16;
      if (SPARSE && sh.s < BN) {
        const int j = (u0 + r) >> sh.ls;
        bytes = ((S.uni[j >> 5] >> (j & 31)) & 1u) ? 16 : 0;
      }
      cp_async16(&S.k[buf][r][c], row_ptr<bf16>(a.k, b, kvh, u0 + r) + c, bytes);
      cp_async16(&S.v[buf][r][c], row_ptr<bf16>(a.v, b, kvh, u0 + r) + c, bytes);
    }
  };

  int kt = next_tile(0);
  if (kt >= 0) load_kv(kt, 0);
  cp_async_commit();

  const int g = lane >> 2, q4 = lane & 3;
  const int r0 = warp * 16;
  const int rl[2] = {r0 + g, r0 + g + 8};
  const float sl2 = sh.scale * kLog2e;
  float lse2[2], Dc[2], Df[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    lse2[i] = a.lse_full[rbase + rl[i]] * kLog2e;
    Dc[i] = a.Dc[rbase + rl[i]];
    Df[i] = SPARSE ? 0.f : a.Df[rbase + rl[i]];
  }
  float dq[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dq[n][e] = 0.f;

  int it = 0;
  while (kt >= 0) {
    const int buf = it & 1;
    const int nxt = next_tile(kt + 1);
    if (nxt >= 0) load_kv(nxt, buf ^ 1);
    cp_async_commit();
    const int u0 = kt * BN;
    if (tid < BM) {
      const int rs = sh.per_token ? tid : ((t0 + tid) >> sh.ls) - ib0;
      S.cm[tid] = tile_keep_mask_p2(sel[rs], u0, sh.ls) & causal_mask(t0 + tid, u0);
    }
    cp_async_wait<1>();
    __syncthreads();

    const bool diag = (u0 == t0);
    unsigned long long cmr[2], dmr[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const unsigned long long causal = diag ? (2ull << rl[i]) - 1ull : ~0ull;
      cmr[i] = S.cm[rl[i]];
      dmr[i] = SPARSE ? 0ull : (causal & ~cmr[i]);
    }
    const bool noneA = __all_sync(0xffffffffu, (cmr[0] | cmr[1]) == 0ull);
    const bool allA = !diag && __all_sync(0xffffffffu, (cmr[0] & cmr[1]) == ~0ull);
    // MODE 0: both sets in the sub-tile (element-wise routing); 1: every pair
    // selected; 2: every pair dropped (both only off the diagonal).
    auto step = [&](auto mode, int ks) {
      constexpr int MODE = decltype(mode)::value;
      if constexpr (SPARSE && MODE == 2) return;
      const int sh0 = ks * NK + 2 * q4;  // bit (n*8 + (e&1)) of the shifted masks: key of element (n, e)
      unsigned long long inA[2] = {0ull, 0ull}, inD[2] = {0ull, 0ull};
      uint32_t fa = MODE == 1 ? (1u << NN) - 1u : 0u;  // bit n: the set has a pair in column group n
      uint32_t fd = MODE == 2 ? (1u << NN) - 1u : 0u;
      if constexpr (MODE == 0) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          inA[i] = cmr[i] >> sh0;
          inD[i] = dmr[i] >> sh0;
        }
#pragma unroll
        for (int n = 0; n < NN; ++n) {
          if (((inA[0] | inA[1]) >> (n * 8)) & 3ull) fa |= 1u << n;
          if (((inD[0] | inD[1]) >> (n * 8)) & 3ull) fd |= 1u << n;
        }
        fa = warp_or(fa);
        fd = warp_or(fd);
      }
      const uint32_t live = fa | fd;
      if (live == 0u) return;

      float sc[NN][4], dpc[NN][4];
      [[maybe_unused]] float dpf[SPARSE ? 1 : NN][4];
#pragma unroll
      for (int n = 0; n < NN; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[n][e] = dpc[n][e] = 0.f;
      if constexpr (!SPARSE) {
#pragma unroll
        for (int n = 0; n < NN; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) dpf[n][e] = 0.f;
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t qa[4], oa[4];
        [[maybe_unused]] uint32_t fa4[4];
        ldsm_x4(qa, &S.q[r0 + (lane & 15)][kk * 16 + (lane >> 4) * 8]);
        if (fa) ldsm_x4(oa, &S.doc[r0 + (lane & 15)][kk * 16 + (lane >> 4) * 8]);
        if constexpr (!SPARSE) {
          if (fd) ldsm_x4(fa4, &S.dhf[r0 + (lane & 15)][kk * 16 + (lane >> 4) * 8]);
        }
#pragma unroll
        for (int j = 0; j < NN / 2; ++j) {
          if (((live >> (2 * j)) & 3u) == 0u) continue;
          const int krow = ks * NK + j * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int kcol = kk * 16 + ((lane >> 3) & 1) * 8;
          uint32_t kb[4], vb[4];
          ldsm_x4(kb, &S.k[buf][krow][kcol]);
          ldsm_x4(vb, &S.v[buf][krow][kcol]);
#pragma unroll
          for (int hn = 0; hn < 2; ++hn) {
            const int n = 2 * j + hn;
            if ((live >> n) & 1u) mma16816(sc[n], qa, kb[2 * hn], kb[2 * hn + 1]);
            if ((fa >> n) & 1u) mma16816(dpc[n], oa, vb[2 * hn], vb[2 * hn + 1]);
            if constexpr (!SPARSE) {
              if ((fd >> n) & 1u) mma16816(dpf[n], fa4, vb[2 * hn], vb[2 * hn + 1]);
            }
          }
        }
      }
      // dS in registers, packed as the A operand of dS K.
      uint32_t da[NN / 2][4];
#pragma unroll
      for (int n = 0; n < NN; ++n) {
        float ds[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = e >> 1, bit = n * 8 + (e & 1);
          const bool isA = MODE == 1 || (MODE == 0 && ((inA[i] >> bit) & 1ull));
          const bool isD = !SPARSE && (MODE == 2 || (MODE == 0 && ((inD[i] >> bit) & 1ull)));
          const float p = fast_ex2((isA || isD) ? fmaf(sc[n][e], sl2, -lse2[i]) : kNegInf);
          float dpd = 0.f;
          if constexpr (!SPARSE) dpd = dpf[n][e];
          ds[e] = isA ? p * (dpc[n][e] - Dc[i]) : (isD ? p * (dpd - Df[i]) : 0.f);
        }
        da[n >> 1][(n & 1) * 2] = pack2(ds[0], ds[1]);
        da[n >> 1][(n & 1) * 2 + 1] = pack2(ds[2], ds[3]);
      }
#pragma unroll
      for (int kq = 0; kq < NN / 2; ++kq) {
        if (((live >> (2 * kq)) & 3u) == 0u) continue;
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
          uint32_t kb[4];
          ldsm_x4_t(kb, &S.k[buf][ks * NK + kq * 16 + (lane & 7) + ((lane >> 3) & 1) * 8][j * 16 + (lane >> 4) * 8]);
          mma16816(dq[2 * j], da[kq], kb[0], kb[1]);
          mma16816(dq[2 * j + 1], da[kq], kb[2], kb[3]);
        }
      }
    };
    if (!(SPARSE && noneA)) {
#pragma unroll
      for (int ks = 0; ks < BN / NK; ++ks) {
        if (allA) step(std::integral_constant<int, 1>{}, ks);
        else if (!SPARSE && noneA && !diag) step(std::integral_constant<int, 2>{}, ks);
        else step(std::integral_constant<int, 0>{}, ks);
      }
    }
    __syncthreads();
    kt = nxt;
    ++it;
  }
  cp_async_wait<0>();
  __syncthreads();

#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int i = 0; i < 2; ++i)
      *reinterpret_cast<uint32_t*>(&S.q[rl[i]][n * 8 + 2 * q4]) =
          pack2(sh.scale * dq[n][2 * i], sh.scale * dq[n][2 * i + 1]);
  __syncwarp();
  for (int c = lane; c < 16 * D / 8; c += 32) {
    const int r = c / (D / 8), col = (c % (D / 8)) * 8;
    *reinterpret_cast<uint4*>(row_ptr_w<bf16>(a.dq, b, h, t0 + r0 + r) + col) =
        *reinterpret_cast<const uint4*>(&S.q[r0 + r][col]);
  }
}

// ================================================================ dK, dV
template <int D, bool SPARSE>
struct DkvSmem {
  static constexpr int LD = D + 8;
  bf16 k[BN][LD];  // the CTA's keys; each warp's rows double as its dK staging
  bf16 v[BN][LD];  // and dV staging
  bf16 q[2][BM][LD];
  bf16 doc[2][BM][LD];
  bf16 dhf[SPARSE ? 1 : 2][BM][LD];
  float lse[2][BM], dc[2][BM], df[2][BM];
  uint32_t word[2][BM];  // per query row: its selection word that covers this key tile
  uint32_t tiles[kMaxHeadsPerCta * 128];  // sparse mode: bit hh*nq + (qt - kt): tile visited
};

template <int D, bool SPARSE>
__global__ void __launch_bounds__(NT, D == 64 ? 2 : 1)
    bwd_dkv_mma_kernel(BwdArgs a, MmaShape sh, const bf16* __restrict__ dhf, const bf16* __restrict__ doc,
                       float* __restrict__ part) {
  constexpr int NQ = 32;  // queries per register sub-tile
  constexpr int NN = NQ / 8;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  DkvSmem<D, SPARSE>& S = *reinterpret_cast<DkvSmem<D, SPARSE>*>(smem_raw);
  const int kt = blockIdx.x;  // the most query tiles first
  const int chunks = sh.g / sh.hpc;
  const int kvh = blockIdx.y / chunks, chunk = blockIdx.y % chunks;
  const int b = blockIdx.z;
  const int Hkv = sh.Hq / sh.g;
  const int u0 = kt * BN;
  const int nqt = sh.N / BM;
  const int nq = nqt - kt;  // causal query tiles of this key tile
  const int rph = sh.per_token ? sh.N : sh.n;
  const int jb = u0 / sh.s;                         // first key block of the tile
  const int wi = jb >> 5;                           // the selection word holding all of the tile's blocks
  const int nbt = sh.s >= BN ? 1 : BN / sh.s;
  const uint32_t tbm = ((nbt == 32 ? 0u : (1u << nbt)) - 1u) << (jb & 31);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int e = tid; e < BN * D / 8; e += NT) {
    const int r = e / (D / 8), c = (e % (D / 8)) * 8;
    cp_async16(&S.k[r][c], row_ptr<bf16>(a.k, b, kvh, u0 + r) + c, 16);
    cp_async16(&S.v[r][c], row_ptr<bf16>(a.v, b, kvh, u0 + r) + c, 16);
  }

  // Sparse mode: which (head, query tile) steps hold a selected pair.
  if (SPARSE) {
    for (int w = tid; w < sh.hpc * 128; w += NT) S.tiles[w] = 0u;
    __syncthreads();
    const int nrow = sh.per_token ? BM : (sh.s >= BM ? 1 : BM / sh.s);
    for (int e = tid; e < sh.hpc * nq; e += NT) {
      const int hh = e / nq, qt = kt + e % nq;
      const int h = (kvh * chunks + chunk) * sh.hpc + hh;
      const int t0 = qt * BM;
      const uint32_t* base = a.mask + ((int64_t)b * sh.Hq + h) * rph * sh.words + wi;
      uint32_t any = 0u;
      for (int r = 0; r < nrow && !any; ++r) {
        const int64_t mrow = sh.per_token ? (int64_t)t0 + r : (int64_t)t0 / sh.s + r;
        any = base[mrow * sh.words] & tbm;
      }
      if (any) atomicOr(&S.tiles[hh * 128 + ((e % nq) >> 5)], 1u << ((e % nq) & 31));
    }
    __syncthreads();
  }
  // Steps are numbered hh * nq + (qt - kt).
  const int nsteps = sh.hpc * nq;
  auto next_step = [&](int from) -> int {
    if constexpr (!SPARSE) {
      return from < nsteps ? from : -1;
    } else {
      while (from < nsteps) {
        const int hh = from / nq, x = from % nq;
        uint32_t bits = S.tiles[hh * 128 + (x >> 5)] & (~0u << (x & 31));
        if (bits) {
          const int y = (x & ~31) + __ffs(bits) - 1;
          if (y < nq) return hh * nq + y;
          from = (hh + 1) * nq;
        } else {
          from = ((x | 31) + 1 < nq) ? hh * nq + (x | 31) + 1 : (hh + 1) * nq;
        }
      }
      return -1;
    }
  };
  auto load_q = [&](int step, int buf) {
    const int hh = step / nq, qt = kt + step % nq;
    const int h = (kvh * chunks + chunk) * sh.hpc + hh;
    const int t0 = qt * BM;
    const int64_t rbase = ((int64_t)b * sh.Hq + h) * sh.N + t0;
    for (int e = tid; e < BM * D / 8; e += NT) {
      const int r = e / (D / 8), c = (e % (D / 8)) * 8;
      cp_async16(&S.q[buf][r][c], row_ptr<bf16>(a.q, b, h, t0 + r) + c, 16);
      cp_async16(&S.doc[buf][r][c], doc + (rbase + r) * D + c, 16);
      if (!SPARSE) cp_async16(&S.dhf[buf][r][c], dhf + (rbase + r) * D + c, 16);
    }
    if (tid < 48) {
      const int arr = tid / 16, c = (tid % 16) * 4;
      const float* src = arr == 0 ? a.lse_full : (arr == 1 ? a.Dc : a.Df);
      float* dst = arr == 0 ? S.lse[buf] : (arr == 1 ? S.dc[buf] : S.df[buf]);
      cp_async16(dst + c, src + rbase + c, 16);
    } else if (tid >= 64) {
      const int r = tid - 64;
      const int64_t mrow = sh.per_token ? (int64_t)t0 + r : (int64_t)((t0 + r) >> sh.ls);
      cp_async4(&S.word[buf][r], a.mask + (((int64_t)b * sh.Hq + h) * rph + mrow) * sh.words + wi);
    }
  };

  int step = next_step(0);
  if (step >= 0) load_q(step, 0);
  cp_async_commit();

  const int g = lane >> 2, q4 = lane & 3;
  const int r0 = warp * 16;
  const int kl[2] = {r0 + g, r0 + g + 8};                        // this thread's keys in the tile
  const int bp = ((u0 + r0) / sh.s) & 31;                         // their block's bit in a selection word
  const float sl2 = sh.scale * kLog2e;
  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;

  uint32_t kfr[D / 16][4], vfr[D / 16][4];  // the warp's K and V rows as A fragments, loaded once
  int it = 0;
  while (step >= 0) {
    const int buf = it & 1;
    const int nxt = next_step(step + 1);
    if (nxt >= 0) load_q(nxt, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const bool diag = (step % nq) == 0;  // query tile == key tile
    if (it == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        ldsm_x4(kfr[kk], &S.k[r0 + (lane & 15)][kk * 16 + (lane >> 4) * 8]);
        ldsm_x4(vfr[kk], &S.v[r0 + (lane & 15)][kk * 16 + (lane >> 4) * 8]);
      }
    }

    // The warp's 16 keys lie in one key block (blocks have 16 keys or more):
    // bit bp of a query row's selection word says whether that row selected it.
    const bool sel0 = (S.word[buf][lane] >> bp) & 1u, sel1 = (S.word[buf][lane + 32] >> bp) & 1u;
    const bool noneA = __all_sync(0xffffffffu, !sel0 && !sel1);
    const bool allA = !diag && __all_sync(0xffffffffu, sel0 && sel1);
    // MODE 0: both sets (element-wise routing); 1: every pair selected;
    // 2: every pair dropped (both only off the diagonal).
    auto step_q = [&](auto mode, int qs) {
      constexpr int MODE = decltype(mode)::value;
      if constexpr (SPARSE && MODE == 2) return;
      const int qb = qs * NQ;
      // Element (n, e): key kl[e >> 1], query qb + n*8 + 2*q4 + (e & 1).
      uint32_t mA = 0, mD = 0;  // bit n*4 + e
      uint32_t fa = MODE == 1 ? (1u << NN) - 1u : 0u, fd = MODE == 2 ? (1u << NN) - 1u : 0u;
      if constexpr (MODE == 0) {
#pragma unroll
        for (int n = 0; n < NN; ++n)
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            const int c = qb + n * 8 + 2 * q4 + c2;
            const bool sel = (S.word[buf][c] >> bp) & 1u;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const bool causal = !diag || kl[i] <= c;
              const int e = 2 * i + c2;
              if (causal && sel) mA |= 1u << (n * 4 + e);
              if (!SPARSE && causal && !sel) mD |= 1u << (n * 4 + e);
            }
          }
#pragma unroll
        for (int n = 0; n < NN; ++n) {
          if ((mA >> (n * 4)) & 15u) fa |= 1u << n;
          if ((mD >> (n * 4)) & 15u) fd |= 1u << n;
        }
        fa = warp_or(fa);
        fd = warp_or(fd);
      }
      const uint32_t live = fa | fd;
      if (live == 0u) return;

      float sc[NN][4], dpc[NN][4];
      [[maybe_unused]] float dpf[SPARSE ? 1 : NN][4];
#pragma unroll
      for (int n = 0; n < NN; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[n][e] = dpc[n][e] = 0.f;
      if constexpr (!SPARSE) {
#pragma unroll
        for (int n = 0; n < NN; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) dpf[n][e] = 0.f;
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t (&ka)[4] = kfr[kk];
        const uint32_t (&va)[4] = vfr[kk];
#pragma unroll
        for (int j = 0; j < NN / 2; ++j) {
          if (((live >> (2 * j)) & 3u) == 0u) continue;
          const int qrow = qb + j * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int qcol = kk * 16 + ((lane >> 3) & 1) * 8;
          uint32_t qf[4], of[4];
          [[maybe_unused]] uint32_t ff[4];
          ldsm_x4(qf, &S.q[buf][qrow][qcol]);
          if ((fa >> (2 * j)) & 3u) ldsm_x4(of, &S.doc[buf][qrow][qcol]);
          if constexpr (!SPARSE) {
            if ((fd >> (2 * j)) & 3u) ldsm_x4(ff, &S.dhf[buf][qrow][qcol]);
          }
#pragma unroll
          for (int hn = 0; hn < 2; ++hn) {
            const int n = 2 * j + hn;
            if ((live >> n) & 1u) mma16816(sc[n], ka, qf[2 * hn], qf[2 * hn + 1]);
            if ((fa >> n) & 1u) mma16816(dpc[n], va, of[2 * hn], of[2 * hn + 1]);
            if constexpr (!SPARSE) {
              if ((fd >> n) & 1u) mma16816(dpf[n], va, ff[2 * hn], ff[2 * hn + 1]);
            }
          }
        }
      }
      // P^T and dS^T in registers, packed as A operands over 16-query steps.
      uint32_t pA[NN / 2][4], dS[NN / 2][4];
      [[maybe_unused]] uint32_t pD[SPARSE ? 1 : NN / 2][4];
#pragma unroll
      for (int n = 0; n < NN; ++n) {
        float wA[4], wD[4], ds[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = qb + n * 8 + 2 * q4 + (e & 1);
          const bool isA = MODE == 1 || (MODE == 0 && ((mA >> (n * 4 + e)) & 1u));
          const bool isD = !SPARSE && (MODE == 2 || (MODE == 0 && ((mD >> (n * 4 + e)) & 1u)));
          const float p = fast_ex2((isA || isD) ? fmaf(sc[n][e], sl2, -S.lse[buf][c] * kLog2e) : kNegInf);
          float dpd = 0.f;
          if constexpr (!SPARSE) dpd = dpf[n][e];
          wA[e] = isA ? p : 0.f;
          wD[e] = isD ? p : 0.f;
          ds[e] = isA ? p * (dpc[n][e] - S.dc[buf][c]) : (isD ? p * (dpd - S.df[buf][c]) : 0.f);
        }
        pA[n >> 1][(n & 1) * 2] = pack2(wA[0], wA[1]);
        pA[n >> 1][(n & 1) * 2 + 1] = pack2(wA[2], wA[3]);
        if constexpr (!SPARSE) {
          pD[n >> 1][(n & 1) * 2] = pack2(wD[0], wD[1]);
          pD[n >> 1][(n & 1) * 2 + 1] = pack2(wD[2], wD[3]);
        }
        dS[n >> 1][(n & 1) * 2] = pack2(ds[0], ds[1]);
        dS[n >> 1][(n & 1) * 2 + 1] = pack2(ds[2], ds[3]);
      }
      // dV += P_A^T dO_c + P_D^T dh_f,  dK += dS^T Q  (B operands: [query][d] rows, transposed loads).
#pragma unroll
      for (int kq = 0; kq < NN / 2; ++kq) {
        const bool useL = (live >> (2 * kq)) & 3u;
        if (!useL) continue;
        const bool useA = (fa >> (2 * kq)) & 3u;
        [[maybe_unused]] const bool useD = !SPARSE && ((fd >> (2 * kq)) & 3u);
        const int qrow = qb + kq * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
          const int col = j * 16 + (lane >> 4) * 8;
          uint32_t qf[4];
          ldsm_x4_t(qf, &S.q[buf][qrow][col]);
          mma16816(dk[2 * j], dS[kq], qf[0], qf[1]);
          mma16816(dk[2 * j + 1], dS[kq], qf[2], qf[3]);
          if (useA) {
            uint32_t of[4];
            ldsm_x4_t(of, &S.doc[buf][qrow][col]);
            mma16816(dv[2 * j], pA[kq], of[0], of[1]);
            mma16816(dv[2 * j + 1], pA[kq], of[2], of[3]);
          }
          if constexpr (!SPARSE) {
            if (useD) {
              uint32_t ff[4];
              ldsm_x4_t(ff, &S.dhf[buf][qrow][col]);
              mma16816(dv[2 * j], pD[kq], ff[0], ff[1]);
              mma16816(dv[2 * j + 1], pD[kq], ff[2], ff[3]);
            }
          }
        }
      }
    };
    if (!(SPARSE && noneA)) {
#pragma unroll
      for (int qs = 0; qs < BM / NQ; ++qs) {
        if (allA) step_q(std::integral_constant<int, 1>{}, qs);
        else if (!SPARSE && noneA && !diag) step_q(std::integral_constant<int, 2>{}, qs);
        else step_q(std::integral_constant<int, 0>{}, qs);
      }
    }
    __syncthreads();
    step = nxt;
    ++it;
  }
  cp_async_wait<0>();
  __syncthreads();

  if (part == nullptr) {
    // One chunk per kv group: bf16 results through the warp's own K / V rows.
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        *reinterpret_cast<uint32_t*>(&S.k[kl[i]][n * 8 + 2 * q4]) =
            pack2(sh.scale * dk[n][2 * i], sh.scale * dk[n][2 * i + 1]);
        *reinterpret_cast<uint32_t*>(&S.v[kl[i]][n * 8 + 2 * q4]) = pack2(dv[n][2 * i], dv[n][2 * i + 1]);
      }
    __syncwarp();
    for (int c = lane; c < 16 * D / 8; c += 32) {
      const int r = c / (D / 8), col = (c % (D / 8)) * 8;
      *reinterpret_cast<uint4*>(row_ptr_w<bf16>(a.dk, b, kvh, u0 + r0 + r) + col) =
          *reinterpret_cast<const uint4*>(&S.k[r0 + r][col]);
      *reinterpret_cast<uint4*>(row_ptr_w<bf16>(a.dv, b, kvh, u0 + r0 + r) + col) =
          *reinterpret_cast<const uint4*>(&S.v[r0 + r][col]);
    }
  } else {
    // fp32 partials [chunk][2][B][Hkv][N][D] (dK unscaled, dV), added by kvsum.
    const int64_t plane = (int64_t)gridDim.z * Hkv * sh.N * D;
    float* pk = part + (int64_t)chunk * 2 * plane + (((int64_t)b * Hkv + kvh) * sh.N + u0) * D;
    float* pv = pk + plane;
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        *reinterpret_cast<float2*>(pk + (int64_t)kl[i] * D + n * 8 + 2 * q4) = make_float2(dk[n][2 * i], dk[n][2 * i + 1]);
        *reinterpret_cast<float2*>(pv + (int64_t)kl[i] * D + n * 8 + 2 * q4) = make_float2(dv[n][2 * i], dv[n][2 * i + 1]);
      }
  }
}

// dK = scale * sum_c part_k[c], dV = sum_c part_v[c], chunks added in order.
template <int D>
__global__ void __launch_bounds__(256) kvsum_kernel(const float* __restrict__ part, int chunks, int Hkv, int N,
                                                   float scale, TensorRef dk, TensorRef dv, int64_t plane) {
  const int64_t e = ((int64_t)blockIdx.x * 256 + threadIdx.x) * 4;  // first of 4 elements
  if (e >= plane) return;
  const int64_t row = e / D;
  const int c = (int)(e % D);
  const int t = (int)(row % N), bh = (int)(row / N), b = bh / Hkv, h = bh % Hkv;
  float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
  for (int q = 0; q < chunks; ++q) {
    const float4 xk = *reinterpret_cast<const float4*>(part + (int64_t)q * 2 * plane + e);
    const float4 xv = *reinterpret_cast<const float4*>(part + (int64_t)q * 2 * plane + plane + e);
    sk.x += xk.x; sk.y += xk.y; sk.z += xk.z; sk.w += xk.w;
    sv.x += xv.x; sv.y += xv.y; sv.z += xv.z; sv.w += xv.w;
  }
  bf16* ok = row_ptr_w<bf16>(dk, b, h, t) + c;
  bf16* ov = row_ptr_w<bf16>(dv, b, h, t) + c;
  *reinterpret_cast<uint2*>(ok) = make_uint2(pack2(scale * sk.x, scale * sk.y), pack2(scale * sk.z, scale * sk.w));
  *reinterpret_cast<uint2*>(ov) = make_uint2(pack2(sv.x, sv.y), pack2(sv.z, sv.w));
}

template <int D, bool SPARSE>
cudaError_t bwd_t(const Dims& Dm, const BwdArgs& a, const bf16* dhf, const bf16* doc, cudaStream_t st) {
  MmaShape sh{Dm.Hq, Dm.g, Dm.N, Dm.s, Dm.n, Dm.k, Dm.scale, Dm.per_token, __builtin_ctz((unsigned)Dm.s),
              a.words, bwd_mma_heads_per_cta(Dm)};
  const int chunks = Dm.g / sh.hpc;
  auto kdq = bwd_dq_mma_kernel<D, SPARSE>;
  auto kkv = bwd_dkv_mma_kernel<D, SPARSE>;
  const size_t sq = sizeof(DqSmem<D, SPARSE>) + (size_t)sel_rows(Dm.per_token, Dm.s) * 64 * sizeof(uint32_t);
  const size_t skv = sizeof(DkvSmem<D, SPARSE>);
  cudaError_t e = cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sq);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)skv);
  if (e != cudaSuccess) return e;
  float* part = chunks > 1 ? a.kvpart : nullptr;
  kkv<<<dim3(Dm.N / BN, Dm.Hkv * chunks, Dm.B), NT, skv, st>>>(a, sh, dhf, doc, part);
  count_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  kdq<<<dim3(Dm.N / BM, Dm.Hq, Dm.B), NT, sq, st>>>(a, sh, dhf, doc);
  count_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (part != nullptr) {
    const int64_t plane = (int64_t)Dm.B * Dm.Hkv * Dm.N * D;
    const unsigned blocks = (unsigned)((plane / 4 + 255) / 256);
    kvsum_kernel<D><<<blocks, 256, 0, st>>>(part, chunks, Dm.Hkv, Dm.N, Dm.scale, a.dk, a.dv, plane);
    count_launches(1);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace

bool bwd_mma_supported(const Dims& D) { return D.dtype == SSA_BF16 && (D.d == 64 || D.d == 128); }

int bwd_mma_heads_per_cta(const Dims& D) {
  // The smallest number of chunks that leaves at most kMaxHeadsPerCta heads
  // per CTA: enough CTAs per key tile to balance the causal triangle.
  for (int chunks = 1; chunks <= D.g; ++chunks)
    if (D.g % chunks == 0 && D.g / chunks <= kMaxHeadsPerCta) return D.g / chunks;
  return 1;
}

size_t bwd_mma_partial_bytes(const Dims& D) {
  const int chunks = D.g / bwd_mma_heads_per_cta(D);
  if (chunks <= 1) return 0;
  return (size_t)chunks * 2 * D.B * D.Hkv * D.N * D.d * sizeof(float);
}

cudaError_t launch_kvsum(const Dims& D, const BwdArgs& a, const float* part, int chunks, cudaStream_t st) {
  const int64_t plane = (int64_t)D.B * D.Hkv * D.N * D.d;
  const unsigned blocks = (unsigned)((plane / 4 + 255) / 256);
  if (D.d == 128) kvsum_kernel<128><<<blocks, 256, 0, st>>>(part, chunks, D.Hkv, D.N, D.scale, a.dk, a.dv, plane);
  else kvsum_kernel<64><<<blocks, 256, 0, st>>>(part, chunks, D.Hkv, D.N, D.scale, a.dk, a.dv, plane);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_bwd_mma(const Dims& D, const BwdArgs& a, int32_t* status, cudaStream_t st) {
  // The fp32 dh_f / dO_c workspace regions hold the bf16 operands in their
  // lower halves.
  bf16* dhf = reinterpret_cast<bf16*>(a.dhf);
  bf16* doc = reinterpret_cast<bf16*>(a.doc);
  const double M = (double)D.B * D.Hq * D.N * D.d;
  const float c2 = (float)(2.0 * (double)a.alpha / M);
  const unsigned blocks = (unsigned)sqdiff_partial_count(D);
  if (D.d == 128) bwd_pre_mma_kernel<128><<<blocks, 256, 0, st>>>(a, D.Hq, D.N, c2, dhf, doc);
  else bwd_pre_mma_kernel<64><<<blocks, 256, 0, st>>>(a, D.Hq, D.N, c2, dhf, doc);
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.align_loss != nullptr) {
    e = launch_finish_mean(a.partials, a.n_partials, M, 2.0f, a.align_loss, 1, st);
    if (e != cudaSuccess) return e;
  }
  // Dual backward at d = 64: the tcgen05 kernels with per-row masks.
  if (!a.sparse_only && bwd_tcm_supported(D))
    return launch_bwd_tcm(D, a, dhf, doc, bwd_mma_heads_per_cta(D), status, st);
  if (D.d == 128)
    return a.sparse_only ? bwd_t<128, true>(D, a, dhf, doc, st) : bwd_t<128, false>(D, a, dhf, doc, st);
  return a.sparse_only ? bwd_t<64, true>(D, a, dhf, doc, st) : bwd_t<64, false>(D, a, dhf, doc, st);
}

}  // namespace ssa
