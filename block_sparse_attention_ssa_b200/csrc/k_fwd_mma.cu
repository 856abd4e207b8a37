// Warp-level tensor-core dual-stream forward and dropped-mass kernels
// (mma.sync m16n8k16, bf16 operands, fp32 accumulation and softmax).
//
// The bf16 path for the shapes the tcgen05 kernels do not take: head dim 64
// (the paper's models), blocks of 16 or 32 keys, and per-token selection.
// It computes what the CUDA-core kernels compute ("SSA: Achieving Sparser
// Attention ...", "Practical Implementation of SSA"; "Technische Samenvatting:
// SSA", "Bidirectionele Uitlijning"): for every query t two online softmaxes
// side by side, over A_t (causal keys in selected blocks) and over D_t (the
// other causal keys), each with its own running max, sum and accumulator, and
// at the end
//   h_sparse = o_A / l_A,
//   h_full   = (e^{m_A-M} o_A + e^{m_D-M} o_D) / (e^{m_A-M} l_A + e^{m_D-M} l_D),
//   delta    = e^{lse_D - lse_full}.
//
// CTA: 64 query rows (4 warps x 16 rows), key tiles of 64 double-buffered in
// shared memory with cp.async.  A warp computes its 16 x 64 logits with mma,
// keeps them in registers, routes every logit to its set with the row's
// kept-key bit mask (selected blocks, per block or per token, and causality),
// and multiplies the bf16 weights of each set by the V tile straight from the
// accumulator registers.  A 16-key step whose weights are all in one set
// skips the other set's product; in the sparse-only mode the CTA visits only
// key tiles that some of its rows selected and never reads the keys of blocks
// none of them selected (those rows are zero-filled in shared memory).
#include "mma_sync.cuh"
#include "ssa_internal.cuh"

namespace ssa {
namespace {

using namespace warp_mma;
using bf16 = __nv_bfloat16;

constexpr int BM = 64;   // query rows per CTA
constexpr int BN = 64;   // keys per tile
constexpr int NT = 128;  // 4 warps
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct MmaShape {
  int Hq, g, N, s, n, k;
  float scale;
  int per_token;
  int ls;  // log2 of the block size
};

template <int D>
struct Smem {
  static constexpr int LD = D + 8;  // row pitch: 8 ldmatrix rows hit 8 distinct 16-byte bank groups
  bf16 q[BM][LD];                   // Q tile; each warp's 16 rows double as its output staging
  bf16 k[2][BN][LD];
  bf16 v[2][BN][LD];
  unsigned long long cm[BM];        // per row: kept keys of the current tile (selected and causal)
  uint32_t uni[64];                 // union of the tile's selection rows
  uint32_t tiles[128];              // bit kt set: key tile kt is visited
  // followed by the selected-block bit sets, 64 words per selection row: one
  // row per query block of the tile, or (per-token selection) per query row
};

// Selection rows a CTA holds.
__host__ __device__ inline int sel_rows(int per_token, int s) { return per_token ? BM : (s >= BM ? 1 : BM / s); }

template <int D, bool WITH_V, bool SPARSE>
__global__ void __launch_bounds__(NT, D == 64 ? 4 : 2) fwd_mma_kernel(FwdArgs a, MmaShape sh) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Smem<D>& S = *reinterpret_cast<Smem<D>*>(smem_raw);
  uint32_t (*sel)[64] = reinterpret_cast<uint32_t (*)[64]>(smem_raw + sizeof(Smem<D>));
  const int qt = gridDim.x - 1 - blockIdx.x;  // the longest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / sh.g;
  const int t0 = qt * BM;
  const int ib0 = t0 / sh.s;
  const int nqb = sh.s >= BM ? 1 : BM / sh.s;
  const int nsel = sh.per_token ? BM : nqb;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int e = tid; e < BM * D / 8; e += NT) {
    const int r = e / (D / 8), c = (e % (D / 8)) * 8;
    cp_async16(&S.q[r][c], row_ptr<bf16>(a.q, b, h, t0 + r) + c, 16);
  }
  for (int w = tid; w < nsel * 64; w += NT) (&sel[0][0])[w] = 0u;
  if (tid < 64) S.uni[tid] = 0u;
  S.tiles[tid] = 0u;
  __syncthreads();
  for (int e = tid; e < nsel * sh.k; e += NT) {
    const int r = e / sh.k;
    const int64_t srow = sh.per_token ? (int64_t)t0 + r : (int64_t)ib0 + r;
    const int iblk = sh.per_token ? (t0 + r) / sh.s : ib0 + r;
    const int j = a.idx[(((int64_t)b * sh.Hq + h) * (sh.per_token ? sh.N : sh.n) + srow) * sh.k + e % sh.k];
    if (j >= 0 && j <= iblk) {
      atomicOr(&sel[r][j >> 5], 1u << (j & 31));
      if (SPARSE) atomicOr(&S.uni[j >> 5], 1u << (j & 31));
    }
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
  auto next_tile = [&](int from) -> int {  // first visited tile >= from, else -1
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
      if (WITH_V) cp_async16(&S.v[buf][r][c], row_ptr<bf16>(a.v, b, kvh, u0 + r) + c, bytes);
    }
  };

  int kt = next_tile(0);
  if (kt >= 0) load_kv(kt, 0);
  cp_async_commit();

  const int g = lane >> 2, q4 = lane & 3;
  const int r0 = warp * 16;
  const int rl[2] = {r0 + g, r0 + g + 8};
  const float sl2 = sh.scale * kLog2e;  // logits in log2 units
  float mA[2] = {kNegInf, kNegInf}, mD[2] = {kNegInf, kNegInf};
  float lA[2] = {0.f, 0.f}, lD[2] = {0.f, 0.f};  // this thread's share of the row sums
  constexpr int ND = SPARSE ? 1 : D / 8;  // the sparse stream keeps no o_D
  float oA[D / 8][4], oD[ND][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) oA[n][e] = 0.f;
#pragma unroll
  for (int n = 0; n < ND; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) oD[n][e] = 0.f;

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
    const unsigned long long cm0 = S.cm[rl[0]], cm1 = S.cm[rl[1]];
    // Warp-uniform shortcuts: none of the warp's pairs in this tile is
    // selected, or (off the diagonal) all of them are.
    const bool noneA = __all_sync(0xffffffffu, (cm0 | cm1) == 0ull);
    const bool allA = !diag && __all_sync(0xffffffffu, (cm0 & cm1) == ~0ull);
    // One set holds every logit of the warp: a plain online-softmax step.
    auto uniform = [&](auto& o, float (&m)[2], float (&l)[2], const float (&sc)[8][4]) {
      // row maxima as balanced trees (short dependency chains)
      float t0[8], t1[8], mx[2], c[2];
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        t0[n] = fmaxf(sc[n][0], sc[n][1]);
        t1[n] = fmaxf(sc[n][2], sc[n][3]);
      }
#pragma unroll
      for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
        for (int n = 0; n < w; ++n) {
          t0[n] = fmaxf(t0[n], t0[n + w]);
          t1[n] = fmaxf(t1[n], t1[n + w]);
        }
      mx[0] = t0[0];
      mx[1] = t1[0];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
        mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
        const float nm = fmaxf(m[i], mx[i] * sl2);
        c[i] = fast_ex2(m[i] - nm);
        m[i] = nm;
        l[i] *= c[i];
      }
      if (WITH_V && __any_sync(0xffffffffu, c[0] != 1.f || c[1] != 1.f)) {
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          o[n][0] *= c[0]; o[n][1] *= c[0];
          o[n][2] *= c[1]; o[n][3] *= c[1];
        }
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t pa[4];
        float w[2][4];
#pragma unroll
        for (int hn = 0; hn < 2; ++hn) {
#pragma unroll
          for (int e = 0; e < 4; ++e) w[hn][e] = fast_ex2(fmaf(sc[2 * kk + hn][e], sl2, -m[e >> 1]));
          pa[hn * 2] = pack2(w[hn][0], w[hn][1]);
          pa[hn * 2 + 1] = pack2(w[hn][2], w[hn][3]);
        }
        l[0] += (w[0][0] + w[0][1]) + (w[1][0] + w[1][1]);
        l[1] += (w[0][2] + w[0][3]) + (w[1][2] + w[1][3]);
        if (WITH_V) {
#pragma unroll
          for (int j = 0; j < D / 16; ++j) {
            uint32_t vb[4];
            ldsm_x4_t(vb, &S.v[buf][kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8][j * 16 + (lane >> 4) * 8]);
            mma16816(o[2 * j], pa, vb[0], vb[1]);
            mma16816(o[2 * j + 1], pa, vb[2], vb[3]);
          }
        }
      }
    };

    if (!(SPARSE && noneA)) {  // the sparse stream has nothing of this tile for the warp
      float sc[8][4];
  #pragma unroll
      for (int n = 0; n < 8; ++n)
  #pragma unroll
        for (int e = 0; e < 4; ++e) sc[n][e] = 0.f;
  #pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t qa[4];
        ldsm_x4(qa, &S.q[r0 + (lane & 15)][kk * 16 + (lane >> 4) * 8]);
  #pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t kb[4];
          ldsm_x4(kb, &S.k[buf][j * 16 + (lane & 7) + ((lane >> 4) << 3)][kk * 16 + ((lane >> 3) & 1) * 8]);
          mma16816(sc[2 * j], qa, kb[0], kb[1]);
          mma16816(sc[2 * j + 1], qa, kb[2], kb[3]);
        }
      }

      if (!diag && (allA || noneA)) {
        if (allA) {
          uniform(oA, mA, lA, sc);
        } else {
          if constexpr (!SPARSE) uniform(oD, mD, lD, sc);
        }
      } else {
        // Set membership of this thread's logits: bit nt*8 + (e & 1) of the
        // row's masks shifted by 2*q4 is the key of sc[nt][e].
        unsigned long long inA[2], inD[2];
    #pragma unroll
        for (int i = 0; i < 2; ++i) {
          const unsigned long long causal = diag ? (2ull << rl[i]) - 1ull : ~0ull;  // rl <= 63
          const unsigned long long cm = i ? cm1 : cm0;
          inA[i] = cm >> (2 * q4);
          inD[i] = (causal & ~cm) >> (2 * q4);
        }
        float mxA[2] = {kNegInf, kNegInf}, mxD[2] = {kNegInf, kNegInf};
    #pragma unroll
        for (int n = 0; n < 8; ++n)
    #pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = e >> 1, bit = n * 8 + (e & 1);
            const float x = sc[n][e] * sl2;
            sc[n][e] = x;
            if ((inA[i] >> bit) & 1ull) mxA[i] = fmaxf(mxA[i], x);
            if (!SPARSE && ((inD[i] >> bit) & 1ull)) mxD[i] = fmaxf(mxD[i], x);
          }
        float bA[2], bD[2], cA[2], cD[2];
    #pragma unroll
        for (int i = 0; i < 2; ++i) {
          mxA[i] = fmaxf(mxA[i], __shfl_xor_sync(0xffffffffu, mxA[i], 1));
          mxA[i] = fmaxf(mxA[i], __shfl_xor_sync(0xffffffffu, mxA[i], 2));
          const float nA = fmaxf(mA[i], mxA[i]);
          bA[i] = (nA == kNegInf) ? 0.f : nA;
          cA[i] = fast_ex2(mA[i] - bA[i]);
          mA[i] = nA;
          lA[i] *= cA[i];
          if (!SPARSE) {
            mxD[i] = fmaxf(mxD[i], __shfl_xor_sync(0xffffffffu, mxD[i], 1));
            mxD[i] = fmaxf(mxD[i], __shfl_xor_sync(0xffffffffu, mxD[i], 2));
            const float nD = fmaxf(mD[i], mxD[i]);
            bD[i] = (nD == kNegInf) ? 0.f : nD;
            cD[i] = fast_ex2(mD[i] - bD[i]);
            mD[i] = nD;
            lD[i] *= cD[i];
          }
        }
        if (WITH_V) {
          if (__any_sync(0xffffffffu, cA[0] != 1.f || cA[1] != 1.f)) {
    #pragma unroll
            for (int n = 0; n < D / 8; ++n) {
              oA[n][0] *= cA[0]; oA[n][1] *= cA[0];
              oA[n][2] *= cA[1]; oA[n][3] *= cA[1];
            }
          }
          if constexpr (!SPARSE) {
            if (__any_sync(0xffffffffu, cD[0] != 1.f || cD[1] != 1.f)) {
    #pragma unroll
              for (int n = 0; n < ND; ++n) {
                oD[n][0] *= cD[0]; oD[n][1] *= cD[0];
                oD[n][2] *= cD[1]; oD[n][3] *= cD[1];
              }
            }
          }
        }
        // Per 16-key step: the weights (one exponential per logit) packed as the
        // A operand, then P V for each set that has a weight in the step.
    #pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t pa[4], pd[4];
    #pragma unroll
          for (int hn = 0; hn < 2; ++hn) {
            const int n = 2 * kk + hn;
            float wA[4], wD[4];
    #pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = e >> 1, bit = n * 8 + (e & 1);
              const bool isA = (inA[i] >> bit) & 1ull;
              const bool isD = !SPARSE && ((inD[i] >> bit) & 1ull);
              const float p = fast_ex2(isA ? sc[n][e] - bA[i] : (isD ? sc[n][e] - bD[i] : kNegInf));
              wA[e] = isA ? p : 0.f;
              wD[e] = isA ? 0.f : p;
              lA[i] += wA[e];
              lD[i] += wD[e];
            }
            pa[hn * 2] = pack2(wA[0], wA[1]);
            pa[hn * 2 + 1] = pack2(wA[2], wA[3]);
            pd[hn * 2] = pack2(wD[0], wD[1]);
            pd[hn * 2 + 1] = pack2(wD[2], wD[3]);
          }
          if (WITH_V) {
            const unsigned long long stepbits = 0x303ull << (16 * kk);
            const bool useA = __any_sync(0xffffffffu, ((inA[0] | inA[1]) & stepbits) != 0ull);
            const bool useD = !SPARSE && __any_sync(0xffffffffu, ((inD[0] | inD[1]) & stepbits) != 0ull);
            if (!useA && !useD) continue;
    #pragma unroll
            for (int j = 0; j < D / 16; ++j) {
              uint32_t vb[4];
              ldsm_x4_t(vb, &S.v[buf][kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8][j * 16 + (lane >> 4) * 8]);
              if (useA) {
                mma16816(oA[2 * j], pa, vb[0], vb[1]);
                mma16816(oA[2 * j + 1], pa, vb[2], vb[3]);
              }
              if constexpr (!SPARSE) {
                if (useD) {
                  mma16816(oD[2 * j], pd, vb[0], vb[1]);
                  mma16816(oD[2 * j + 1], pd, vb[2], vb[3]);
                }
              }
            }
          }
        }
      }
    }
    __syncthreads();
    kt = nxt;
    ++it;
  }
  cp_async_wait<0>();
  __syncthreads();  // every Q copy has landed before a warp reuses its rows for staging

#pragma unroll
  for (int i = 0; i < 2; ++i) {
    lA[i] += __shfl_xor_sync(0xffffffffu, lA[i], 1);
    lA[i] += __shfl_xor_sync(0xffffffffu, lA[i], 2);
    lD[i] += __shfl_xor_sync(0xffffffffu, lD[i], 1);
    lD[i] += __shfl_xor_sync(0xffffffffu, lD[i], 2);
  }

  if (WITH_V) {
    float inv_s[2], wa[2], wd[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      inv_s[i] = lA[i] > 0.f ? 1.0f / lA[i] : 0.f;
      const float M = fmaxf(mA[i], mD[i]);
      wa[i] = lA[i] > 0.f ? fast_ex2(mA[i] - M) : 0.f;
      wd[i] = lD[i] > 0.f ? fast_ex2(mD[i] - M) : 0.f;
      const float inv_f = 1.0f / (wa[i] * lA[i] + wd[i] * lD[i]);
      wa[i] *= inv_f;
      wd[i] *= inv_f;
    }
    // h_sparse through the warp's own Q rows, then 16-byte row stores.
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
#pragma unroll
      for (int i = 0; i < 2; ++i)
        *reinterpret_cast<uint32_t*>(&S.q[rl[i]][n * 8 + 2 * q4]) =
            pack2(oA[n][2 * i] * inv_s[i], oA[n][2 * i + 1] * inv_s[i]);
    __syncwarp();
    for (int c = lane; c < 16 * D / 8; c += 32) {
      const int r = c / (D / 8), col = (c % (D / 8)) * 8;
      *reinterpret_cast<uint4*>(row_ptr_w<bf16>(a.hs, b, h, t0 + r0 + r) + col) =
          *reinterpret_cast<const uint4*>(&S.q[r0 + r][col]);
    }
    if constexpr (!SPARSE) {
      __syncwarp();
#pragma unroll
      for (int n = 0; n < ND; ++n)
#pragma unroll
        for (int i = 0; i < 2; ++i)
          *reinterpret_cast<uint32_t*>(&S.q[rl[i]][n * 8 + 2 * q4]) =
              pack2(wa[i] * oA[n][2 * i] + wd[i] * oD[n][2 * i], wa[i] * oA[n][2 * i + 1] + wd[i] * oD[n][2 * i + 1]);
      __syncwarp();
      for (int c = lane; c < 16 * D / 8; c += 32) {
        const int r = c / (D / 8), col = (c % (D / 8)) * 8;
        *reinterpret_cast<uint4*>(row_ptr_w<bf16>(a.hf, b, h, t0 + r0 + r) + col) =
            *reinterpret_cast<const uint4*>(&S.q[r0 + r][col]);
      }
    }
  }
  if (q4 == 0) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int64_t o = ((int64_t)b * sh.Hq + h) * sh.N + t0 + rl[i];
      const float lse_a = lA[i] > 0.f ? mA[i] * kLn2 + logf(lA[i]) : kNegInf;
      const float lse_d = lD[i] > 0.f ? mD[i] * kLn2 + logf(lD[i]) : kNegInf;
      const float hi = fmaxf(lse_a, lse_d), lo = fminf(lse_a, lse_d);
      const float lse_f = (lo == kNegInf) ? hi : hi + log1pf(expf(lo - hi));
      if (WITH_V) {
        a.lse_sel[o] = lse_a;
        if (!SPARSE) {
          a.lse_full[o] = lse_f;
          a.delta[o] = lD[i] > 0.f ? expf(lse_d - lse_f) : 0.f;
        }
      } else if (a.lse_in != nullptr) {
        a.delta[o] = lD[i] > 0.f ? lD[i] * expf(mD[i] * kLn2 - a.lse_in[o]) : 0.f;
      } else {
        a.delta[o] = lD[i] > 0.f ? expf(lse_d - lse_f) : 0.f;
      }
    }
  }
}

template <int D, bool WITH_V, bool SPARSE>
cudaError_t launch_t(const Dims& Dm, const FwdArgs& a, cudaStream_t st) {
  auto kern = fwd_mma_kernel<D, WITH_V, SPARSE>;
  const size_t smem = sizeof(Smem<D>) + (size_t)sel_rows(Dm.per_token, Dm.s) * 64 * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  MmaShape sh{Dm.Hq, Dm.g, Dm.N, Dm.s, Dm.n, Dm.k, Dm.scale, Dm.per_token, __builtin_ctz((unsigned)Dm.s)};
  dim3 grid(Dm.N / BM, Dm.Hq, Dm.B);
  kern<<<grid, NT, smem, st>>>(a, sh);
  count_launches(1);
  return cudaGetLastError();
}

template <int D>
cudaError_t dispatch(const Dims& Dm, const FwdArgs& a, bool with_v, cudaStream_t st) {
  if (!with_v) return launch_t<D, false, false>(Dm, a, st);
  return a.sparse_only ? launch_t<D, true, true>(Dm, a, st) : launch_t<D, true, false>(Dm, a, st);
}

}  // namespace

bool fwd_mma_supported(const Dims& D) { return D.dtype == SSA_BF16 && (D.d == 64 || D.d == 128); }

cudaError_t launch_fwd_mma(const Dims& D, const FwdArgs& a, cudaStream_t st) {
  return D.d == 128 ? dispatch<128>(D, a, true, st) : dispatch<64>(D, a, true, st);
}

cudaError_t launch_dropped_mma(const Dims& D, const FwdArgs& a, cudaStream_t st) {
  return D.d == 128 ? dispatch<128>(D, a, false, st) : dispatch<64>(D, a, false, st);
}

}  // namespace ssa
