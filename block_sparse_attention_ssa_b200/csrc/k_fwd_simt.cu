// CUDA-core dual-stream forward and dropped-mass kernels (fp32 arithmetic).
//
// This is the path for fp32 inputs (tensor cores have no fp32-input kind
// accurate enough for a 1e-4 tolerance) and for shapes outside the tensor-core
// kernel's envelope.
//
// What it computes ("SSA: Achieving Sparser Attention ...", "Practical
// Implementation of SSA"; "Technische Samenvatting: SSA", sections
// "1. Probleemstelling" and "Bidirectionele Uitlijning"): for each query t,
// two softmaxes over disjoint key sets, A_t (keys in selected blocks) and D_t
// (the other causal keys), are kept online side by side, each with its own
// running max, sum and output accumulator.  Tiles are 64 x 64; with blocks of
// 64 or more keys a tile lies in one query block and one key block and
// belongs wholly to A or to D, with smaller blocks (16, 32) every row carries
// a 64-bit mask of its selected keys in the tile and each weight goes to the
// accumulator of its own set.  At the end:
//   h_sparse = o_A / l_A,
//   h_full   = (e^{m_A-M} o_A + e^{m_D-M} o_D) / (e^{m_A-M} l_A + e^{m_D-M} l_D),
//   delta    = e^{lse_D - lse_full},  lse_full = logaddexp(lse_A, lse_D).
#include "ssa_internal.cuh"

namespace ssa {
namespace {

constexpr int BM = 64;   // query rows per CTA
constexpr int BN = 64;   // keys per tile
constexpr int NT = 256;  // threads

struct SimtShape {
  int Hq, g, N, s, n, k;
  float scale;
  int per_token;  // selection rows are tokens (1) or query blocks (0)
};

template <int D>
struct FwdSmem {
  float q[BM][D];
  float kt[D][BN];       // K tile, transposed
  float v[BN][D];
  float p[BM][BN + 1];   // logits, then the weights of set A
  float pd[BM][BN + 1];  // weights of set D
  float m[2][BM], l[2][BM], corr[2][BM];
  unsigned long long cm[BM];  // per row: keys of the tile in selected blocks (causal ones only)
  uint32_t sel[BM][64];       // selected-block bit sets: per query block of the tile, or per row
};

// o = corr * o + P V for the 4 x CW patch this thread owns.
template <int D, int CW>
__device__ __forceinline__ void pv_update(float (&o)[4][CW], const float (&cr)[4],
                                          const float (*p)[BN + 1], const float (*v)[D], int pr,
                                          int pc) {
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < CW; ++c) o[r][c] *= cr[r];
#pragma unroll 4
  for (int kk = 0; kk < BN; ++kk) {
    float pv[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) pv[r] = p[pr * 4 + r][kk];
#pragma unroll
    for (int c = 0; c < CW; ++c) {
      const float vv = v[kk][pc * CW + c];
#pragma unroll
      for (int r = 0; r < 4; ++r) o[r][c] = fmaf(pv[r], vv, o[r][c]);
    }
  }
}

template <typename T, int D, bool WITH_V>
__global__ void __launch_bounds__(NT) fwd_simt_kernel(FwdArgs a, SimtShape sh) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  FwdSmem<D>& S = *reinterpret_cast<FwdSmem<D>*>(smem_raw);
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / sh.g;
  const int t0 = qt * BM;
  const int ib0 = t0 / sh.s;                       // first query block of the tile
  const int nqb = sh.s >= BM ? 1 : BM / sh.s;      // query blocks in the tile
  const int tid = threadIdx.x;

  // Selected-block bits of the tile's selection rows: its query blocks, or
  // (per-token selection) its 64 tokens.
  for (int w = tid; w < BM * 64; w += NT) (&S.sel[0][0])[w] = 0u;
  __syncthreads();
  const int nsel = sh.per_token ? BM : nqb;
  for (int e = tid; e < nsel * sh.k; e += NT) {
    const int r = e / sh.k;
    const int64_t srow = sh.per_token ? (int64_t)t0 + r : (int64_t)ib0 + r;  // selection row within the head
    const int iblk = sh.per_token ? (t0 + r) / sh.s : ib0 + r;               // its query block
    const int j = a.idx[(((int64_t)b * sh.Hq + h) * (sh.per_token ? sh.N : sh.n) + srow) * sh.k + e % sh.k];
    if (j >= 0 && j <= iblk) atomicOr(&S.sel[r][j >> 5], 1u << (j & 31));
  }
  // Q tile -> fp32 smem.
  constexpr int VEC = Vec16<T>::kN;
  for (int e = tid; e < BM * D / VEC; e += NT) {
    const int r = e / (D / VEC), c = (e % (D / VEC)) * VEC;
    Vec16<T>::load(row_ptr<T>(a.q, b, h, t0 + r) + c, &S.q[r][c]);
  }
  if (tid < BM) {
    S.m[0][tid] = S.m[1][tid] = kNegInf;
    S.l[0][tid] = S.l[1][tid] = 0.f;
  }

  // PV ownership: rows pr*4..+3, columns pc*CW..+CW-1.
  constexpr int CW = D / 16;
  const int pr = tid / 16, pc = tid % 16;
  float oA[4][CW], oD[4][CW];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < CW; ++c) oA[r][c] = oD[r][c] = 0.f;

  // Score ownership: rows ty*4..+3, keys tx*4..+3.
  const int ty = tid / 16, tx = tid % 16;
  // Softmax ownership: row sr, 16 keys starting at sq*16.
  const int sr = tid / 4, sq = tid % 4;

  for (int kt = 0; kt <= qt; ++kt) {
    const int u0 = kt * BN;
    __syncthreads();  // previous tile fully consumed; sel bits visible
    bool myA = false, myD = false;
    if (tid < BM) {
      const unsigned long long causal = causal_mask(t0 + tid, u0);
      const int r = sh.per_token ? tid : (t0 + tid) / sh.s - ib0;
      const unsigned long long cm = tile_keep_mask(S.sel[r], u0, sh.s) & causal;
      S.cm[tid] = cm;
      myA = cm != 0ull;
      myD = (causal & ~cm) != 0ull;
    }
    const bool anyA = __syncthreads_or(myA), anyD = __syncthreads_or(myD);
    if (a.sparse_only && !anyA) continue;  // the sparse stream reads selected keys only
    for (int e = tid; e < BN * D / VEC; e += NT) {
      const int r = e / (D / VEC), c = (e % (D / VEC)) * VEC;
      float tmp[VEC];
      Vec16<T>::load(row_ptr<T>(a.k, b, kvh, u0 + r) + c, tmp);
#pragma unroll
      for (int x = 0; x < VEC; ++x) S.kt[c + x][r] = tmp[x];
      if (WITH_V) Vec16<T>::load(row_ptr<T>(a.v, b, kvh, u0 + r) + c, &S.v[r][c]);
    }
    __syncthreads();

    // x = scale * Q K^T for a 4x4 patch.
    float acc[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
#pragma unroll 8
    for (int c = 0; c < D; ++c) {
      const float4 kv = *reinterpret_cast<const float4*>(&S.kt[c][tx * 4]);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float qv = S.q[ty * 4 + r][c];
        acc[r][0] = fmaf(qv, kv.x, acc[r][0]);
        acc[r][1] = fmaf(qv, kv.y, acc[r][1]);
        acc[r][2] = fmaf(qv, kv.z, acc[r][2]);
        acc[r][3] = fmaf(qv, kv.w, acc[r][3]);
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int row = ty * 4 + r, col = tx * 4 + c;
        const bool ok = (u0 + col) <= (t0 + row);
        S.p[row][col] = ok ? sh.scale * acc[r][c] : kNegInf;
      }
    __syncthreads();

    // Online softmax update of both sets: each logit joins the set its key's
    // block belongs to for this row (causal mask already applied).
    {
      const unsigned long long cm = S.cm[sr] >> (sq * 16);
      float mA = kNegInf, mD = kNegInf;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float x = S.p[sr][sq * 16 + c];
        if ((cm >> c) & 1ull) mA = fmaxf(mA, x);
        else mD = fmaxf(mD, x);
      }
      mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 1));
      mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 2));
      mD = fmaxf(mD, __shfl_xor_sync(0xffffffffu, mD, 1));
      mD = fmaxf(mD, __shfl_xor_sync(0xffffffffu, mD, 2));
      const float oldA = S.m[0][sr], oldD = S.m[1][sr];
      const float newA = fmaxf(oldA, mA), newD = fmaxf(oldD, mD);
      float sumA = 0.f, sumD = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float x = S.p[sr][sq * 16 + c];
        float pA = 0.f, pD = 0.f;
        if (x != kNegInf) {
          if ((cm >> c) & 1ull) pA = expf(x - newA);
          else pD = expf(x - newD);
        }
        S.p[sr][sq * 16 + c] = pA;
        S.pd[sr][sq * 16 + c] = pD;
        sumA += pA;
        sumD += pD;
      }
      sumA += __shfl_xor_sync(0xffffffffu, sumA, 1);
      sumA += __shfl_xor_sync(0xffffffffu, sumA, 2);
      sumD += __shfl_xor_sync(0xffffffffu, sumD, 1);
      sumD += __shfl_xor_sync(0xffffffffu, sumD, 2);
      if (sq == 0) {
        const float cA = (oldA == kNegInf) ? 0.f : expf(oldA - newA);
        const float cD = (oldD == kNegInf) ? 0.f : expf(oldD - newD);
        S.corr[0][sr] = cA;
        S.corr[1][sr] = cD;
        S.l[0][sr] = S.l[0][sr] * cA + sumA;
        S.l[1][sr] = S.l[1][sr] * cD + sumD;
        S.m[0][sr] = newA;
        S.m[1][sr] = newD;
      }
    }
    __syncthreads();

    if (WITH_V) {
      // a set with no pair in this tile keeps its max (factor 1) and gains nothing
      float cr[4];
      if (anyA) {
#pragma unroll
        for (int r = 0; r < 4; ++r) cr[r] = S.corr[0][pr * 4 + r];
        pv_update<D, CW>(oA, cr, S.p, S.v, pr, pc);
      }
      if (anyD && !a.sparse_only) {
#pragma unroll
        for (int r = 0; r < 4; ++r) cr[r] = S.corr[1][pr * 4 + r];
        pv_update<D, CW>(oD, cr, S.pd, S.v, pr, pc);
      }
    }
  }
  __syncthreads();

  // Epilogue.
  if (WITH_V) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = pr * 4 + r;
      const float mA = S.m[0][row], lA = S.l[0][row], mD = S.m[1][row], lD = S.l[1][row];
      const float M = fmaxf(mA, mD);
      const float wa = (lA > 0.f) ? expf(mA - M) : 0.f;
      const float wd = (lD > 0.f) ? expf(mD - M) : 0.f;
      const float inv_full = 1.0f / (wa * lA + wd * lD);
      const float inv_sel = (lA > 0.f) ? 1.0f / lA : 0.f;
      T* hs = row_ptr_w<T>(a.hs, b, h, t0 + row) + pc * CW;
#pragma unroll
      for (int c = 0; c < CW; ++c) hs[c] = from_f32<T>(oA[r][c] * inv_sel);
      if (!a.sparse_only) {
        T* hf = row_ptr_w<T>(a.hf, b, h, t0 + row) + pc * CW;
#pragma unroll
        for (int c = 0; c < CW; ++c) hf[c] = from_f32<T>((wa * oA[r][c] + wd * oD[r][c]) * inv_full);
      }
    }
  }
  if (tid < BM) {
    const int row = tid;
    const int64_t o = ((int64_t)b * sh.Hq + h) * sh.N + t0 + row;
    const float mA = S.m[0][row], lA = S.l[0][row], mD = S.m[1][row], lD = S.l[1][row];
    const float lse_a = (lA > 0.f) ? mA + logf(lA) : kNegInf;
    const float lse_d = (lD > 0.f) ? mD + logf(lD) : kNegInf;
    const float hi = fmaxf(lse_a, lse_d), lo = fminf(lse_a, lse_d);
    const float lse_f = (lo == kNegInf) ? hi : hi + log1pf(expf(lo - hi));
    if (WITH_V) {
      a.lse_sel[o] = lse_a;
      if (!a.sparse_only) {
        a.lse_full[o] = lse_f;
        a.delta[o] = (lD > 0.f) ? expf(lse_d - lse_f) : 0.f;
      }
    } else if (a.lse_in != nullptr) {
      a.delta[o] = (lD > 0.f) ? lD * expf(mD - a.lse_in[o]) : 0.f;
    } else {
      a.delta[o] = (lD > 0.f) ? expf(lse_d - lse_f) : 0.f;
    }
  }
}

template <typename T, int D, bool WITH_V>
cudaError_t launch_t(const Dims& Dm, const FwdArgs& a, cudaStream_t st) {
  auto kern = fwd_simt_kernel<T, D, WITH_V>;
  const size_t smem = sizeof(FwdSmem<D>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  SimtShape sh{Dm.Hq, Dm.g, Dm.N, Dm.s, Dm.n, Dm.k, Dm.scale, Dm.per_token};
  dim3 grid(Dm.N / BM, Dm.Hq, Dm.B);
  kern<<<grid, NT, smem, st>>>(a, sh);
  count_launches(1);
  return cudaGetLastError();
}

template <bool WITH_V>
cudaError_t dispatch(const Dims& D, const FwdArgs& a, cudaStream_t st) {
  if (D.dtype == SSA_BF16)
    return D.d == 128 ? launch_t<__nv_bfloat16, 128, WITH_V>(D, a, st)
                      : launch_t<__nv_bfloat16, 64, WITH_V>(D, a, st);
  return D.d == 128 ? launch_t<float, 128, WITH_V>(D, a, st) : launch_t<float, 64, WITH_V>(D, a, st);
}

}  // namespace

cudaError_t launch_fwd_simt(const Dims& D, const FwdArgs& a, cudaStream_t st) {
  return dispatch<true>(D, a, st);
}

cudaError_t launch_dropped_simt(const Dims& D, const FwdArgs& a, cudaStream_t st) {
  return dispatch<false>(D, a, st);
}

}  // namespace ssa
