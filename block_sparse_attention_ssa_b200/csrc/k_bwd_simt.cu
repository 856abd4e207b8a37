// Backward of both attention streams with the alignment loss folded in.
//
// Objective ("Technische Samenvatting: SSA", "Bidirectionele Uitlijning";
// "SSA: Achieving Sparser Attention ...", "Bidirectional Attention
// Alignment"):  L = <g_f, h_full> + <g_s, h_sparse> + alpha (L_sp + L_cm),
// L_sp = mean((h_full - sg h_sparse)^2), L_cm = mean((h_sparse - sg h_full)^2).
// With M = B*Hq*N*d:
//   dh_f = g_f + 2 alpha (h_f - h_s) / M,   dh_s = g_s + 2 alpha (h_s - h_f) / M.
//
// One combined pass.  On A_t the sparse softmax is a rescaled copy of the full
// one, P_s = r_t P_f with r_t = exp(lse_full - lse_sel) = 1 / (1 - delta_t), so
// the two streams' contributions collapse into a single softmax backward:
//   selected key u (u in A_t):  dX = P_f (dO_c . v_u - D_c),  dV_u += P_f dO_c,
//   dropped key u  (u in D_t):  dX = P_f (dh_f . v_u - D_f),  dV_u += P_f dh_f,
// with dO_c = dh_f + r dh_s, D_f = dh_f . h_f, D_c = D_f + r dh_s . h_s, and
// dQ_t = scale sum_u dX K_u, dK_u = scale sum_t dX Q_t.  The selection is held
// fixed (no gradient through idx or delta).
#include "ssa_internal.cuh"

namespace ssa {
namespace {

constexpr int NT = 256;
constexpr int BT = 64;  // tile edge (query rows / keys)

// ------------------------------------------------------------------ preprocess
// One warp per row (b, h, t); 8 rows per CTA.  Also leaves one partial sum of
// (h_f - h_s)^2 per CTA for the alignment loss (fixed-order reduction later).
template <typename T, int D>
__global__ void __launch_bounds__(NT) bwd_pre_kernel(BwdArgs a, int Hq, int N, float c2) {
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t row = (int64_t)blockIdx.x * 8 + w;  // row in [0, B*Hq*N)
  const int t = (int)(row % N);
  const int bh = (int)(row / N);
  const int b = bh / Hq, h = bh % Hq;
  const T* hf = row_ptr<T>(a.hf, b, h, t);
  const T* hs = row_ptr<T>(a.hs, b, h, t);
  const T* gf = a.gf.p ? row_ptr<T>(a.gf, b, h, t) : nullptr;
  const T* gs = a.gs.p ? row_ptr<T>(a.gs, b, h, t) : nullptr;
  const float lf = a.lse_full[row], ls = a.lse_sel[row];
  const float r = (ls == kNegInf) ? 0.f : expf(lf - ls);
  float sq = 0.f, df = 0.f, ds = 0.f;
  float* dhf = a.dhf + row * D;
  float* doc = a.doc + row * D;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const int c = lane + 32 * e;
    const float xf = to_f32(hf[c]), xs = to_f32(hs[c]);
    const float diff = xf - xs;
    sq = fmaf(diff, diff, sq);
    const float vf = (gf ? to_f32(gf[c]) : 0.f) + c2 * diff;
    const float vs = (gs ? to_f32(gs[c]) : 0.f) - c2 * diff;
    df = fmaf(vf, xf, df);
    ds = fmaf(vs, xs, ds);
    dhf[c] = vf;
    doc[c] = fmaf(r, vs, vf);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    sq += __shfl_xor_sync(0xffffffffu, sq, off);
    df += __shfl_xor_sync(0xffffffffu, df, off);
    ds += __shfl_xor_sync(0xffffffffu, ds, off);
  }
  __shared__ float part[8];
  if (lane == 0) {
    a.Df[row] = df;
    a.Dc[row] = fmaf(r, ds, df);
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

// ------------------------------------------------------------------ dQ
// grid (N/64, Hq, B).  For its 64 query rows the CTA walks every causal key
// tile.  With blocks of 64 or more keys a tile belongs to A or to D for all
// 64 rows; with smaller blocks each row's 64-bit mask of selected keys picks,
// element by element, the combined (dO_c, D_c) or the full-stream
// (dh_f, D_f) gradient.

template <int D>
struct DqSmem {
  float q[BT][D];
  float doc[BT][D];
  float dhf[BT][D];
  float k[BT][D + 1];
  float v[BT][D + 1];
  float p[BT][BT + 1];
  float lse[BT], dc[BT], df[BT];
  unsigned long long cm[BT];  // per query row: keys of the tile in selected blocks
};

// xs = Q K^T, dpc = dO_c V^T, dpf = dh_f V^T for a 4 x 4 patch (only the
// products a tile needs).
template <int D, bool NC, bool NF>
__device__ __forceinline__ void dq_dots(const DqSmem<D>& S, int ty, int tx, float (&xs)[4][4], float (&dpc)[4][4],
                                        float (&dpf)[4][4]) {
#pragma unroll 4
  for (int c = 0; c < D; ++c) {
    float kv[4], vv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      kv[j] = S.k[tx * 4 + j][c];
      vv[j] = S.v[tx * 4 + j][c];
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float qv = S.q[ty * 4 + r][c];
      const float oc = NC ? S.doc[ty * 4 + r][c] : 0.f;
      const float of = NF ? S.dhf[ty * 4 + r][c] : 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        xs[r][j] = fmaf(qv, kv[j], xs[r][j]);
        if (NC) dpc[r][j] = fmaf(oc, vv[j], dpc[r][j]);
        if (NF) dpf[r][j] = fmaf(of, vv[j], dpf[r][j]);
      }
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(NT) bwd_dq_kernel(BwdArgs a, int Hq, int g, int N, int s, int n,
                                                   float scale, int per_token) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  DqSmem<D>& S = *reinterpret_cast<DqSmem<D>*>(smem_raw);
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z, kvh = h / g;
  const int t0 = qt * BT, tid = threadIdx.x;
  const int64_t rbase = ((int64_t)b * Hq + h) * N + t0;
  const int rph = per_token ? N : n;  // selection rows per head
  constexpr int VEC = Vec16<T>::kN;

  for (int e = tid; e < BT * D / VEC; e += NT) {
    const int r = e / (D / VEC), c = (e % (D / VEC)) * VEC;
    Vec16<T>::load(row_ptr<T>(a.q, b, h, t0 + r) + c, &S.q[r][c]);
  }
  for (int e = tid; e < BT * D; e += NT) {
    const int r = e / D, c = e % D;
    S.doc[r][c] = a.doc[(rbase + r) * D + c];
    S.dhf[r][c] = a.dhf[(rbase + r) * D + c];
  }
  if (tid < BT) {
    S.lse[tid] = a.lse_full[rbase + tid];
    S.dc[tid] = a.Dc[rbase + tid];
    S.df[tid] = a.Df[rbase + tid];
  }

  constexpr int CW = D / 16;
  const int pr = tid / 16, pc = tid % 16;  // dQ patch: rows pr*4.., cols pc*CW..
  const int ty = tid / 16, tx = tid % 16;  // score patch: rows ty*4.., keys tx*4..
  float dq[4][CW];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < CW; ++c) dq[r][c] = 0.f;

  for (int kt = 0; kt <= qt; ++kt) {
    const int u0 = kt * BT;
    __syncthreads();
    bool myA = false, myD = false;
    if (tid < BT) {
      const int t = t0 + tid;
      const uint32_t* blocks = a.mask + (((int64_t)b * Hq + h) * rph + (per_token ? t : t / s)) * a.words;
      const unsigned long long causal = causal_mask(t, u0);
      const unsigned long long cm = tile_keep_mask(blocks, u0, s) & causal;
      S.cm[tid] = cm;
      myA = cm != 0ull;
      myD = (causal & ~cm) != 0ull;
    }
    const bool anyA = __syncthreads_or(myA);
    const bool anyD = __syncthreads_or(myD) && !a.sparse_only;  // dropped pairs: no sparse-stream gradient
    if (!anyA && !anyD) continue;  // uniform over the CTA
    for (int e = tid; e < BT * D / VEC; e += NT) {
      const int r = e / (D / VEC), c = (e % (D / VEC)) * VEC;
      float tk[VEC], tv[VEC];
      Vec16<T>::load(row_ptr<T>(a.k, b, kvh, u0 + r) + c, tk);
      Vec16<T>::load(row_ptr<T>(a.v, b, kvh, u0 + r) + c, tv);
#pragma unroll
      for (int x = 0; x < VEC; ++x) {
        S.k[r][c + x] = tk[x];
        S.v[r][c + x] = tv[x];
      }
    }
    __syncthreads();
    float xs[4][4], dpc[4][4], dpf[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) xs[r][c] = dpc[r][c] = dpf[r][c] = 0.f;
    if (anyA && anyD) dq_dots<D, true, true>(S, ty, tx, xs, dpc, dpf);
    else if (anyA) dq_dots<D, true, false>(S, ty, tx, xs, dpc, dpf);
    else dq_dots<D, false, true>(S, ty, tx, xs, dpc, dpf);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = ty * 4 + r;
      const unsigned long long cm = S.cm[row];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = tx * 4 + j;
        float ds = 0.f;
        if (u0 + col <= t0 + row) {
          const bool in_a = (cm >> col) & 1ull;
          if (in_a || anyD) {
            const float p = expf(scale * xs[r][j] - S.lse[row]);
            ds = in_a ? p * (dpc[r][j] - S.dc[row]) : p * (dpf[r][j] - S.df[row]);
          }
        }
        S.p[row][col] = ds;
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < BT; ++kk) {
      float dsv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) dsv[r] = S.p[pr * 4 + r][kk];
#pragma unroll
      for (int c = 0; c < CW; ++c) {
        const float kv = S.k[kk][pc * CW + c];
#pragma unroll
        for (int r = 0; r < 4; ++r) dq[r][c] = fmaf(dsv[r], kv, dq[r][c]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    T* out = row_ptr_w<T>(a.dq, b, h, t0 + pr * 4 + r) + pc * CW;
#pragma unroll
    for (int c = 0; c < CW; ++c) out[c] = from_f32<T>(scale * dq[r][c]);
  }
}

// ------------------------------------------------------------------ dK, dV
// grid (N/64, Hkv, B).  For its 64 keys the CTA walks the g query heads of the
// group and every causal query tile.  Each query row's 64-bit mask of
// selected keys (from its query block's bit set) decides, element by
// element, whether the pair is selected (combined gradient dO_c, D_c) or
// dropped (dh_f, D_f); dV takes P_A^T dO_c + P_D^T dh_f.
template <int D>
struct DkvSmem {
  float k[BT][D + 1];
  float v[BT][D + 1];
  float q[BT][D + 1];
  float doc[BT][D + 1];
  float dhf[BT][D + 1];
  float p[BT][BT + 1];   // P^T on selected pairs: [key][query]
  float pd[BT][BT + 1];  // P^T on dropped pairs
  float ds[BT][BT + 1];  // dS^T
  float lse[BT], dc[BT], df[BT];
  unsigned long long cm[BT];  // per query row: keys of this tile in selected blocks (causal ones)
};

template <int D, bool NC, bool NF>
__device__ __forceinline__ void dkv_dots(const DkvSmem<D>& S, int ty, int tx, float (&xs)[4][4],
                                         float (&dpc)[4][4], float (&dpf)[4][4]) {
#pragma unroll 4
  for (int c = 0; c < D; ++c) {
    float qv[4], oc[4], of[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      qv[j] = S.q[tx * 4 + j][c];
      oc[j] = NC ? S.doc[tx * 4 + j][c] : 0.f;
      of[j] = NF ? S.dhf[tx * 4 + j][c] : 0.f;
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float kv = S.k[ty * 4 + r][c];
      const float vv = S.v[ty * 4 + r][c];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        xs[r][j] = fmaf(kv, qv[j], xs[r][j]);
        if (NC) dpc[r][j] = fmaf(vv, oc[j], dpc[r][j]);
        if (NF) dpf[r][j] = fmaf(vv, of[j], dpf[r][j]);
      }
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(NT) bwd_dkv_kernel(BwdArgs a, int Hq, int g, int N, int s, int n,
                                                    float scale, int per_token) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  DkvSmem<D>& S = *reinterpret_cast<DkvSmem<D>*>(smem_raw);
  const int kt = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int u0 = kt * BT, tid = threadIdx.x;
  const int nqt = N / BT;
  constexpr int VEC = Vec16<T>::kN;
  for (int e = tid; e < BT * D / VEC; e += NT) {
    const int r = e / (D / VEC), c = (e % (D / VEC)) * VEC;
    float tk[VEC], tv[VEC];
    Vec16<T>::load(row_ptr<T>(a.k, b, kvh, u0 + r) + c, tk);
    Vec16<T>::load(row_ptr<T>(a.v, b, kvh, u0 + r) + c, tv);
#pragma unroll
    for (int x = 0; x < VEC; ++x) {
      S.k[r][c + x] = tk[x];
      S.v[r][c + x] = tv[x];
    }
  }
  constexpr int CW = D / 16;
  const int pr = tid / 16, pc = tid % 16;  // dK/dV patch: keys pr*4.., cols pc*CW..
  const int ty = tid / 16, tx = tid % 16;  // S^T patch: keys ty*4.., queries tx*4..
  float dk[4][CW], dv[4][CW];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < CW; ++c) dk[r][c] = dv[r][c] = 0.f;

  for (int hh = 0; hh < g; ++hh) {
    const int h = kvh * g + hh;
    for (int qt = kt; qt < nqt; ++qt) {
      const int t0 = qt * BT;
      const int64_t rbase = ((int64_t)b * Hq + h) * N + t0;
      __syncthreads();
      bool myA = false, myD = false;
      if (tid < BT) {
        const int t = t0 + tid;
        const uint32_t* blocks =
            a.mask + (((int64_t)b * Hq + h) * (per_token ? N : n) + (per_token ? t : t / s)) * a.words;
        const unsigned long long causal = causal_mask(t, u0);
        const unsigned long long cm = tile_keep_mask(blocks, u0, s) & causal;
        S.cm[tid] = cm;
        myA = cm != 0ull;
        myD = (causal & ~cm) != 0ull;
      }
      const bool anyA = __syncthreads_or(myA);
      const bool anyD = __syncthreads_or(myD) && !a.sparse_only;  // dropped pairs: no sparse-stream gradient
      if (!anyA && !anyD) continue;  // uniform over the CTA
      for (int e = tid; e < BT * D / VEC; e += NT) {
        const int r = e / (D / VEC), c = (e % (D / VEC)) * VEC;
        float tq[VEC];
        Vec16<T>::load(row_ptr<T>(a.q, b, h, t0 + r) + c, tq);
#pragma unroll
        for (int x = 0; x < VEC; ++x) S.q[r][c + x] = tq[x];
      }
      for (int e = tid; e < BT * D; e += NT) {
        const int r = e / D, c = e % D;
        if (anyA) S.doc[r][c] = a.doc[(rbase + r) * D + c];
        if (anyD) S.dhf[r][c] = a.dhf[(rbase + r) * D + c];
      }
      if (tid < BT) {
        S.lse[tid] = a.lse_full[rbase + tid];
        S.dc[tid] = a.Dc[rbase + tid];
        S.df[tid] = a.Df[rbase + tid];
      }
      __syncthreads();
      float xs[4][4], dpc[4][4], dpf[4][4];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) xs[r][c] = dpc[r][c] = dpf[r][c] = 0.f;
      if (anyA && anyD) dkv_dots<D, true, true>(S, ty, tx, xs, dpc, dpf);
      else if (anyA) dkv_dots<D, true, false>(S, ty, tx, xs, dpc, dpf);
      else dkv_dots<D, false, true>(S, ty, tx, xs, dpc, dpf);
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int key = ty * 4 + r, qr = tx * 4 + j;
          float pa = 0.f, pdv = 0.f, ds = 0.f;
          if (u0 + key <= t0 + qr) {
            const bool in_a = (S.cm[qr] >> key) & 1ull;
            if (in_a || anyD) {
              const float p = expf(scale * xs[r][j] - S.lse[qr]);
              if (in_a) {
                pa = p;
                ds = p * (dpc[r][j] - S.dc[qr]);
              } else {
                pdv = p;
                ds = p * (dpf[r][j] - S.df[qr]);
              }
            }
          }
          S.p[key][qr] = pa;
          S.pd[key][qr] = pdv;
          S.ds[key][qr] = ds;
        }
      __syncthreads();
#pragma unroll 4
      for (int qq = 0; qq < BT; ++qq) {
        float pv[4], pdv[4], dsv[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          pv[r] = S.p[pr * 4 + r][qq];
          pdv[r] = S.pd[pr * 4 + r][qq];
          dsv[r] = S.ds[pr * 4 + r][qq];
        }
#pragma unroll
        for (int c = 0; c < CW; ++c) {
          const float oc = anyA ? S.doc[qq][pc * CW + c] : 0.f;
          const float of = anyD ? S.dhf[qq][pc * CW + c] : 0.f;
          const float qv = S.q[qq][pc * CW + c];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            dv[r][c] = fmaf(pv[r], oc, fmaf(pdv[r], of, dv[r][c]));
            dk[r][c] = fmaf(dsv[r], qv, dk[r][c]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    T* ok = row_ptr_w<T>(a.dk, b, kvh, u0 + pr * 4 + r) + pc * CW;
    T* ov = row_ptr_w<T>(a.dv, b, kvh, u0 + pr * 4 + r) + pc * CW;
#pragma unroll
    for (int c = 0; c < CW; ++c) {
      ok[c] = from_f32<T>(scale * dk[r][c]);
      ov[c] = from_f32<T>(dv[r][c]);
    }
  }
}

// ------------------------------------------------------------------ reductions
template <typename T, int D>
__global__ void __launch_bounds__(NT) sqdiff_kernel(TensorRef x, TensorRef y, int Hq, int N,
                                                   float* partials) {
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t row = (int64_t)blockIdx.x * 8 + w;
  const int t = (int)(row % N), bh = (int)(row / N), b = bh / Hq, h = bh % Hq;
  const T* px = row_ptr<T>(x, b, h, t);
  const T* py = row_ptr<T>(y, b, h, t);
  float sq = 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const float dlt = to_f32(px[lane + 32 * e]) - to_f32(py[lane + 32 * e]);
    sq = fmaf(dlt, dlt, sq);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
  __shared__ float part[8];
  if (lane == 0) part[w] = sq;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) s += part[q];
    partials[blockIdx.x] = s;
  }
}

// One CTA: fixed-order tree sum of the partials in double precision.
__global__ void __launch_bounds__(1024) finish_kernel(const float* partials, int np, double inv_count,
                                                     float mult, float* out, int n_out) {
  __shared__ double red[1024];
  double s = 0.0;
  for (int q = threadIdx.x; q < np; q += 1024) s += (double)partials[q];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int off = 512; off > 0; off >>= 1) {
    if ((int)threadIdx.x < off) red[threadIdx.x] += red[threadIdx.x + off];
    __syncthreads();
  }
  if ((int)threadIdx.x < n_out) out[threadIdx.x] = (float)(red[0] * inv_count * mult);
}

template <typename T, int D>
cudaError_t bwd_t(const Dims& Dm, const BwdArgs& a, cudaStream_t st) {
  auto kq = bwd_dq_kernel<T, D>;
  auto kkv = bwd_dkv_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sizeof(DqSmem<D>));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(DkvSmem<D>));
  if (e != cudaSuccess) return e;
  kq<<<dim3(Dm.N / BT, Dm.Hq, Dm.B), NT, sizeof(DqSmem<D>), st>>>(a, Dm.Hq, Dm.g, Dm.N, Dm.s, Dm.n,
                                                                 Dm.scale, Dm.per_token);
  count_launches(1);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  kkv<<<dim3(Dm.N / BT, Dm.Hkv, Dm.B), NT, sizeof(DkvSmem<D>), st>>>(a, Dm.Hq, Dm.g, Dm.N, Dm.s,
                                                                    Dm.n, Dm.scale, Dm.per_token);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

int sqdiff_partial_count(const Dims& D) {
  return (int)(((int64_t)D.B * D.Hq * D.N + 7) / 8);
}

cudaError_t launch_bwd_pre(const Dims& D, const BwdArgs& a, cudaStream_t st) {
  const double M = (double)D.B * D.Hq * D.N * D.d;
  const float c2 = (float)(2.0 * (double)a.alpha / M);
  const unsigned blocks = (unsigned)sqdiff_partial_count(D);
  if (D.dtype == SSA_BF16) {
    if (D.d == 128) bwd_pre_kernel<__nv_bfloat16, 128><<<blocks, NT, 0, st>>>(a, D.Hq, D.N, c2);
    else bwd_pre_kernel<__nv_bfloat16, 64><<<blocks, NT, 0, st>>>(a, D.Hq, D.N, c2);
  } else {
    if (D.d == 128) bwd_pre_kernel<float, 128><<<blocks, NT, 0, st>>>(a, D.Hq, D.N, c2);
    else bwd_pre_kernel<float, 64><<<blocks, NT, 0, st>>>(a, D.Hq, D.N, c2);
  }
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || a.align_loss == nullptr) return e;
  // L_align = L_sp + L_cm = 2 * mean((h_f - h_s)^2)
  return launch_finish_mean(a.partials, a.n_partials, M, 2.0f, a.align_loss, 1, st);
}

cudaError_t launch_bwd_simt(const Dims& D, const BwdArgs& a, cudaStream_t st) {
  if (D.dtype == SSA_BF16)
    return D.d == 128 ? bwd_t<__nv_bfloat16, 128>(D, a, st) : bwd_t<__nv_bfloat16, 64>(D, a, st);
  return D.d == 128 ? bwd_t<float, 128>(D, a, st) : bwd_t<float, 64>(D, a, st);
}

cudaError_t launch_sqdiff_partials(const Dims& D, const TensorRef& x, const TensorRef& y,
                                   float* partials, int n_partials, cudaStream_t st) {
  (void)n_partials;
  const unsigned blocks = (unsigned)sqdiff_partial_count(D);
  if (D.dtype == SSA_BF16) {
    if (D.d == 128) sqdiff_kernel<__nv_bfloat16, 128><<<blocks, NT, 0, st>>>(x, y, D.Hq, D.N, partials);
    else sqdiff_kernel<__nv_bfloat16, 64><<<blocks, NT, 0, st>>>(x, y, D.Hq, D.N, partials);
  } else {
    if (D.d == 128) sqdiff_kernel<float, 128><<<blocks, NT, 0, st>>>(x, y, D.Hq, D.N, partials);
    else sqdiff_kernel<float, 64><<<blocks, NT, 0, st>>>(x, y, D.Hq, D.N, partials);
  }
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_finish_mean(const float* partials, int n_partials, double count, float mult,
                               float* out, int n_out, cudaStream_t st) {
  finish_kernel<<<1, 1024, 0, st>>>(partials, n_partials, 1.0 / count, mult, out, n_out);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace ssa
