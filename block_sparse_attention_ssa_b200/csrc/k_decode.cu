// Sparse-stream decode: one new token per (batch, query head) attends through
// a pooled-key cache ("SSA: Achieving Sparser Attention ...", sections
// "Practical Implementation of SSA" and "Training Efficiency Considerations":
// at inference the sparse stream alone runs; "SSA: Sparse Sparse Attention"
// skill page, "6. Inference with Sparse or Full Mode": generation appends one
// token at a time).
//
// Token t lies in block i = t / s.  The selection rule is the forward's, with
// the query side read as the mean of the queries of block i seen so far
// (positions i*s .. t; at the last token of a block this is the forward's
// block mean exactly):
//   qbar   = (sum of q_u, u = i*s .. t) / (t - i*s + 1),
//   score_j = scale * qbar . kbar_j for j < i (kbar_j = mean of key block j),
//   Sel     = {i} + the k-1 largest scores (ties to the smaller j), or
//             {0..i} when i + 1 <= k,
//   h_t     = softmax over A_t = {u <= t : u / s in Sel} of scale q_t . k_u,
//             applied to V.
// State kept by the caller between calls: qsum [B,Hq,d] (running sum of the
// current block's queries) and kbar [B,Hkv,n,d] (means of complete blocks);
// the call folds q_t into qsum and, when t closes block i, writes kbar_i.
//
// One CTA per (kv head, batch) serves the g query heads that share the kv
// head: it scores and selects per query head, then walks the union of the
// selected blocks once, 64 keys at a time, so every K/V row is read once per
// CTA.  CUDA cores, fp32 arithmetic: the work per token is a few MB of K/V.
#include <climits>

#include "ssa_internal.cuh"

namespace ssa {
namespace {

constexpr int NT = 256;
constexpr int CH = 64;  // keys per chunk

struct DecodeShape {
  int Hq, g, N, s, n, k, t;
  float scale;
};

// Byte offsets of the shared-memory regions (host and device agree on them).
struct DecodeLayout {
  size_t q, qbar, o, sc, mx, sum, x, sel, uni, cnt, list, k, v, bytes;
  __host__ __device__ DecodeLayout(int g, int n, int D) {
    size_t at = 0;
    auto take = [&](size_t nbytes) {
      const size_t r = at;
      at = (at + nbytes + 15) / 16 * 16;
      return r;
    };
    q = take((size_t)g * D * 4);        // [g][D] q_t
    qbar = take((size_t)g * D * 4);     // [g][D] block-prefix query mean
    o = take((size_t)g * D * 4);        // [g][D] output accumulator
    sc = take((size_t)g * n * 4);       // [g][n] block scores
    mx = take((size_t)g * 4);           // [g] running max
    sum = take((size_t)g * 4);          // [g] running sum
    x = take((size_t)g * CH * 4);       // [g][CH] logits / weights of a chunk
    sel = take((size_t)g * 64 * 4);     // [g][64] selected-block bits
    uni = take(64 * 4);                 // [64] union of the bits over the g heads
    cnt = take(16);                     // union count
    list = take((size_t)n * 2);         // [n] union, ascending
    k = take((size_t)CH * (D + 1) * 4); // [CH][D+1] K chunk (also pooled keys)
    v = take((size_t)CH * D * 4);       // [CH][D] V chunk
    bytes = at;
  }
};

template <typename T, int D>
__global__ void __launch_bounds__(NT) decode_kernel(TensorRef q, TensorRef K, TensorRef V, TensorRef hout,
                                                    float* lse, int32_t* idx, float* qsum, float* kbar,
                                                    DecodeShape sh) {
  constexpr int VEC = Vec16<T>::kN;
  const int kvh = blockIdx.x, b = blockIdx.y;
  const int G = sh.g, n = sh.n, s = sh.s, t = sh.t;
  const int i = t / s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hkv = sh.Hq / G;

  extern __shared__ __align__(16) uint8_t smem[];
  const DecodeLayout L(G, n, D);
  float* sq = reinterpret_cast<float*>(smem + L.q);
  float* sqbar = reinterpret_cast<float*>(smem + L.qbar);
  float* so = reinterpret_cast<float*>(smem + L.o);
  float* ssc = reinterpret_cast<float*>(smem + L.sc);
  float* smax = reinterpret_cast<float*>(smem + L.mx);
  float* ssum = reinterpret_cast<float*>(smem + L.sum);
  float* sx = reinterpret_cast<float*>(smem + L.x);
  uint32_t* ssel = reinterpret_cast<uint32_t*>(smem + L.sel);
  uint32_t* suni = reinterpret_cast<uint32_t*>(smem + L.uni);
  int* snu = reinterpret_cast<int*>(smem + L.cnt);
  uint16_t* slist = reinterpret_cast<uint16_t*>(smem + L.list);
  float* sk = reinterpret_cast<float*>(smem + L.k);
  float* sv = reinterpret_cast<float*>(smem + L.v);
  (void)suni;

  // ---- q_t, the running block sum of queries, and its mean
  const float cnt = (float)(t - i * s + 1);
  for (int e = tid; e < G * D; e += NT) {
    const int hh = e / D, c = e % D;
    const int h = kvh * G + hh;
    const float x = to_f32(row_ptr<T>(q, b, h, 0)[c]);
    float* qs = qsum + ((int64_t)b * sh.Hq + h) * D + c;
    const float acc = (t % s == 0 ? 0.f : *qs) + x;
    *qs = acc;
    sq[e] = x;
    sqbar[e] = acc / cnt;
    so[e] = 0.f;
  }
  if (tid < G) {
    smax[tid] = kNegInf;
    ssum[tid] = 0.f;
  }
  __syncthreads();

  // ---- scores of the complete blocks j < i, 64 pooled keys at a time
  const float* kb = kbar + ((int64_t)b * Hkv + kvh) * n * D;
  for (int j0 = 0; j0 < i; j0 += CH) {
    const int rows = min(CH, i - j0);
    for (int e = tid; e < rows * D; e += NT) sk[(e / D) * (D + 1) + e % D] = kb[(int64_t)(j0 + e / D) * D + e % D];
    __syncthreads();
    for (int e = tid; e < G * rows; e += NT) {
      const int hh = e / rows, jj = e % rows;
      const float* qv = sqbar + hh * D;
      const float* kv = sk + jj * (D + 1);
      float acc = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) acc = fmaf(qv[c], kv[c], acc);
      ssc[(size_t)hh * n + j0 + jj] = sh.scale * acc;
    }
    __syncthreads();
  }

  // ---- per-head top-(k-1) of the scores plus the diagonal block
  for (int hh = warp; hh < G; hh += NT / 32) {
    uint32_t* sel = ssel + hh * 64;
    for (int w = lane; w < 64; w += 32) sel[w] = 0u;
    __syncwarp();
    if (i + 1 <= sh.k) {
      for (int j = lane; j <= i; j += 32) atomicOr(&sel[j >> 5], 1u << (j & 31));
    } else {
      if (lane == 0) atomicOr(&sel[i >> 5], 1u << (i & 31));
      const float* sc = ssc + (size_t)hh * n;
      for (int r = 0; r < sh.k - 1; ++r) {
        __syncwarp();
        float best = kNegInf;
        int bj = INT_MAX;
        for (int j = lane; j < i; j += 32) {
          if ((sel[j >> 5] >> (j & 31)) & 1u) continue;
          float v = sc[j];
          if (v != v) v = kNegInf;  // NaN ranks last
          if (v > best || (v == best && j < bj)) {
            best = v;
            bj = j;
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, best, off);
          const int oj = __shfl_xor_sync(0xffffffffu, bj, off);
          if (ov > best || (ov == best && oj < bj)) {
            best = ov;
            bj = oj;
          }
        }
        if (lane == 0 && bj < i) sel[bj >> 5] |= 1u << (bj & 31);
      }
    }
    __syncwarp();
    if (lane == 0) {  // Sel ascending, -1 padded
      int32_t* out = idx + ((int64_t)b * sh.Hq + kvh * G + hh) * sh.k;
      int c = 0;
      for (int w = 0; w <= (i >> 5); ++w)
        for (uint32_t x = sel[w]; x && c < sh.k; x &= x - 1) out[c++] = 32 * w + __ffs(x) - 1;
      for (; c < sh.k; ++c) out[c] = -1;
    }
  }
  __syncthreads();

  // ---- union of the selected blocks over the g heads, ascending
  if (warp == 0) {
    uint32_t w0 = 0, w1 = 0;
    for (int hh = 0; hh < G; ++hh) {
      w0 |= ssel[hh * 64 + 2 * lane];
      w1 |= ssel[hh * 64 + 2 * lane + 1];
    }
    const int c = __popc(w0) + __popc(w1);
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    int pos = incl - c;
    for (uint32_t x = w0; x; x &= x - 1) slist[pos++] = (uint16_t)(64 * lane + __ffs(x) - 1);
    for (uint32_t x = w1; x; x &= x - 1) slist[pos++] = (uint16_t)(64 * lane + 32 + __ffs(x) - 1);
    if (lane == 31) snu[0] = incl;
  }
  __syncthreads();
  const int nu = snu[0];

  // ---- attention over the union, CH keys at a time (online softmax per head)
  for (int e = 0; e < nu; ++e) {
    const int j = slist[e];
    const int u_end = min(j * s + s, t + 1);
    for (int c0 = j * s; c0 < u_end; c0 += CH) {
      const int rows = min(CH, u_end - c0);
      for (int x = tid; x < rows * (D / VEC); x += NT) {
        const int r = x / (D / VEC), c = (x % (D / VEC)) * VEC;
        float tk[VEC], tv[VEC];
        Vec16<T>::load(row_ptr<T>(K, b, kvh, (int64_t)c0 + r) + c, tk);
        Vec16<T>::load(row_ptr<T>(V, b, kvh, (int64_t)c0 + r) + c, tv);
#pragma unroll
        for (int y = 0; y < VEC; ++y) {
          sk[r * (D + 1) + c + y] = tk[y];
          sv[r * D + c + y] = tv[y];
        }
      }
      __syncthreads();
      for (int x = tid; x < G * CH; x += NT) {
        const int hh = x / CH, uu = x % CH;
        float v = kNegInf;
        if (uu < rows && ((ssel[hh * 64 + (j >> 5)] >> (j & 31)) & 1u)) {
          const float* qv = sq + hh * D;
          const float* kv = sk + uu * (D + 1);
          float acc = 0.f;
#pragma unroll 8
          for (int c = 0; c < D; ++c) acc = fmaf(qv[c], kv[c], acc);
          v = sh.scale * acc;
        }
        sx[x] = v;
      }
      __syncthreads();
      for (int hh = warp; hh < G; hh += NT / 32) {
        if (!((ssel[hh * 64 + (j >> 5)] >> (j & 31)) & 1u)) continue;
        float* xs = sx + hh * CH;
        float mt = fmaxf(xs[lane], xs[lane + 32]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
        const float m_old = smax[hh];
        const float m_new = fmaxf(m_old, mt);
        const float p0 = (xs[lane] == kNegInf) ? 0.f : __expf(xs[lane] - m_new);
        const float p1 = (xs[lane + 32] == kNegInf) ? 0.f : __expf(xs[lane + 32] - m_new);
        float ps = p0 + p1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        const float corr = (m_old == kNegInf) ? 0.f : __expf(m_old - m_new);
        __syncwarp();
        xs[lane] = p0;
        xs[lane + 32] = p1;
        __syncwarp();
        float* o = so + hh * D;
#pragma unroll
        for (int r = 0; r < D / 32; ++r) {
          const int c = lane + 32 * r;
          float acc = o[c] * corr;
          for (int uu = 0; uu < rows; ++uu) acc = fmaf(xs[uu], sv[uu * D + c], acc);
          o[c] = acc;
        }
        if (lane == 0) {
          smax[hh] = m_new;
          ssum[hh] = ssum[hh] * corr + ps;
        }
      }
      __syncthreads();
    }
  }

  // ---- outputs
  for (int e = tid; e < G * D; e += NT) {
    const int hh = e / D, c = e % D;
    const float l = ssum[hh];
    row_ptr_w<T>(hout, b, kvh * G + hh, 0)[c] = from_f32<T>(l > 0.f ? so[e] / l : 0.f);
  }
  if (tid < G) {
    const float l = ssum[tid];
    lse[(int64_t)b * sh.Hq + kvh * G + tid] = l > 0.f ? smax[tid] + logf(l) : kNegInf;
  }

  // ---- the token closes block i: its key mean joins the pooled cache
  if (t % s == s - 1) {
    for (int c = tid; c < D; c += NT) {
      float acc = 0.f;
      for (int u = i * s; u < i * s + s; ++u) acc += to_f32(row_ptr<T>(K, b, kvh, u)[c]);
      kbar[(((int64_t)b * Hkv + kvh) * n + i) * D + c] = acc / (float)s;
    }
  }
}

// Prefill of the decode state from a prompt of t0 tokens: kbar of the
// complete blocks 0 .. t0/s - 1 and qsum of the partial block (rows
// (t0/s)*s .. t0-1; zero when t0 is a multiple of s).  grid (n + 1, Hq, B):
// x < t0/s pools key block x (heads < Hkv), x == n sums the queries.
template <typename T, int D>
__global__ void __launch_bounds__(128) decode_prefill_kernel(TensorRef Q, TensorRef K, float* qsum, float* kbar,
                                                             int Hq, int Hkv, int s, int n, int t0) {
  const int x = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int full = t0 / s;
  for (int c = threadIdx.x; c < D; c += 128) {
    if (x < full && h < Hkv) {
      float acc = 0.f;
      for (int u = x * s; u < x * s + s; ++u) acc += to_f32(row_ptr<T>(K, b, h, u)[c]);
      kbar[(((int64_t)b * Hkv + h) * n + x) * D + c] = acc / (float)s;
    } else if (x == n) {
      float acc = 0.f;
      for (int u = full * s; u < t0; ++u) acc += to_f32(row_ptr<T>(Q, b, h, u)[c]);
      qsum[((int64_t)b * Hq + h) * D + c] = acc;
    }
  }
}

template <typename T, int D>
cudaError_t decode_t(const Dims& Dm, const DecodeArgs& a, cudaStream_t st) {
  const size_t smem = DecodeLayout(Dm.g, Dm.n, D).bytes;
  auto kern = decode_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  DecodeShape sh{Dm.Hq, Dm.g, Dm.N, Dm.s, Dm.n, Dm.k, a.t, Dm.scale};
  kern<<<dim3(Dm.Hkv, Dm.B), NT, smem, st>>>(a.q, a.k, a.v, a.h, a.lse, a.idx, a.qsum, a.kbar, sh);
  count_launches(1);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t prefill_t(const Dims& Dm, const DecodeArgs& a, cudaStream_t st) {
  decode_prefill_kernel<T, D><<<dim3(Dm.n + 1, Dm.Hq, Dm.B), 128, 0, st>>>(a.q, a.k, a.qsum, a.kbar, Dm.Hq, Dm.Hkv,
                                                                          Dm.s, Dm.n, a.t);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

size_t decode_smem_bytes(const Dims& D) { return DecodeLayout(D.g, D.n, D.d).bytes; }

cudaError_t launch_decode(const Dims& D, const DecodeArgs& a, cudaStream_t st) {
  if (D.dtype == SSA_BF16)
    return D.d == 128 ? decode_t<__nv_bfloat16, 128>(D, a, st) : decode_t<__nv_bfloat16, 64>(D, a, st);
  return D.d == 128 ? decode_t<float, 128>(D, a, st) : decode_t<float, 64>(D, a, st);
}

cudaError_t launch_decode_prefill(const Dims& D, const DecodeArgs& a, cudaStream_t st) {
  if (D.dtype == SSA_BF16)
    return D.d == 128 ? prefill_t<__nv_bfloat16, 128>(D, a, st) : prefill_t<__nv_bfloat16, 64>(D, a, st);
  return D.d == 128 ? prefill_t<float, 128>(D, a, st) : prefill_t<float, 64>(D, a, st);
}

}  // namespace ssa
