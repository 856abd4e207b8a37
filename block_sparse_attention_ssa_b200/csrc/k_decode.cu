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
// block mean exactly), or, with per-token selection, q_t itself:
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
// Two launches per token (CUDA cores, fp32 arithmetic; a token moves a few MB):
//   select: one CTA per (query head, batch) scores the pooled blocks and
//     keeps its top-k (block-wide arg-max rounds), leaving the kept-block
//     bits in the workspace;
//   attend: the union of the g query heads' kept blocks is split BPC blocks
//     per CTA (flash-decoding style); each CTA reads its K/V rows once for
//     all g heads, leaves a partial (o, max, sum) per head, and the last CTA
//     of a (kv head, batch) to finish -- an atomic counter, no waiting --
//     merges the partials.
#include <algorithm>
#include <climits>

#include "ssa_internal.cuh"

namespace ssa {
namespace {

constexpr int NT = 256;
constexpr int CH = 64;   // keys per chunk
constexpr int BPC = 2;   // selected blocks per attention CTA

struct DecodeShape {
  int Hq, g, N, s, n, k, t, splits;
  float scale;
  int per_token;  // the query side of the score is q_t itself (per-token selection)
};

// Per-call scratch in the caller's workspace.
struct DecodeWs {
  unsigned* counter;  // [B*Hkv]         attention CTAs finished (reset by the select kernel)
  uint32_t* sel;      // [B*Hkv][g][64]  selected-block bits per query head
  float* part;        // [B*Hq][splits][D+2] partial (o, m, l) per attention CTA
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

inline DecodeWs decode_ws(void* ws, const Dims& Dm) {
  char* p = static_cast<char*>(ws);
  const size_t bk = (size_t)Dm.B * Dm.Hkv;
  DecodeWs w;
  size_t o = 0;
  w.counter = reinterpret_cast<unsigned*>(p + o); o += align256(bk * 4);
  w.sel = reinterpret_cast<uint32_t*>(p + o); o += align256(bk * Dm.g * 64 * 4);
  w.part = reinterpret_cast<float*>(p + o);
  return w;
}

int decode_splits(const Dims& Dm) {
  const int most = std::min(Dm.g * Dm.k, Dm.n);  // blocks in a union
  return (most + BPC - 1) / BPC;
}

// Byte offsets of the select kernel's shared memory.
struct SelectLayout {
  size_t qbar, sc, sel, red, bytes;
  __host__ __device__ SelectLayout(int n, int D) {
    size_t at = 0;
    auto take = [&](size_t nbytes) {
      const size_t r = at;
      at = (at + nbytes + 15) / 16 * 16;
      return r;
    };
    qbar = take((size_t)D * 4);   // [D] block-prefix query mean
    sc = take((size_t)n * 4);     // [n] block scores
    sel = take(64 * 4);           // [64] selected-block bits
    red = take((size_t)NT * 8);   // per-warp arg-max candidates / key-sum staging
    bytes = at;
  }
};

// ---- step 1: query-block mean, block scores and top-k of one query head.
// grid (Hq, B).  Also folds q_t into qsum; the first head of each kv head
// resets the attention counter and, when t closes block i, writes the
// block's key mean into kbar.
template <typename T, int D>
__global__ void __launch_bounds__(NT) decode_select_kernel(TensorRef q, TensorRef K, int32_t* idx, float* qsum,
                                                           float* kbar, DecodeWs ws, DecodeShape sh) {
  const int h = blockIdx.x, b = blockIdx.y;
  const int G = sh.g, n = sh.n, s = sh.s, t = sh.t;
  const int kvh = h / G, hh = h % G;
  const int i = t / s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hkv = sh.Hq / G;
  const int bk = b * Hkv + kvh;

  extern __shared__ __align__(16) uint8_t smem[];
  const SelectLayout L(n, D);
  float* sqbar = reinterpret_cast<float*>(smem + L.qbar);
  float* ssc = reinterpret_cast<float*>(smem + L.sc);
  uint32_t* sel = reinterpret_cast<uint32_t*>(smem + L.sel);
  float* rv = reinterpret_cast<float*>(smem + L.red);
  int* rj = reinterpret_cast<int*>(rv + NT);

  if (tid < D) {
    float* qs = qsum + ((int64_t)b * sh.Hq + h) * D + tid;
    const float x = to_f32(row_ptr<T>(q, b, h, 0)[tid]);
    const float acc = (t % s == 0 ? 0.f : *qs) + x;
    *qs = acc;
    sqbar[tid] = sh.per_token ? x : acc / (float)(t - i * s + 1);
  }
  if (tid < 64) sel[tid] = 0u;
  if (hh == 0 && tid == 0) ws.counter[bk] = 0u;
  __syncthreads();

  // scores of the complete blocks j < i: a warp takes RPW pooled keys at a
  // time (a lane holds PER consecutive dims of each), so RPW coalesced row
  // loads are in flight before the dot products and lane reductions
  constexpr int PER = D / 32, RPW = 4;
  const float* kb = kbar + (int64_t)bk * n * D;
  float qv[PER];
#pragma unroll
  for (int c = 0; c < PER; ++c) qv[c] = sqbar[lane * PER + c];
  for (int j0 = warp * RPW; j0 < i; j0 += (NT / 32) * RPW) {
    float kv[RPW][PER];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
#pragma unroll
      for (int c = 0; c < PER; ++c) kv[r][c] = (j0 + r < i) ? kb[(int64_t)(j0 + r) * D + lane * PER + c] : 0.f;
    }
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      float p = 0.f;
#pragma unroll
      for (int c = 0; c < PER; ++c) p = fmaf(qv[c], kv[r][c], p);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
      if (lane == 0 && j0 + r < i) ssc[j0 + r] = sh.scale * p;
    }
  }
  __syncthreads();

  // top-(k-1) of the scores plus the diagonal block; each round is a
  // block-wide arg-max (score descending, index ascending)
  if (i + 1 <= sh.k) {
    for (int j = tid; j <= i; j += NT) atomicOr(&sel[j >> 5], 1u << (j & 31));
  } else {
    if (tid == 0) sel[i >> 5] |= 1u << (i & 31);
    for (int r = 0; r < sh.k - 1; ++r) {
      __syncthreads();
      float best = kNegInf;
      int bj = INT_MAX;
      for (int j = tid; j < i; j += NT) {
        if ((sel[j >> 5] >> (j & 31)) & 1u) continue;
        float v = ssc[j];
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
      if (lane == 0) {
        rv[warp] = best;
        rj[warp] = bj;
      }
      __syncthreads();
      if (warp == 0) {
        best = lane < NT / 32 ? rv[lane] : kNegInf;
        bj = lane < NT / 32 ? rj[lane] : INT_MAX;
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
  }
  __syncthreads();
  if (tid < 64) ws.sel[((size_t)bk * G + hh) * 64 + tid] = sel[tid];
  if (tid == 0) {  // Sel ascending, -1 padded
    int32_t* out = idx + ((int64_t)b * sh.Hq + h) * sh.k;
    int c = 0;
    for (int w = 0; w <= (i >> 5); ++w)
      for (uint32_t x = sel[w]; x && c < sh.k; x &= x - 1) out[c++] = 32 * w + __ffs(x) - 1;
    for (; c < sh.k; ++c) out[c] = -1;
  }

  // the token closes block i: its key mean joins the pooled cache (no
  // reader of this call uses kbar[i]); the kv head's first query head does it
  if (t % s == s - 1 && hh == 0) {
    // NT / D row groups sum interleaved rows (8 loads in flight each), then fold
    constexpr int RG = NT / D;
    const int c = tid % D, rg = tid / D;
    float acc = 0.f;
    for (int u0 = i * s + rg * 8; u0 < i * s + s; u0 += RG * 8) {
      float v[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) v[r] = to_f32(row_ptr<T>(K, b, kvh, u0 + r)[c]);
#pragma unroll
      for (int r = 0; r < 8; ++r) acc += v[r];
    }
    rv[tid] = acc;
    __syncthreads();
    if (tid < D) {
      float sum = 0.f;
      for (int g2 = 0; g2 < RG; ++g2) sum += rv[g2 * D + tid];
      kbar[((int64_t)bk * n + i) * D + tid] = sum / (float)s;
    }
  }
}

// Byte offsets of the attention kernel's shared memory.
struct AttendLayout {
  size_t q, o, mx, sum, x, k, v, lst, bytes;
  __host__ __device__ AttendLayout(int g, int D) {
    size_t at = 0;
    auto take = [&](size_t nbytes) {
      const size_t r = at;
      at = (at + nbytes + 15) / 16 * 16;
      return r;
    };
    q = take((size_t)g * D * 4);         // [g][D] q_t
    o = take((size_t)g * D * 4);         // [g][D] partial output
    mx = take((size_t)g * 4);            // [g] running max
    sum = take((size_t)g * 4);           // [g] running sum
    x = take((size_t)g * CH * 4);        // [g][CH] logits / weights of a chunk
    k = take((size_t)CH * (D + 1) * 4);  // [CH][D+1] K chunk
    v = take((size_t)CH * D * 4);        // [CH][D] V chunk
    lst = take(16 + 4 * BPC);            // this CTA's blocks of the union, flag
    bytes = at;
  }
};

// ---- step 2: attention over the union of the g heads' selected blocks,
// BPC blocks per CTA.  The next chunk's K/V rows are loaded into registers
// while the current chunk is processed.  Each CTA leaves a partial
// (o, m, l) per query head and the last CTA of a (batch, kv head) to finish
// merges them.  grid (splits, Hkv, B).
template <typename T, int D>
__global__ void __launch_bounds__(NT) decode_attend_kernel(TensorRef q, TensorRef K, TensorRef V, TensorRef hout,
                                                           float* lse, DecodeWs ws, DecodeShape sh) {
  constexpr int VEC = Vec16<T>::kN;
  constexpr int ITERS = CH * (D / VEC) / NT;  // 16-byte loads per thread per chunk and tensor
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int G = sh.g, s = sh.s, t = sh.t;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hkv = sh.Hq / G;
  const int bk = b * Hkv + kvh;

  extern __shared__ __align__(16) uint8_t smem[];
  const AttendLayout L(G, D);
  float* sq = reinterpret_cast<float*>(smem + L.q);
  float* so = reinterpret_cast<float*>(smem + L.o);
  float* smax = reinterpret_cast<float*>(smem + L.mx);
  float* ssum = reinterpret_cast<float*>(smem + L.sum);
  float* sx = reinterpret_cast<float*>(smem + L.x);
  float* sk = reinterpret_cast<float*>(smem + L.k);
  float* sv = reinterpret_cast<float*>(smem + L.v);
  int* slst = reinterpret_cast<int*>(smem + L.lst);  // [0] count, [1..] blocks, [1 + BPC] last flag

  const uint32_t* selw = ws.sel + (size_t)bk * G * 64;
  // this CTA's entries [split*BPC, split*BPC + BPC) of the ascending union
  if (warp == 0) {
    uint32_t w0 = 0, w1 = 0;
#pragma unroll 4
    for (int hh = 0; hh < G; ++hh) {
      const uint2 wv = *reinterpret_cast<const uint2*>(selw + hh * 64 + 2 * lane);
      w0 |= wv.x;
      w1 |= wv.y;
    }
    const int c = __popc(w0) + __popc(w1);
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    const int e0 = split * BPC;
    int pos = incl - c;
    for (uint32_t x = w0; x; x &= x - 1, ++pos)
      if (pos >= e0 && pos < e0 + BPC) slst[1 + pos - e0] = 64 * lane + __ffs(x) - 1;
    for (uint32_t x = w1; x; x &= x - 1, ++pos)
      if (pos >= e0 && pos < e0 + BPC) slst[1 + pos - e0] = 64 * lane + 32 + __ffs(x) - 1;
    if (lane == 31) slst[0] = max(0, min(BPC, incl - e0));
  }
  for (int e = tid; e < G * D; e += NT) {
    sq[e] = to_f32(row_ptr<T>(q, b, kvh * G + e / D, 0)[e % D]);
    so[e] = 0.f;
  }
  if (tid < G) {
    smax[tid] = kNegInf;
    ssum[tid] = 0.f;
  }
  __syncthreads();
  const int nb = slst[0];
  const int cpb = (s + CH - 1) / CH;  // chunks per block
  const int nch = nb * cpb;
  auto chunk_rows = [&](int ch, int& j, int& c0) {
    j = slst[1 + ch / cpb];
    c0 = j * s + (ch % cpb) * CH;
    return max(0, min(CH, min(j * s + s, t + 1) - c0));
  };

  float tk[ITERS][VEC], tv[ITERS][VEC];
  auto load_chunk = [&](int ch) {
    int j, c0;
    const int rows = chunk_rows(ch, j, c0);
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      const int x = tid + it * NT, r = x / (D / VEC), c = (x % (D / VEC)) * VEC;
      if (r < rows) {
        Vec16<T>::load(row_ptr<T>(K, b, kvh, (int64_t)c0 + r) + c, tk[it]);
        Vec16<T>::load(row_ptr<T>(V, b, kvh, (int64_t)c0 + r) + c, tv[it]);
      }
    }
  };
  if (nch > 0) load_chunk(0);
  for (int ch = 0; ch < nch; ++ch) {
    int j, c0;
    const int rows = chunk_rows(ch, j, c0);
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      const int x = tid + it * NT, r = x / (D / VEC), c = (x % (D / VEC)) * VEC;
      if (r < rows) {
#pragma unroll
        for (int y = 0; y < VEC; ++y) {
          sk[r * (D + 1) + c + y] = tk[it][y];
          sv[r * D + c + y] = tv[it][y];
        }
      }
    }
    if (ch + 1 < nch) load_chunk(ch + 1);  // in flight while this chunk is used
    __syncthreads();
    for (int x = tid; x < G * CH; x += NT) {
      const int hh = x / CH, uu = x % CH;
      float v = kNegInf;
      if (uu < rows && ((selw[hh * 64 + (j >> 5)] >> (j & 31)) & 1u)) {
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
      if (!((selw[hh * 64 + (j >> 5)] >> (j & 31)) & 1u)) continue;
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

  // partial (o, m, l) of this CTA for each of the g heads
  for (int e = tid; e < G * (D + 2); e += NT) {
    const int hh = e / (D + 2), c = e % (D + 2);
    const float v = c < D ? so[hh * D + c] : (c == D ? smax[hh] : ssum[hh]);
    ws.part[(((size_t)b * sh.Hq + kvh * G + hh) * sh.splits + split) * (D + 2) + c] = v;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) slst[1 + BPC] = (atomicAdd(&ws.counter[bk], 1u) == (unsigned)sh.splits - 1) ? 1 : 0;
  __syncthreads();
  if (!slst[1 + BPC]) return;
  __threadfence();

  // last CTA: merge the splits; warp hh merges head hh (lanes over splits for
  // the statistics, over dims for the output, four splits' rows in flight)
  constexpr int PER = D / 32;
  for (int hh = warp; hh < G; hh += NT / 32) {
    const float* p = ws.part + ((size_t)b * sh.Hq + kvh * G + hh) * sh.splits * (D + 2);
    float M = kNegInf;
    for (int x = lane; x < sh.splits; x += 32) M = fmaxf(M, __ldcg(p + (size_t)x * (D + 2) + D));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float Lsum = 0.f;
    for (int x = lane; x < sh.splits; x += 32) {
      const float m = __ldcg(p + (size_t)x * (D + 2) + D);
      if (m != kNegInf) Lsum += __ldcg(p + (size_t)x * (D + 2) + D + 1) * __expf(m - M);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, off);
    float acc[PER];
#pragma unroll
    for (int c = 0; c < PER; ++c) acc[c] = 0.f;
    for (int x0 = 0; x0 < sh.splits; x0 += 4) {
      float m[4], o[4][PER];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int x = x0 + r;
        m[r] = x < sh.splits ? __ldcg(p + (size_t)x * (D + 2) + D) : kNegInf;
#pragma unroll
        for (int c = 0; c < PER; ++c) o[r][c] = x < sh.splits ? __ldcg(p + (size_t)x * (D + 2) + lane * PER + c) : 0.f;
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (m[r] == kNegInf) continue;
        const float wgt = __expf(m[r] - M);
#pragma unroll
        for (int c = 0; c < PER; ++c) acc[c] = fmaf(o[r][c], wgt, acc[c]);
      }
    }
    T* dst = row_ptr_w<T>(hout, b, kvh * G + hh, 0) + lane * PER;
#pragma unroll
    for (int c = 0; c < PER; ++c) dst[c] = from_f32<T>(Lsum > 0.f ? acc[c] / Lsum : 0.f);
    if (lane == 0) lse[(int64_t)b * sh.Hq + kvh * G + hh] = Lsum > 0.f ? M + logf(Lsum) : kNegInf;
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
  const int splits = decode_splits(Dm);
  const DecodeWs ws = decode_ws(a.ws, Dm);
  DecodeShape sh{Dm.Hq, Dm.g, Dm.N, Dm.s, Dm.n, Dm.k, a.t, splits, Dm.scale, Dm.per_token};
  const size_t sm1 = SelectLayout(Dm.n, D).bytes, sm2 = AttendLayout(Dm.g, D).bytes;
  auto k1 = decode_select_kernel<T, D>;
  auto k2 = decode_attend_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
  if (e != cudaSuccess) return e;
  k1<<<dim3(Dm.Hq, Dm.B), NT, sm1, st>>>(a.q, a.k, a.idx, a.qsum, a.kbar, ws, sh);
  count_launches(1);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k2<<<dim3(splits, Dm.Hkv, Dm.B), NT, sm2, st>>>(a.q, a.k, a.v, a.h, a.lse, ws, sh);
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

size_t decode_smem_bytes(const Dims& D) {
  const size_t a = SelectLayout(D.n, D.d).bytes, b = AttendLayout(D.g, D.d).bytes;
  return a > b ? a : b;
}

size_t decode_ws_bytes(const Dims& D) {
  const size_t bk = (size_t)D.B * D.Hkv;
  return align256(bk * 4) + align256(bk * D.g * 64 * 4) +
         align256((size_t)D.B * D.Hq * decode_splits(D) * (D.d + 2) * 4);
}

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
