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
// One launch per token (a token moves a few MB): a thread-block cluster of CL
// CTAs per (batch, kv head) selects the blocks of the g query heads (every CTA
// scores a slice of the pooled blocks for every head, fp32 on CUDA cores, and
// keeps each head's best k-1 of its slice; the head's owner merges the CL
// lists), attends the union of their kept blocks split CL ways (each K/V row
// read once for all g heads; bf16 on mma.sync with the heads as the rows of
// one fragment, fp32 on CUDA cores) and merges the partials, exchanging the
// candidate lists, the selections and the partials through distributed shared
// memory between cluster barriers (no workspace, no atomics, no waiting on
// flags; the only waits are the bounded ones on the copies into shared
// memory).
#include <algorithm>
#include <climits>
#include <type_traits>

#include <cooperative_groups.h>

#include "mma_sync.cuh"
#include "sm100_ptx.cuh"
#include "ssa_internal.cuh"

namespace ssa {
namespace {

constexpr int NT = 256;
constexpr int CH = 64;   // keys per chunk
constexpr int CL = 8;    // CTAs per cluster: one cluster per (batch, kv head)

struct DecodeShape {
  int Hq, g, N, s, n, k, t;
  float scale;
  int per_token;   // the query side of the score is q_t itself (per-token selection)
  int mma;         // attention on mma.sync with TMA-loaded bf16 K / V chunks (bf16, g <= 16)
  int chr;         // rows of a chunk on that path: min(CH, s)
  int kbs;         // this CTA's slice of the pooled keys comes into shared memory by one bulk copy
  int32_t* status; // per-device status report (a bounded wait that ran out)
};

// The bf16 attention phase stages a chunk's K and V as 64-column halves of
// CH rows x 128 B in the TMA 128-byte swizzle (the 16-byte piece c of row r
// sits at piece c ^ (r & 7): the 8 rows of an ldmatrix hit different banks),
// two chunks in flight; the ring needs 1024-byte alignment.
template <int D>
constexpr int kTileBytes = (D / 64) * CH * 128;  // one tensor of one chunk
template <int D>
constexpr int kRingBytes = 2 * 2 * kTileBytes<D>;

// Byte offsets of the decode kernel's shared memory.
struct DecodeLayout {
  size_t qbar, sc, cand, red, q, o, mx, sum, x, k, v, lst, usel, corr, bar, bytes;
  __host__ __device__ DecodeLayout(int n, int g, int k_eff, int D) {
    size_t at = 0;
    auto take = [&](size_t nbytes) {
      const size_t r = at;
      at = (at + nbytes + 15) / 16 * 16;
      return r;
    };
    const int most = (std::min(g * k_eff, n) + CL - 1) / CL;  // union blocks this CTA attends
    const int slice = (n + CL - 1) / CL;                    // pooled blocks this CTA scores
    qbar = take((size_t)g * D * 4);       // [g][D] query side of the block scores
    sc = take((size_t)g * slice * 4);     // [g][slice] block scores of this CTA's slice
    cand = take((size_t)g * 64 * 8);      // [g][64] best k-1 (score, block) of the slice
    red = take((size_t)NT * 8);           // arg-max candidates / key-sum staging
    q = take((size_t)g * D * 4);          // [g][D] q_t
    o = take((size_t)g * D * 4);          // [g][D] partial output
    mx = take((size_t)g * 4);             // [g] running max
    sum = take((size_t)g * 4);            // [g] running sum
    x = take((size_t)g * CH * 4);         // [g][CH] logits / weights of a chunk
    // [CH][D+1] K chunk and [CH][D] V chunk (fp32), or, contiguous with it,
    // the bf16 ring of two chunks (K rows, then V rows, kRowPitch bytes each)
    const size_t kv32 = (size_t)CH * (D + 1) * 4 + (size_t)CH * D * 4;
    const size_t ring = (size_t)2 * 2 * (D / 64) * CH * 128 + 1024;
    k = take(std::max((size_t)CH * (D + 1) * 4, (ring > kv32 ? ring - kv32 : 0) + (size_t)CH * (D + 1) * 4));
    v = take((size_t)CH * D * 4);
    lst = take((size_t)(1 + most) * 4);   // this CTA's blocks of the union
    usel = take((size_t)g * 64 * 4);      // [g][64] every head's selected-block bits
    corr = take((size_t)g * 4);           // [g] rescale factor of a chunk
    bar = take(32);                       // the ring's two mbarriers, the pooled-key slice's, an abort flag
    bytes = at;
  }
};

// Attention phase of the bf16 decode step on mma.sync: the g <= 16 query heads
// of the kv head are the 16 rows of one A fragment, so a 64-key chunk is read
// from shared memory once for every head.  Warp w forms the logits of keys
// 8w .. 8w + 7 (S = q_t K^T, fp32 accumulation of exact bf16 products), a warp
// per head updates the online softmax, and warp w adds P V for the columns
// 16w .. 16w + 15 (P rounded to bf16 for the product, as in the other
// tensor-core kernels).  The chunk's K / V rows arrive by bulk copies into a
// two-slot ring (one mbarrier per slot, bounded waits); the partial (o, max,
// sum) lands where the merge phase reads it.
template <int D, typename RowsF, typename IssueF>
__device__ __forceinline__ void decode_attend_mma(const DecodeShape& sh, int G, int rank, int t, int tid, int lane,
                                                  int warp, const int* slst, const uint32_t* usel, const float* sq,
                                                  float* so, float* smax, float* ssum, float* scorr, float* sx,
                                                  uint8_t* ring, uint64_t* cbar, int* cabort, RowsF chunk_rows,
                                                  IssueF issue_chunk, int cpb) {
  using namespace warp_mma;
  (void)rank;
  (void)t;
  const int g8 = lane >> 2, q4 = lane & 3;
  // byte offset of the 16-byte piece `pc` (0..7) of row r in the 64-column half hh
  auto swz = [](int hh, int r, int pc) { return hh * CH * 128 + r * 128 + ((pc ^ (r & 7)) << 4); };
  const bool r0ok = g8 < G, r1ok = g8 + 8 < G;  // fragment rows g8, g8 + 8 are heads
  const int nch = slst[0] * cpb;
  auto frag = [&](const float* base, int pitch, int c, uint32_t (&a)[4]) {  // rows g8 / g8 + 8, columns c.., c + 8..
    const float2 z = make_float2(0.f, 0.f);
    const float2 x0 = r0ok ? *reinterpret_cast<const float2*>(base + g8 * pitch + c) : z;
    const float2 x1 = r1ok ? *reinterpret_cast<const float2*>(base + (g8 + 8) * pitch + c) : z;
    const float2 x2 = r0ok ? *reinterpret_cast<const float2*>(base + g8 * pitch + c + 8) : z;
    const float2 x3 = r1ok ? *reinterpret_cast<const float2*>(base + (g8 + 8) * pitch + c + 8) : z;
    a[0] = pack2(x0.x, x0.y);
    a[1] = pack2(x1.x, x1.y);
    a[2] = pack2(x2.x, x2.y);
    a[3] = pack2(x3.x, x3.y);
  };
  float o[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  bool ok = true;
  for (int chk = 0; chk < nch; ++chk) {
    const int slot = chk & 1;
    ok = sm100::mbar_wait(&cbar[slot], (uint32_t)(chk >> 1) & 1u, cabort) && ok;
    int j, c0;
    const int rows = chunk_rows(chk, j, c0);
    const uint8_t* kb = ring + slot * 2 * kTileBytes<D>;
    uint8_t* vb = ring + slot * 2 * kTileBytes<D> + kTileBytes<D>;
    if (rows < CH) {  // V rows past the chunk's end (a later block, or beyond t) become zeros
      for (int e = tid; e < (CH - rows) * (D / 8); e += NT) {
        const int r = rows + e / (D / 8), c = e % (D / 8);
        *reinterpret_cast<uint4*>(vb + swz(c / 8, r, c % 8)) = make_uint4(0u, 0u, 0u, 0u);
      }
      sm100::fence_proxy_async_smem();  // before a later TMA load into the same bytes
    }
    {  // logits of keys 8w .. 8w + 7 for every head
      float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
      if (8 * warp < rows) {
#pragma unroll
        for (int kk = 0; kk < D / 16; kk += 2) {
          uint32_t kf[4], qa[4], qb[4];
          ldsm_x4_addr(kf, saddr(kb + swz(kk / 4, 8 * warp + (lane & 7), (kk % 4) * 2 + (lane >> 3))));
          frag(sq, D, kk * 16 + 2 * q4, qa);
          frag(sq, D, (kk + 1) * 16 + 2 * q4, qb);
          mma16816(a0, qa, kf[0], kf[1]);
          mma16816(a1, qb, kf[2], kf[3]);
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hh = g8 + 8 * (e >> 1), key = 8 * warp + 2 * q4 + (e & 1);
        if (hh < G) {
          const bool selh = (usel[hh * 64 + (j >> 5)] >> (j & 31)) & 1u;
          sx[hh * CH + key] = (selh && key < rows) ? sh.scale * (a0[e] + a1[e]) : kNegInf;
        }
      }
    }
    __syncthreads();
    // softmax statistics: a warp per head; the weights go back over the logits
    for (int hh = warp; hh < G; hh += NT / 32) {
      float* xs = sx + hh * CH;
      if (!((usel[hh * 64 + (j >> 5)] >> (j & 31)) & 1u)) {  // the head skips this block
        xs[lane] = 0.f;
        xs[lane + 32] = 0.f;
        if (lane == 0) scorr[hh] = 1.f;
        continue;
      }
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
      if (lane == 0) {
        smax[hh] = m_new;
        ssum[hh] = ssum[hh] * corr + ps;
        scorr[hh] = corr;
      }
    }
    __syncthreads();
    // o = o * corr + P V for the columns 16w .. 16w + 15
    if (16 * warp < D) {
      const float f0 = r0ok ? scorr[g8] : 1.f, f1 = r1ok ? scorr[g8 + 8] : 1.f;
#pragma unroll
      for (int n = 0; n < 2; ++n) {
        o[n][0] *= f0;
        o[n][1] *= f0;
        o[n][2] *= f1;
        o[n][3] *= f1;
      }
      const int nks = (rows + 15) / 16;
      for (int ks = 0; ks < nks; ++ks) {
        uint32_t pa[4], vf[4];
        frag(sx, CH, ks * 16 + 2 * q4, pa);
        ldsm_x4_t_addr(vf, saddr(vb + swz(warp / 4, ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, (warp % 4) * 2 + (lane >> 4))));
        mma16816(o[0], pa, vf[0], vf[1]);
        mma16816(o[1], pa, vf[2], vf[3]);
      }
    }
    __syncthreads();  // every warp is done with the slot and the weights
    if (tid == 0 && chk + 2 < nch) issue_chunk(chk + 2, slot);
  }
  if (16 * warp < D) {
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int hh = g8 + 8 * r;
        if (hh < G) {
          const int c = 16 * warp + 8 * n + 2 * q4;
          so[hh * D + c] = o[n][2 * r];
          so[hh * D + c + 1] = o[n][2 * r + 1];
        }
      }
  }
  if (!ok) atomicCAS(sh.status, 0, (int)SSA_ERR_TIMEOUT);
}

// grid (CL, Hkv, B), one cluster of CL CTAs per (batch, kv head).
//   1. selection: CTA r scores the pooled blocks for the query heads
//      r, r + CL, .. of the group (folding q_t into qsum) and keeps each
//      head's top-k in its shared memory; CTA 0 writes the key mean of a
//      block the token closes;
//   2. after a cluster barrier every CTA reads all heads' selections from
//      the selecting CTAs (distributed shared memory), forms their union and
//      attends its share of the union's blocks (CL-way split, ascending),
//      reading each K/V row once for all g heads and keeping a partial
//      (o, max, sum) per head;
//   3. after a second barrier CTA r merges the partials of heads r, r + CL,
//      .. from the CL CTAs and writes h and lse; a last barrier keeps every
//      CTA's shared memory alive until the merges have read it.
// k_eff <= 64 (each slice keeps at most 63 candidates per head).
// Two CTAs fit an SM (registers and shared memory), so that the clusters
// of every (batch, kv head) are resident at once.
template <typename T, int D>
__global__ void __cluster_dims__(CL, 1, 1) __launch_bounds__(NT, 2)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, TensorRef q,
                  TensorRef K, TensorRef V, TensorRef hout, float* lse, int32_t* idx, float* qsum, float* kbar,
                  DecodeShape sh) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int kvh = blockIdx.y, b = blockIdx.z;
  const int G = sh.g, n = sh.n, s = sh.s, t = sh.t;
  const int i = t / s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hkv = sh.Hq / G;
  const int bk = b * Hkv + kvh;

  extern __shared__ __align__(16) uint8_t smem[];
  const DecodeLayout L(n, G, sh.k, D);
  float* sqbar = reinterpret_cast<float*>(smem + L.qbar);
  float* ssc = reinterpret_cast<float*>(smem + L.sc);
  float2* scand = reinterpret_cast<float2*>(smem + L.cand);  // (score, block index bits)
  float* scorr = reinterpret_cast<float*>(smem + L.corr);
  float* rv = reinterpret_cast<float*>(smem + L.red);
  float* sq = reinterpret_cast<float*>(smem + L.q);
  float* so = reinterpret_cast<float*>(smem + L.o);
  float* smax = reinterpret_cast<float*>(smem + L.mx);
  float* ssum = reinterpret_cast<float*>(smem + L.sum);
  float* sx = reinterpret_cast<float*>(smem + L.x);
  float* sk = reinterpret_cast<float*>(smem + L.k);
  float* sv = reinterpret_cast<float*>(smem + L.v);
  int* slst = reinterpret_cast<int*>(smem + L.lst);
  uint32_t* usel = reinterpret_cast<uint32_t*>(smem + L.usel);

  // ================================================================ 1. selection
  // (a) the query side of every head (q_t folded into the block's query sum;
  //     the head's owner, rank hh % CL, writes the sum back after the first
  //     cluster barrier, when every CTA has read the old value)
  const int slice = (n + CL - 1) / CL;
  const int j0 = min(i, i * rank / CL), j1 = min(i, i * (rank + 1) / CL);  // this CTA's blocks of [0, i)
  // The slice's pooled keys (j1 - j0 rows of D floats, contiguous) start
  // towards the idle attention ring at once, in flight during (a).
  uint64_t* cbar = reinterpret_cast<uint64_t*>(smem + L.bar);  // [0], [1]: the attention ring; [2]: the slice
  int* cabort = reinterpret_cast<int*>(smem + L.bar + 24);
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem + L.k) + 1023) & ~uintptr_t(1023));
  const bool kb_copy = sh.kbs && j1 > j0;
  if (tid == 0) {
    *cabort = 0;
    if (kb_copy) {
      sm100::mbar_init(&cbar[2], 1);
      sm100::fence_mbar_init();
      const uint32_t bytes = (uint32_t)((j1 - j0) * D * 4);
      sm100::mbar_expect_tx(&cbar[2], bytes);
      sm100::bulk_load(ring, kbar + ((int64_t)bk * n + j0) * D, bytes, &cbar[2]);
    }
  }
  // (loads of four elements per thread issued before their use; q_t is
  //  kept in the partial-output buffer until the attention phase)
  for (int base = 0; base < G * D; base += 4 * NT) {
    float xq[4], old[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = base + u * NT + tid;
      xq[u] = old[u] = 0.f;
      if (e < G * D) {
        const int hh = e / D, c = e % D, h = kvh * G + hh;
        xq[u] = to_f32(row_ptr<T>(q, b, h, 0)[c]);
        if (t % s != 0) old[u] = qsum[((int64_t)b * sh.Hq + h) * D + c];
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = base + u * NT + tid;
      if (e < G * D) {
        const float acc = old[u] + xq[u];
        sqbar[e] = sh.per_token ? xq[u] : acc / (float)(t - i * s + 1);
        sq[e] = acc;  // the new sum, written back by the owner below
        so[e] = xq[u];
      }
    }
  }
  for (int e = tid; e < G * 64; e += NT) usel[e] = 0u;
  __syncthreads();
  // (b) scores of this CTA's slice for every head: a thread per (head,
  //     block), the whole pooled key row loaded at once as 16-byte vectors
  //     (the slice's rows stay in L1 across the heads)
  const float* kb = kbar + (int64_t)bk * n * D;
  const int ns = j1 - j0;  // <= slice <= NT
  const float* kslice = kb + (int64_t)j0 * D;  // the slice's rows: in shared memory, or read from global
  bool ok_slice = true;
  if (kb_copy) {
    ok_slice = sm100::mbar_wait(&cbar[2], 0, cabort);
    if (!ok_slice) atomicCAS(sh.status, 0, (int)SSA_ERR_TIMEOUT);
    kslice = reinterpret_cast<const float*>(ring);
  }
  // a thread per (block, head group): the block's row is loaded once and
  // dotted with the queries of heads hg, hg + HG, ..
  const int HG = ns > 0 ? min(G, max(1, NT / ns)) : 1;
  if (tid < ns * HG) {
    const int jj = tid % ns, hg = tid / ns;
    const float4* row = reinterpret_cast<const float4*>(kslice + (int64_t)jj * D);
    // the row in pieces of 32 floats (registers); partial dots per head in
    // the score slots.  Row jj starts at its own 16-byte piece, so that the
    // rows of a warp read different shared-memory banks.
    constexpr int P4 = 8;
#pragma unroll 1
    for (int p0 = 0; p0 < D / 4; p0 += P4) {
      float4 kv[P4];
#pragma unroll
      for (int c4 = 0; c4 < P4; ++c4) kv[c4] = row[(p0 + c4 + jj) & (D / 4 - 1)];
      for (int hh = hg; hh < G; hh += HG) {
        const float4* qv = reinterpret_cast<const float4*>(sqbar + hh * D);
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int c4 = 0; c4 < P4; ++c4) {
          const float4 qq = qv[(p0 + c4 + jj) & (D / 4 - 1)];
          a0 = fmaf(qq.x, kv[c4].x, fmaf(qq.y, kv[c4].y, a0));
          a1 = fmaf(qq.z, kv[c4].z, fmaf(qq.w, kv[c4].w, a1));
        }
        float* slot = ssc + hh * slice + jj;
        *slot = (p0 == 0 ? 0.f : *slot) + (a0 + a1);
      }
    }
    for (int hh = hg; hh < G; hh += HG) {
      const float x = sh.scale * ssc[hh * slice + jj];
      ssc[hh * slice + jj] = (x != x) ? kNegInf : x;  // NaN ranks last
    }
  }
  __syncthreads();
  // (c) per head, the best k-1 of the slice, sorted: each candidate's rank
  //     is the number of slice entries that beat it (score descending, block
  //     ascending); ranks below k-1 are kept, at their rank.  Unfilled list
  //     entries are NaN (compares false with everything).
  const float kOut = __int_as_float(0x7fffffff);
  const int km1 = sh.k - 1;
  if (i + 1 > sh.k && ns <= 64) {
    // A warp per head sorts the slice's (score, block) pairs with a bitonic
    // network, score descending and block ascending (the rank rule's order),
    // two pairs per lane (elements 2 lane and 2 lane + 1; missing ones rank
    // last), and keeps the first k-1.
    for (int hh = warp; hh < G; hh += NT / 32) {
      const float* sc = ssc + hh * slice;
      float v[2];
      int jb[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int e = 2 * lane + q;
        v[q] = e < ns ? sc[e] : kNegInf;
        jb[q] = e < ns ? j0 + e : INT_MAX;
      }
      auto better = [](float va, int ja, float vb, int jbb) { return va > vb || (va == vb && ja < jbb); };
#pragma unroll
      for (int sz = 2; sz <= 64; sz <<= 1) {
#pragma unroll
        for (int d = sz >> 1; d > 0; d >>= 1) {
          if (d == 1) {  // both elements in this lane
            const bool desc = ((2 * lane) & sz) == 0;
            if (better(v[1], jb[1], v[0], jb[0]) == desc) {
              const float tv = v[0];
              v[0] = v[1];
              v[1] = tv;
              const int tj = jb[0];
              jb[0] = jb[1];
              jb[1] = tj;
            }
          } else {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int e = 2 * lane + q;
              const float ov = __shfl_xor_sync(0xffffffffu, v[q], d >> 1);
              const int oj = __shfl_xor_sync(0xffffffffu, jb[q], d >> 1);
              const bool low = (e & d) == 0;       // the lower index of the pair
              const bool desc = (e & sz) == 0;     // this run sorts descending
              // the lower index keeps the better pair in a descending run, the worse in an ascending one
              const bool take = better(ov, oj, v[q], jb[q]) == (low == desc);
              if (take) {
                v[q] = ov;
                jb[q] = oj;
              }
            }
          }
        }
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int e = 2 * lane + q;
        if (e < km1) scand[hh * 64 + e] = e < ns ? make_float2(v[q], __int_as_float(jb[q]))
                                                 : make_float2(kOut, __int_as_float(INT_MAX));
      }
    }
  } else if (i + 1 > sh.k) {
    for (int e = tid; e < G * km1; e += NT) scand[(e / km1) * 64 + e % km1] = make_float2(kOut, __int_as_float(INT_MAX));
    __syncthreads();
    for (int e = tid; e < G * ns; e += NT) {
      const int hh = e / ns, jj = e % ns;
      const float* sc = ssc + hh * slice;
      const float v = sc[jj];
      int rk0 = 0, rk1 = 0, o = 0;
      for (; o + 8 <= ns; o += 8) {  // eight loads in flight, two counters
#pragma unroll
        for (int u = 0; u < 8; u += 2) {
          const float w0 = sc[o + u], w1 = sc[o + u + 1];
          rk0 += (w0 > v || (w0 == v && o + u < jj)) ? 1 : 0;
          rk1 += (w1 > v || (w1 == v && o + u + 1 < jj)) ? 1 : 0;
        }
      }
      for (; o < ns; ++o) {
        const float w = sc[o];
        rk0 += (w > v || (w == v && o < jj)) ? 1 : 0;
      }
      const int rk = rk0 + rk1;
      if (rk < km1) scand[hh * 64 + rk] = make_float2(v, __int_as_float(j0 + jj));
    }
  }
  cluster.sync();  // every CTA's candidate lists are visible to the cluster
  // (d) every CTA merges every head's CL sorted lists, read straight from the
  //     peers' shared memory: a warp per head sorts the CL lists' candidates
  //     (score descending, block ascending) with a bitonic network and keeps
  //     the k-1 best with the diagonal block in this CTA's copy of every
  //     head's selection bits (k <= 16: four pairs per lane in registers;
  //     larger k: the warp's share of the idle attention ring).  No selection
  //     has to cross the cluster afterwards.  The head's owner (CTA hh mod CL)
  //     writes its query sum and idx row.
  auto better = [](float va, int ja, float vb, int jb) { return va > vb || (va == vb && ja < jb); };
  auto merge_heads = [&]() {
    constexpr int E = 4;
    constexpr int PER_LIST = 32 * E / CL;  // 16 candidate slots per list (>= k - 1)
    for (int hh = warp; hh < G; hh += NT / 32) {
      // Each list is sorted already: odd lists are read in reverse, so every
      // pair of lists is a bitonic sequence and the network starts at the
      // merges of 32.
      float v[E];
      int jb[E];
#pragma unroll
      for (int q = 0; q < E; ++q) {
        const int e = E * lane + q, r = e / PER_LIST, c0 = e % PER_LIST;
        const int c = (r & 1) ? PER_LIST - 1 - c0 : c0;
        float2 x = make_float2(kNegInf, __int_as_float(INT_MAX));
        if (c < km1) x = cluster.map_shared_rank(scand, r)[hh * 64 + c];
        jb[q] = __float_as_int(x.y);
        v[q] = jb[q] == INT_MAX ? kNegInf : x.x;  // unfilled entries rank last
      }
#pragma unroll
      for (int sz = 2 * PER_LIST; sz <= 32 * E; sz <<= 1) {
#pragma unroll
        for (int d = sz >> 1; d > 0; d >>= 1) {
          if (d < E) {  // both elements of a pair in this lane
#pragma unroll
            for (int q = 0; q < E; ++q) {
              if (q & d) continue;
              const int hi = q | d;
              const bool desc = ((E * lane + q) & sz) == 0;
              if (better(v[hi], jb[hi], v[q], jb[q]) == desc) {
                const float tv = v[q];
                v[q] = v[hi];
                v[hi] = tv;
                const int tj = jb[q];
                jb[q] = jb[hi];
                jb[hi] = tj;
              }
            }
          } else {
#pragma unroll
            for (int q = 0; q < E; ++q) {
              const int e = E * lane + q;
              const float ov = __shfl_xor_sync(0xffffffffu, v[q], d / E);
              const int oj = __shfl_xor_sync(0xffffffffu, jb[q], d / E);
              const bool low = (e & d) == 0, desc = (e & sz) == 0;
              // the lower index keeps the better pair in a descending run, the worse in an ascending one
              if (better(ov, oj, v[q], jb[q]) == (low == desc)) {
                v[q] = ov;
                jb[q] = oj;
              }
            }
          }
        }
      }
#pragma unroll
      for (int q = 0; q < E; ++q)
        if (E * lane + q < km1 && jb[q] != INT_MAX) atomicOr(&usel[hh * 64 + (jb[q] >> 5)], 1u << (jb[q] & 31));
      if (lane == 0) atomicOr(&usel[hh * 64 + (i >> 5)], 1u << (i & 31));
    }
  };
  if (i + 1 <= sh.k) {
    for (int e = tid; e < G * (i + 1); e += NT) {
      const int hh = e / (i + 1), j = e % (i + 1);
      atomicOr(&usel[hh * 64 + (j >> 5)], 1u << (j & 31));
    }
  } else if (km1 <= 15) {
    merge_heads();
  } else {
    const int per_list = km1 <= 31 ? 32 : 64, n2 = CL * per_list;  // 256 or 512 candidates
    float2* buf = reinterpret_cast<float2*>(ring) + warp * 512;   // the ring is idle until phase 2
    for (int hh = warp; hh < G; hh += NT / 32) {
      for (int e = lane; e < n2; e += 32) {
        const int r = e / per_list, c = e % per_list;
        float2 x = make_float2(kNegInf, __int_as_float(INT_MAX));
        if (c < km1) x = cluster.map_shared_rank(scand, r)[hh * 64 + c];
        if (__float_as_int(x.y) == INT_MAX) x.x = kNegInf;  // unfilled entries rank last
        buf[e] = x;
      }
      __syncwarp();
      for (int sz = 2; sz <= n2; sz <<= 1)
        for (int d = sz >> 1; d > 0; d >>= 1) {
          for (int pr = lane; pr < n2 / 2; pr += 32) {
            const int lo = 2 * d * (pr / d) + pr % d, hi = lo + d;  // the pr-th pair at stride d
            const bool desc = (lo & sz) == 0;
            const float2 xa = buf[lo], xb = buf[hi];
            if (better(xb.x, __float_as_int(xb.y), xa.x, __float_as_int(xa.y)) == desc) {
              buf[lo] = xb;
              buf[hi] = xa;
            }
          }
          __syncwarp();
        }
      for (int e = lane; e < km1; e += 32) {
        const int jx = __float_as_int(buf[e].y);
        if (jx != INT_MAX) atomicOr(&usel[hh * 64 + (jx >> 5)], 1u << (jx & 31));
      }
      if (lane == 0) atomicOr(&usel[hh * 64 + (i >> 5)], 1u << (i & 31));
      __syncwarp();  // the buffer is read before the next head refills it
    }
  }
  __syncthreads();
  const int nown = rank < G ? (G - 1 - rank) / CL + 1 : 0;  // heads rank, rank + CL, ..
  for (int e = tid; e < nown * D; e += NT) {
    const int hh = rank + CL * (e / D), c = e % D;
    qsum[((int64_t)b * sh.Hq + kvh * G + hh) * D + c] = sq[hh * D + c];
  }
  // idx rows, ascending and -1 padded: warp hl writes head rank + CL*hl's
  // (lane l places the blocks of words 2l and 2l + 1 after a prefix count)
  if (warp < nown) {
    const uint32_t* sel = usel + (rank + CL * warp) * 64;
    int32_t* out = idx + ((int64_t)b * sh.Hq + kvh * G + rank + CL * warp) * sh.k;
    const uint32_t w0 = sel[2 * lane], w1 = sel[2 * lane + 1];
    const int c = __popc(w0) + __popc(w1);
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    const int cnt = __shfl_sync(0xffffffffu, incl, 31);
    int pos = incl - c;
    for (uint32_t xw = w0; xw; xw &= xw - 1, ++pos)
      if (pos < sh.k) out[pos] = 64 * lane + __ffs(xw) - 1;
    for (uint32_t xw = w1; xw; xw &= xw - 1, ++pos)
      if (pos < sh.k) out[pos] = 64 * lane + 32 + __ffs(xw) - 1;
    for (int q = cnt + lane; q < sh.k; q += 32) out[q] = -1;
  }
  // the token closes block i: its key mean joins the pooled cache (no
  // reader of this call uses kbar[i])
  if (rank == 0 && t % s == s - 1) {
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
  // (no cluster barrier here: every CTA holds every head's selection, and the
  //  peers' candidate lists stay untouched until the last barrier)

  // ================================================================ 2. attention
  // (every head's selection was pushed into usel by its owner; q_t waits in so)
  for (int e = tid; e < G * D; e += NT) {
    sq[e] = so[e];
    so[e] = 0.f;
  }
  if (tid < G) {
    smax[tid] = kNegInf;
    ssum[tid] = 0.f;
  }
  if (sh.mma) {
    // the ring held the pooled-key slice and the merge's list copies (generic
    // accesses) before the TMA loads write it
    sm100::fence_proxy_async_smem();
    if (tid == 0) {
      sm100::mbar_init(&cbar[0], 1);
      sm100::mbar_init(&cbar[1], 1);
      sm100::fence_mbar_init();
    }
  }
  // chunks of the CTA's union blocks: CH rows (chr rows of a block of s < CH
  // on the bf16 path), the last one cut at t
  const int crows = sh.mma ? sh.chr : CH;
  const int cpb = (s + crows - 1) / crows;  // chunks per block
  auto chunk_rows = [&](int chk, int& j, int& c0) {
    j = slst[1 + chk / cpb];
    c0 = j * s + (chk % cpb) * crows;
    return max(0, min(crows, min(j * s + s, t + 1) - c0));
  };
  // bf16 path: one thread loads a chunk's K and V halves into ring slot
  // `slot` by TMA (the slot's barrier counts the bytes; rows past N read zeros)
  auto issue_chunk = [&](int chk, int slot) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
      int j, c0;
      chunk_rows(chk, j, c0);
      uint8_t* base = ring + slot * 2 * kTileBytes<D>;
      sm100::mbar_expect_tx(&cbar[slot], (uint32_t)(2 * (D / 64) * sh.chr * 128));
#pragma unroll
      for (int hh = 0; hh < D / 64; ++hh) {
        sm100::tma_load_4d(base + hh * CH * 128, &tmK, &cbar[slot], hh * 64, c0, kvh, b);
        sm100::tma_load_4d(base + kTileBytes<D> + hh * CH * 128, &tmV, &cbar[slot], hh * 64, c0, kvh, b);
      }
    }
  };
  __syncthreads();
  // this CTA's entries [cnt*rank/CL, cnt*(rank+1)/CL) of the ascending union
  if (warp == 0) {
    uint32_t w0 = 0, w1 = 0;
    for (int hh = 0; hh < G; ++hh) {
      w0 |= usel[hh * 64 + 2 * lane];
      w1 |= usel[hh * 64 + 2 * lane + 1];
    }
    const int c = __popc(w0) + __popc(w1);
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    const int cnt = __shfl_sync(0xffffffffu, incl, 31);
    const int lo = cnt * rank / CL, hi = cnt * (rank + 1) / CL;
    int pos = incl - c;
    for (uint32_t xw = w0; xw; xw &= xw - 1, ++pos)
      if (pos >= lo && pos < hi) slst[1 + pos - lo] = 64 * lane + __ffs(xw) - 1;
    for (uint32_t xw = w1; xw; xw &= xw - 1, ++pos)
      if (pos >= lo && pos < hi) slst[1 + pos - lo] = 64 * lane + 32 + __ffs(xw) - 1;
    if (lane == 0) slst[0] = hi - lo;
    if (sh.mma) {  // the first two chunks start at once
      __syncwarp();
      const int nch0 = slst[0] * cpb;
      if (lane == 0)
        for (int c2 = 0; c2 < 2 && c2 < nch0; ++c2) issue_chunk(c2, c2);
    }
  }
  __syncthreads();
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    if (sh.mma) decode_attend_mma<D>(sh, G, rank, t, tid, lane, warp, slst, usel, sq, so, smax, ssum, scorr, sx,
                                     ring, cbar, cabort, chunk_rows, issue_chunk, cpb);
  }
  if (!sh.mma) {
    constexpr int VEC = Vec16<T>::kN;
    constexpr int ITERS = CH * (D / VEC) / NT;  // 16-byte loads per thread per chunk and tensor
    const int nb = slst[0];
    const int nch = nb * cpb;
    float tk[ITERS][VEC], tv[ITERS][VEC];
    auto load_chunk = [&](int chk) {
      int j, c0;
      const int rows = chunk_rows(chk, j, c0);
#pragma unroll
      for (int it = 0; it < ITERS; ++it) {
        const int xx = tid + it * NT, r = xx / (D / VEC), c = (xx % (D / VEC)) * VEC;
        if (r < rows) {
          Vec16<T>::load(row_ptr<T>(K, b, kvh, (int64_t)c0 + r) + c, tk[it]);
          Vec16<T>::load(row_ptr<T>(V, b, kvh, (int64_t)c0 + r) + c, tv[it]);
        }
      }
    };
    if (nch > 0) load_chunk(0);
    for (int chk = 0; chk < nch; ++chk) {
      int j, c0;
      const int rows = chunk_rows(chk, j, c0);
#pragma unroll
      for (int it = 0; it < ITERS; ++it) {
        const int xx = tid + it * NT, r = xx / (D / VEC), c = (xx % (D / VEC)) * VEC;
        if (r < rows) {
#pragma unroll
          for (int y = 0; y < VEC; ++y) {
            sk[r * (D + 1) + c + y] = tk[it][y];
            sv[r * D + c + y] = tv[it][y];
          }
        }
      }
      if (chk + 1 < nch) load_chunk(chk + 1);  // in flight while this chunk is used
      __syncthreads();
      for (int xx = tid; xx < G * CH; xx += NT) {
        const int hh = xx / CH, uu = xx % CH;
        float v = kNegInf;
        if (uu < rows && ((usel[hh * 64 + (j >> 5)] >> (j & 31)) & 1u)) {
          const float* qvv = sq + hh * D;
          const float* kvv = sk + uu * (D + 1);
          float acc = 0.f;
#pragma unroll 8
          for (int c = 0; c < D; ++c) acc = fmaf(qvv[c], kvv[c], acc);
          v = sh.scale * acc;
        }
        sx[xx] = v;
      }
      __syncthreads();
      // softmax statistics: a warp per head; the weights go back over the logits
      for (int hh = warp; hh < G; hh += NT / 32) {
        if (!((usel[hh * 64 + (j >> 5)] >> (j & 31)) & 1u)) continue;
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
        if (lane == 0) {
          smax[hh] = m_new;
          ssum[hh] = ssum[hh] * corr + ps;
          scorr[hh] = corr;
        }
      }
      __syncthreads();
      // o += P V: a thread per (head, column), every warp busy
      for (int xx = tid; xx < G * D; xx += NT) {
        const int hh = xx / D, c = xx % D;
        if (!((usel[hh * 64 + (j >> 5)] >> (j & 31)) & 1u)) continue;
        const float* xs = sx + hh * CH;
        float acc = so[xx] * scorr[hh];
        for (int uu = 0; uu < rows; ++uu) acc = fmaf(xs[uu], sv[uu * D + c], acc);
        so[xx] = acc;
      }
      __syncthreads();
    }
  }
  cluster.sync();  // every CTA's partial (o, max, sum) is visible to the cluster

  // ================================================================ 3. merge
  for (int hh = rank; hh < G; hh += CL) {
    float M = kNegInf;
#pragma unroll
    for (int r = 0; r < CL; ++r) M = fmaxf(M, *cluster.map_shared_rank(smax + hh, r));
    float Lsum = 0.f, wgt[CL];
#pragma unroll
    for (int r = 0; r < CL; ++r) {
      const float m = *cluster.map_shared_rank(smax + hh, r);
      wgt[r] = (m == kNegInf) ? 0.f : __expf(m - M);
      Lsum += *cluster.map_shared_rank(ssum + hh, r) * wgt[r];
    }
    for (int c = tid; c < D; c += NT) {
      float acc = 0.f;
#pragma unroll
      for (int r = 0; r < CL; ++r)
        if (wgt[r] != 0.f) acc = fmaf(*cluster.map_shared_rank(so + hh * D + c, r), wgt[r], acc);
      row_ptr_w<T>(hout, b, kvh * G + hh, 0)[c] = from_f32<T>(Lsum > 0.f ? acc / Lsum : 0.f);
    }
    if (tid == 0) lse[(int64_t)b * sh.Hq + kvh * G + hh] = Lsum > 0.f ? M + logf(Lsum) : kNegInf;
  }
  cluster.sync();  // peers' shared memory stays alive until every merge has read it
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
cudaError_t decode_t(const Dims& Dm, const DecodeArgs& a, int32_t* status, cudaStream_t st) {
  // the bf16 path reads chunks of min(CH, s) rows through TMA maps (which
  // need 16-byte aligned rows and strides; otherwise the CUDA-core path runs)
  const int chr = std::min(CH, Dm.s);
  CUtensorMap mk{}, mv{};
  const int mma = std::is_same<T, __nv_bfloat16>::value && Dm.g <= 16 &&
                  make_tma_map_bf16(&mk, a.k, Dm.B, Dm.Hkv, Dm.N, chr, D) &&
                  make_tma_map_bf16(&mv, a.v, Dm.B, Dm.Hkv, Dm.N, chr, D);
  // the pooled-key slice of a CTA fits the ring and starts 16-byte aligned
  const int kbs = reinterpret_cast<uintptr_t>(a.kbar) % 16 == 0 &&
                  (size_t)((Dm.n + CL - 1) / CL) * D * 4 <= (size_t)kRingBytes<D>;
  DecodeShape sh{Dm.Hq, Dm.g, Dm.N, Dm.s, Dm.n, Dm.k, a.t, Dm.scale, Dm.per_token, mma, chr, kbs, status};
  const size_t smem = DecodeLayout(Dm.n, Dm.g, Dm.k, D).bytes;
  auto run = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3(CL, Dm.Hkv, Dm.B), NT, smem, st>>>(mk, mv, a.q, a.k, a.v, a.h, a.lse, a.idx, a.qsum, a.kbar, sh);
    count_launches(1);
    return cudaGetLastError();
  };
  return run(decode_kernel<T, D>);
}

template <typename T, int D>
cudaError_t prefill_t(const Dims& Dm, const DecodeArgs& a, cudaStream_t st) {
  decode_prefill_kernel<T, D><<<dim3(Dm.n + 1, Dm.Hq, Dm.B), 128, 0, st>>>(a.q, a.k, a.qsum, a.kbar, Dm.Hq, Dm.Hkv,
                                                                          Dm.s, Dm.n, a.t);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

size_t decode_smem_bytes(const Dims& D) { return DecodeLayout(D.n, D.g, D.k, D.d).bytes; }

bool decode_supported(const Dims& D) { return D.k <= 64 && decode_smem_bytes(D) <= 232448; }

size_t decode_ws_bytes(const Dims& D) {
  (void)D;
  return 0;  // the decode step keeps its scratch in the cluster's shared memory
}

cudaError_t launch_decode(const Dims& D, const DecodeArgs& a, int32_t* dev_status, cudaStream_t st) {
  if (D.dtype == SSA_BF16)
    return D.d == 128 ? decode_t<__nv_bfloat16, 128>(D, a, dev_status, st)
                      : decode_t<__nv_bfloat16, 64>(D, a, dev_status, st);
  return D.d == 128 ? decode_t<float, 128>(D, a, dev_status, st) : decode_t<float, 64>(D, a, dev_status, st);
}

cudaError_t launch_decode_prefill(const Dims& D, const DecodeArgs& a, cudaStream_t st) {
  if (D.dtype == SSA_BF16)
    return D.d == 128 ? prefill_t<__nv_bfloat16, 128>(D, a, st) : prefill_t<__nv_bfloat16, 64>(D, a, st);
  return D.d == 128 ? prefill_t<float, 128>(D, a, st) : prefill_t<float, 64>(D, a, st);
}

}  // namespace ssa
