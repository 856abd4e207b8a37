// Sparse-stream forward for blocks of 16 or 32 keys with per-block
// selection: every query block walks its own selected key blocks.
//
// What it computes ("SSA: Achieving Sparser Attention ...", "Practical
// Implementation of SSA": the sparse stream attends, for query t in block i,
// the causal keys of the blocks in Sel(i); "Training Efficiency
// Considerations": at inference the sparse stream runs alone):
//   h_sparse[t] = softmax_{u in A_t}(scale q_t . k_u) V,   lse_sel[t] = log sum_{u in A_t} e^{scale q_t . k_u}.
//
// With blocks of 16 or 32 keys the rows of one 64-row tile select up to
// 4 x k different blocks, so a tile-wide walk over the union of their key
// tiles reads and multiplies mostly keys that no row of the tile attends.
// Here the unit is the query block: one warp (blocks of 16) or a pair of
// warps (blocks of 32, 16 rows each) holds the block's query rows as mma.sync
// A fragments in registers and visits exactly the key blocks of Sel(i), in
// ascending order, each one S-key step of an online softmax (S x d keys and
// values, double or triple buffered with cp.async in the group's own shared
// memory).  Only the diagonal block needs the causal mask.  The rows of a CTA
// share nothing but the launch; the key and value rows of a kv head are read
// from L2 by every query head that selected them.
#include "mma_sync.cuh"
#include "ssa_internal.cuh"

namespace ssa {
namespace {

using namespace warp_mma;
using bf16 = __nv_bfloat16;

constexpr int BM = 64;   // query rows per CTA
constexpr int NT = 128;  // 4 warps of 16 rows
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct WalkShape {
  int Hq, g, N, n, k;
  float scale;
};

template <int D, int S>
struct WalkCfg {
  static constexpr int W = S / 16;                 // warps per query block
  static constexpr int G = 4 / W;                  // query blocks per CTA
  static constexpr int NS = D == 64 ? 3 : 2;       // K/V stages per query block
  static constexpr int LD = D + 8;                 // row pitch (conflict-free ldmatrix)
  static constexpr int STAGE = S * LD * 2;         // one key (or value) block; stage 0 stages the output
  static constexpr int GRP_BYTES = NS * 2 * STAGE;
  static constexpr int SEL_OFF = G * GRP_BYTES;
  static constexpr int SMEM = SEL_OFF + G * 64 * 4;  // + one 2048-bit selection set per query block
};

// Barrier of the W warps that share a query block.
template <int W>
__device__ __forceinline__ void group_sync(int grp) {
  if constexpr (W == 1) {
    __syncwarp();
  } else {
    asm volatile("bar.sync %0, %1;\n" ::"r"(grp + 1), "n"(32 * W) : "memory");
  }
}

template <int D, int S>
__global__ void __launch_bounds__(NT, D == 64 ? 4 : 2) fwd_walk_kernel(FwdArgs a, WalkShape sh) {
  using C = WalkCfg<D, S>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grp = warp / C::W, gt = (warp % C::W) * 32 + lane;  // query block of the CTA, thread in it
  const int qt = gridDim.x - 1 - blockIdx.x;                     // the longest rows first
  const int h = blockIdx.y, b = blockIdx.z, kvh = h / sh.g;
  const int t0 = qt * BM;
  const int i = t0 / S + grp;      // this group's query block
  const int r0 = t0 + warp * 16;   // this warp's first row

  unsigned char* gbase = smem + grp * C::GRP_BYTES;
  uint32_t* sel = reinterpret_cast<uint32_t*>(smem + C::SEL_OFF) + grp * 64;
  auto kbuf = [&](int st) { return reinterpret_cast<bf16 (*)[C::LD]>(gbase + (2 * st) * C::STAGE); };
  auto vbuf = [&](int st) { return reinterpret_cast<bf16 (*)[C::LD]>(gbase + (2 * st + 1) * C::STAGE); };

  for (int w = gt; w < 64; w += 32 * C::W) sel[w] = 0u;
  group_sync<C::W>(grp);
  const int32_t* irow = a.idx + (((int64_t)b * sh.Hq + h) * sh.n + i) * sh.k;
  for (int e = gt; e < sh.k; e += 32 * C::W) {
    const int j = irow[e];
    if (j >= 0 && j <= i) atomicOr(&sel[j >> 5], 1u << (j & 31));  // duplicates and invalid entries drop out
  }
  group_sync<C::W>(grp);

  const int nw = i / 32 + 1;
  auto next_blk = [&](int from) -> int {  // first selected block >= from, else -1
    for (int w = from >> 5; w < nw; ++w) {
      uint32_t bits = sel[w];
      if (w == (from >> 5)) bits &= ~0u << (from & 31);
      if (bits) return w * 32 + __ffs(bits) - 1;
    }
    return -1;
  };
  auto load_blk = [&](int j, int st) {
    bf16 (*ks)[C::LD] = kbuf(st);
    bf16 (*vs)[C::LD] = vbuf(st);
    for (int e = gt; e < S * D / 8; e += 32 * C::W) {
      const int r = e / (D / 8), c = (e % (D / 8)) * 8;
      cp_async16(&ks[r][c], row_ptr<bf16>(a.k, b, kvh, (int64_t)j * S + r) + c, 16);
      cp_async16(&vs[r][c], row_ptr<bf16>(a.v, b, kvh, (int64_t)j * S + r) + c, 16);
    }
  };

  int issued = -1;
#pragma unroll
  for (int p = 0; p < C::NS - 1; ++p) {
    const int j = next_blk(issued + 1);
    if (j >= 0) {
      load_blk(j, p);
      issued = j;
    }
    cp_async_commit();
  }

  const int g8 = lane >> 2, q4 = lane & 3;
  const float sl2 = sh.scale * kLog2e;  // logits in log2 units
  float m[2] = {kNegInf, kNegInf}, l[2] = {0.f, 0.f};
  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
  uint32_t qa[D / 16][4];  // the warp's Q rows as A fragments, straight from global memory
  {
    const bf16* q0p = row_ptr<bf16>(a.q, b, h, r0 + g8);
    const bf16* q1p = row_ptr<bf16>(a.q, b, h, r0 + g8 + 8);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int c = kk * 16 + 2 * q4;
      qa[kk][0] = *reinterpret_cast<const uint32_t*>(q0p + c);
      qa[kk][1] = *reinterpret_cast<const uint32_t*>(q1p + c);
      qa[kk][2] = *reinterpret_cast<const uint32_t*>(q0p + c + 8);
      qa[kk][3] = *reinterpret_cast<const uint32_t*>(q1p + c + 8);
    }
  }

  int cur = next_blk(0);
  for (int it = 0; cur >= 0; ++it) {
    cp_async_wait<C::NS - 2>();
    group_sync<C::W>(grp);  // block `it` has landed for the group; stage (it - 1) is free
    {
      const int j = next_blk(issued + 1);
      if (j >= 0) {
        load_blk(j, (it + C::NS - 1) % C::NS);
        issued = j;
      }
      cp_async_commit();
    }
    const int st = it % C::NS;
    bf16 (*ks)[C::LD] = kbuf(st);
    bf16 (*vs)[C::LD] = vbuf(st);

    float sc[S / 8][4];
#pragma unroll
    for (int n = 0; n < S / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[n][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
      for (int jn = 0; jn < S / 16; ++jn) {
        uint32_t kb[4];
        ldsm_x4(kb, &ks[jn * 16 + (lane & 7) + ((lane >> 4) << 3)][kk * 16 + ((lane >> 3) & 1) * 8]);
        mma16816(sc[2 * jn], qa[kk], kb[0], kb[1]);
        mma16816(sc[2 * jn + 1], qa[kk], kb[2], kb[3]);
      }
    if (cur == i) {  // the diagonal block: keys after the row are not causal
#pragma unroll
      for (int n = 0; n < S / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int u = cur * S + n * 8 + 2 * q4 + (e & 1);
          const int t = r0 + g8 + 8 * (e >> 1);
          if (u > t) sc[n][e] = kNegInf;
        }
    }
    float c[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float mx = kNegInf;
#pragma unroll
      for (int n = 0; n < S / 8; ++n) mx = fmaxf(mx, fmaxf(sc[n][2 * r], sc[n][2 * r + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float nm = fmaxf(m[r], mx * sl2);  // finite: every row keeps a key in every visited block
      c[r] = fast_ex2(m[r] - nm);
      m[r] = nm;
      l[r] *= c[r];
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      o[n][0] *= c[0]; o[n][1] *= c[0];
      o[n][2] *= c[1]; o[n][3] *= c[1];
    }
#pragma unroll
    for (int kk = 0; kk < S / 16; ++kk) {
      uint32_t pa[4];
#pragma unroll
      for (int hn = 0; hn < 2; ++hn) {
        float w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) w[e] = fast_ex2(fmaf(sc[2 * kk + hn][e], sl2, -m[e >> 1]));
        l[0] += w[0] + w[1];
        l[1] += w[2] + w[3];
        pa[hn * 2] = pack2(w[0], w[1]);
        pa[hn * 2 + 1] = pack2(w[2], w[3]);
      }
#pragma unroll
      for (int jd = 0; jd < D / 16; ++jd) {
        uint32_t vb[4];
        ldsm_x4_t(vb, &vs[kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8][jd * 16 + (lane >> 4) * 8]);
        mma16816(o[2 * jd], pa, vb[0], vb[1]);
        mma16816(o[2 * jd + 1], pa, vb[2], vb[3]);
      }
    }
    cur = next_blk(cur + 1);
  }
  cp_async_wait<0>();
  group_sync<C::W>(grp);  // every warp of the group is done with the stages
  bf16 (*qs)[C::LD] = kbuf(0) + (warp % C::W) * 16;  // this warp's 16 output rows

  float inv[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
    inv[r] = l[r] > 0.f ? 1.0f / l[r] : 0.f;
  }
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int r = 0; r < 2; ++r)
      *reinterpret_cast<uint32_t*>(&qs[g8 + 8 * r][n * 8 + 2 * q4]) = pack2(o[n][2 * r] * inv[r], o[n][2 * r + 1] * inv[r]);
  __syncwarp();
  for (int e = lane; e < 16 * D / 8; e += 32) {
    const int r = e / (D / 8), col = (e % (D / 8)) * 8;
    *reinterpret_cast<uint4*>(row_ptr_w<bf16>(a.hs, b, h, r0 + r) + col) = *reinterpret_cast<const uint4*>(&qs[r][col]);
  }
  if (q4 == 0) {
#pragma unroll
    for (int r = 0; r < 2; ++r)
      a.lse_sel[((int64_t)b * sh.Hq + h) * sh.N + r0 + g8 + 8 * r] = l[r] > 0.f ? m[r] * kLn2 + logf(l[r]) : kNegInf;
  }
}

template <int D, int S>
cudaError_t launch_t(const Dims& Dm, const FwdArgs& a, cudaStream_t st) {
  using C = WalkCfg<D, S>;
  auto kern = fwd_walk_kernel<D, S>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  WalkShape sh{Dm.Hq, Dm.g, Dm.N, Dm.n, Dm.k, Dm.scale};
  dim3 grid(Dm.N / BM, Dm.Hq, Dm.B);
  kern<<<grid, NT, C::SMEM, st>>>(a, sh);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

bool fwd_walk_supported(const Dims& D) {
  return D.dtype == SSA_BF16 && !D.per_token && (D.s == 16 || D.s == 32) && (D.d == 64 || D.d == 128);
}

cudaError_t launch_fwd_walk(const Dims& D, const FwdArgs& a, cudaStream_t st) {
  if (D.d == 64) return D.s == 16 ? launch_t<64, 16>(D, a, st) : launch_t<64, 32>(D, a, st);
  return D.s == 16 ? launch_t<128, 16>(D, a, st) : launch_t<128, 32>(D, a, st);
}

}  // namespace ssa
