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
#include "sm100_ptx.cuh"
#include "ssa_internal.cuh"

namespace ssa {
namespace {

using namespace warp_mma;
using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int BM = 64;   // query rows per CTA
constexpr int NT = 128;  // 4 warps of 16 rows
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// The running row maximum moves only when a block's maximum exceeds it by
// more than this (log2 units): the exponentials then stay below 2^8, and a
// rescale of the accumulators is rare.  Numerator and denominator share the
// stale maximum, so the result is the same softmax.
constexpr float kLazy = 8.0f;

struct WalkShape {
  int Hq, g, N, n, k;
  float scale;
  int32_t* status;
};

// Shared memory of one query block (one group of W warps): NS slots, each
// the K block then the V block of one selected key block, stored as
// 64-column halves of S rows x 128 B in the TMA 128-byte swizzle (the 16-byte
// chunk c of row r sits at chunk c ^ (r & 7)), so that ldmatrix reads are
// conflict-free without padding.
template <int D, int S>
struct WalkCfg {
  static constexpr int W = S / 16;         // warps per query block
  static constexpr int G = 4 / W;          // query blocks per CTA
  static constexpr int NS = 3;             // slots: block it (P V), block it + 1 (its logits), one load ahead
  static constexpr int HALF = S * 128;     // 64 columns of one block
  static constexpr int TILE = (D / 64) * HALF;
  static constexpr int SLOT = 2 * TILE;    // K, then V
  static constexpr int GRP_BYTES = NS * SLOT;
  static constexpr int BAR_OFF = G * GRP_BYTES;            // NS mbarriers per query block
  static constexpr int FLAG_OFF = BAR_OFF + G * NS * 8;    // one abort flag per query block
  static constexpr int SEL_OFF = FLAG_OFF + G * 4;         // one 2048-bit selection set per query block
  static constexpr int SMEM = SEL_OFF + G * 64 * 4 + 1024;  // + alignment slack
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

// Byte offset of the 16-byte chunk `ch` (0..7) of row r in a swizzled half.
__device__ __forceinline__ uint32_t swz(int r, int ch) { return (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4)); }

template <int D, int S>
__global__ void __launch_bounds__(NT, D == 64 ? 4 : 2)
    fwd_walk_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, FwdArgs a,
                    WalkShape sh) {
  using C = WalkCfg<D, S>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grp = warp / C::W, wig = warp % C::W, gt = wig * 32 + lane;  // query block of the CTA, thread in it
  const int qt = gridDim.x - 1 - blockIdx.x;                               // the longest rows first
  const int h = blockIdx.y, b = blockIdx.z, kvh = h / sh.g;
  const int t0 = qt * BM;
  const int i = t0 / S + grp;     // this group's query block
  const int r0 = t0 + warp * 16;  // this warp's first row

  unsigned char* gbase = smem + grp * C::GRP_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF) + grp * C::NS;
  int* abort_flag = reinterpret_cast<int*>(smem + C::FLAG_OFF) + grp;
  uint32_t* sel = reinterpret_cast<uint32_t*>(smem + C::SEL_OFF) + grp * 64;

  for (int w = gt; w < 64; w += 32 * C::W) sel[w] = 0u;
  if (gt == 0) {
#pragma unroll
    for (int s = 0; s < C::NS; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  group_sync<C::W>(grp);
  const int32_t* irow = a.idx + (((int64_t)b * sh.Hq + h) * sh.n + i) * sh.k;
  for (int e = gt; e < sh.k; e += 32 * C::W) {
    const int j = irow[e];
    if (j >= 0 && j <= i) atomicOr(&sel[j >> 5], 1u << (j & 31));  // duplicates and invalid entries drop out
  }
  group_sync<C::W>(grp);

  // Number of selected blocks, and whether the diagonal one (always the last
  // in ascending order) is among them.
  const int nw = i / 32 + 1;
  int cnt = 0;
  for (int w = lane; w < nw; w += 32) cnt += __popc(sel[w]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  const bool diag_sel = (sel[i >> 5] >> (i & 31)) & 1u;

  // Thread gt == 0 issues the loads, in ascending block order.
  int iw = 0;
  uint32_t ibits = sel[0];
  int issued = 0;
  auto issue_next = [&](int slot) {
    while (ibits == 0u) ibits = sel[++iw];  // bounded: issued < cnt blocks remain
    const int j = iw * 32 + __ffs(ibits) - 1;
    ibits &= ibits - 1u;
    unsigned char* dst = gbase + slot * C::SLOT;
    mbar_expect_tx(&full[slot], C::SLOT);
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh) {
      tma_load_4d(dst + hh * C::HALF, &tmK, &full[slot], hh * 64, j * S, kvh, b);
      tma_load_4d(dst + C::TILE + hh * C::HALF, &tmV, &full[slot], hh * 64, j * S, kvh, b);
    }
    ++issued;
  };
  if (gt == 0) {
#pragma unroll
    for (int s = 0; s < C::NS - 1; ++s)
      if (issued < cnt) issue_next(s);
  }

  const int g8 = lane >> 2, q4 = lane & 3;
  const float sl2 = sh.scale * kLog2e;  // logits in log2 units
  float m[2] = {kNegInf, kNegInf};
  float l[2] = {0.f, 0.f};  // this thread's share of the row sums (fp32, before the bf16 rounding of P)
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

  bool ok = true;
  auto wait_slot = [&](int slot, uint32_t ph) {
    ok = __all_sync(0xffffffffu, mbar_wait(&full[slot], ph, abort_flag)) && ok;
  };
  // Logits of one key block: s = Q K^T (16 rows x S keys).
  auto logits = [&](float (&s)[S / 8][4], int slot) {
    const uint32_t kt = smem_u32(gbase + slot * C::SLOT);
#pragma unroll
    for (int n = 0; n < S / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[n][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
      for (int jn = 0; jn < S / 16; ++jn) {
        uint32_t kb[4];
        const int r = jn * 16 + (lane & 7) + ((lane >> 4) << 3);
        ldsm_x4_addr(kb, kt + (kk / 4) * C::HALF + swz(r, (kk % 4) * 2 + ((lane >> 3) & 1)));
        mma16816(s[2 * jn], qa[kk], kb[0], kb[1]);
        mma16816(s[2 * jn + 1], qa[kk], kb[2], kb[3]);
      }
  };
  // Online-softmax step of one key block, then O += P V.
  auto attend = [&](float (&s)[S / 8][4], int slot, bool diag) {
    if (diag) {  // the diagonal block: keys after the row are not causal
#pragma unroll
      for (int n = 0; n < S / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int u = i * S + n * 8 + 2 * q4 + (e & 1);
          const int t = r0 + g8 + 8 * (e >> 1);
          if (u > t) s[n][e] = kNegInf;
        }
    }
    float nm[2];
    bool need = false;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float mx = kNegInf;
#pragma unroll
      for (int n = 0; n < S / 8; ++n) mx = fmaxf(mx, fmaxf(s[n][2 * r], s[n][2 * r + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      nm[r] = fmaxf(m[r], mx * sl2);  // finite: every row keeps a key in every visited block
      need |= nm[r] > m[r] + kLazy;
    }
    if (__any_sync(0xffffffffu, need)) {
      float c[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        c[r] = fast_ex2(m[r] - nm[r]);
        m[r] = nm[r];
      }
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        o[n][0] *= c[0]; o[n][1] *= c[0];
        o[n][2] *= c[1]; o[n][3] *= c[1];
      }
      l[0] *= c[0];
      l[1] *= c[1];
    }
    const uint32_t vt = smem_u32(gbase + slot * C::SLOT + C::TILE);
#pragma unroll
    for (int kk = 0; kk < S / 16; ++kk) {
      uint32_t pa[4];
#pragma unroll
      for (int hn = 0; hn < 2; ++hn) {
        float w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) w[e] = fast_ex2(fmaf(s[2 * kk + hn][e], sl2, -m[e >> 1]));
        l[0] += w[0] + w[1];
        l[1] += w[2] + w[3];
        pa[hn * 2] = pack2(w[0], w[1]);
        pa[hn * 2 + 1] = pack2(w[2], w[3]);
      }
      const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int jd = 0; jd < D / 16; ++jd) {
        uint32_t vb[4];
        ldsm_x4_t_addr(vb, vt + (jd / 4) * C::HALF + swz(r, (jd % 4) * 2 + (lane >> 4)));
        mma16816(o[2 * jd], pa, vb[0], vb[1]);
        mma16816(o[2 * jd + 1], pa, vb[2], vb[3]);
      }
    }
  };

  // Software pipeline: the logits of block it + 1 are issued before the
  // softmax and P V of block it, so that the tensor core works on one while
  // the exponentials of the other run.
  float sa[S / 8][4], sb[S / 8][4];
  int st = 0;
  uint32_t ph = 0;
  auto step = [&](float (&cur)[S / 8][4], float (&nxt)[S / 8][4], int it) {
    const int st1 = st + 1 == C::NS ? 0 : st + 1;
    const uint32_t ph1 = st1 == 0 ? ph ^ 1u : ph;
    group_sync<C::W>(grp);  // every warp of the group is done with block it - 1's slot
    if (gt == 0 && issued < cnt) issue_next(st == 0 ? C::NS - 1 : st - 1);
    if (it + 1 < cnt) {
      wait_slot(st1, ph1);
      logits(nxt, st1);
    }
    attend(cur, st, diag_sel && it == cnt - 1);
    st = st1;
    ph = ph1;
  };
  if (cnt > 0) {
    wait_slot(0, 0);
    logits(sa, 0);
  }
  for (int it = 0; it < cnt; it += 2) {
    step(sa, sb, it);
    if (it + 1 < cnt) step(sb, sa, it + 1);
  }
  group_sync<C::W>(grp);  // every warp of the group is done with the slots

  // Epilogue: O / l through a swizzled staging tile in slot 0, 16-byte stores.
  unsigned char* stage = gbase;
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
    for (int r = 0; r < 2; ++r) {
      const int rr = wig * 16 + g8 + 8 * r;
      *reinterpret_cast<uint32_t*>(stage + (n / 8) * C::HALF + swz(rr, n % 8) + q4 * 4) =
          pack2(o[n][2 * r] * inv[r], o[n][2 * r + 1] * inv[r]);
    }
  __syncwarp();
  for (int e = lane; e < 16 * D / 8; e += 32) {
    const int r = e / (D / 8), c = e % (D / 8);
    *reinterpret_cast<uint4*>(row_ptr_w<bf16>(a.hs, b, h, r0 + r) + c * 8) =
        *reinterpret_cast<const uint4*>(stage + (c / 8) * C::HALF + swz(wig * 16 + r, c % 8));
  }
  if (q4 == 0) {
#pragma unroll
    for (int r = 0; r < 2; ++r)
      a.lse_sel[((int64_t)b * sh.Hq + h) * sh.N + r0 + g8 + 8 * r] = l[r] > 0.f ? m[r] * kLn2 + logf(l[r]) : kNegInf;
  }
  if (!ok && lane == 0) atomicCAS(sh.status, 0, (int)SSA_ERR_TIMEOUT);
}

template <int D, int S>
cudaError_t launch_t(const Dims& Dm, const FwdArgs& a, int32_t* status, cudaStream_t st) {
  using C = WalkCfg<D, S>;
  CUtensorMap mk, mv;
  if (!make_tma_map_bf16(&mk, a.k, Dm.B, Dm.Hkv, Dm.N, S, D) || !make_tma_map_bf16(&mv, a.v, Dm.B, Dm.Hkv, Dm.N, S, D))
    return cudaErrorInvalidValue;
  auto kern = fwd_walk_kernel<D, S>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  WalkShape sh{Dm.Hq, Dm.g, Dm.N, Dm.n, Dm.k, Dm.scale, status};
  dim3 grid(Dm.N / BM, Dm.Hq, Dm.B);
  kern<<<grid, NT, C::SMEM, st>>>(mk, mv, a, sh);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

bool fwd_walk_supported(const Dims& D) {
  return D.dtype == SSA_BF16 && !D.per_token && (D.s == 16 || D.s == 32) && (D.d == 64 || D.d == 128);
}

cudaError_t launch_fwd_walk(const Dims& D, const FwdArgs& a, int32_t* dev_status, cudaStream_t st) {
  if (D.d == 64) return D.s == 16 ? launch_t<64, 16>(D, a, dev_status, st) : launch_t<64, 32>(D, a, dev_status, st);
  return D.s == 16 ? launch_t<128, 16>(D, a, dev_status, st) : launch_t<128, 32>(D, a, dev_status, st);
}

}  // namespace ssa
