// Sparse-stream backward for blocks of 16 or 32 keys with per-block
// selection: dQ by walking each query block's own selected key blocks, dK and
// dV by walking, for each key block, the query blocks that selected it.
//
// What it computes (the gradient of <g_s, h_sparse> with the selection held
// fixed; "SSA: Achieving Sparser Attention ...", "Practical Implementation of
// SSA" and "Technische Samenvatting: SSA", "Bidirectionele Uitlijning": the
// sparse stream alone gives gradient only to the pairs it attends): with
// P_tu = e^{scale q_t.k_u - lse_sel[t]} on A_t and D_t = sum_d g_s[t,d] h_s[t,d],
//   dS_tu = P_tu (g_s[t] . v_u - D_t),
//   dQ_t  = scale sum_u dS_tu k_u,  dK_u = scale sum_t dS_tu q_t,  dV_u = sum_t P_tu g_s[t].
//
// dQ: like the forward walk, one warp (blocks of 16) or a pair of warps
// (blocks of 32) per query block holds its Q and g_s rows as mma.sync A
// fragments and visits the selected key blocks with a cp.async ring; the
// first launch also writes D_t for the second.
//
// dK, dV: the selections are skewed (a few key blocks are chosen by almost
// every later query block), so the unit is a (query head, 16-key slice) CTA
// of four warps.  It lists the query blocks whose selection holds the key
// block (ballots over the selection bit masks, ascending), deals them to its
// warps in turn, adds the four warps' accumulators in shared memory in a
// fixed order and writes one fp32 partial per query head; the GQA group's
// partials are then added in head order.  No atomics: bit-reproducible.
#include "mma_sync.cuh"
#include "sm100_ptx.cuh"
#include "ssa_internal.cuh"

namespace ssa {
namespace {

using namespace warp_mma;
using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int BM = 64;   // query rows per dQ CTA
constexpr int NT = 128;  // 4 warps
constexpr float kLog2e = 1.4426950408889634f;

struct WalkShape {
  int Hq, g, N, n, words;
  float scale;
  int32_t* status;
};

template <int W>
__device__ __forceinline__ void group_sync(int grp) {
  if constexpr (W == 1) {
    __syncwarp();
  } else {
    asm volatile("bar.sync %0, %1;\n" ::"r"(grp + 1), "n"(32 * W) : "memory");
  }
}

// ---------------------------------------------------------------- dQ -----

// Shared memory of a dQ CTA, per query block (group of W warps): NS slots,
// each the K block then the V block of one selected key block, stored as
// 64-column halves of S rows x 128 B in the TMA 128-byte swizzle (the 16-byte
// chunk c of row r sits at chunk c ^ (r & 7)).
template <int D, int S>
struct DqCfg {
  static constexpr int W = S / 16;
  static constexpr int G = 4 / W;
  static constexpr int NS = 3;             // block it (dS K), block it + 1 (its products), one load ahead
  static constexpr int HALF = S * 128;     // 64 columns of one block
  static constexpr int TILE = (D / 64) * HALF;
  static constexpr int SLOT = 2 * TILE;    // K, then V
  static constexpr int GRP_BYTES = NS * SLOT;
  static constexpr int BAR_OFF = G * GRP_BYTES;          // NS mbarriers per query block
  static constexpr int FLAG_OFF = BAR_OFF + G * NS * 8;  // one abort flag per query block
  static constexpr int SEL_OFF = FLAG_OFF + G * 4;       // one 2048-bit selection set per query block
  static constexpr int SMEM = SEL_OFF + G * 64 * 4 + 1024;  // + alignment slack
};

// Byte offset of the 16-byte chunk `ch` (0..7) of row r in a swizzled half.
__device__ __forceinline__ uint32_t swz(int r, int ch) { return (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4)); }

template <int D, int S>
__global__ void __launch_bounds__(NT, D == 64 ? (S == 16 ? 4 : 3) : 2)
    bwd_dq_walk_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, BwdArgs a,
                       WalkShape sh) {
  using C = DqCfg<D, S>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grp = warp / C::W, wig = warp % C::W, gt = wig * 32 + lane;
  const int qt = gridDim.x - 1 - blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z, kvh = h / sh.g;
  const int t0 = qt * BM;
  const int i = t0 / S + grp;
  const int r0 = t0 + warp * 16;
  const int64_t rowbase = ((int64_t)b * sh.Hq + h) * sh.N;

  unsigned char* gbase = smem + grp * C::GRP_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF) + grp * C::NS;
  int* abort_flag = reinterpret_cast<int*>(smem + C::FLAG_OFF) + grp;
  uint32_t* sel = reinterpret_cast<uint32_t*>(smem + C::SEL_OFF) + grp * 64;

  const uint32_t* mrow = a.mask + (rowbase / sh.N * sh.n + i) * sh.words;
  for (int w = gt; w < 64; w += 32 * C::W) sel[w] = w < sh.words ? mrow[w] : 0u;
  if (gt == 0) {
#pragma unroll
    for (int s = 0; s < C::NS; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_mbar_init();
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
  int iw = 0, issued = 0;
  uint32_t ibits = sel[0];
  auto issue_next = [&](int slot) {
    while (ibits == 0u) ibits = sel[++iw];  // bounded: fewer than cnt blocks issued
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

  // D_t = g_s[t] . h_s[t]: two lanes per row, then to the fragment rows.
  const int g8 = lane >> 2, q4 = lane & 3;
  float Dt[2], lse2[2];
  {
    const int rr = lane >> 1, half = lane & 1;
    const bf16* gp = row_ptr<bf16>(a.gs, b, h, r0 + rr) + half * (D / 2);
    const bf16* hp = row_ptr<bf16>(a.hs, b, h, r0 + rr) + half * (D / 2);
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < D / 2; c += 8) {
      const uint4 gv = *reinterpret_cast<const uint4*>(gp + c);
      const uint4 hv = *reinterpret_cast<const uint4*>(hp + c);
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hv);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 gf = __bfloat1622float2(g2[q]), hf = __bfloat1622float2(h2[q]);
        acc = fmaf(gf.x, hf.x, acc);
        acc = fmaf(gf.y, hf.y, acc);
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    if (half == 0) a.Dc[rowbase + r0 + rr] = acc;
    Dt[0] = __shfl_sync(0xffffffffu, acc, 2 * g8);
    Dt[1] = __shfl_sync(0xffffffffu, acc, 2 * (g8 + 8));
#pragma unroll
    for (int r = 0; r < 2; ++r) lse2[r] = a.lse_sel[rowbase + r0 + g8 + 8 * r] * kLog2e;
  }

  // Q and g_s rows of the warp as A fragments, straight from global memory.
  uint32_t qa[D / 16][4], ga[D / 16][4];
  {
    const bf16* q0p = row_ptr<bf16>(a.q, b, h, r0 + g8);
    const bf16* q1p = row_ptr<bf16>(a.q, b, h, r0 + g8 + 8);
    const bf16* g0p = row_ptr<bf16>(a.gs, b, h, r0 + g8);
    const bf16* g1p = row_ptr<bf16>(a.gs, b, h, r0 + g8 + 8);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int c = kk * 16 + 2 * q4;
      qa[kk][0] = *reinterpret_cast<const uint32_t*>(q0p + c);
      qa[kk][1] = *reinterpret_cast<const uint32_t*>(q1p + c);
      qa[kk][2] = *reinterpret_cast<const uint32_t*>(q0p + c + 8);
      qa[kk][3] = *reinterpret_cast<const uint32_t*>(q1p + c + 8);
      ga[kk][0] = *reinterpret_cast<const uint32_t*>(g0p + c);
      ga[kk][1] = *reinterpret_cast<const uint32_t*>(g1p + c);
      ga[kk][2] = *reinterpret_cast<const uint32_t*>(g0p + c + 8);
      ga[kk][3] = *reinterpret_cast<const uint32_t*>(g1p + c + 8);
    }
  }

  bool ok = true;
  auto wait_slot = [&](int slot, uint32_t ph) {
    ok = __all_sync(0xffffffffu, mbar_wait(&full[slot], ph, abort_flag)) && ok;
  };
  // S = Q K^T and dP = g_s V^T of one key block (16 rows x S keys).
  auto products = [&](float (&sc)[S / 8][4], float (&dp)[S / 8][4], int slot) {
    const uint32_t kt = smem_u32(gbase + slot * C::SLOT), vt = kt + C::TILE;
#pragma unroll
    for (int n = 0; n < S / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[n][e] = dp[n][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
      for (int jn = 0; jn < S / 16; ++jn) {
        uint32_t kb[4], vb[4];
        const int r = jn * 16 + (lane & 7) + ((lane >> 4) << 3);
        const uint32_t off = (kk / 4) * C::HALF + swz(r, (kk % 4) * 2 + ((lane >> 3) & 1));
        ldsm_x4_addr(kb, kt + off);
        ldsm_x4_addr(vb, vt + off);
        mma16816(sc[2 * jn], qa[kk], kb[0], kb[1]);
        mma16816(sc[2 * jn + 1], qa[kk], kb[2], kb[3]);
        mma16816(dp[2 * jn], ga[kk], vb[0], vb[1]);
        mma16816(dp[2 * jn + 1], ga[kk], vb[2], vb[3]);
      }
  };
  const float sl2 = sh.scale * kLog2e;
  float dq[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dq[n][e] = 0.f;
  // dS = P (dP - D), then dQ += dS K.
  auto grads = [&](float (&sc)[S / 8][4], const float (&dp)[S / 8][4], int slot, bool diag) {
    const uint32_t kt = smem_u32(gbase + slot * C::SLOT);
#pragma unroll
    for (int n = 0; n < S / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = e >> 1;
        float p = fast_ex2(fmaf(sc[n][e], sl2, -lse2[r]));
        if (diag && i * S + n * 8 + 2 * q4 + (e & 1) > r0 + g8 + 8 * r) p = 0.f;
        sc[n][e] = p * (dp[n][e] - Dt[r]);
      }
#pragma unroll
    for (int kk = 0; kk < S / 16; ++kk) {
      uint32_t da[4];
      da[0] = pack2(sc[2 * kk][0], sc[2 * kk][1]);
      da[1] = pack2(sc[2 * kk][2], sc[2 * kk][3]);
      da[2] = pack2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
      da[3] = pack2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
      const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int jd = 0; jd < D / 16; ++jd) {
        uint32_t kb[4];
        ldsm_x4_t_addr(kb, kt + (jd / 4) * C::HALF + swz(r, (jd % 4) * 2 + (lane >> 4)));
        mma16816(dq[2 * jd], da, kb[0], kb[1]);
        mma16816(dq[2 * jd + 1], da, kb[2], kb[3]);
      }
    }
  };

  // Software pipeline: the products of block it + 1 are issued before the
  // gradients of block it.
  float sc[S / 8][4], dp[S / 8][4];
  int st = 0;
  uint32_t ph = 0;
  if (cnt > 0) {
    wait_slot(0, 0);
    products(sc, dp, 0);
  }
  for (int it = 0; it < cnt; ++it) {
    const int st1 = st + 1 == C::NS ? 0 : st + 1;
    const uint32_t ph1 = st1 == 0 ? ph ^ 1u : ph;
    group_sync<C::W>(grp);  // every warp of the group is done with block it - 1's slot
    if (gt == 0 && issued < cnt) issue_next(st == 0 ? C::NS - 1 : st - 1);
    float sn[S / 8][4], dn[S / 8][4];
    if (it + 1 < cnt) {
      wait_slot(st1, ph1);
      products(sn, dn, st1);
    }
    grads(sc, dp, st, diag_sel && it == cnt - 1);
#pragma unroll
    for (int n = 0; n < S / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        sc[n][e] = sn[n][e];
        dp[n][e] = dn[n][e];
      }
    st = st1;
    ph = ph1;
  }
  group_sync<C::W>(grp);  // every warp of the group is done with the slots

  // Epilogue: scale * dQ through a swizzled staging tile in slot 0, 16-byte stores.
  unsigned char* stage = gbase;
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int rr = wig * 16 + g8 + 8 * r;
      *reinterpret_cast<uint32_t*>(stage + (n / 8) * C::HALF + swz(rr, n % 8) + q4 * 4) =
          pack2(sh.scale * dq[n][2 * r], sh.scale * dq[n][2 * r + 1]);
    }
  __syncwarp();
  for (int e = lane; e < 16 * D / 8; e += 32) {
    const int r = e / (D / 8), c = e % (D / 8);
    *reinterpret_cast<uint4*>(row_ptr_w<bf16>(a.dq, b, h, r0 + r) + c * 8) =
        *reinterpret_cast<const uint4*>(stage + (c / 8) * C::HALF + swz(wig * 16 + r, c % 8));
  }
  if (!ok && lane == 0) atomicCAS(sh.status, 0, (int)SSA_ERR_TIMEOUT);
}

// ------------------------------------------------------------- dK, dV -----

// maskT[b,h,j] = the set of query blocks i whose selection holds key block j:
// the selection bit matrix of every head transposed in 32 x 32 tiles, one warp
// per (32 query blocks, head) with ballots.
__global__ void __launch_bounds__(32) mask_transpose_kernel(const uint32_t* __restrict__ mask,
                                                            uint32_t* __restrict__ maskT, int n, int words) {
  const int it = blockIdx.x, lane = threadIdx.x;
  const int64_t base = (int64_t)blockIdx.y * n * words;
  const int i = it * 32 + lane;
  for (int jt = 0; jt < words; ++jt) {
    const uint32_t w = (i < n && jt <= it) ? mask[base + (int64_t)i * words + jt] : 0u;  // j <= i only
    uint32_t mine = 0u;
#pragma unroll
    for (int bit = 0; bit < 32; ++bit) {
      const uint32_t col = __ballot_sync(0xffffffffu, (w >> bit) & 1u);
      if (lane == bit) mine = col;
    }
    const int j = jt * 32 + lane;
    if (j < n) maskT[base + (int64_t)j * words + it] = mine;
  }
}

// Shared memory of a dK / dV CTA: per warp a ring of NS query blocks (Q,
// then g_s, each as 64-column halves of S rows x 128 B in the TMA 128-byte
// swizzle: the 16-byte chunk c of row r sits at chunk c ^ (r & 7), so ldmatrix
// reads are conflict-free without padding), the 16-key K and V slice in the
// same layout, and the ascending list of query blocks that chose the key
// block.  The rings become the reduction buffer at the end.
template <int D, int S>
struct KvCfg {
  static constexpr int NW = 4;                  // warps, dealt the list in turn
  static constexpr int NS = D == 64 ? 3 : 2;    // query blocks in a warp's ring
  static constexpr int HALF = S * 128;          // 64 columns of S query rows
  static constexpr int QT = (D / 64) * HALF;    // one Q (or g_s) block
  static constexpr int SLOT = 2 * QT;           // Q, then g_s
  static constexpr int RING = NS * SLOT;
  static constexpr int KHALF = 16 * 128;        // 64 columns of the 16-key slice
  static constexpr int KT = (D / 64) * KHALF;   // the K (or V) slice
  static constexpr int RED = NW * 2 * 16 * D * 4;  // the warps' dK, dV (fp32)
  static constexpr int KV_OFF = NW * RING > RED ? NW * RING : RED;
  static constexpr int LIST_OFF = KV_OFF + 2 * KT;
  static constexpr int BAR_OFF = LIST_OFF + 2048 * 2 + 16;   // query-block list (n <= 2048) + its length
  static constexpr int FLAG_OFF = BAR_OFF + (NW * NS + 1) * 8;  // NW rings' barriers, the slice barrier
  static constexpr int SMEM = FLAG_OFF + 16 + 1024;              // abort flag, alignment slack
  static constexpr int MINB = (D == 64 && S == 16) ? 3 : (D == 128 && S == 32) ? 1 : 2;  // resident CTAs per SM the registers are sized for
};

// One CTA per (query head, 16-key slice u0 .. u0 + 15 of key block j), heads
// innermost so that every head's early key blocks (the ones most query
// blocks choose) start first.  The ascending list of query blocks whose
// selection holds j is dealt to the four warps in turn; per query block:
// S^T = K Q^T and dP^T = V g_s^T (16 keys x S rows), P^T from lse_sel,
// dS^T = P^T (dP^T - D), then dV += P^T g_s and dK += dS^T Q.  A warp issues
// the products of its next query block before the gradients of the current
// one, so the tensor core has independent work while the exponentials run.
// The four warps' sums are added in a fixed order into one fp32 partial per
// query head (dK unscaled, dV); the GQA group's partials are added in head
// order afterwards.
template <int D, int S>
__global__ void __launch_bounds__(NT, KvCfg<D, S>::MINB)
    bwd_dkv_walk_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
                        const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        BwdArgs a, WalkShape sh, float* part) {
  using C = KvCfg<D, S>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.x, j = blockIdx.y / (S / 16), b = blockIdx.z, kvh = h / sh.g;
  const int u0 = j * S + (blockIdx.y % (S / 16)) * 16;  // first key of the slice
  const int64_t rowbase = ((int64_t)b * sh.Hq + h) * sh.N;
  uint16_t* list = reinterpret_cast<uint16_t*>(smem + C::LIST_OFF);
  int* list_len = reinterpret_cast<int*>(smem + C::LIST_OFF + 2048 * 2);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF) + warp * C::NS;  // this warp's ring
  uint64_t* kvbar = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF) + C::NW * C::NS;
  int* abort_flag = reinterpret_cast<int*>(smem + C::FLAG_OFF);
  unsigned char* ring = smem + warp * C::RING;

  if (tid == 0) {
    for (int s = 0; s <= C::NW * C::NS; ++s) mbar_init(reinterpret_cast<uint64_t*>(smem + C::BAR_OFF) + s, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Query blocks whose selection holds j, ascending: lane l of warp 0 takes
  // words 2l and 2l+1 of the transposed mask row, a warp scan places them.
  if (warp == 0) {
    const uint32_t* trow = a.maskT + (rowbase / sh.N * sh.n + j) * sh.words;
    const uint32_t w0 = 2 * lane < sh.words ? trow[2 * lane] : 0u;
    const uint32_t w1 = 2 * lane + 1 < sh.words ? trow[2 * lane + 1] : 0u;
    const int c = __popc(w0) + __popc(w1);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int pos = incl - c;
    for (uint32_t bits = w0; bits; bits &= bits - 1u) list[pos++] = (uint16_t)(64 * lane + __ffs(bits) - 1);
    for (uint32_t bits = w1; bits; bits &= bits - 1u) list[pos++] = (uint16_t)(64 * lane + 32 + __ffs(bits) - 1);
    if (lane == 31) *list_len = incl;
  }
  __syncthreads();  // the list and the barriers are in place
  if (tid == 0) {  // the slice's K and V rows
    mbar_expect_tx(kvbar, 2 * C::KT);
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh) {
      unsigned char* dst = smem + C::KV_OFF + hh * C::KHALF;
      tma_load_4d(dst, &tmK, kvbar, hh * 64, u0, kvh, b);
      tma_load_4d(dst + C::KT, &tmV, kvbar, hh * 64, u0, kvh, b);
    }
  }
  const int total = *list_len;
  const int mine = total > warp ? (total - warp + C::NW - 1) / C::NW : 0;  // list[warp + NW p], p < mine

  // Lane 0 of each warp issues its own ring's loads.
  int issued = 0;
  auto issue_next = [&](int slot) {
    const int i = list[warp + C::NW * issued];
    unsigned char* dst = ring + slot * C::SLOT;
    mbar_expect_tx(&full[slot], C::SLOT);
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh) {
      tma_load_4d(dst + hh * C::HALF, &tmQ, &full[slot], hh * 64, i * S, h, b);
      tma_load_4d(dst + C::QT + hh * C::HALF, &tmG, &full[slot], hh * 64, i * S, h, b);
    }
    ++issued;
  };
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < C::NS - 1; ++s)
      if (issued < mine) issue_next(s);
  }

  const int g8 = lane >> 2, q4 = lane & 3;
  const float sl2 = sh.scale * kLog2e;
  // lse_sel (log2 units) and D of the query rows n*8 + 2*q4 + {0, 1}.
  auto load_rows = [&](int i, float2 (&ls)[S / 8], float2 (&dd)[S / 8]) {
#pragma unroll
    for (int n = 0; n < S / 8; ++n) {
      const int64_t o = rowbase + (int64_t)i * S + n * 8 + 2 * q4;
      const float2 l = *reinterpret_cast<const float2*>(a.lse_sel + o);
      ls[n] = make_float2(l.x * kLog2e, l.y * kLog2e);
      dd[n] = *reinterpret_cast<const float2*>(a.Dc + o);
    }
  };

  bool ok = true;
  auto wait_bar = [&](uint64_t* bar, uint32_t ph) {
    ok = __all_sync(0xffffffffu, mbar_wait(bar, ph, abort_flag)) && ok;
  };
  const uint32_t kt = smem_u32(smem + C::KV_OFF), vt = kt + C::KT;
  auto products = [&](float (&sT)[S / 8][4], float (&pT)[S / 8][4], int slot) {
    const uint32_t qt = smem_u32(ring + slot * C::SLOT), gq = qt + C::QT;
#pragma unroll
    for (int n = 0; n < S / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) sT[n][e] = pT[n][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t ka[4], va[4];  // the slice's K and V rows as A fragments
      const uint32_t aoff = (kk / 4) * C::KHALF + swz(lane & 15, (kk % 4) * 2 + (lane >> 4));
      ldsm_x4_addr(ka, kt + aoff);
      ldsm_x4_addr(va, vt + aoff);
#pragma unroll
      for (int jn = 0; jn < S / 16; ++jn) {
        uint32_t qb[4], gb[4];
        const int r = jn * 16 + (lane & 7) + ((lane >> 4) << 3);
        const uint32_t boff = (kk / 4) * C::HALF + swz(r, (kk % 4) * 2 + ((lane >> 3) & 1));
        ldsm_x4_addr(qb, qt + boff);
        ldsm_x4_addr(gb, gq + boff);
        mma16816(sT[2 * jn], ka, qb[0], qb[1]);
        mma16816(sT[2 * jn + 1], ka, qb[2], qb[3]);
        mma16816(pT[2 * jn], va, gb[0], gb[1]);
        mma16816(pT[2 * jn + 1], va, gb[2], gb[3]);
      }
    }
  };
  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;
  auto grads = [&](float (&sT)[S / 8][4], float (&pT)[S / 8][4], int slot, const float2 (&ls)[S / 8],
                   const float2 (&dd)[S / 8], int i) {
    const uint32_t qt = smem_u32(ring + slot * C::SLOT), gq = qt + C::QT;
    const bool diag = i == j;
#pragma unroll
    for (int n = 0; n < S / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = n * 8 + 2 * q4 + (e & 1);  // query row within the block
        float p_ = fast_ex2(fmaf(sT[n][e], sl2, -((e & 1) ? ls[n].y : ls[n].x)));
        if (diag && u0 + g8 + 8 * (e >> 1) > i * S + c) p_ = 0.f;
        sT[n][e] = p_;
        pT[n][e] = p_ * (pT[n][e] - ((e & 1) ? dd[n].y : dd[n].x));  // dS^T
      }
#pragma unroll
    for (int kk = 0; kk < S / 16; ++kk) {
      uint32_t pa[4], da[4];
      pa[0] = pack2(sT[2 * kk][0], sT[2 * kk][1]);
      pa[1] = pack2(sT[2 * kk][2], sT[2 * kk][3]);
      pa[2] = pack2(sT[2 * kk + 1][0], sT[2 * kk + 1][1]);
      pa[3] = pack2(sT[2 * kk + 1][2], sT[2 * kk + 1][3]);
      da[0] = pack2(pT[2 * kk][0], pT[2 * kk][1]);
      da[1] = pack2(pT[2 * kk][2], pT[2 * kk][3]);
      da[2] = pack2(pT[2 * kk + 1][0], pT[2 * kk + 1][1]);
      da[3] = pack2(pT[2 * kk + 1][2], pT[2 * kk + 1][3]);
      const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int jd = 0; jd < D / 16; ++jd) {
        uint32_t gb[4], qb[4];
        const uint32_t off = (jd / 4) * C::HALF + swz(r, (jd % 4) * 2 + (lane >> 4));
        ldsm_x4_t_addr(gb, gq + off);
        ldsm_x4_t_addr(qb, qt + off);
        mma16816(dv[2 * jd], pa, gb[0], gb[1]);
        mma16816(dv[2 * jd + 1], pa, gb[2], gb[3]);
        mma16816(dk[2 * jd], da, qb[0], qb[1]);
        mma16816(dk[2 * jd + 1], da, qb[2], qb[3]);
      }
    }
  };

  float sc[S / 8][4], pc[S / 8][4];  // products of the current query block
  float2 lc[S / 8], dc[S / 8];
  int ic = 0;
  int st = 0;
  uint32_t ph = 0;
  wait_bar(kvbar, 0);
  if (mine > 0) {
    ic = list[warp];
    load_rows(ic, lc, dc);
    wait_bar(&full[0], 0);
    products(sc, pc, 0);
  }
  for (int p = 0; p < mine; ++p) {
    const int st1 = st + 1 == C::NS ? 0 : st + 1;
    const uint32_t ph1 = st1 == 0 ? ph ^ 1u : ph;
    __syncwarp();  // the warp is done with query block p - 1's slot
    if (lane == 0 && issued < mine) issue_next(st == 0 ? C::NS - 1 : st - 1);
    float sn[S / 8][4], pn[S / 8][4];
    float2 ln[S / 8], dn[S / 8];
    int in = 0;
    if (p + 1 < mine) {
      in = list[warp + C::NW * (p + 1)];
      load_rows(in, ln, dn);
      wait_bar(&full[st1], ph1);
      products(sn, pn, st1);
    }
    grads(sc, pc, st, lc, dc, ic);
#pragma unroll
    for (int n = 0; n < S / 8; ++n) {
      lc[n] = ln[n];
      dc[n] = dn[n];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        sc[n][e] = sn[n][e];
        pc[n][e] = pn[n][e];
      }
    }
    ic = in;
    st = st1;
    ph = ph1;
  }
  __syncthreads();  // every warp is done with its ring: it becomes the reduction buffer

  float* red = reinterpret_cast<float*>(smem);  // [warp][2][16][D]
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float* rk = red + ((warp * 2 + 0) * 16 + g8 + 8 * r) * D + n * 8 + 2 * q4;
      float* rv = red + ((warp * 2 + 1) * 16 + g8 + 8 * r) * D + n * 8 + 2 * q4;
      *reinterpret_cast<float2*>(rk) = make_float2(dk[n][2 * r], dk[n][2 * r + 1]);
      *reinterpret_cast<float2*>(rv) = make_float2(dv[n][2 * r], dv[n][2 * r + 1]);
    }
  __syncthreads();
  // fp32 partials [head in group][2][B][Hkv][N][D] (dK unscaled, dV)
  const int64_t plane = (int64_t)gridDim.z * (sh.Hq / sh.g) * sh.N * D;
  float* pk = part + (int64_t)(h % sh.g) * 2 * plane + (((int64_t)b * (sh.Hq / sh.g) + kvh) * sh.N + u0) * D;
  for (int e = tid * 4; e < 2 * 16 * D; e += NT * 4) {
    const int which = e / (16 * D), off = e % (16 * D);
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < C::NW; ++w) {
      const float4 x = *reinterpret_cast<const float4*>(red + (w * 2 + which) * 16 * D + off);
      s.x += x.x; s.y += x.y; s.z += x.z; s.w += x.w;
    }
    *reinterpret_cast<float4*>(pk + which * plane + off) = s;
  }
  if (!ok && lane == 0) atomicCAS(sh.status, 0, (int)SSA_ERR_TIMEOUT);
}

template <int D, int S>
cudaError_t launch_t(const Dims& Dm, const BwdArgs& a, int32_t* status, cudaStream_t st) {
  WalkShape sh{Dm.Hq, Dm.g, Dm.N, Dm.n, a.words, Dm.scale, status};
  {
    using C = DqCfg<D, S>;
    CUtensorMap mk, mv;
    if (!make_tma_map_bf16(&mk, a.k, Dm.B, Dm.Hkv, Dm.N, S, D) || !make_tma_map_bf16(&mv, a.v, Dm.B, Dm.Hkv, Dm.N, S, D))
      return cudaErrorInvalidValue;
    auto kern = bwd_dq_walk_kernel<D, S>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    kern<<<dim3(Dm.N / BM, Dm.Hq, Dm.B), NT, C::SMEM, st>>>(mk, mv, a, sh);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    mask_transpose_kernel<<<dim3((Dm.n + 31) / 32, Dm.B * Dm.Hq), 32, 0, st>>>(a.mask, a.maskT, Dm.n, a.words);
    count_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  float* part = a.dhf;  // the dh_f and dO_c regions, unused by the sparse stream alone, hold g partials
  {
    using C = KvCfg<D, S>;
    CUtensorMap mq, mg, mk, mv;
    if (!make_tma_map_bf16(&mq, a.q, Dm.B, Dm.Hq, Dm.N, S, D) || !make_tma_map_bf16(&mg, a.gs, Dm.B, Dm.Hq, Dm.N, S, D) ||
        !make_tma_map_bf16(&mk, a.k, Dm.B, Dm.Hkv, Dm.N, 16, D) || !make_tma_map_bf16(&mv, a.v, Dm.B, Dm.Hkv, Dm.N, 16, D))
      return cudaErrorInvalidValue;
    auto kern = bwd_dkv_walk_kernel<D, S>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    kern<<<dim3(Dm.Hq, Dm.n * (S / 16), Dm.B), NT, C::SMEM, st>>>(mq, mg, mk, mv, a, sh, part);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return launch_kvsum(Dm, a, part, Dm.g, st);
}

}  // namespace

bool bwd_walk_supported(const Dims& D) {
  return D.dtype == SSA_BF16 && !D.per_token && (D.s == 16 || D.s == 32) && (D.d == 64 || D.d == 128);
}

cudaError_t launch_bwd_walk(const Dims& D, const BwdArgs& a, int32_t* dev_status, cudaStream_t st) {
  if (D.d == 64) return D.s == 16 ? launch_t<64, 16>(D, a, dev_status, st) : launch_t<64, 32>(D, a, dev_status, st);
  return D.s == 16 ? launch_t<128, 16>(D, a, dev_status, st) : launch_t<128, 32>(D, a, dev_status, st);
}

}  // namespace ssa
