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
#include "ssa_internal.cuh"

namespace ssa {
namespace {

using namespace warp_mma;
using bf16 = __nv_bfloat16;

constexpr int BM = 64;   // query rows per dQ CTA
constexpr int NT = 128;  // 4 warps
constexpr float kLog2e = 1.4426950408889634f;

struct WalkShape {
  int Hq, g, N, n, words;
  float scale;
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

template <int D, int S>
struct DqCfg {
  static constexpr int W = S / 16;
  static constexpr int G = 4 / W;
  static constexpr int NS = D == 64 ? 3 : 2;
  static constexpr int LD = D + 8;
  static constexpr int STAGE = S * LD * 2;  // stage 0 later stages the output
  static constexpr int GRP_BYTES = NS * 2 * STAGE;
  static constexpr int SEL_OFF = G * GRP_BYTES;
  static constexpr int SMEM = SEL_OFF + G * 64 * 4;
};

template <int D, int S>
__global__ void __launch_bounds__(NT, D == 64 ? 4 : 2) bwd_dq_walk_kernel(BwdArgs a, WalkShape sh) {
  using C = DqCfg<D, S>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grp = warp / C::W, gt = (warp % C::W) * 32 + lane;
  const int qt = gridDim.x - 1 - blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z, kvh = h / sh.g;
  const int t0 = qt * BM;
  const int i = t0 / S + grp;
  const int r0 = t0 + warp * 16;
  const int64_t rowbase = ((int64_t)b * sh.Hq + h) * sh.N;

  unsigned char* gbase = smem + grp * C::GRP_BYTES;
  uint32_t* sel = reinterpret_cast<uint32_t*>(smem + C::SEL_OFF) + grp * 64;
  auto kbuf = [&](int st) { return reinterpret_cast<bf16 (*)[C::LD]>(gbase + (2 * st) * C::STAGE); };
  auto vbuf = [&](int st) { return reinterpret_cast<bf16 (*)[C::LD]>(gbase + (2 * st + 1) * C::STAGE); };

  const uint32_t* mrow = a.mask + (rowbase / sh.N * sh.n + i) * sh.words;
  for (int w = gt; w < 64; w += 32 * C::W) sel[w] = w < sh.words ? mrow[w] : 0u;
  group_sync<C::W>(grp);

  const int nw = i / 32 + 1;
  auto next_blk = [&](int from) -> int {
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

  const float sl2 = sh.scale * kLog2e;
  float dq[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dq[n][e] = 0.f;

  int cur = next_blk(0);
  for (int it = 0; cur >= 0; ++it) {
    cp_async_wait<C::NS - 2>();
    group_sync<C::W>(grp);
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

    float sc[S / 8][4], dp[S / 8][4];
#pragma unroll
    for (int n = 0; n < S / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[n][e] = dp[n][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
      for (int jn = 0; jn < S / 16; ++jn) {
        uint32_t kb[4], vb[4];
        const int rr = jn * 16 + (lane & 7) + ((lane >> 4) << 3), cc = kk * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x4(kb, &ks[rr][cc]);
        ldsm_x4(vb, &vs[rr][cc]);
        mma16816(sc[2 * jn], qa[kk], kb[0], kb[1]);
        mma16816(sc[2 * jn + 1], qa[kk], kb[2], kb[3]);
        mma16816(dp[2 * jn], ga[kk], vb[0], vb[1]);
        mma16816(dp[2 * jn + 1], ga[kk], vb[2], vb[3]);
      }
    const bool diag = (cur == i);
#pragma unroll
    for (int n = 0; n < S / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = e >> 1;
        float p = fast_ex2(fmaf(sc[n][e], sl2, -lse2[r]));
        if (diag && cur * S + n * 8 + 2 * q4 + (e & 1) > r0 + g8 + 8 * r) p = 0.f;
        sc[n][e] = p * (dp[n][e] - Dt[r]);  // dS
      }
#pragma unroll
    for (int kk = 0; kk < S / 16; ++kk) {
      uint32_t da[4];
      da[0] = pack2(sc[2 * kk][0], sc[2 * kk][1]);
      da[1] = pack2(sc[2 * kk][2], sc[2 * kk][3]);
      da[2] = pack2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
      da[3] = pack2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
      for (int jd = 0; jd < D / 16; ++jd) {
        uint32_t kb[4];
        ldsm_x4_t(kb, &ks[kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8][jd * 16 + (lane >> 4) * 8]);
        mma16816(dq[2 * jd], da, kb[0], kb[1]);
        mma16816(dq[2 * jd + 1], da, kb[2], kb[3]);
      }
    }
    cur = next_blk(cur + 1);
  }
  cp_async_wait<0>();
  group_sync<C::W>(grp);  // every warp of the group is done with the stages
  bf16 (*qs)[C::LD] = kbuf(0) + (warp % C::W) * 16;  // this warp's 16 output rows
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int r = 0; r < 2; ++r)
      *reinterpret_cast<uint32_t*>(&qs[g8 + 8 * r][n * 8 + 2 * q4]) =
          pack2(sh.scale * dq[n][2 * r], sh.scale * dq[n][2 * r + 1]);
  __syncwarp();
  for (int e = lane; e < 16 * D / 8; e += 32) {
    const int r = e / (D / 8), col = (e % (D / 8)) * 8;
    *reinterpret_cast<uint4*>(row_ptr_w<bf16>(a.dq, b, h, r0 + r) + col) = *reinterpret_cast<const uint4*>(&qs[r][col]);
  }
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

template <int D, int S>
struct KvCfg {
  static constexpr int NS = (D == 64 && S == 16) ? 3 : 2;
  static constexpr int LD = D + 8;
  static constexpr int ROWS = S * LD * 2;                     // S query rows
  static constexpr int STAGE = 2 * ROWS + 2 * S * 4;          // Q, g_s, lse, D
  static constexpr int RING = 4 * NS * STAGE;
  static constexpr int RED = 2 * 4 * 16 * D * 4;              // four warps' dK, dV (fp32)
  static constexpr int KV_OFF = RING > RED ? RING : RED;
  static constexpr int LIST_OFF = KV_OFF + 2 * 16 * LD * 2;   // K and V slice staging
  static constexpr int SMEM = LIST_OFF + 2048 * 2 + 16;       // query-block list (n <= 2048) + its length
};

template <int D, int S>
__global__ void __launch_bounds__(NT) bwd_dkv_walk_kernel(BwdArgs a, WalkShape sh, float* part) {
  using C = KvCfg<D, S>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j = blockIdx.x / (S / 16), half = blockIdx.x % (S / 16);
  const int h = blockIdx.y, b = blockIdx.z, kvh = h / sh.g;
  const int u0 = j * S + half * 16;  // first key of the slice
  const int64_t rowbase = ((int64_t)b * sh.Hq + h) * sh.N;
  bf16 (*kvs)[C::LD] = reinterpret_cast<bf16 (*)[C::LD]>(smem + C::KV_OFF);  // rows 0-15 K, 16-31 V
  uint16_t* list = reinterpret_cast<uint16_t*>(smem + C::LIST_OFF);
  int* list_len = reinterpret_cast<int*>(smem + C::LIST_OFF + 2048 * 2);

  for (int e = tid; e < 2 * 16 * D / 8; e += NT) {
    const int r = e / (D / 8), c = (e % (D / 8)) * 8;
    const TensorRef& t = r < 16 ? a.k : a.v;
    cp_async16(&kvs[r][c], row_ptr<bf16>(t, b, kvh, u0 + (r & 15)) + c, 16);
  }
  cp_async_commit();

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
  cp_async_wait<0>();
  __syncthreads();  // the list and the K / V slice (copied by every thread) are in place
  const int total = *list_len;

  unsigned char* ring = smem + warp * C::NS * C::STAGE;
  auto qbuf = [&](int st) { return reinterpret_cast<bf16 (*)[C::LD]>(ring + st * C::STAGE); };
  auto gbuf = [&](int st) { return reinterpret_cast<bf16 (*)[C::LD]>(ring + st * C::STAGE + C::ROWS); };
  auto lbuf = [&](int st) { return reinterpret_cast<float*>(ring + st * C::STAGE + 2 * C::ROWS); };
  auto dbuf = [&](int st) { return reinterpret_cast<float*>(ring + st * C::STAGE + 2 * C::ROWS + S * 4); };
  auto load_pair = [&](int i, int st) {
    bf16 (*qs)[C::LD] = qbuf(st);
    bf16 (*gs)[C::LD] = gbuf(st);
    for (int e = lane; e < S * D / 8; e += 32) {
      const int r = e / (D / 8), c = (e % (D / 8)) * 8;
      cp_async16(&qs[r][c], row_ptr<bf16>(a.q, b, h, (int64_t)i * S + r) + c, 16);
      cp_async16(&gs[r][c], row_ptr<bf16>(a.gs, b, h, (int64_t)i * S + r) + c, 16);
    }
    if (lane < S / 4) {
      cp_async16(lbuf(st) + 4 * lane, a.lse_sel + rowbase + (int64_t)i * S + 4 * lane, 16);
      cp_async16(dbuf(st) + 4 * lane, a.Dc + rowbase + (int64_t)i * S + 4 * lane, 16);
    }
  };
  // this warp's pairs: list[warp], list[warp + 4], ...
  const int mine = total > warp ? (total - warp + 3) / 4 : 0;
#pragma unroll
  for (int p = 0; p < C::NS - 1; ++p) {
    if (p < mine) load_pair(list[warp + 4 * p], p);
    cp_async_commit();
  }

  const int g8 = lane >> 2, q4 = lane & 3;
  const float sl2 = sh.scale * kLog2e;
  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;

  for (int p = 0; p < mine; ++p) {
    cp_async_wait<C::NS - 2>();
    __syncwarp();
    if (p + C::NS - 1 < mine) load_pair(list[warp + 4 * (p + C::NS - 1)], (p + C::NS - 1) % C::NS);
    cp_async_commit();
    const int st = p % C::NS;
    const int i = list[warp + 4 * p];
    bf16 (*qs)[C::LD] = qbuf(st);
    bf16 (*gs)[C::LD] = gbuf(st);
    const float* ls = lbuf(st);
    const float* ds = dbuf(st);

    // S^T (16 keys x S rows) and dP^T
    float sT[S / 8][4], pT[S / 8][4];
#pragma unroll
    for (int n = 0; n < S / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) sT[n][e] = pT[n][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t ka[4], va[4];  // the key slice's K and V rows as A fragments
      ldsm_x4(ka, &kvs[lane & 15][kk * 16 + (lane >> 4) * 8]);
      ldsm_x4(va, &kvs[16 + (lane & 15)][kk * 16 + (lane >> 4) * 8]);
#pragma unroll
      for (int jn = 0; jn < S / 16; ++jn) {
        uint32_t qb[4], gb[4];
        const int rr = jn * 16 + (lane & 7) + ((lane >> 4) << 3), cc = kk * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x4(qb, &qs[rr][cc]);
        ldsm_x4(gb, &gs[rr][cc]);
        mma16816(sT[2 * jn], ka, qb[0], qb[1]);
        mma16816(sT[2 * jn + 1], ka, qb[2], qb[3]);
        mma16816(pT[2 * jn], va, gb[0], gb[1]);
        mma16816(pT[2 * jn + 1], va, gb[2], gb[3]);
      }
    }
    const bool diag = (i == j);
#pragma unroll
    for (int n = 0; n < S / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = n * 8 + 2 * q4 + (e & 1);  // query row within the block
        float p_ = fast_ex2(fmaf(sT[n][e], sl2, -ls[c] * kLog2e));
        if (diag && u0 + g8 + 8 * (e >> 1) > i * S + c) p_ = 0.f;
        sT[n][e] = p_;
        pT[n][e] = p_ * (pT[n][e] - ds[c]);  // dS^T
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
#pragma unroll
      for (int jd = 0; jd < D / 16; ++jd) {
        uint32_t gb[4], qb[4];
        const int rr = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, cc = jd * 16 + (lane >> 4) * 8;
        ldsm_x4_t(gb, &gs[rr][cc]);
        ldsm_x4_t(qb, &qs[rr][cc]);
        mma16816(dv[2 * jd], pa, gb[0], gb[1]);
        mma16816(dv[2 * jd + 1], pa, gb[2], gb[3]);
        mma16816(dk[2 * jd], da, qb[0], qb[1]);
        mma16816(dk[2 * jd + 1], da, qb[2], qb[3]);
      }
    }
    __syncwarp();  // the stage is read before a later load_pair refills it
  }
  cp_async_wait<0>();
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
    for (int w = 0; w < 4; ++w) {
      const float4 x = *reinterpret_cast<const float4*>(red + (w * 2 + which) * 16 * D + off);
      s.x += x.x; s.y += x.y; s.z += x.z; s.w += x.w;
    }
    *reinterpret_cast<float4*>(pk + which * plane + off) = s;
  }
}

template <int D, int S>
cudaError_t launch_t(const Dims& Dm, const BwdArgs& a, cudaStream_t st) {
  WalkShape sh{Dm.Hq, Dm.g, Dm.N, Dm.n, a.words, Dm.scale};
  {
    using C = DqCfg<D, S>;
    auto kern = bwd_dq_walk_kernel<D, S>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    kern<<<dim3(Dm.N / BM, Dm.Hq, Dm.B), NT, C::SMEM, st>>>(a, sh);
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
    auto kern = bwd_dkv_walk_kernel<D, S>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    kern<<<dim3(Dm.n * (S / 16), Dm.Hq, Dm.B), NT, C::SMEM, st>>>(a, sh, part);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return launch_kvsum(Dm, a, part, Dm.g, st);
}

}  // namespace

bool bwd_walk_supported(const Dims& D) {
  return D.dtype == SSA_BF16 && !D.per_token && (D.s == 16 || D.s == 32) && (D.d == 64 || D.d == 128);
}

cudaError_t launch_bwd_walk(const Dims& D, const BwdArgs& a, cudaStream_t st) {
  if (D.d == 64) return D.s == 16 ? launch_t<64, 16>(D, a, st) : launch_t<64, 32>(D, a, st);
  return D.s == 16 ? launch_t<128, 16>(D, a, st) : launch_t<128, 32>(D, a, st);
}

}  // namespace ssa
