// libssa C ABI: argument checks, workspace layout, kernel dispatch.
// Every check runs on the host before anything is enqueued; see include/ssa.h.
#include <atomic>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include "ssa_internal.cuh"

namespace ssa {

// One NVTX range per entry-point call, named after the call, so a profiler
// timeline (nsys, ncu --nvtx) shows which call enqueued which kernels.
// Header-only NVTX 3: without an attached tool the push / pop are no-ops.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

namespace {

// Status word that kernels with bounded waits write when a wait runs out.
__device__ int32_t g_device_status = 0;

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

ssa_status_t check_dims(const ssa_dims_t* in, Dims* out, bool* empty) {
  if (in == nullptr) return SSA_ERR_INVALID_ARG;
  Dims D{};
  D.B = in->B; D.Hq = in->Hq; D.Hkv = in->Hkv; D.N = in->N; D.d = in->d;
  D.s = in->block; D.topk = in->topk; D.scale = in->scale; D.dtype = in->dtype;
  if (D.B < 0 || D.Hq < 0 || D.N < 0 || D.Hkv < 1 || D.topk < 1) return SSA_ERR_INVALID_ARG;
  if (D.dtype != SSA_F32 && D.dtype != SSA_BF16) return SSA_ERR_INVALID_ARG;
  if (in->per_token != 0 && in->per_token != 1) return SSA_ERR_INVALID_ARG;
  D.per_token = in->per_token;
  if (!(D.scale > 0.f) || D.scale == __builtin_huge_valf()) return SSA_ERR_INVALID_ARG;
  if (D.Hq % D.Hkv != 0) return SSA_ERR_INVALID_ARG;
  if (D.s != 16 && D.s != 32 && D.s != 64 && D.s != 128) return SSA_ERR_UNSUPPORTED;
  if (D.d != 64 && D.d != 128) return SSA_ERR_UNSUPPORTED;
  if (D.N % D.s != 0 || D.N % 64 != 0) return SSA_ERR_UNSUPPORTED;
  D.n = D.N / D.s;
  if (D.n > 2048) return SSA_ERR_UNSUPPORTED;
  D.k = D.topk < D.n ? D.topk : D.n;
  D.g = D.Hkv > 0 ? D.Hq / D.Hkv : 0;
  D.rows_sel = D.per_token ? D.N : D.n;
  *empty = ((int64_t)D.B * D.Hq * D.N == 0);
  if (*empty) D.k = D.topk;
  *out = D;
  return SSA_OK;
}

size_t elem_size(const Dims& D) { return D.dtype == SSA_BF16 ? 2 : 4; }

ssa_status_t check_tensor(const Dims& D, const ssa_tensor_t* t, bool nullable, TensorRef* out) {
  if (t == nullptr) {
    if (!nullable) return SSA_ERR_INVALID_ARG;
    *out = TensorRef{nullptr, 0, 0, 0};
    return SSA_OK;
  }
  if (t->ptr == nullptr) return SSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(t->ptr) % 16 != 0) return SSA_ERR_INVALID_ARG;
  const int64_t es = (int64_t)elem_size(D);
  if (t->stride_b < 0 || t->stride_h < 0 || t->stride_n < 0) return SSA_ERR_INVALID_ARG;
  if ((t->stride_b * es) % 16 || (t->stride_h * es) % 16 || (t->stride_n * es) % 16)
    return SSA_ERR_INVALID_ARG;
  if (t->stride_n < D.d) return SSA_ERR_INVALID_ARG;  // rows may not overlap
  *out = TensorRef{t->ptr, t->stride_b, t->stride_h, t->stride_n};
  return SSA_OK;
}

ssa_status_t check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SSA_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SSA_ERR_CUDA;
  if (major != 10 || minor != 0) return SSA_ERR_UNSUPPORTED;
  return SSA_OK;
}

ssa_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? SSA_OK : SSA_ERR_CUDA; }

// ---------------------------------------------------------------- workspace
struct Layout {
  size_t qbar, kbar;          // block scores
  size_t dhf, doc, Df, Dc, mask, partials, kvpart, maskT;  // backward
  size_t lse;                 // dropped mass
  size_t bytes_scores, bytes_bwd, bytes_dropped, bytes_align, bytes_decode;
  int words, n_partials;
};

Layout layout(const Dims& D) {
  Layout L{};
  const size_t rows = (size_t)D.B * D.Hq * D.N;
  L.words = (D.n + 31) / 32;
  L.n_partials = sqdiff_partial_count(D);
  size_t o = 0;
  L.qbar = o; o = align_up(o + (size_t)D.B * D.Hq * D.n * D.d * 4);
  L.kbar = o; o = align_up(o + (size_t)D.B * D.Hkv * D.n * D.d * 4);
  L.bytes_scores = o;
  o = 0;
  L.dhf = o; o = align_up(o + rows * D.d * 4);
  L.doc = o; o = align_up(o + rows * D.d * 4);
  L.Df = o; o = align_up(o + rows * 4);
  L.Dc = o; o = align_up(o + rows * 4);
  L.mask = o; o = align_up(o + (size_t)D.B * D.Hq * D.rows_sel * L.words * 4);
  L.partials = o; o = align_up(o + (size_t)L.n_partials * 4);
  L.kvpart = o;
  if (bwd_tc_supported(D) || bwd_mma_supported(D)) o = align_up(o + bwd_mma_partial_bytes(D));
  L.maskT = o;
  if (bwd_walk_supported(D)) o = align_up(o + (size_t)D.B * D.Hq * D.n * L.words * 4);
  L.bytes_bwd = o;
  L.lse = 0;
  L.bytes_dropped = align_up(rows * 4);
  L.bytes_align = align_up((size_t)L.n_partials * 4);
  L.bytes_decode = align_up(decode_ws_bytes(D));
  return L;
}

size_t total_bytes(const Layout& L) {
  size_t m = L.bytes_scores;
  if (L.bytes_bwd > m) m = L.bytes_bwd;
  if (L.bytes_dropped > m) m = L.bytes_dropped;
  if (L.bytes_align > m) m = L.bytes_align;
  if (L.bytes_decode > m) m = L.bytes_decode;
  return m;
}

ssa_status_t check_ws(const Dims& D, const void* ws, size_t ws_bytes) {
  const size_t need = total_bytes(layout(D));
  if (ws == nullptr || ws_bytes < need) return SSA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % kAlign != 0) return SSA_ERR_INVALID_ARG;
  return SSA_OK;
}

template <typename P>
P* at(void* ws, size_t off) { return reinterpret_cast<P*>(static_cast<char*>(ws) + off); }

int32_t* device_status_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
  return static_cast<int32_t*>(p);
}

}  // namespace
}  // namespace ssa

using namespace ssa;

extern "C" {

int ssa_version(void) { return 110; }

uint64_t ssa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* ssa_status_string(ssa_status_t s) {
  switch (s) {
    case SSA_OK: return "SSA_OK";
    case SSA_ERR_INVALID_ARG: return "SSA_ERR_INVALID_ARG";
    case SSA_ERR_UNSUPPORTED: return "SSA_ERR_UNSUPPORTED";
    case SSA_ERR_CUDA: return "SSA_ERR_CUDA";
    case SSA_ERR_TIMEOUT: return "SSA_ERR_TIMEOUT";
    case SSA_ERR_WORKSPACE: return "SSA_ERR_WORKSPACE";
  }
  return "SSA_ERR_UNKNOWN";
}

size_t ssa_workspace_bytes(const ssa_dims_t* dims) {
  Dims D;
  bool empty = false;
  if (check_dims(dims, &D, &empty) != SSA_OK || empty) return 0;
  return total_bytes(layout(D));
}

ssa_status_t ssa_block_scores(const ssa_dims_t* dims, const ssa_tensor_t* Q, const ssa_tensor_t* K,
                              float* scores, void* ws, size_t ws_bytes, ssa_stream_t stream) {
  const NvtxRange nvtx_range("ssa_block_scores");
  Dims D;
  bool empty = false;
  ssa_status_t s = check_dims(dims, &D, &empty);
  if (s != SSA_OK) return s;
  if (D.per_token) return SSA_ERR_INVALID_ARG;  // per-token selection: ssa_select_tokens
  if (empty) return SSA_OK;
  TensorRef q, k;
  if ((s = check_tensor(D, Q, false, &q)) != SSA_OK) return s;
  if ((s = check_tensor(D, K, false, &k)) != SSA_OK) return s;
  if (scores == nullptr || reinterpret_cast<uintptr_t>(scores) % 4) return SSA_ERR_INVALID_ARG;
  if ((s = check_ws(D, ws, ws_bytes)) != SSA_OK) return s;
  if ((s = check_device()) != SSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Layout L = layout(D);
  float* qbar = at<float>(ws, L.qbar);
  float* kbar = at<float>(ws, L.kbar);
  cudaError_t e = launch_pool(D, q, D.Hq, qbar, st);
  if (e == cudaSuccess) e = launch_pool(D, k, D.Hkv, kbar, st);
  if (e == cudaSuccess) e = launch_scores(D, qbar, kbar, scores, st);
  return from_cuda(e);
}

ssa_status_t ssa_select_topk(const ssa_dims_t* dims, const float* scores, int32_t* idx,
                             ssa_stream_t stream) {
  const NvtxRange nvtx_range("ssa_select_topk");
  Dims D;
  bool empty = false;
  ssa_status_t s = check_dims(dims, &D, &empty);
  if (s != SSA_OK) return s;
  if (D.per_token) return SSA_ERR_INVALID_ARG;  // per-token selection: ssa_select_tokens
  if (empty) return SSA_OK;
  if (scores == nullptr || idx == nullptr) return SSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(scores) % 4 || reinterpret_cast<uintptr_t>(idx) % 4)
    return SSA_ERR_INVALID_ARG;
  if ((s = check_device()) != SSA_OK) return s;
  return from_cuda(launch_select(D, scores, idx, static_cast<cudaStream_t>(stream)));
}

ssa_status_t ssa_fwd_dual(const ssa_dims_t* dims, const ssa_tensor_t* Q, const ssa_tensor_t* K,
                          const ssa_tensor_t* V, const int32_t* idx, const ssa_tensor_t* h_full,
                          const ssa_tensor_t* h_sparse, float* lse_full, float* lse_sel,
                          float* delta, ssa_stream_t stream) {
  const NvtxRange nvtx_range("ssa_fwd_dual");
  Dims D;
  bool empty = false;
  ssa_status_t s = check_dims(dims, &D, &empty);
  if (s != SSA_OK) return s;
  if (empty) return SSA_OK;
  FwdArgs a{};
  if ((s = check_tensor(D, Q, false, &a.q)) != SSA_OK) return s;
  if ((s = check_tensor(D, K, false, &a.k)) != SSA_OK) return s;
  if ((s = check_tensor(D, V, false, &a.v)) != SSA_OK) return s;
  if ((s = check_tensor(D, h_full, false, &a.hf)) != SSA_OK) return s;
  if ((s = check_tensor(D, h_sparse, false, &a.hs)) != SSA_OK) return s;
  if (!idx || !lse_full || !lse_sel || !delta) return SSA_ERR_INVALID_ARG;
  if ((s = check_device()) != SSA_OK) return s;
  a.idx = idx;
  a.lse_full = lse_full;
  a.lse_sel = lse_sel;
  a.delta = delta;
  a.lse_in = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (fwd_tc_supported(D) || fwd_tcm_supported(D)) {
    int32_t* status = device_status_ptr();
    if (status == nullptr) return SSA_ERR_CUDA;
    return from_cuda(fwd_tc_supported(D) ? launch_fwd_ord(D, a, status, st) : launch_fwd_tcm(D, a, status, st));
  }
  if (fwd_mma_supported(D)) return from_cuda(launch_fwd_mma(D, a, st));
  return from_cuda(launch_fwd_simt(D, a, st));
}

ssa_status_t ssa_bwd_dual(const ssa_dims_t* dims, const ssa_tensor_t* Q, const ssa_tensor_t* K,
                          const ssa_tensor_t* V, const int32_t* idx, const ssa_tensor_t* h_full,
                          const ssa_tensor_t* h_sparse, const float* lse_full,
                          const float* lse_sel, const ssa_tensor_t* g_full,
                          const ssa_tensor_t* g_sparse, float alpha, float* align_loss,
                          const ssa_tensor_t* dQ, const ssa_tensor_t* dK, const ssa_tensor_t* dV,
                          void* ws, size_t ws_bytes, ssa_stream_t stream) {
  const NvtxRange nvtx_range("ssa_bwd_dual");
  Dims D;
  bool empty = false;
  ssa_status_t s = check_dims(dims, &D, &empty);
  if (s != SSA_OK) return s;
  if (empty) return SSA_OK;
  BwdArgs a{};
  if ((s = check_tensor(D, Q, false, &a.q)) != SSA_OK) return s;
  if ((s = check_tensor(D, K, false, &a.k)) != SSA_OK) return s;
  if ((s = check_tensor(D, V, false, &a.v)) != SSA_OK) return s;
  if ((s = check_tensor(D, h_full, false, &a.hf)) != SSA_OK) return s;
  if ((s = check_tensor(D, h_sparse, false, &a.hs)) != SSA_OK) return s;
  if ((s = check_tensor(D, g_full, true, &a.gf)) != SSA_OK) return s;
  if ((s = check_tensor(D, g_sparse, true, &a.gs)) != SSA_OK) return s;
  if ((s = check_tensor(D, dQ, false, &a.dq)) != SSA_OK) return s;
  if ((s = check_tensor(D, dK, false, &a.dk)) != SSA_OK) return s;
  if ((s = check_tensor(D, dV, false, &a.dv)) != SSA_OK) return s;
  if (!(alpha == alpha)) return SSA_ERR_INVALID_ARG;
  if (!idx || !lse_full || !lse_sel) return SSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(lse_full) % 16 || reinterpret_cast<uintptr_t>(lse_sel) % 16)
    return SSA_ERR_INVALID_ARG;
  if ((s = check_ws(D, ws, ws_bytes)) != SSA_OK) return s;
  if ((s = check_device()) != SSA_OK) return s;
  const Layout L = layout(D);
  a.idx = idx;
  a.lse_full = lse_full;
  a.lse_sel = lse_sel;
  a.alpha = alpha;
  a.align_loss = align_loss;
  a.dhf = at<float>(ws, L.dhf);
  a.doc = at<float>(ws, L.doc);
  a.Df = at<float>(ws, L.Df);
  a.Dc = at<float>(ws, L.Dc);
  a.mask = at<uint32_t>(ws, L.mask);
  a.words = L.words;
  a.partials = at<float>(ws, L.partials);
  a.n_partials = L.n_partials;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_build_mask(D, idx, a.mask, L.words, st);
  if (e != cudaSuccess) return from_cuda(e);
  if (bwd_tc_supported(D)) {
    int32_t* status = device_status_ptr();
    if (status == nullptr) return SSA_ERR_CUDA;
    a.kvpart = at<float>(ws, L.kvpart);
    return from_cuda(launch_bwd_tc(D, a, status, st));
  }
  if (bwd_mma_supported(D)) {
    a.kvpart = at<float>(ws, L.kvpart);
    int32_t* status = device_status_ptr();
    if (status == nullptr) return SSA_ERR_CUDA;
    return from_cuda(launch_bwd_mma(D, a, status, st));
  }
  e = launch_bwd_pre(D, a, st);
  if (e == cudaSuccess) e = launch_bwd_simt(D, a, st);
  return from_cuda(e);
}

ssa_status_t ssa_select_tokens(const ssa_dims_t* dims, const ssa_tensor_t* Q, const ssa_tensor_t* K,
                               int32_t* idx, void* ws, size_t ws_bytes, ssa_stream_t stream) {
  const NvtxRange nvtx_range("ssa_select_tokens");
  Dims D;
  bool empty = false;
  ssa_status_t s = check_dims(dims, &D, &empty);
  if (s != SSA_OK) return s;
  if (!D.per_token) return SSA_ERR_INVALID_ARG;  // per-block selection: ssa_block_scores + ssa_select_topk
  if (empty) return SSA_OK;
  TensorRef q, k;
  if ((s = check_tensor(D, Q, false, &q)) != SSA_OK) return s;
  if ((s = check_tensor(D, K, false, &k)) != SSA_OK) return s;
  if (idx == nullptr || reinterpret_cast<uintptr_t>(idx) % 4) return SSA_ERR_INVALID_ARG;
  if ((s = check_ws(D, ws, ws_bytes)) != SSA_OK) return s;
  if ((s = check_device()) != SSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Layout L = layout(D);
  float* kbar = at<float>(ws, L.kbar);
  cudaError_t e = launch_pool(D, k, D.Hkv, kbar, st);
  if (e == cudaSuccess) e = launch_select_tokens(D, q, kbar, idx, st);
  return from_cuda(e);
}

ssa_status_t ssa_fwd_sparse(const ssa_dims_t* dims, const ssa_tensor_t* Q, const ssa_tensor_t* K,
                            const ssa_tensor_t* V, const int32_t* idx, const ssa_tensor_t* h_sparse,
                            float* lse_sel, ssa_stream_t stream) {
  const NvtxRange nvtx_range("ssa_fwd_sparse");
  Dims D;
  bool empty = false;
  ssa_status_t s = check_dims(dims, &D, &empty);
  if (s != SSA_OK) return s;
  if (empty) return SSA_OK;
  FwdArgs a{};
  if ((s = check_tensor(D, Q, false, &a.q)) != SSA_OK) return s;
  if ((s = check_tensor(D, K, false, &a.k)) != SSA_OK) return s;
  if ((s = check_tensor(D, V, false, &a.v)) != SSA_OK) return s;
  if ((s = check_tensor(D, h_sparse, false, &a.hs)) != SSA_OK) return s;
  if (!idx || !lse_sel) return SSA_ERR_INVALID_ARG;
  if ((s = check_device()) != SSA_OK) return s;
  a.hf = TensorRef{nullptr, 0, 0, 0};
  a.idx = idx;
  a.lse_sel = lse_sel;
  a.sparse_only = true;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (fwd_tc_supported(D)) {
    int32_t* status = device_status_ptr();
    if (status == nullptr) return SSA_ERR_CUDA;
    return from_cuda(launch_fwd_ord(D, a, status, st));
  }
  if (fwd_walk_supported(D)) {
    int32_t* status = device_status_ptr();
    if (status == nullptr) return SSA_ERR_CUDA;
    return from_cuda(launch_fwd_walk(D, a, status, st));
  }
  if (fwd_mma_supported(D)) return from_cuda(launch_fwd_mma(D, a, st));
  return from_cuda(launch_fwd_simt(D, a, st));
}

ssa_status_t ssa_bwd_sparse(const ssa_dims_t* dims, const ssa_tensor_t* Q, const ssa_tensor_t* K,
                            const ssa_tensor_t* V, const int32_t* idx, const ssa_tensor_t* h_sparse,
                            const float* lse_sel, const ssa_tensor_t* g_sparse, const ssa_tensor_t* dQ,
                            const ssa_tensor_t* dK, const ssa_tensor_t* dV, void* ws, size_t ws_bytes,
                            ssa_stream_t stream) {
  const NvtxRange nvtx_range("ssa_bwd_sparse");
  Dims D;
  bool empty = false;
  ssa_status_t s = check_dims(dims, &D, &empty);
  if (s != SSA_OK) return s;
  if (empty) return SSA_OK;
  BwdArgs a{};
  if ((s = check_tensor(D, Q, false, &a.q)) != SSA_OK) return s;
  if ((s = check_tensor(D, K, false, &a.k)) != SSA_OK) return s;
  if ((s = check_tensor(D, V, false, &a.v)) != SSA_OK) return s;
  if ((s = check_tensor(D, h_sparse, false, &a.hs)) != SSA_OK) return s;
  if ((s = check_tensor(D, g_sparse, false, &a.gs)) != SSA_OK) return s;
  if ((s = check_tensor(D, dQ, false, &a.dq)) != SSA_OK) return s;
  if ((s = check_tensor(D, dK, false, &a.dk)) != SSA_OK) return s;
  if ((s = check_tensor(D, dV, false, &a.dv)) != SSA_OK) return s;
  if (!idx || !lse_sel) return SSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(lse_sel) % 16) return SSA_ERR_INVALID_ARG;
  if ((s = check_ws(D, ws, ws_bytes)) != SSA_OK) return s;
  if ((s = check_device()) != SSA_OK) return s;
  const Layout L = layout(D);
  // The sparse stream alone is the dual backward with h_full := h_sparse,
  // lse_full := lse_sel, no full-stream gradient and no alignment term
  // (dh_f = 0, r = 1), restricted to the selected pairs.
  a.hf = a.hs;
  a.gf = TensorRef{nullptr, 0, 0, 0};
  a.idx = idx;
  a.lse_full = lse_sel;
  a.lse_sel = lse_sel;
  a.alpha = 0.f;
  a.align_loss = nullptr;
  a.dhf = at<float>(ws, L.dhf);
  a.doc = at<float>(ws, L.doc);
  a.Df = at<float>(ws, L.Df);
  a.Dc = at<float>(ws, L.Dc);
  a.mask = at<uint32_t>(ws, L.mask);
  a.words = L.words;
  a.partials = at<float>(ws, L.partials);
  a.n_partials = L.n_partials;
  a.sparse_only = true;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_build_mask(D, idx, a.mask, L.words, st);
  if (e != cudaSuccess) return from_cuda(e);
  if (bwd_walk_supported(D)) {
    // The walk's g per-head fp32 dK / dV partials fill the adjacent dh_f and
    // dO_c regions (2 x B*Hq*N*d floats), which the sparse stream leaves unused.
    if (L.Df - L.dhf < 2 * (size_t)D.B * D.Hq * D.N * D.d * sizeof(float)) return SSA_ERR_WORKSPACE;
    a.maskT = at<uint32_t>(ws, L.maskT);
    int32_t* status = device_status_ptr();
    if (status == nullptr) return SSA_ERR_CUDA;
    return from_cuda(launch_bwd_walk(D, a, status, st));
  }
  if (bwd_tc_supported(D)) {
    int32_t* status = device_status_ptr();
    if (status == nullptr) return SSA_ERR_CUDA;
    a.kvpart = at<float>(ws, L.kvpart);
    return from_cuda(launch_bwd_tc(D, a, status, st));
  }
  if (bwd_mma_supported(D)) {
    a.kvpart = at<float>(ws, L.kvpart);
    int32_t* status = device_status_ptr();
    if (status == nullptr) return SSA_ERR_CUDA;
    return from_cuda(launch_bwd_mma(D, a, status, st));
  }
  e = launch_bwd_pre(D, a, st);
  if (e == cudaSuccess) e = launch_bwd_simt(D, a, st);
  return from_cuda(e);
}

ssa_status_t ssa_decode_prefill(const ssa_dims_t* dims, const ssa_tensor_t* Q, const ssa_tensor_t* K,
                                int32_t t0, float* qsum, float* kbar, ssa_stream_t stream) {
  const NvtxRange nvtx_range("ssa_decode_prefill");
  Dims D;
  bool empty = false;
  ssa_status_t s = check_dims(dims, &D, &empty);
  if (s != SSA_OK) return s;
  if (empty) return SSA_OK;
  DecodeArgs a{};
  if ((s = check_tensor(D, Q, false, &a.q)) != SSA_OK) return s;
  if ((s = check_tensor(D, K, false, &a.k)) != SSA_OK) return s;
  if (t0 < 0 || t0 > D.N) return SSA_ERR_INVALID_ARG;
  if (!qsum || !kbar || reinterpret_cast<uintptr_t>(qsum) % 4 || reinterpret_cast<uintptr_t>(kbar) % 4)
    return SSA_ERR_INVALID_ARG;
  if ((s = check_device()) != SSA_OK) return s;
  a.qsum = qsum;
  a.kbar = kbar;
  a.t = t0;
  return from_cuda(launch_decode_prefill(D, a, static_cast<cudaStream_t>(stream)));
}

ssa_status_t ssa_decode_step(const ssa_dims_t* dims, const ssa_tensor_t* q, const ssa_tensor_t* K,
                             const ssa_tensor_t* V, int32_t t, float* qsum, float* kbar,
                             const ssa_tensor_t* h, float* lse, int32_t* idx, void* ws, size_t ws_bytes,
                             ssa_stream_t stream) {
  const NvtxRange nvtx_range("ssa_decode_step");
  Dims D;
  bool empty = false;
  ssa_status_t s = check_dims(dims, &D, &empty);
  if (s != SSA_OK) return s;
  if (empty) return SSA_OK;
  DecodeArgs a{};
  if ((s = check_tensor(D, q, false, &a.q)) != SSA_OK) return s;
  if ((s = check_tensor(D, K, false, &a.k)) != SSA_OK) return s;
  if ((s = check_tensor(D, V, false, &a.v)) != SSA_OK) return s;
  if ((s = check_tensor(D, h, false, &a.h)) != SSA_OK) return s;
  if (t < 0 || t >= D.N) return SSA_ERR_INVALID_ARG;
  if (!qsum || !kbar || !lse || !idx) return SSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(qsum) % 4 || reinterpret_cast<uintptr_t>(kbar) % 16 ||
      reinterpret_cast<uintptr_t>(lse) % 4 || reinterpret_cast<uintptr_t>(idx) % 4)
    return SSA_ERR_INVALID_ARG;
  if (!decode_supported(D)) return SSA_ERR_UNSUPPORTED;
  if ((s = check_ws(D, ws, ws_bytes)) != SSA_OK) return s;
  if ((s = check_device()) != SSA_OK) return s;
  a.ws = ws;
  a.lse = lse;
  a.idx = idx;
  a.qsum = qsum;
  a.kbar = kbar;
  a.t = t;
  int32_t* status = device_status_ptr();
  if (status == nullptr) return SSA_ERR_CUDA;
  return from_cuda(launch_decode(D, a, status, static_cast<cudaStream_t>(stream)));
}

ssa_status_t ssa_dropped_mass(const ssa_dims_t* dims, const ssa_tensor_t* Q, const ssa_tensor_t* K,
                              const int32_t* idx, const float* lse_full, float* delta, void* ws,
                              size_t ws_bytes, ssa_stream_t stream) {
  const NvtxRange nvtx_range("ssa_dropped_mass");
  Dims D;
  bool empty = false;
  ssa_status_t s = check_dims(dims, &D, &empty);
  if (s != SSA_OK) return s;
  if (empty) return SSA_OK;
  FwdArgs a{};
  if ((s = check_tensor(D, Q, false, &a.q)) != SSA_OK) return s;
  if ((s = check_tensor(D, K, false, &a.k)) != SSA_OK) return s;
  if (!idx || !delta) return SSA_ERR_INVALID_ARG;
  if ((s = check_ws(D, ws, ws_bytes)) != SSA_OK) return s;
  if ((s = check_device()) != SSA_OK) return s;
  a.v = a.k;  // unused
  a.idx = idx;
  a.delta = delta;
  a.lse_in = lse_full;
  if (fwd_tc_supported(D) || fwd_tcm_supported(D)) {
    int32_t* status = device_status_ptr();
    if (status == nullptr) return SSA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return from_cuda(fwd_tc_supported(D) ? launch_dropped_tc(D, a, status, st) : launch_dropped_tcm(D, a, status, st));
  }
  if (fwd_mma_supported(D)) return from_cuda(launch_dropped_mma(D, a, static_cast<cudaStream_t>(stream)));
  return from_cuda(launch_dropped_simt(D, a, static_cast<cudaStream_t>(stream)));
}

ssa_status_t ssa_align_mse(const ssa_dims_t* dims, const ssa_tensor_t* h_full,
                           const ssa_tensor_t* h_sparse, float* loss, void* ws, size_t ws_bytes,
                           ssa_stream_t stream) {
  const NvtxRange nvtx_range("ssa_align_mse");
  Dims D;
  bool empty = false;
  ssa_status_t s = check_dims(dims, &D, &empty);
  if (s != SSA_OK) return s;
  if (empty) return SSA_OK;
  TensorRef hf, hs;
  if ((s = check_tensor(D, h_full, false, &hf)) != SSA_OK) return s;
  if ((s = check_tensor(D, h_sparse, false, &hs)) != SSA_OK) return s;
  if (loss == nullptr) return SSA_ERR_INVALID_ARG;
  if ((s = check_ws(D, ws, ws_bytes)) != SSA_OK) return s;
  if ((s = check_device()) != SSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Layout L = layout(D);
  float* partials = static_cast<float*>(ws);
  const double M = (double)D.B * D.Hq * D.N * D.d;
  cudaError_t e = launch_sqdiff_partials(D, hf, hs, partials, L.n_partials, st);
  if (e == cudaSuccess) e = launch_finish_mean(partials, L.n_partials, M, 1.0f, loss, 2, st);
  return from_cuda(e);
}

ssa_status_t ssa_selftest_timeout(ssa_stream_t stream) {
  ssa_status_t s = check_device();
  if (s != SSA_OK) return s;
  int32_t* status = device_status_ptr();
  if (status == nullptr) return SSA_ERR_CUDA;
  // ~10 ms at the B200's clock: long enough to be a real wait, short for a test
  return from_cuda(launch_selftest_timeout(status, 20000000LL, static_cast<cudaStream_t>(stream)));
}

ssa_status_t ssa_device_status(int32_t* status, int clear, ssa_stream_t stream) {
  if (status == nullptr) return SSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return SSA_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return SSA_ERR_CUDA;
  *status = v;
  if (clear) {
    const int32_t zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess) return SSA_ERR_CUDA;
  }
  return SSA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- no-alloc variant
// Fixed device scratch for ssa_block_scores_noalloc (see include/ssa.h).  In
// host code this name is only a stand-in for the symbol, never a device
// address: the address is looked up per device with cudaGetSymbolAddress.
static __device__ __align__(256) float g_noalloc_scratch[SSA_NOALLOC_SCRATCH_FLOATS];

namespace ssa {
namespace {

constexpr int kMaxDevices = 128;
float* g_noalloc_ptr[kMaxDevices] = {};
unsigned long long g_noalloc_ctx[kMaxDevices] = {};  // context the cached address belongs to
std::mutex g_noalloc_mu;

// Unique id of the calling thread's current CUDA context (0 if unavailable).
// cudaDeviceReset destroys a device's primary context; the next runtime call
// creates a new one with a new id, in which the library's module -- and with
// it the scratch array -- is loaded again, possibly at another address.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur == nullptr || get_id == nullptr || get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_noalloc_scratch on the current device: looked up once
// per device, and again whenever the device's context has been replaced since.
ssa_status_t noalloc_scratch(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  const unsigned long long ctx = current_context_id();
  if (g_noalloc_ptr[dev] == nullptr || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return SSA_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<float*>(p);
    // cudaGetSymbolAddress made the primary context current if it was not.
    g_noalloc_ctx[dev] = ctx != 0 ? ctx : current_context_id();
  }
  *out = g_noalloc_ptr[dev];
  return SSA_OK;
}

}  // namespace
}  // namespace ssa

extern "C" ssa_status_t ssa_block_scores_noalloc(const ssa_dims_t* dims, const ssa_tensor_t* Q,
                                                 const ssa_tensor_t* K, float* scores,
                                                 ssa_stream_t stream) {
  const NvtxRange nvtx_range("ssa_block_scores_noalloc");
  Dims D;
  bool empty = false;
  ssa_status_t s = check_dims(dims, &D, &empty);
  if (s != SSA_OK) return s;
  if (D.per_token) return SSA_ERR_INVALID_ARG;  // block scores only
  if (empty) return SSA_OK;
  TensorRef q, k;
  if ((s = check_tensor(D, Q, false, &q)) != SSA_OK) return s;
  if ((s = check_tensor(D, K, false, &k)) != SSA_OK) return s;
  if (scores == nullptr || reinterpret_cast<uintptr_t>(scores) % 4) return SSA_ERR_INVALID_ARG;
  const uint64_t q_floats = (uint64_t)D.B * D.Hq * D.n * D.d;
  const uint64_t k_floats = (uint64_t)D.B * D.Hkv * D.n * D.d;
  if (q_floats + k_floats > (uint64_t)SSA_NOALLOC_SCRATCH_FLOATS) return SSA_ERR_WORKSPACE;
  if ((s = check_device()) != SSA_OK) return s;
  float* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != SSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // q-bar at the start, k-bar after it (256-byte aligned, like the workspace layout).
  float* qbar = scratch;
  float* kbar = scratch + (q_floats + 63) / 64 * 64;
  if ((uint64_t)(kbar - scratch) + k_floats > (uint64_t)SSA_NOALLOC_SCRATCH_FLOATS) return SSA_ERR_WORKSPACE;
  cudaError_t e = launch_pool(D, q, D.Hq, qbar, st);
  if (e == cudaSuccess) e = launch_pool(D, k, D.Hkv, kbar, st);
  if (e == cudaSuccess) e = launch_scores(D, qbar, kbar, scores, st);
  return from_cuda(e);
}
