// TMA tensor maps over the [B, H, N, d] bf16 tensors of the tensor-core
// kernels (encoded on the host through the driver entry point, so that the
// library needs no libcuda at link time).
#include "ssa_internal.cuh"

#include <cudaTypedefs.h>

namespace ssa {

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 4-D map over a [B, H, N, d] bf16 tensor: dims (d, N, H, B), box (64, rows, 1, 1).
bool make_tma_map_bf16(CUtensorMap* map, const TensorRef& t, int B, int H, int N, int rows, int d) {
  auto enc = get_encode();
  if (enc == nullptr || (d != 64 && d != 128)) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)t.sn * 2, (cuuint64_t)t.sh * 2, (cuuint64_t)t.sb * 2};
  // A zero stride (a broadcast dimension of size 1) is not accepted; any
  // positive multiple of 16 describes the same single slice.
  for (int i = 0; i < 3; ++i)
    if (strides[i] == 0) strides[i] = 16;
  cuuint32_t box[4] = {64, (cuuint32_t)rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(t.p), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool fwd_tc_supported(const Dims& D) {
  return D.dtype == SSA_BF16 && D.d == 128 && (D.s == 64 || D.s == 128) && D.n <= 2048 && !D.per_token;
}

}  // namespace ssa
