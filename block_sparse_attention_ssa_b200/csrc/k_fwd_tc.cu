// Tensor-core (tcgen05 / TMEM / TMA) dual-stream forward: not built yet.
#include "ssa_internal.cuh"

namespace ssa {

bool fwd_tc_supported(const Dims&) { return false; }

cudaError_t launch_fwd_tc(const Dims&, const FwdArgs&, int32_t*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace ssa
