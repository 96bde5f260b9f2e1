// Tensor-core (tcgen05 / TMEM / TMA) encode and decode kernels: placeholder
// until the sm_100a kernels land; the dispatcher does not select them yet.
#include "flare_internal.cuh"

namespace flare {

cudaError_t launch_tc_encode(const void*, int64_t, const void*, const void*, const Dims&, float,
                             const ChunkPlan&, float*, float*, uint32_t*, cudaStream_t) {
  return cudaErrorNotSupported;
}

cudaError_t launch_tc_decode(const void*, int64_t, const void*, const __nv_bfloat16*, void*,
                             const Dims&, float, const ChunkPlan&, uint32_t*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace flare
