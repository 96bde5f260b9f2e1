// FLARE forward for callers that cannot allocate device memory.
//
// flare_fwd needs a caller-provided workspace for its scratch: the per-chunk
// softmax records of the encode, the merged Z and its bf16 copy, and an
// error word.  Some callers have no way to provide one: a plugin inside a
// host framework that owns every device allocation and hands its plugins no
// workspace, or a latency-critical loop that must not call cudaMalloc (it
// can synchronise the device) once it is running.  flare_fwd_noalloc serves
// them by keeping that scratch in one file-scope device array of fixed size,
// which every GPU that loads this library holds until the process exits.
//
// The array is shared by every call on a device and keeps whatever the last
// call left in it.  Everything that must start at zero (the error word) is
// cleared by each call on its stream, and every other byte is written before
// it is read.  Two calls whose work overlaps on the GPU (different streams,
// or different host threads, same device) race on the array.
#include <mutex>

#include "flare_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_flare_noalloc_scratch[FLARE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
// Per device: the context the address was resolved in, and the address.
void* g_scratch_ctx[kMaxDevices];
void* g_scratch_ptr[kMaxDevices];

// The current context (the driver's cuCtxGetCurrent, reached through the
// runtime's entry-point query so that no driver library is linked).
void* current_context() {
  typedef int (*GetCtx)(void**);
  static GetCtx fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return (GetCtx)p;
  }();
  void* ctx = nullptr;
  if (fn == nullptr || fn(&ctx) != 0) return nullptr;
  return ctx;
}

// Device address of the scratch array on the current device.  The first
// call on a device resolves it with cudaGetSymbolAddress (which also loads
// the module on that device); later calls reuse the cached address while
// the device's context is the one it was resolved in (after a
// cudaDeviceReset the context, and possibly the address, are new, so it is
// resolved again).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  // NULL on a host thread where the runtime has not yet made the device's
  // context current: the address is then resolved again, which does that
  void* ctx = current_context();
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr || ctx == nullptr || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_flare_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = current_context();
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" flare_status_t flare_fwd_noalloc(const void* Q, int64_t q_batch_stride, const void* K,
                                            const void* V, void* Y, int64_t B, int64_t H,
                                            int64_t N, int64_t M, int64_t D,
                                            flare_dtype_t dtype, float scale, float* Z_save,
                                            float* lse_save, void* stream) {
  const size_t need = flare_workspace_size(FLARE_OP_FWD, B, H, N, M, D, dtype);
  if (need == 0) {
    // invalid or unsupported sizes: let flare_fwd report which
    return flare_fwd(Q, q_batch_stride, K, V, Y, B, H, N, M, D, dtype, scale, Z_save, lse_save,
                     nullptr, 0, stream);
  }
  if (need > (size_t)FLARE_NOALLOC_SCRATCH_BYTES) {
    flare::note_error(
        "flare_fwd_noalloc: these sizes need %zu bytes of scratch, above the fixed %u-byte "
        "array; use flare_fwd with a caller workspace",
        need, (unsigned)FLARE_NOALLOC_SCRATCH_BYTES);
    return FLARE_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) {
    cudaGetLastError();
    flare::note_error("flare_fwd_noalloc: cudaGetSymbolAddress of the scratch array failed");
    return FLARE_ERR_CUDA;
  }
  return flare_fwd(Q, q_batch_stride, K, V, Y, B, H, N, M, D, dtype, scale, Z_save, lse_save,
                   scratch, (size_t)FLARE_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" flare_status_t flare_noalloc_device_status(uint32_t* detail, void* stream) {
  if (detail) *detail = 0;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) {
    cudaGetLastError();
    flare::note_error("flare_noalloc_device_status: cudaGetSymbolAddress of the scratch array failed");
    return FLARE_ERR_CUDA;
  }
  return flare_device_status(scratch, (size_t)FLARE_NOALLOC_SCRATCH_BYTES, detail, stream);
}
