// gdn_noalloc.cu -- gdn_prefill_noalloc: the prefill with a built-in scratch array instead
// of a caller-provided workspace, for callers that cannot allocate device memory at call
// time (their device memory is owned by another allocator, or they must not take the
// device-wide synchronisation of cudaMalloc / cudaFree inside a latency-critical loop).
#include <cuda_runtime.h>

#include <atomic>

#include "gdn.h"

namespace {

// The scratch itself: one fixed array per GPU that loads the library, alive until exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GDN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices];
std::atomic<bool> g_scratch_ready[kMaxDevices];

// Device address of the scratch array on the current device.  In host code the array's
// name is only a host-side stand-in, so the address is looked up once per device (with
// that device current) and cached.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_CUDA;
  if (!g_scratch_ready[dev].load(std::memory_order_acquire)) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return GDN_ERR_CUDA;
    g_scratch_ptr[dev] = p;
    g_scratch_ready[dev].store(true, std::memory_order_release);
  }
  *out = g_scratch_ptr[dev];
  return GDN_OK;
}

}  // namespace

extern "C" int gdn_prefill_noalloc(const gdn_dims_t* d, const void* q, const void* k,
                                   const void* v, const void* z, const float* a, const float* b,
                                   const float* A_log, const float* dt_bias, const float* conv_w,
                                   const float* norm_w, const float* init_state,
                                   const int32_t* cu_seqlens, void* y, float* final_state,
                                   gdn_stream_t stream) {
  if (!d) return GDN_ERR_NULL;
  const size_t need = gdn_prefill_workspace_size(d);
  if (need == 0) return GDN_ERR_SHAPE;
  if (need > GDN_NOALLOC_SCRATCH_BYTES) return GDN_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != GDN_OK) return rc;
  return gdn_prefill(d, q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w, init_state, cu_seqlens,
                     y, final_state, scratch, GDN_NOALLOC_SCRATCH_BYTES, stream);
}
