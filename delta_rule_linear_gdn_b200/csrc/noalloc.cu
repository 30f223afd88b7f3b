// Allocation-free chunked prefill: the tensor-core prefill with its device
// scratch taken from a fixed array that lives in this library's device image,
// for callers that cannot allocate device memory when they call us.
//
// The scratch is a file-scope __device__ array. Its host-side name is only a
// stand-in for the device symbol, so host code never passes it to a kernel:
// the device address is looked up once per device with cudaGetSymbolAddress
// (with that device current) and cached. Every GPU that loads the library
// holds the array until the process exits.

#include <mutex>

#include "common.cuh"

namespace {

// Stated maximum scratch of the allocation-free call: 32 MiB per GPU.
constexpr size_t kNoAllocScratchBytes = 32u << 20;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::once_flag g_once[kMaxDevices];
void* g_scratch[kMaxDevices];
cudaError_t g_setup_status[kMaxDevices];

// Device address of the scratch array on the current device; the first call
// per device performs the lookup.
cudaError_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_once[dev], [dev]() {
    void* p = nullptr;
    g_setup_status[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    g_scratch[dev] = p;
  });
  if (g_setup_status[dev] != cudaSuccess) return g_setup_status[dev];
  *out = g_scratch[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" GDN2_API gdn2_status gdn2_chunk_fwd_noalloc(const gdn2_params* p, const void* q, const void* k,
                                                       const void* v, const float* alpha, const float* b,
                                                       const float* w, const float* S0, void* o, float* S_T,
                                                       void* stream) {
  if (!p) return GDN2_ERR_INVALID_ARG;
  if (p->cu_seqlens) return GDN2_ERR_UNSUPPORTED;   // packed sequences need every chunk's slot at once
  // Only the tensor-core prefill uses scratch; it is the configuration this
  // call serves (every other configuration runs without scratch through
  // gdn2_chunk_fwd).
  if (gdn2_chunk_fwd_workspace(p) == 0) return GDN2_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return GDN2_ERR_CUDA;
  // The array holds as many chunks per (sequence, value head) as fit; the
  // sequence runs in segments of that many chunks. A problem whose single
  // chunk slot per sequence-head exceeds the array gets GDN2_ERR_WORKSPACE.
  return gdn2::chunk_fwd_checked(p, q, k, v, alpha, b, w, S0, o, S_T, scratch, kNoAllocScratchBytes, stream,
                                 /*segmented_ok=*/true);
}
