// Allocation-free chunked prefill: the tensor-core prefill with its device
// scratch taken from a fixed array that lives in this library's device image,
// for callers that cannot allocate device memory when they call us.
//
// The scratch is a file-scope __device__ array. Its host-side name is only a
// stand-in for the device symbol, so host code never passes it to a kernel:
// the device address is looked up per device with cudaGetSymbolAddress (with
// that device current) and cached once the lookup has succeeded. The first
// call on a device also loads the library's device code there, which is when
// the array is reserved; every GPU that has done so holds it until the
// process exits.

#include <mutex>

#include "common.cuh"

namespace {

// Stated maximum scratch of the allocation-free call: 32 MiB per GPU.
constexpr size_t kNoAllocScratchBytes = 32u << 20;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_lock;
void* g_scratch[kMaxDevices];   // device address per device, NULL until a lookup succeeded

// Device address of the scratch array on the current device. A failed lookup
// is not cached: the next call tries again.
cudaError_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> guard(g_lock);
  if (g_scratch[dev] == nullptr) {
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_noalloc_scratch)) != cudaSuccess) return e;
    g_scratch[dev] = p;
  }
  *out = g_scratch[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" GDN2_API gdn2_status gdn2_chunk_fwd_noalloc(const gdn2_params* p, const void* q, const void* k,
                                                       const void* v, const float* alpha, const float* b,
                                                       const float* w, const float* S0, void* o, float* S_T,
                                                       void* stream) {
  // invalid parameters get the statuses of gdn2_chunk_fwd
  const gdn2_status st = gdn2::check_chunk_params(p);
  if (st != GDN2_OK) return st;
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

extern "C" GDN2_API gdn2_status gdn2_chunk_fwd_noalloc_status(void* stream) {
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return GDN2_ERR_CUDA;
  return gdn2::read_device_status(scratch, static_cast<cudaStream_t>(stream));
}
