// noalloc.cu -- slora_lora_delta_noalloc: the decode delta with its scratch in
// a fixed device array that the library owns, so the caller does not have to
// provide (or allocate) any scratch memory for the call.
//
// Who needs this: code that cannot allocate device memory at the point where
// it runs the delta -- for instance a plug-in whose host framework owns every
// device allocation and hands it only its inputs and outputs, or a
// latency-critical serving loop that must not risk an allocation blocking on
// the device.  Such a caller still passes the pool, x, y and the index vector;
// everything else the kernels need comes from the array below.
//
// The array is a file-scope __device__ object: every GPU that loads this
// library reserves kNoAllocScratchBytes for it until the process exits.  Host
// code must not pass the symbol itself to a kernel (on the host it is only a
// stand-in); the device address is looked up with cudaGetSymbolAddress once per
// device, on the first call made while that device is current, and kept for the
// life of the process: resetting a device (cudaDeviceReset) while the library
// is loaded is not supported.
#include <mutex>
#include <nvtx3/nvToolsExt.h>
#include <string>

#include "slora_internal.h"

namespace slora {
slora_status_t lora_delta_on_scratch(slora_pool* P, int32_t n, const int32_t* projs,
                                     const void* const* x, const int64_t* ldx, void* const* y,
                                     const int64_t* ldy, const int32_t* idx, int32_t T,
                                     cudaStream_t st, void* scratch, size_t scratch_cap);
}  // namespace slora

namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;  // 8 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_lookup_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_lookup_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" size_t slora_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" slora_status_t slora_lora_delta_noalloc(slora_pool* pool, int32_t n,
                                                   const int32_t* projs, const void* const* x,
                                                   const int64_t* ldx, void* const* y,
                                                   const int64_t* ldy, const int32_t* idx,
                                                   int32_t T, void* stream) {
  if (!pool) return SLORA_ERR_INVALID_ARG;
  nvtxRangePushA("slora_lora_delta_noalloc");
  void* scratch = nullptr;
  slora_status_t st = SLORA_ERR_CUDA;
  if (scratch_address(&scratch) == cudaSuccess)
    st = slora::lora_delta_on_scratch(pool, n, projs, x, ldx, y, ldy, idx, T,
                                      static_cast<cudaStream_t>(stream), scratch,
                                      kNoAllocScratchBytes);
  nvtxRangePop();
  return st;
}
