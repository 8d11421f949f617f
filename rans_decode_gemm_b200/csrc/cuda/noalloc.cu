// noalloc.cu -- device-resident scratch for the allocation-free fused GEMM
// entry point (ans_gemm_noalloc).
//
// The fused GEMM needs scratch memory (split-K counters and partial sums, and
// the staged copy of X).  ans_gemm takes it from the caller; ans_gemm_noalloc
// takes it from this file-scope array instead, so that callers which cannot
// call cudaMalloc can still run the kernel.  Every GPU that loads the library
// holds the array until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.h"

namespace ansdev {

// Fixed maximum of the allocation-free path's scratch (see kNoAllocScratchBytes).
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_mutex;
void* g_ptr[64];  // device address of g_noalloc_scratch, per device ordinal
}  // namespace

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device with cudaGetSymbolAddress (with that device current).
cudaError_t noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_ptr[dev] = p;
  }
  *ptr = g_ptr[dev];
  return cudaSuccess;
}

}  // namespace ansdev
