// q3d_noalloc.cu -- the fixed weight-staging area behind
// conv3d_implicit_gemm_noalloc.
//
// Some callers may not allocate device memory while a convolution is being
// enqueued: a runtime that divides the device's memory among its own pools at
// start-up and keeps its steady-state footprint fixed, or a host thread that
// must not take the allocator's locks or wait on a pool to grow.  For weights
// that cannot be read in place (dtype other than BF16, K not a multiple of 8,
// or a base address that is not 16-byte aligned) the regular entry point
// takes a stream-ordered allocation for the BF16 copy; the no-alloc entry
// point copies them into this array instead.  The array lives in its own
// translation unit, so its device memory is reserved only when this module
// is first used on a device.
#include <mutex>

#include <cuda_runtime.h>

#include "q3d_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_weights[q3d::kNoAllocStagingBytes];

constexpr int kMaxDevices = 64;
void* g_area[kMaxDevices];
std::mutex g_area_mu;

}  // namespace

namespace q3d {

cudaError_t noalloc_staging_area(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_area_mu);
  if (!g_area[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_weights);
    if (e != cudaSuccess) return e;
    g_area[dev] = p;
  }
  *out = g_area[dev];
  return cudaSuccess;
}

}  // namespace q3d
