// act_amax.cu -- the global amax of an activation tensor, max |x| over all
// elements, as one binary32 value on the device.
//
// The Model-Optimizer "Conv3D Implicit GEMM CUDA kernel" article feeds the
// fused quantiser a scalar act_amax: its usage example (sec. 7.2) passes
// x.abs().max(), and in the quantised inference path (sec. 8.3) the input
// quantizer supplies it.  Reading one more pass over x is HBM-bound work, so
// this kernel only streams: each thread issues up to eight 16-byte loads
// before it folds any of them (one DRAM round trip per batch; the grid is
// sized so that an input of up to 64 KB per thread block needs a single
// batch), at most four CTAs per SM, one atomic per CTA.
//
// Exactness: the maximum of |x| is one of the inputs, so no rounding is
// involved.  For a non-negative IEEE value (binary32, binary16 or bfloat16)
// the magnitude bits order like unsigned integers, so each thread keeps the
// largest magnitude bit pattern of its own format (packed 16-bit halves with
// a SIMD unsigned max), widens it to binary32 once (exact for both 16-bit
// formats), and the CTA maxima meet in an unsigned atomicMax on the binary32
// bits of the output word, which the launcher zeroes first on the same
// stream.  A NaN input has the largest magnitude pattern and comes out as a
// NaN; the quantiser's result for NaN input is unspecified anyway.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "q3d_internal.h"

namespace q3d {
namespace {

constexpr int kAmaxThreads = 512;
constexpr int kAmaxUnroll = 8;  // 16-byte loads in flight per thread

__device__ __forceinline__ uint4 ld_stream_v4(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Per-format magnitude folding: fold(acc, w) keeps, per element lane of the
// 32-bit word w, the larger magnitude bit pattern; widen() turns the
// folded word into the binary32 bits of its largest magnitude.
template <typename T>
struct Mag;
template <>
struct Mag<float> {
  static __device__ __forceinline__ uint32_t fold(uint32_t acc, uint32_t w) { return max(acc, w & 0x7FFFFFFFu); }
  static __device__ __forceinline__ uint32_t widen(uint32_t acc) { return acc; }
};
template <>
struct Mag<__nv_bfloat16> {
  static __device__ __forceinline__ uint32_t fold(uint32_t acc, uint32_t w) { return __vmaxu2(acc, w & 0x7FFF7FFFu); }
  static __device__ __forceinline__ uint32_t widen(uint32_t acc) {
    return max(acc & 0xFFFFu, acc >> 16) << 16;  // bfloat16 -> binary32 is a shift
  }
};
template <>
struct Mag<__half> {
  static __device__ __forceinline__ uint32_t fold(uint32_t acc, uint32_t w) { return __vmaxu2(acc, w & 0x7FFF7FFFu); }
  static __device__ __forceinline__ uint32_t widen(uint32_t acc) {
    const unsigned short h = static_cast<unsigned short>(max(acc & 0xFFFFu, acc >> 16));
    return __float_as_uint(__half2float(__ushort_as_half(h)));
  }
};

// Fold one element given as its raw bits in the low bits of a word.
template <typename T>
__device__ __forceinline__ uint32_t fold_scalar(uint32_t acc, const T* p) {
  if constexpr (sizeof(T) == 4) {
    return Mag<T>::fold(acc, __ldg(reinterpret_cast<const uint32_t*>(p)));
  } else {
    return Mag<T>::fold(acc, static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short*>(p))));
  }
}

// kVec: x is 16-byte aligned; n_vec 16-byte vectors are read vectorised and
// the n - n_vec * (16 / sizeof(T)) trailing elements one by one.  Otherwise
// every element is read one by one (still coalesced).
template <typename T, bool kVec>
__global__ void __launch_bounds__(kAmaxThreads) act_amax_kernel(const T* __restrict__ x, int64_t n,
                                                                unsigned int* __restrict__ amax_bits) {
  constexpr int kPer = 16 / static_cast<int>(sizeof(T));
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthr = static_cast<int64_t>(gridDim.x) * blockDim.x;
  uint32_t acc = 0;
  int64_t scalar_from = 0;
  if constexpr (kVec) {
    const int64_t n_vec = n / kPer;
    const uint4* xv = reinterpret_cast<const uint4*>(x);
    for (int64_t i = tid; i < n_vec; i += kAmaxUnroll * nthr) {
      // every load of the batch is issued before any is folded; a vector past
      // the end reads as zeros, which fold to nothing
      uint4 v[kAmaxUnroll];
#pragma unroll
      for (int u = 0; u < kAmaxUnroll; ++u) {
        const int64_t j = i + u * nthr;
        v[u] = j < n_vec ? ld_stream_v4(xv + j) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kAmaxUnroll; ++u) {
        acc = Mag<T>::fold(acc, v[u].x);
        acc = Mag<T>::fold(acc, v[u].y);
        acc = Mag<T>::fold(acc, v[u].z);
        acc = Mag<T>::fold(acc, v[u].w);
      }
    }
    scalar_from = n_vec * kPer;
  }
  for (int64_t i = scalar_from + tid; i < n; i += nthr) acc = fold_scalar<T>(acc, x + i);

  uint32_t m = Mag<T>::widen(acc);
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  __shared__ uint32_t warp_max[kAmaxThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) warp_max[warp] = m;
  __syncthreads();
  if (warp == 0) {
    m = lane < static_cast<int>(blockDim.x >> 5) ? warp_max[lane] : 0u;
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if (lane == 0 && m != 0u) atomicMax(amax_bits, m);
  }
}

template <typename T>
cudaError_t launch_amax_typed(const void* x, int64_t n, float* amax, cudaStream_t s, int sm_count) {
  unsigned int* bits = reinterpret_cast<unsigned int*>(amax);
  cudaError_t e = cudaMemsetAsync(bits, 0, sizeof(unsigned int), s);
  if (e != cudaSuccess || n == 0) return e;
  constexpr int64_t kPer = 16 / static_cast<int64_t>(sizeof(T));
  const bool vec = reinterpret_cast<uintptr_t>(x) % 16 == 0;
  // vectorised: enough threads for one batch of kAmaxUnroll vectors each;
  // element by element: one element each; at most 4 CTAs per SM either way
  const int64_t per_cta = vec ? static_cast<int64_t>(kAmaxThreads) * kAmaxUnroll : kAmaxThreads;
  const int64_t units = vec ? (n + kPer - 1) / kPer : n;
  const int64_t want = (units + per_cta - 1) / per_cta;
  const int64_t cap = static_cast<int64_t>(sm_count) * 4;
  const unsigned grid = static_cast<unsigned>(want < cap ? (want < 1 ? 1 : want) : cap);
  if (vec)
    act_amax_kernel<T, true><<<grid, kAmaxThreads, 0, s>>>(static_cast<const T*>(x), n, bits);
  else
    act_amax_kernel<T, false><<<grid, kAmaxThreads, 0, s>>>(static_cast<const T*>(x), n, bits);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_act_amax(const void* x, int dtype, int64_t n, float* amax, cudaStream_t s, int sm_count) {
  switch (dtype) {
    case 0: return launch_amax_typed<float>(x, n, amax, s, sm_count);
    case 1: return launch_amax_typed<__half>(x, n, amax, s, sm_count);
    default: return launch_amax_typed<__nv_bfloat16>(x, n, amax, s, sm_count);
  }
}

}  // namespace q3d
