// fp4_fake_quant.cu -- standalone NVFP4 fake-quantisation (Model-Optimizer
// "Conv3D Implicit GEMM CUDA kernel" article, sec. 6.4 and 7.3), with the
// block sizes its call accepts (16, 32, 64, 128, 256; sec. 7.1).
//
// B200 design: the op is a pure stream over HBM (read 16 elements, write 16
// elements, ~40 ALU ops per element-block).  One thread owns one block of 16
// consecutive elements, so the block maximum is a register reduction (no
// warp shuffles, no shared memory), and each thread moves its block with
// 16-byte vector loads/stores.  A grid-stride loop over a grid sized to the
// SM count keeps every SM streaming.
#include <cstdint>
#include <cuda_runtime.h>

#include "nvfp4.cuh"
#include "q3d_internal.h"

namespace q3d {

namespace {

template <typename T, bool kVec>
struct BlockIO;

// 16 elements of a 16-bit type = two 16-byte vectors.
template <typename T>
struct BlockIO<T, true> {
  static_assert(sizeof(T) == 2, "16-bit types");
  static __device__ __forceinline__ void load(const T* p, float (&v)[16]) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
    uint4 a = __ldcs(q), b = __ldcs(q + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      T lo, hi;
      const unsigned short l16 = static_cast<unsigned short>(w[i] & 0xFFFFu);
      const unsigned short h16 = static_cast<unsigned short>(w[i] >> 16);
      memcpy(&lo, &l16, 2);
      memcpy(&hi, &h16, 2);
      v[2 * i] = DTypeOps<T>::to_f32(lo);
      v[2 * i + 1] = DTypeOps<T>::to_f32(hi);
    }
  }
  static __device__ __forceinline__ void store(T* p, const float (&v)[16]) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const T lo = DTypeOps<T>::from_f32(v[2 * i]);
      const T hi = DTypeOps<T>::from_f32(v[2 * i + 1]);
      unsigned short l16, h16;
      memcpy(&l16, &lo, 2);
      memcpy(&h16, &hi, 2);
      w[i] = static_cast<uint32_t>(l16) | (static_cast<uint32_t>(h16) << 16);
    }
    uint4* q = reinterpret_cast<uint4*>(p);
    __stcs(q, make_uint4(w[0], w[1], w[2], w[3]));
    __stcs(q + 1, make_uint4(w[4], w[5], w[6], w[7]));
  }
};

// 16 fp32 = four 16-byte vectors.
template <>
struct BlockIO<float, true> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[16]) {
    const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 a = __ldcs(q + i);
      v[4 * i] = a.x; v[4 * i + 1] = a.y; v[4 * i + 2] = a.z; v[4 * i + 3] = a.w;
    }
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[16]) {
    float4* q = reinterpret_cast<float4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) __stcs(q + i, make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]));
  }
};

// Unaligned storage: element-wise accesses.
template <typename T>
struct BlockIO<T, false> {
  static __device__ __forceinline__ void load(const T* p, float (&v)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = DTypeOps<T>::to_f32(p[i]);
  }
  static __device__ __forceinline__ void store(T* p, const float (&v)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) p[i] = DTypeOps<T>::from_f32(v[i]);
  }
};

// One thread per 16 consecutive elements; a quantisation block of 16 * G
// elements is held by G consecutive lanes (G = 1, 2, 4, 8, 16; the article's
// block sizes 16 .. 256, sec. 7.1), whose |v| maxima meet in xor shuffles
// within the lane group.  The loop is uniform per warp (a warp covers 512
// consecutive elements, a whole number of blocks), so every lane of a group
// reaches the shuffles; lanes past the end take zeros and store nothing.
template <typename T, bool kVec, int G>
__global__ void __launch_bounds__(256) fp4_fake_quant_kernel(const T* x, T* y,
                                                             const float* __restrict__ amax, int64_t nunits) {
  const Nvfp4Global gs = nvfp4_global(__ldg(amax));
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int lane = threadIdx.x & 31;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b - lane < nunits; b += stride) {
    const bool live = b < nunits;
    float v[16];
    if (live) {
      BlockIO<T, kVec>::load(x + b * 16, v);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = 0.0f;
    }
    float bmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
    if constexpr (G > 1) {
#pragma unroll
      for (int o = 1; o < G; o <<= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
    }
    float scale, inv;
    nvfp4_block_scale(bmax, gs, scale, inv);
    float o[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) nvfp4_pair(v[2 * i], v[2 * i + 1], inv, scale, o[2 * i], o[2 * i + 1]);
    if (live) BlockIO<T, kVec>::store(y + b * 16, o);
  }
}

__global__ void selftest_formats_kernel(const float* __restrict__ in, int64_t n, float* __restrict__ e2m1,
                                        float* __restrict__ e4m3) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float v = in[i];
  float q0, q1;
  // scale 1, inverse 1: the pair helper reduces to the bare E2M1 rounding
  nvfp4_pair(v, 0.0f, 1.0f, 1.0f, q0, q1);
  e2m1[i] = q0;
  e4m3[i] = e4m3_round_trip(fabsf(v));
}

__global__ void selftest_ratio_kernel(const float* __restrict__ bmax, const float* __restrict__ t, int64_t n,
                                      float* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float ti = t[i];
  out[i] = nvfp4_ratio(bmax[i], ti, __frcp_rn(ti));
}

template <typename T, bool kVec>
cudaError_t launch_fq_groups(const void* x, void* y, int64_t nunits, const float* amax, int group, int grid,
                             cudaStream_t s) {
  const T* xi = static_cast<const T*>(x);
  T* yo = static_cast<T*>(y);
  switch (group) {
    case 1: fp4_fake_quant_kernel<T, kVec, 1><<<grid, 256, 0, s>>>(xi, yo, amax, nunits); break;
    case 2: fp4_fake_quant_kernel<T, kVec, 2><<<grid, 256, 0, s>>>(xi, yo, amax, nunits); break;
    case 4: fp4_fake_quant_kernel<T, kVec, 4><<<grid, 256, 0, s>>>(xi, yo, amax, nunits); break;
    case 8: fp4_fake_quant_kernel<T, kVec, 8><<<grid, 256, 0, s>>>(xi, yo, amax, nunits); break;
    default: fp4_fake_quant_kernel<T, kVec, 16><<<grid, 256, 0, s>>>(xi, yo, amax, nunits); break;
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_fq_typed(const void* x, void* y, int64_t numel, int block, const float* amax, cudaStream_t s,
                            int sm_count) {
  const int64_t nunits = numel / 16;
  const int threads = 256;
  int64_t want = (nunits + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(sm_count) * 8;
  const int grid = static_cast<int>(want < cap ? (want < 1 ? 1 : want) : cap);
  const bool vec = (reinterpret_cast<uintptr_t>(x) % 16 == 0) && (reinterpret_cast<uintptr_t>(y) % 16 == 0);
  return vec ? launch_fq_groups<T, true>(x, y, nunits, amax, block / 16, grid, s)
             : launch_fq_groups<T, false>(x, y, nunits, amax, block / 16, grid, s);
}

}  // namespace

cudaError_t launch_fp4_fake_quant(const void* x, void* y, int dtype, int64_t numel, int block, const float* amax,
                                  cudaStream_t s, int sm_count) {
  if (numel == 0) return cudaSuccess;
  switch (dtype) {
    case 0: return launch_fq_typed<float>(x, y, numel, block, amax, s, sm_count);
    case 1: return launch_fq_typed<__half>(x, y, numel, block, amax, s, sm_count);
    default: return launch_fq_typed<__nv_bfloat16>(x, y, numel, block, amax, s, sm_count);
  }
}

cudaError_t launch_selftest_formats(const float* in, int64_t n, float* e2m1, float* e4m3, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t grid = (n + threads - 1) / threads;
  selftest_formats_kernel<<<static_cast<unsigned>(grid), threads, 0, s>>>(in, n, e2m1, e4m3);
  return cudaGetLastError();
}

cudaError_t launch_selftest_ratio(const float* bmax, const float* t, int64_t n, float* out, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t grid = (n + threads - 1) / threads;
  selftest_ratio_kernel<<<static_cast<unsigned>(grid), threads, 0, s>>>(bmax, t, n, out);
  return cudaGetLastError();
}

}  // namespace q3d
