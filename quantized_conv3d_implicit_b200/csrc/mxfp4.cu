// mxfp4.cu -- MXFP4 quantisation and fake-quantisation: E2M1 values in
// groups of 32 consecutive elements sharing one power-of-two scale 2^E,
// stored as an E8M0 byte (E + 127).
//
// Follows the CANN aclnnFlatQuantV2 page (its per-group route with
// FLOAT4_E2M1 output, steps 3 and 4):
//   dst_max == 0  E = floor(log2(group max |v|)) - 2 (E2M1's largest
//                 magnitude 6 is 1.5 * 2^2);
//   dst_max != 0  S = group max / dst_max (binary32 division); E is the
//                 exponent of S, raised by one when S is normal, below the
//                 top binade and not a power of two;
//   E is clamped to the E8M0 range [-127, 127] (a zero or subnormal maximum
//   or S gives -127); each element becomes E2M1(v * 2^-E) with round to
//   nearest, ties to even, saturating at 6, and dequantises to E2M1 * 2^E.
//
// B200 design: a pure stream over HBM, like the NVFP4 call: one thread per 16
// consecutive elements (16-byte vector loads when aligned), a group held by
// two adjacent lanes whose maxima meet in one xor shuffle; the scaling is an
// exact multiply by a power of two built from exponent bits, and the E2M1
// rounding is the hardware conversion (cvt.rn.satfinite.e2m1x2), which also
// yields the packed codes (element 2i in the low nibble).
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "nvfp4.cuh"
#include "q3d_internal.h"

namespace q3d {

namespace {

template <typename T, bool kVec>
struct Io16;
template <typename T>
struct Io16<T, true> {
  static_assert(sizeof(T) == 2, "16-bit types");
  static __device__ __forceinline__ void load(const T* p, float (&v)[16]) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
    const uint4 a = __ldcs(q), b = __ldcs(q + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      T lo, hi;
      const unsigned short l16 = static_cast<unsigned short>(w[i] & 0xFFFFu), h16 = static_cast<unsigned short>(w[i] >> 16);
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
      const T lo = DTypeOps<T>::from_f32(v[2 * i]), hi = DTypeOps<T>::from_f32(v[2 * i + 1]);
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
template <>
struct Io16<float, true> {
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
template <typename T>
struct Io16<T, false> {
  static __device__ __forceinline__ void load(const T* p, float (&v)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = DTypeOps<T>::to_f32(p[i]);
  }
  static __device__ __forceinline__ void store(T* p, const float (&v)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) p[i] = DTypeOps<T>::from_f32(v[i]);
  }
};

// One thread per 16 elements; lanes 2j, 2j+1 hold one group of 32.  The
// loop is uniform per warp (a warp spans 512 elements, 16 whole groups), so
// both lanes of a group reach the shuffle; lanes past the end take zeros and
// write nothing.
template <typename T, bool kVec>
__global__ void __launch_bounds__(256) mxfp4_kernel(const T* x, T* y, uint8_t* scales, uint8_t* codes, float dst_max,
                                                    int64_t nunits) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int lane = threadIdx.x & 31;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b - lane < nunits; b += stride) {
    const bool live = b < nunits;
    float v[16];
    if (live) {
      Io16<T, kVec>::load(x + b * 16, v);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = 0.0f;
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    const int e = mx_scale_exp(amax, dst_max);
    const float down = mx_exp2i(-e), up = mx_exp2i(e);
    uint32_t packed[2] = {0u, 0u};
    float o[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float a0 = __fmul_rn(v[2 * i], down), a1 = __fmul_rn(v[2 * i + 1], down);  // exact: powers of two
      uint32_t h2;
      uint16_t c16;
      asm("{\n\t.reg .b8 q;\n\t"
          "cvt.rn.satfinite.e2m1x2.f32 q, %2, %3;\n\t"
          "cvt.rn.f16x2.e2m1x2 %0, q;\n\t"
          "cvt.u16.u8 %1, q;\n\t}"
          : "=r"(h2), "=h"(c16)
          : "f"(a1), "f"(a0));
      packed[i >> 2] |= static_cast<uint32_t>(c16 & 0xFFu) << (8 * (i & 3));
      o[2 * i] = __fmul_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu))), up);
      o[2 * i + 1] = __fmul_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16))), up);
    }
    if (live) {
      if (y) Io16<T, kVec>::store(y + b * 16, o);
      if (codes) {
        uint8_t* c = codes + b * 8;
        if ((reinterpret_cast<uintptr_t>(c) & 7u) == 0) {
          *reinterpret_cast<uint2*>(c) = make_uint2(packed[0], packed[1]);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) c[i] = static_cast<uint8_t>(packed[i >> 2] >> (8 * (i & 3)));
        }
      }
      if (scales && (lane & 1) == 0) scales[b >> 1] = static_cast<uint8_t>(e + 127);
    }
  }
}

template <typename T>
cudaError_t launch_mx_typed(const void* x, void* y, uint8_t* scales, uint8_t* codes, float dst_max, int64_t numel,
                            cudaStream_t s, int sm_count) {
  const int64_t nunits = numel / 16;
  const int threads = 256;
  const int64_t want = (nunits + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(sm_count) * 8;
  const int grid = static_cast<int>(want < cap ? (want < 1 ? 1 : want) : cap);
  const bool vec = (reinterpret_cast<uintptr_t>(x) % 16 == 0) && (reinterpret_cast<uintptr_t>(y) % 16 == 0);
  if (vec)
    mxfp4_kernel<T, true><<<grid, threads, 0, s>>>(static_cast<const T*>(x), static_cast<T*>(y), scales, codes,
                                                   dst_max, nunits);
  else
    mxfp4_kernel<T, false><<<grid, threads, 0, s>>>(static_cast<const T*>(x), static_cast<T*>(y), scales, codes,
                                                    dst_max, nunits);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mxfp4(const void* x, void* y, uint8_t* scales, uint8_t* codes, int dtype, int64_t numel,
                         float dst_max, cudaStream_t s, int sm_count) {
  if (numel == 0) return cudaSuccess;
  switch (dtype) {
    case 0: return launch_mx_typed<float>(x, y, scales, codes, dst_max, numel, s, sm_count);
    case 1: return launch_mx_typed<__half>(x, y, scales, codes, dst_max, numel, s, sm_count);
    default: return launch_mx_typed<__nv_bfloat16>(x, y, scales, codes, dst_max, numel, s, sm_count);
  }
}

}  // namespace q3d
