// conv3d_igemm_basic.cu -- straightforward tcgen05 implicit-GEMM Conv3D.
//
// GEMM view (Model-Optimizer "Conv3D Implicit GEMM CUDA kernel" article,
// sec. 5.1): row m = ((n*OD + od)*OH + oh)*OW + ow, column k =
// ((c*KD + kd)*KH + kh)*KW + kw, A[m,k] = x[n, c, od*sd + kd*dd - pd, ...]
// (zero outside x), B[co,k] = w[co, c, kd, kh, kw], y[n, co, od, oh, ow] =
// sum_k A[m,k] B[co,k] + bias[co].
//
// This is the general-purpose path: any shape, stride, dilation, padding
// and alignment.  One CTA of 128 threads computes a 128 x n_tile output tile:
//   - B (BF16 weights, K-major) arrives by TMA in 128-byte-swizzled 64-wide
//     K slices;
//   - every thread builds one row of the A slice: it gathers 64 im2col
//     values of its output position straight from global memory (index math
//     on the fly, no lookup tables), fake-quantises them in blocks of 16
//     when requested (sec. 6.3; the block is a register reduction because
//     the thread owns the whole row segment), rounds to BF16 and writes the
//     swizzled layout the tensor core reads; the quantiser's other formats
//     (NVFP4 blocks of 32..256, MXFP4 groups of 32) take each block's
//     maximum in a gather pass over the block's columns before its first
//     16-column piece;
//   - one thread issues tcgen05.mma (M=128, N=n_tile, K=16) x 4 per slice
//     into an FP32 accumulator in tensor memory, two slices in flight;
//   - the epilogue reads the accumulator with tcgen05.ld, adds the bias in
//     FP32, rounds to the output dtype and stores NCDHW with bounds checks.
// The high-throughput specialised kernel lives in conv3d_igemm_fast.cu.
#include <cstdint>
#include <cuda_runtime.h>

#include "nvfp4.cuh"
#include "q3d_internal.h"
#include "sm100_ptx.cuh"

namespace q3d {

namespace {

constexpr int kBlockM = 128;
constexpr int kBlockK = 64;
constexpr int kStages = 2;
constexpr int kThreads = 128;
constexpr uint32_t kATileBytes = kBlockM * kBlockK * 2;

struct BasicParams {
  ConvGeom g;
  const void* x;
  const void* bias;
  void* y;
  const float* act_amax;
  unsigned int* err;
  int quant;
  int qfmt;        // 1: NVFP4 blocks of qblock, 2: MXFP4 groups of 32 (when quant)
  int qblock;
  float dst_max;   // MXFP4 only
  int n_tile;
  int tmem_cols;
  int num_k_stages;
};

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
    conv3d_igemm_basic_kernel(const __grid_constant__ BasicParams p, const __grid_constant__ CUtensorMap tmap_w) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t b_bytes = static_cast<uint32_t>(p.n_tile) * 128u;
  const uint32_t a_off = 0;
  const uint32_t b_off = kStages * kATileBytes;
  const uint32_t bar_off = b_off + kStages * b_bytes;
  const uint32_t bar_tma = base + bar_off;
  const uint32_t bar_mma = bar_tma + 8u * kStages;
  const uint32_t bar_acc = bar_mma + 8u * kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + bar_off + 8u * (2 * kStages + 1));

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const ConvGeom& g = p.g;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_tma + 8u * s, 1);
      mbar_init(bar_mma + 8u * s, 1);
    }
    mbar_init(bar_acc, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmap_w);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), static_cast<uint32_t>(p.tmem_cols));
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_slot;

  // this thread's output row
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kBlockM;
  const int n0 = blockIdx.y * p.n_tile;
  const int64_t m = m0 + tid;
  const bool row_ok = m < g.M;
  int nb = 0, od = 0, oh = 0, ow = 0;
  if (row_ok) {
    int64_t r = m;
    ow = static_cast<int>(r % g.OW); r /= g.OW;
    oh = static_cast<int>(r % g.OH); r /= g.OH;
    od = static_cast<int>(r % g.OD);
    nb = static_cast<int>(r / g.OD);
  }
  const int id0 = od * g.sd - g.pd, ih0 = oh * g.sh - g.ph, iw0 = ow * g.sw - g.pw;
  const T* xn = static_cast<const T*>(p.x) + static_cast<int64_t>(nb) * g.C * g.D * g.H * g.W;
  Nvfp4Global G{0.0f, 0.0f, 0.0f};
  if (p.quant && p.qfmt == 1) G = nvfp4_global(__ldg(p.act_amax));  // MXFP4 takes no global amax
  const int khw = g.KH * g.KW;
  const uint32_t idesc = umma_idesc_bf16_f32(kBlockM, static_cast<uint32_t>(p.n_tile));

  // A[m, kk] of this row (column kk of the implicit im2col matrix)
  auto im2col_at = [&](int kk) -> float {
    const int c = kk / g.taps;
    int r = kk - c * g.taps;
    const int kd = r / khw;
    r -= kd * khw;
    const int kh = r / g.KW, kw = r - (r / g.KW) * g.KW;
    const int id = id0 + kd * g.dd, ih = ih0 + kh * g.dh, iw = iw0 + kw * g.dw;
    if (static_cast<unsigned>(id) < static_cast<unsigned>(g.D) && static_cast<unsigned>(ih) < static_cast<unsigned>(g.H) &&
        static_cast<unsigned>(iw) < static_cast<unsigned>(g.W))
      return DTypeOps<T>::to_f32(xn[((static_cast<int64_t>(c) * g.D + id) * g.H + ih) * g.W + iw]);
    return 0.0f;
  };
  // scale of the current quantisation block of the other formats: NVFP4
  // (q_a, q_b) = (1/scale, scale), MXFP4 (2^-E, 2^E)
  float q_a = 1.0f, q_b = 1.0f;
  bool aborted = false;
  bool tma_wait_failed = false;
  int last_tma_stage = -1;
  for (int s = 0; s < p.num_k_stages; ++s) {
    const int st = s % kStages;
    const uint32_t use = static_cast<uint32_t>(s / kStages);
    bool fail = tma_wait_failed;
    if (s >= kStages) fail |= !mbar_wait(bar_mma + 8u * st, (use - 1u) & 1u, p.err, kSiteMmaDone);
    if (__syncthreads_or(fail)) { aborted = true; break; }

    if (tid == 0) {
      mbar_arrive_expect_tx(bar_tma + 8u * st, b_bytes);
      tma_load_2d(base + b_off + st * b_bytes, &tmap_w, bar_tma + 8u * st, s * kBlockK, n0);
      last_tma_stage = s;
    }

    // A slice: columns k0 .. k0+63 of row m
    uint8_t* a_tile = smem + a_off + st * kATileBytes;
    const int k0 = s * kBlockK;
    int c = k0 / g.taps;
    int r = k0 - c * g.taps;
    int kd = r / khw;
    r -= kd * khw;
    int kh = r / g.KW;
    int kw = r - kh * g.KW;
#pragma unroll 1
    for (int blk = 0; blk < kBlockK / 16; ++blk) {
      float v[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int k = k0 + blk * 16 + j;
        float val = 0.0f;
        if (row_ok && k < g.K) {
          const int id = id0 + kd * g.dd, ih = ih0 + kh * g.dh, iw = iw0 + kw * g.dw;
          if (static_cast<unsigned>(id) < static_cast<unsigned>(g.D) &&
              static_cast<unsigned>(ih) < static_cast<unsigned>(g.H) &&
              static_cast<unsigned>(iw) < static_cast<unsigned>(g.W))
            val = DTypeOps<T>::to_f32(xn[((static_cast<int64_t>(c) * g.D + id) * g.H + ih) * g.W + iw]);
        }
        v[j] = val;
        if (++kw == g.KW) {
          kw = 0;
          if (++kh == g.KH) {
            kh = 0;
            if (++kd == g.KD) { kd = 0; ++c; }
          }
        }
      }
      if (p.quant && p.qfmt == 1 && p.qblock == 16) {
        float bmax = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j) bmax = fmaxf(bmax, fabsf(v[j]));
        float scale, inv;
        nvfp4_block_scale(bmax, G, scale, inv);
#pragma unroll
        for (int i = 0; i < 8; ++i) nvfp4_pair(v[2 * i], v[2 * i + 1], inv, scale, v[2 * i], v[2 * i + 1]);
      } else if (p.quant) {
        // a quantisation block of qblock columns (a multiple of 16) starts
        // here: its |v| maximum over all its columns (a short last block as
        // if zero-filled) sets the scale its 16-column pieces share
        const int kb = k0 + blk * 16;
        if (kb % p.qblock == 0) {
          float bm = 0.0f;
          const int ke = min(kb + p.qblock, g.K);
          for (int kk = kb; kk < ke && row_ok; ++kk) bm = fmaxf(bm, fabsf(im2col_at(kk)));
          if (p.qfmt == 2) {
            const int e = mx_scale_exp(bm, p.dst_max);
            q_a = mx_exp2i(-e);
            q_b = mx_exp2i(e);
          } else {
            nvfp4_block_scale(bm, G, q_b, q_a);
          }
        }
        if (p.qfmt == 2) {
#pragma unroll
          for (int i = 0; i < 8; ++i) mx_pair(v[2 * i], v[2 * i + 1], q_a, q_b, v[2 * i], v[2 * i + 1]);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) nvfp4_pair(v[2 * i], v[2 * i + 1], q_a, q_b, v[2 * i], v[2 * i + 1]);
        }
      }
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
      *reinterpret_cast<uint4*>(a_tile + sw128_offset(tid, 2 * blk)) = make_uint4(w[0], w[1], w[2], w[3]);
      *reinterpret_cast<uint4*>(a_tile + sw128_offset(tid, 2 * blk + 1)) = make_uint4(w[4], w[5], w[6], w[7]);
    }
    fence_proxy_async_smem();
    __syncthreads();

    if (tid == 0) {
      if (!mbar_wait(bar_tma + 8u * st, use & 1u, p.err, kSiteTmaFull)) {
        tma_wait_failed = true;
      } else {
        last_tma_stage = -1;
        tc_fence_after();
        const uint64_t adesc = umma_desc_kmajor_sw128(base + a_off + st * kATileBytes);
        const uint64_t bdesc = umma_desc_kmajor_sw128(base + b_off + st * b_bytes);
#pragma unroll
        for (int j = 0; j < kBlockK / 16; ++j)
          umma_bf16(tmem_acc, adesc + 2u * j, bdesc + 2u * j, idesc, (s > 0 || j > 0) ? 1u : 0u);
        umma_commit(bar_mma + 8u * st);
      }
    }
  }
  if (!aborted && tid == 0 && tma_wait_failed) aborted = true;  // only thread 0 knows; handled below

  // accumulator complete (also drains every MMA issued so far)
  if (tid == 0) umma_commit(bar_acc);
  bool acc_ok = mbar_wait(bar_acc, 0, p.err, kSiteAccFull);
  if (tid == 0 && last_tma_stage >= 0) {
    // a TMA load whose wait gave up may still be in flight: wait once more
    const int st = last_tma_stage % kStages;
    mbar_wait(bar_tma + 8u * st, static_cast<uint32_t>(last_tma_stage / kStages) & 1u, p.err, kSiteDrain);
  }
  const bool skip = __syncthreads_or(aborted || !acc_ok || tma_wait_failed);
  tc_fence_after();

  if (!skip) {
    const int64_t S = static_cast<int64_t>(g.OD) * g.OH * g.OW;
    int64_t ybase = 0;
    if (row_ok) {
      const int64_t ni = m / S;
      ybase = ni * g.Cout * S + (m - ni * S);
    }
    T* y = static_cast<T*>(p.y);
    const T* bias = static_cast<const T*>(p.bias);
    for (int c0 = 0; c0 < p.n_tile; c0 += 16) {
      uint32_t r[16];
      tmem_ld16(tmem_acc + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(c0), r);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int co = n0 + c0 + j;
        if (row_ok && co < g.Cout) {
          float v = __uint_as_float(r[j]);
          if (bias) v = __fadd_rn(v, DTypeOps<T>::to_f32(bias[co]));
          y[ybase + static_cast<int64_t>(co) * S] = DTypeOps<T>::from_f32(v);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem_acc, static_cast<uint32_t>(p.tmem_cols));
}

template <typename T>
__global__ void stage_weights_kernel(const T* __restrict__ w, int32_t Cout, int32_t K, int64_t ld,
                                     __nv_bfloat16* __restrict__ out) {
  const int64_t total = static_cast<int64_t>(Cout) * ld;
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += step) {
    const int64_t r = i / ld;
    const int64_t c = i - r * ld;
    out[i] = c < K ? __float2bfloat16_rn(DTypeOps<T>::to_f32(w[r * K + c])) : __float2bfloat16_rn(0.0f);
  }
}

template <typename T>
cudaError_t launch_basic_typed(const BasicParams& p, const CUtensorMap& tmap, dim3 grid, size_t smem,
                               cudaStream_t s) {
  auto kern = conv3d_igemm_basic_kernel<T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, s>>>(p, tmap);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_stage_weights(const void* w, int dtype, int32_t Cout, int32_t K, int64_t ld, void* w_bf16,
                                 cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(Cout) * ld;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 4096) blocks = 4096;
  auto* out = static_cast<__nv_bfloat16*>(w_bf16);
  switch (dtype) {
    case 0: stage_weights_kernel<float><<<static_cast<unsigned>(blocks), threads, 0, s>>>(
                static_cast<const float*>(w), Cout, K, ld, out); break;
    case 1: stage_weights_kernel<__half><<<static_cast<unsigned>(blocks), threads, 0, s>>>(
                static_cast<const __half*>(w), Cout, K, ld, out); break;
    default: stage_weights_kernel<__nv_bfloat16><<<static_cast<unsigned>(blocks), threads, 0, s>>>(
                static_cast<const __nv_bfloat16*>(w), Cout, K, ld, out); break;
  }
  return cudaGetLastError();
}

// Split Cout into the fewest tiles of at most 256 columns (the largest
// M=128 tcgen05 N), each a multiple of 16.
static void pick_n_tiles(int cout, int& n_tile, int& n_tiles) {
  n_tiles = (cout + 255) / 256;
  const int per = (cout + n_tiles - 1) / n_tiles;
  n_tile = (per + 15) / 16 * 16;
}

cudaError_t launch_conv3d_basic(const ConvGeom& g, const ConvLaunch& L, cudaStream_t s, const char** why) {
  int n_tile, n_tiles;
  pick_n_tiles(g.Cout, n_tile, n_tiles);
  int tmem_cols = 32;
  while (tmem_cols < n_tile) tmem_cols <<= 1;
  const int64_t m_tiles = (g.M + kBlockM - 1) / kBlockM;
  if (m_tiles > 0x7FFFFFFF) { *why = "too many output rows"; return cudaErrorInvalidValue; }

  EncodeTiledFn encode = get_encode_tiled();
  if (!encode) { *why = "cuTensorMapEncodeTiled unavailable"; return cudaErrorNotSupported; }
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(g.K), static_cast<cuuint64_t>(g.Cout)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(L.w_ld) * 2u};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBlockK), static_cast<cuuint32_t>(n_tile)};
  const cuuint32_t es[2] = {1, 1};
  CUresult cr = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(L.w_bf16), dims, strides, box,
                       es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) { *why = "weight tensor map rejected"; return cudaErrorInvalidValue; }

  BasicParams p;
  p.g = g;
  p.x = L.x; p.bias = L.bias; p.y = L.y; p.act_amax = L.act_amax; p.err = L.err;
  p.quant = L.quant; p.qfmt = L.qfmt; p.qblock = L.qblock; p.dst_max = L.dst_max;
  p.n_tile = n_tile; p.tmem_cols = tmem_cols;
  p.num_k_stages = (g.K + kBlockK - 1) / kBlockK;
  size_t smem = 1024 + kStages * kATileBytes + kStages * static_cast<size_t>(n_tile) * 128 + 128;
  // Keep (CTAs per SM) x tmem_cols <= 512 so no CTA ever waits in
  // tcgen05.alloc: request enough shared memory that at most 512/tmem_cols
  // CTAs fit in the SM's 228 KB (1 KB of which is reserved per CTA).
  const size_t max_ctas = 512 / static_cast<size_t>(tmem_cols);
  const size_t min_smem = 233472 / (max_ctas + 1) + 1;
  if (max_ctas < 16 && smem + 1024 < min_smem) smem = min_smem - 1024;
  const dim3 grid(static_cast<unsigned>(m_tiles), static_cast<unsigned>(n_tiles));
  switch (L.dtype) {
    case 0: return launch_basic_typed<float>(p, tmap, grid, smem, s);
    case 1: return launch_basic_typed<__half>(p, tmap, grid, smem, s);
    default: return launch_basic_typed<__nv_bfloat16>(p, tmap, grid, smem, s);
  }
}

}  // namespace q3d
