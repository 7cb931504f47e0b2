// conv3d_igemm_fast.cu -- warp-specialised persistent implicit-GEMM Conv3D
// for sm_100a.
//
// GEMM view as in the Model-Optimizer "Conv3D Implicit GEMM CUDA kernel"
// article, sec. 5.1 (rows (n, od, oh, ow), columns (c, kd, kh, kw)), with the
// NVFP4 activation quantiser of sec. 6.3 fused into the A-operand producer.
//
// One CTA per SM walks output tiles of 128 positions (TH x TW rectangle of
// one (n, od) plane) x n_tile output channels.  Roles (16 warps):
//   warp 0       TMA producer: for every tile, 5-D halo boxes of x (C_slot
//                channels x KD_ext x H_ext x W_box, out-of-range coordinates
//                zero-filled, which is exactly the convolution padding) into
//                a ring of channel slots, and 128B-swizzled 64-wide K slices
//                of the BF16 weights;
//   warp 1       TMEM owner and MMA issuer: tcgen05.mma kind::f16, M=128,
//                N = n_tile (split into <= 256 wide instructions), K = 16
//                (one quantisation block), FP32 accumulators in TMEM, double
//                buffered when 2 * n_tile <= 512 columns;
//   warps 4-7    epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//                lanes 32*(w%4)..+31), bias add in FP32, rounding to the
//                output dtype, bounds-checked NCDHW stores;
//   warps 8-15   transform: thread (half h, row r) builds the 32 columns
//                [32h, 32h+32) of row r of each 64-wide A slice from the halo
//                (on-the-fly (c, kd, kh, kw) decomposition, no tables), and
//                fake-quantises each 16-column block as a register reduction
//                (the thread owns the whole block), then writes BF16 in the
//                swizzled K-major layout; rows of a warp are consecutive so
//                the 16-byte stores are bank-conflict free.
// Pipelines: halo ring (full/empty), A stages (full: 8 transform warps,
// empty: tcgen05.commit), B stages (full: TMA tx, empty: commit),
// accumulators (full: commit, empty: 4 epilogue warps).  Every wait is
// bounded and any timeout aborts all roles through a shared flag.
#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <cuda_runtime.h>

#include "nvfp4.cuh"
#include "q3d_internal.h"
#include "sm100_ptx.cuh"

namespace q3d {

namespace {

constexpr int kThreads = 512;
constexpr int kWarpProducer = 0;
constexpr int kWarpMma = 1;
constexpr int kWarpEpi0 = 4;
constexpr int kWarpXf0 = 8;
constexpr int kNumXfWarps = 8;
constexpr int kBlockM = 128;
constexpr int kBlockK = 64;
constexpr uint32_t kATileBytes = kBlockM * kBlockK * 2;
constexpr int kMaxSmem = 232448;  // 227 KB dynamic shared memory per CTA

struct FastParams {
  ConvGeom g;
  const void* bias;
  void* y;
  const float* act_amax;
  unsigned int* err;
  int quant;
  // output tiling
  int TH, TW, n_ohb, n_owb;
  int n_tile, n_ntiles, n_sub, sub_n;
  int64_t num_tiles;
  int ks;  // 64-wide K slices per tile
  // halo staging
  int align_elems;  // 16 bytes in elements
  int w_box, h_ext, kd_ext, c_slot, q_slots, chan_elems;
  uint32_t slot_bytes, slot_tx;
  int ring;
  // pipeline depths
  int sa, sb, n_acc, tmem_cols;
  uint32_t b_stage_bytes;
  // shared memory map (bytes from the 1024-aligned base)
  uint32_t off_a, off_b, off_halo, off_bar;
};

struct TileCoord {
  int n, od, oh0, ow0, nt;
};

// Tile order: output-channel tile fastest, then the frame od, then the
// spatial blocks; consecutive tiles (running concurrently on neighbouring
// SMs) share two of their three input frames and their halo columns in L2.
__device__ __forceinline__ TileCoord decode_tile(const FastParams& p, int64_t t) {
  TileCoord c;
  c.nt = static_cast<int>(t % p.n_ntiles); t /= p.n_ntiles;
  c.od = static_cast<int>(t % p.g.OD); t /= p.g.OD;
  const int owb = static_cast<int>(t % p.n_owb); t /= p.n_owb;
  const int ohb = static_cast<int>(t % p.n_ohb);
  c.n = static_cast<int>(t / p.n_ohb);
  c.oh0 = ohb * p.TH;
  c.ow0 = owb * p.TW;
  return c;
}

__device__ __forceinline__ int floor_div(int a, int b) { return (a >= 0) ? a / b : -((-a + b - 1) / b); }

// First input column covered by the halo of a tile: the leftmost tap,
// rounded down to a 16-byte boundary (the TMA start coordinate rule).
__device__ __forceinline__ int halo_w0(const FastParams& p, int ow0) {
  return floor_div(ow0 * p.g.sw - p.g.pw, p.align_elems) * p.align_elems;
}

// Wait that also gives up early when another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, unsigned int* err, unsigned int site,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0u) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kQ3dWaitTimeoutNs) {
        if (err) atomicOr(err, site);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

template <typename T>
__device__ __forceinline__ float lds_as_f32(const uint8_t* p);
template <>
__device__ __forceinline__ float lds_as_f32<float>(const uint8_t* p) { return *reinterpret_cast<const float*>(p); }
template <>
__device__ __forceinline__ float lds_as_f32<__half>(const uint8_t* p) {
  return __half2float(*reinterpret_cast<const __half*>(p));
}
template <>
__device__ __forceinline__ float lds_as_f32<__nv_bfloat16>(const uint8_t* p) {
  return __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const unsigned short*>(p)) << 16);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
    conv3d_igemm_fast_kernel(const __grid_constant__ FastParams p, const __grid_constant__ CUtensorMap tmap_x,
                             const __grid_constant__ CUtensorMap tmap_w) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);

  // barrier map
  const uint32_t bar0 = base + p.off_bar;
  const uint32_t bar_halo_full = bar0;
  const uint32_t bar_halo_empty = bar_halo_full + 8u * p.ring;
  const uint32_t bar_b_full = bar_halo_empty + 8u * p.ring;
  const uint32_t bar_b_empty = bar_b_full + 8u * p.sb;
  const uint32_t bar_a_full = bar_b_empty + 8u * p.sb;
  const uint32_t bar_a_empty = bar_a_full + 8u * p.sa;
  const uint32_t bar_acc_full = bar_a_empty + 8u * p.sa;
  const uint32_t bar_acc_empty = bar_acc_full + 16u;
  const uint32_t bar_drain = bar_acc_empty + 16u;
  const uint32_t bar_end = bar_drain + 8u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + (bar_end - base));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + (bar_end - base) + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const ConvGeom& g = p.g;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.ring; ++i) {
      mbar_init(bar_halo_full + 8u * i, 1);
      mbar_init(bar_halo_empty + 8u * i, kNumXfWarps);
    }
    for (int i = 0; i < p.sb; ++i) {
      mbar_init(bar_b_full + 8u * i, 1);
      mbar_init(bar_b_empty + 8u * i, 1);
    }
    for (int i = 0; i < p.sa; ++i) {
      mbar_init(bar_a_full + 8u * i, kNumXfWarps);
      mbar_init(bar_a_empty + 8u * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_acc_full + 8u * i, 1);
      mbar_init(bar_acc_empty + 8u * i, 4);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), static_cast<uint32_t>(p.tmem_cols));
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kWarpProducer) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t slot_ctr = 0, bst = 0;
      int64_t last_slot = -1, last_b = -1;
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        const TileCoord tc = decode_tile(p, t);
        const int w0 = halo_w0(p, tc.ow0);
        const int h0 = tc.oh0 * g.sh - g.ph;
        const int d0 = tc.od * g.sd - g.pd;
        int q_issued = 0;
        for (int s = 0; ok && s < p.ks; ++s) {
          const int k_last = min(kBlockK * s + kBlockK - 1, g.K - 1);
          const int q_need = (k_last / g.taps) / p.c_slot;
          while (q_issued <= q_need) {
            const uint32_t e = slot_ctr % p.ring, u = slot_ctr / p.ring;
            if (u > 0 && !wait_or_abort(bar_halo_empty + 8u * e, (u - 1u) & 1u, p.err, kSiteHaloEmpty, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar_halo_full + 8u * e, p.slot_tx);
            tma_load_5d(base + p.off_halo + e * p.slot_bytes, &tmap_x, bar_halo_full + 8u * e, w0, h0, d0,
                        q_issued * p.c_slot, tc.n);
            last_slot = slot_ctr;
            ++q_issued;
            ++slot_ctr;
          }
          if (!ok) break;
          const uint32_t e = bst % p.sb, u = bst / p.sb;
          if (u > 0 && !wait_or_abort(bar_b_empty + 8u * e, (u - 1u) & 1u, p.err, kSiteProducerEmpty, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar_b_full + 8u * e, p.b_stage_bytes);
          for (int i = 0; i < p.n_sub; ++i)
            tma_load_2d(base + p.off_b + e * p.b_stage_bytes + static_cast<uint32_t>(i * p.sub_n) * 128u, &tmap_w,
                        bar_b_full + 8u * e, kBlockK * s, tc.nt * p.n_tile + i * p.sub_n);
          last_b = bst;
          ++bst;
        }
      }
      if (!ok) {
        // let the last copies of each kind land before the CTA exits
        if (last_slot >= 0)
          mbar_wait(bar_halo_full + 8u * static_cast<uint32_t>(last_slot % p.ring),
                    static_cast<uint32_t>(last_slot / p.ring) & 1u, p.err, kSiteDrain);
        if (last_b >= 0)
          mbar_wait(bar_b_full + 8u * static_cast<uint32_t>(last_b % p.sb), static_cast<uint32_t>(last_b / p.sb) & 1u,
                    p.err, kSiteDrain);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16_f32(kBlockM, static_cast<uint32_t>(p.sub_n));
      uint32_t ast = 0, bst = 0, acc_ctr = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        const uint32_t eb = acc_ctr % p.n_acc, ub = acc_ctr / p.n_acc;
        if (ub > 0 && !wait_or_abort(bar_acc_empty + 8u * eb, (ub - 1u) & 1u, p.err, kSiteAccEmpty, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + eb * static_cast<uint32_t>(p.n_tile);
        for (int s = 0; s < p.ks; ++s) {
          const uint32_t ea = ast % p.sa, eB = bst % p.sb;
          if (!wait_or_abort(bar_a_full + 8u * ea, (ast / p.sa) & 1u, p.err, kSiteAStageFull, abort_flag) ||
              !wait_or_abort(bar_b_full + 8u * eB, (bst / p.sb) & 1u, p.err, kSiteTmaFull, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = umma_desc_kmajor_sw128(base + p.off_a + ea * kATileBytes);
          const uint64_t bdesc = umma_desc_kmajor_sw128(base + p.off_b + eB * p.b_stage_bytes);
#pragma unroll
          for (int j = 0; j < kBlockK / 16; ++j)
            for (int i = 0; i < p.n_sub; ++i)
              umma_bf16(d_tmem + static_cast<uint32_t>(i * p.sub_n), adesc + 2u * j,
                        bdesc + static_cast<uint64_t>(i * p.sub_n * 8) + 2u * j, idesc, (s > 0 || j > 0) ? 1u : 0u);
          umma_commit(bar_a_empty + 8u * ea);
          umma_commit(bar_b_empty + 8u * eB);
          ++ast;
          ++bst;
        }
        if (!ok) break;
        umma_commit(bar_acc_full + 8u * eb);
        ++acc_ctr;
      }
      if (!ok) {
        umma_commit(bar_drain);
        mbar_wait(bar_drain, 0, p.err, kSiteDrain);
      }
    }
  } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + 4) {
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - kWarpEpi0;
    const int r = ew * 32 + lane;
    const int S_hw = g.OH * g.OW;
    const int64_t S = static_cast<int64_t>(g.OD) * S_hw;
    T* y = static_cast<T*>(p.y);
    const T* bias = static_cast<const T*>(p.bias);
    uint32_t acc_ctr = 0;
    for (int64_t t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
      const uint32_t eb = acc_ctr % p.n_acc;
      if (!wait_or_abort(bar_acc_full + 8u * eb, (acc_ctr / p.n_acc) & 1u, p.err, kSiteAccFull, abort_flag)) break;
      tc_fence_after();
      const TileCoord tc = decode_tile(p, t);
      const int oh = tc.oh0 + r / p.TW, ow = tc.ow0 + r % p.TW;
      const bool valid = oh < g.OH && ow < g.OW;
      const int64_t ybase = (static_cast<int64_t>(tc.n) * g.Cout) * S + static_cast<int64_t>(tc.od) * S_hw +
                            static_cast<int64_t>(oh) * g.OW + ow;
      const int co0 = tc.nt * p.n_tile;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + eb * static_cast<uint32_t>(p.n_tile);
      for (int c0 = 0; c0 < p.n_tile; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(taddr + static_cast<uint32_t>(c0), v);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int co = co0 + c0 + j;
            if (co < g.Cout) {
              float f = __uint_as_float(v[j]);
              if (bias) f = __fadd_rn(f, DTypeOps<T>::to_f32(bias[co]));
              y[ybase + static_cast<int64_t>(co) * S] = DTypeOps<T>::from_f32(f);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_acc_empty + 8u * eb);
      ++acc_ctr;
    }
  } else if (warp >= kWarpXf0) {
    // ------------------------------------------------------------------ transform
    const int xw = warp - kWarpXf0;
    const int h = xw >> 2;
    const int r = (xw & 3) * 32 + lane;
    const int th = r / p.TW, tw = r % p.TW;
    const int khw = g.KH * g.KW;
    const int esz = static_cast<int>(sizeof(T));
    const int hstride = g.dh * p.w_box;                 // elements between kh taps
    const int dstride = g.dd * p.h_ext * p.w_box;       // elements between kd taps
    Nvfp4Global G{0.0f, 0.0f};
    if (p.quant) G = nvfp4_global(__ldg(p.act_amax));
    uint32_t slot_base = 0, ast = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
      const TileCoord tc = decode_tile(p, t);
      const int w0 = halo_w0(p, tc.ow0);
      const int thr_off = th * g.sh * p.w_box + tw * g.sw + (tc.ow0 * g.sw - g.pw - w0);
      int waited = -1, released = 0;
      for (int s = 0; s < p.ks; ++s) {
        const uint32_t ea = ast % p.sa, ua = ast / p.sa;
        if (ua > 0 && !wait_or_abort(bar_a_empty + 8u * ea, (ua - 1u) & 1u, p.err, kSiteMmaDone, abort_flag)) {
          ok = false;
          break;
        }
        const int k_last = min(kBlockK * s + kBlockK - 1, g.K - 1);
        const int q_need = (k_last / g.taps) / p.c_slot;
        while (waited < q_need) {
          ++waited;
          const uint32_t gs = slot_base + static_cast<uint32_t>(waited);
          if (!wait_or_abort(bar_halo_full + 8u * (gs % p.ring), (gs / p.ring) & 1u, p.err, kSiteHaloFull,
                             abort_flag)) {
            ok = false;
            break;
          }
        }
        if (!ok) break;
        uint8_t* a_tile = smem + p.off_a + ea * kATileBytes;
#pragma unroll 1
        for (int bb = 0; bb < 2; ++bb) {
          const int blk = 2 * h + bb;
          const int kb = kBlockK * s + 16 * blk;
          int c = kb / g.taps;
          int rr = kb - c * g.taps;
          int kd = rr / khw;
          rr -= kd * khw;
          int kh = rr / g.KW;
          int kw = rr - kh * g.KW;
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float val = 0.0f;
            if (kb + j < g.K) {
              const int q = c / p.c_slot;
              const uint32_t e = (slot_base + static_cast<uint32_t>(q)) % p.ring;
              const int off = (c - q * p.c_slot) * p.chan_elems + kd * dstride + kh * hstride + kw * g.dw + thr_off;
              val = lds_as_f32<T>(smem + p.off_halo + e * p.slot_bytes + off * esz);
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
          if (p.quant) {
            float bmax = 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) bmax = fmaxf(bmax, fabsf(v[j]));
            float scale, inv;
            nvfp4_block_scale(bmax, G, scale, inv);
#pragma unroll
            for (int i = 0; i < 8; ++i) nvfp4_pair(v[2 * i], v[2 * i + 1], inv, scale, v[2 * i], v[2 * i + 1]);
          }
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
          *reinterpret_cast<uint4*>(a_tile + sw128_offset(r, 2 * blk)) = make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(a_tile + sw128_offset(r, 2 * blk + 1)) = make_uint4(w[4], w[5], w[6], w[7]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_a_full + 8u * ea);
        ++ast;
        // halo slots below the first one the next slice needs are done
        const int q_keep = (s + 1 < p.ks) ? ((kBlockK * (s + 1)) / g.taps) / p.c_slot : p.q_slots;
        while (released < q_keep) {
          if (lane == 0) mbar_arrive(bar_halo_empty + 8u * ((slot_base + static_cast<uint32_t>(released)) % p.ring));
          ++released;
        }
      }
      slot_base += static_cast<uint32_t>(p.q_slots);
    }
  }

  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, static_cast<uint32_t>(p.tmem_cols));
  }
}

template <typename T>
cudaError_t launch_fast_typed(const FastParams& p, const CUtensorMap& tx, const CUtensorMap& tw, int grid,
                              size_t smem, cudaStream_t s) {
  auto kern = conv3d_igemm_fast_kernel<T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, s>>>(p, tx, tw);
  return cudaGetLastError();
}

// Q3D_KERNEL=basic|fast selects a kernel explicitly (both compute the same
// result); unset selects the specialised kernel when it applies.
int kernel_choice() {
  const char* v = getenv("Q3D_KERNEL");
  if (!v) return 1;
  if (!strcmp(v, "basic")) return 1;
  if (!strcmp(v, "fast")) return 2;
  return 1;
}

}  // namespace

cudaError_t launch_conv3d_fast(const ConvGeom& g, const ConvLaunch& L, cudaStream_t s, const char** why,
                               bool* handled) {
  *handled = false;
  if (kernel_choice() == 1) return cudaSuccess;
  const int esz = L.dtype == 0 ? 4 : 2;
  const int align = 16 / esz;
  // TMA needs 16-byte aligned base and strides for x
  if (reinterpret_cast<uintptr_t>(L.x) % 16 != 0 || (static_cast<int64_t>(g.W) * esz) % 16 != 0) return cudaSuccess;
  if (g.Cout > 512 * 64) return cudaSuccess;

  FastParams p;
  memset(&p, 0, sizeof(p));
  p.g = g;
  p.bias = L.bias; p.y = L.y; p.act_amax = L.act_amax; p.err = L.err; p.quant = L.quant;
  p.align_elems = align;

  // output channels per tile: all of Cout up to 512, else tiles of 256
  int n_ntiles = 1, n_tile = (g.Cout + 15) / 16 * 16;
  if (n_tile > 512) {
    n_ntiles = (g.Cout + 255) / 256;
    n_tile = ((g.Cout + n_ntiles - 1) / n_ntiles + 15) / 16 * 16;
  }
  const int n_sub = (n_tile + 255) / 256;
  const int sub_n = ((n_tile / n_sub) + 15) / 16 * 16;
  n_tile = sub_n * n_sub;
  p.n_tile = n_tile; p.n_ntiles = n_ntiles; p.n_sub = n_sub; p.sub_n = sub_n;
  p.n_acc = (2 * n_tile <= 512) ? 2 : 1;
  int tmem = 32;
  while (tmem < p.n_acc * n_tile) tmem <<= 1;
  p.tmem_cols = tmem;

  // spatial tile: TH x TW = 128 with the least padding waste
  const int kd_ext = (g.KD - 1) * g.dd + 1;
  double best = 1e30;
  int bTW = 0;
  for (int TW = 128; TW >= 8; TW /= 2) {
    const int TH = 128 / TW;
    const int h_ext = (TH - 1) * g.sh + (g.KH - 1) * g.dh + 1;
    const int w_ext = (TW - 1) * g.sw + (g.KW - 1) * g.dw + 1;
    const int w_box = (w_ext + align - 1 + align - 1) / align * align;  // worst-case start misalignment
    if (w_box > 256 || h_ext > 256 || kd_ext > 256) continue;
    const double waste = (double)((g.OH + TH - 1) / TH * TH) * ((g.OW + TW - 1) / TW * TW) / ((double)g.OH * g.OW);
    const double halo = (double)h_ext * w_box / 128.0;
    const double score = waste * (1.0 + 0.02 * halo);
    if (score < best - 1e-9) { best = score; bTW = TW; }
  }
  if (bTW == 0) return cudaSuccess;
  p.TW = bTW; p.TH = 128 / bTW;
  p.n_owb = (g.OW + p.TW - 1) / p.TW;
  p.n_ohb = (g.OH + p.TH - 1) / p.TH;
  p.h_ext = (p.TH - 1) * g.sh + (g.KH - 1) * g.dh + 1;
  const int w_ext = (p.TW - 1) * g.sw + (g.KW - 1) * g.dw + 1;
  p.w_box = (w_ext + 2 * (align - 1)) / align * align;
  p.kd_ext = kd_ext;
  p.chan_elems = p.kd_ext * p.h_ext * p.w_box;
  const int chan_bytes = p.chan_elems * esz;
  p.c_slot = 8192 / chan_bytes;
  if (p.c_slot < 1) p.c_slot = 1;
  if (p.c_slot > 256) p.c_slot = 256;
  if (p.c_slot > g.C) p.c_slot = g.C;
  p.q_slots = (g.C + p.c_slot - 1) / p.c_slot;
  p.slot_tx = static_cast<uint32_t>(p.c_slot) * chan_bytes;
  p.slot_bytes = (p.slot_tx + 127u) / 128u * 128u;
  p.ks = (g.K + kBlockK - 1) / kBlockK;
  p.num_tiles = static_cast<int64_t>(g.N) * g.OD * p.n_ohb * p.n_owb * n_ntiles;
  p.b_stage_bytes = static_cast<uint32_t>(n_tile) * 128u;

  // widest span of halo slots one K slice needs at once
  int span = 1;
  for (int s0 = 0; s0 < p.ks; ++s0) {
    const int qlo = ((kBlockK * s0) / g.taps) / p.c_slot;
    const int qhi = ((std::min(kBlockK * s0 + kBlockK - 1, g.K - 1)) / g.taps) / p.c_slot;
    span = std::max(span, qhi - qlo + 1);
  }
  // pipeline depths under the shared-memory budget
  int sa = 4, sb = 4, ring = std::max(span + 3, 4);
  auto total = [&](int a, int b, int r) {
    const int nbar = 2 * r + 2 * b + 2 * a + 4 + 1;
    return 1024 + a * static_cast<int>(kATileBytes) + b * static_cast<int>(p.b_stage_bytes) +
           r * static_cast<int>(p.slot_bytes) + nbar * 8 + 16;
  };
  while (total(sa, sb, ring) > kMaxSmem) {
    if (sb > 2) --sb;
    else if (ring > span + 1) --ring;
    else if (sa > 2) --sa;
    else return cudaSuccess;  // does not fit: use the general kernel
  }
  p.sa = sa; p.sb = sb; p.ring = ring;
  p.off_a = 0;
  p.off_b = p.off_a + sa * kATileBytes;
  p.off_halo = p.off_b + sb * p.b_stage_bytes;
  p.off_bar = (p.off_halo + ring * p.slot_bytes + 7u) / 8u * 8u;
  size_t smem = static_cast<size_t>(total(sa, sb, ring));
  // at most 512 / tmem_cols CTAs may share an SM, so tcgen05.alloc never waits
  const size_t max_ctas = 512 / static_cast<size_t>(p.tmem_cols);
  const size_t min_smem = 233472 / (max_ctas + 1) + 1;
  if (max_ctas < 4 && smem + 1024 < min_smem) smem = min_smem - 1024;

  EncodeTiledFn encode = get_encode_tiled();
  if (!encode) { *why = "cuTensorMapEncodeTiled unavailable"; return cudaErrorNotSupported; }
  CUtensorMap tmap_x, tmap_w;
  {
    const CUtensorMapDataType dt = L.dtype == 0 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : L.dtype == 1 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                  : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const cuuint64_t dims[5] = {(cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.D, (cuuint64_t)g.C, (cuuint64_t)g.N};
    const cuuint64_t st[4] = {(cuuint64_t)g.W * esz, (cuuint64_t)g.H * g.W * esz, (cuuint64_t)g.D * g.H * g.W * esz,
                              (cuuint64_t)g.C * g.D * g.H * g.W * esz};
    const cuuint32_t box[5] = {(cuuint32_t)p.w_box, (cuuint32_t)p.h_ext, (cuuint32_t)p.kd_ext, (cuuint32_t)p.c_slot, 1};
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    CUresult cr = encode(&tmap_x, dt, 5, const_cast<void*>(L.x), dims, st, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return cudaSuccess;  // shape the TMA unit cannot describe: general kernel
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)g.K, (cuuint64_t)g.Cout};
    const cuuint64_t st[1] = {(cuuint64_t)L.w_ld * 2u};
    const cuuint32_t box[2] = {(cuuint32_t)kBlockK, (cuuint32_t)p.sub_n};
    const cuuint32_t es[2] = {1, 1};
    CUresult cr = encode(&tmap_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(L.w_bf16), dims, st, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) { *why = "weight tensor map rejected"; return cudaErrorInvalidValue; }
  }
  const int64_t grid64 = std::min<int64_t>(p.num_tiles, L.sm_count);
  *handled = true;
  switch (L.dtype) {
    case 0: return launch_fast_typed<float>(p, tmap_x, tmap_w, static_cast<int>(grid64), smem, s);
    case 1: return launch_fast_typed<__half>(p, tmap_x, tmap_w, static_cast<int>(grid64), smem, s);
    default: return launch_fast_typed<__nv_bfloat16>(p, tmap_x, tmap_w, static_cast<int>(grid64), smem, s);
  }
}

}  // namespace q3d
