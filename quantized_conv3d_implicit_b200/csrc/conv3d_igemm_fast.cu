// conv3d_igemm_fast.cu -- warp-specialised persistent implicit-GEMM Conv3D
// for sm_100a.
//
// GEMM view as in the Model-Optimizer "Conv3D Implicit GEMM CUDA kernel"
// article, sec. 5.1 (rows (n, od, oh, ow), columns (c, kd, kh, kw)), with the
// NVFP4 activation quantiser of sec. 6.3 fused into the A-operand producer.
//
// One CTA per SM walks output tiles.  A tile is n_mt M-subtiles of 128
// output positions (each a TH x TW rectangle of one (n, od) plane, stacked
// along oh) times n_tile output channels.  Every 64-wide K slice of the BF16
// weights is loaded once per tile and feeds all n_mt subtiles, so the weight
// traffic per tensor-core cycle shrinks by n_mt; the accumulators of the
// subtiles (n_mt * n_tile <= 512 FP32 columns) live in tensor memory.
//
// Roles (16 warps):
//   warp 0     weight producer: TMA of 128B-swizzled K-major weight slices;
//   warp 1     TMEM owner and MMA issuer: tcgen05.mma kind::f16, M = 128,
//              N = n_tile in <= 256-wide instructions, K = 16 (one
//              quantisation block), per subtile;
//   warp 2     halo producer: 5-D TMA boxes of x (C_slot channels x KD_ext x
//              H_ext x W_box; out-of-range coordinates are zero-filled, which
//              is exactly the convolution padding) into a ring of slots;
//   warps 4-7  epilogue: tcgen05.ld (warp w reads TMEM lanes 32*(w%4)..+31),
//              bias in FP32, rounding to the output dtype, bounds-checked
//              NCDHW stores; each (subtile, N-part) accumulator is handed
//              back as soon as it is drained, so the next tile's MMAs start
//              while the rest is still being written;
//   warps 8-15 transform: a thread owns 8 consecutive output rows and one
//              16-column quantisation block.  It walks the block's taps
//              (c, kd, kh, kw) incrementally (no divisions, no tables),
//              reads the 8 rows of each tap with 32-bit shared loads and a
//              byte permute, takes the block maximum of each row as a packed
//              register reduction, derives the E4M3 scale with an IEEE
//              division and a per-CTA table of
//              (scale, 1/scale) per E4M3 code, and writes BF16 in the
//              MN-major 128B-swizzled layout (one conflict-free 16-byte store
//              per tap).
// All waits are bounded; a timeout in any role aborts all roles.
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
constexpr int kWarpB = 0;
constexpr int kWarpMma = 1;
constexpr int kWarpHalo = 2;
constexpr int kWarpEpi0 = 4;
constexpr int kWarpXf0 = 8;
constexpr int kNumXfWarps = 8;
constexpr int kBlockK = 64;
constexpr uint32_t kASubBytes = 128u * kBlockK * 2u;  // one 128-row subtile of one K slice
constexpr int kMaxSmem = 232448;                      // 227 KB dynamic shared memory per CTA
constexpr int kMaxAcc = 8;

struct FastParams {
  ConvGeom g;
  const void* bias;
  void* y;
  const float* act_amax;
  unsigned int* err;
  int quant;
  // tiling
  int TH, TW, n_mt;       // subtile = TH x TW = 128 positions; a tile stacks n_mt subtiles along oh
  int n_ohb, n_owb;
  int n_tile, n_ntiles, n_sub, sub_n;
  int64_t num_tiles;
  int ks;                 // K slices per tile
  // halo staging
  int align;              // 16 bytes in elements
  int w_box, h_ext, kd_ext, c_slot, q_slots, chan_elems;
  uint32_t slot_bytes, slot_tx;
  int ring;
  // pipelines
  int sa, sb, groups;     // A stages, B stages, transform groups working on separate slices
  uint32_t a_stage_bytes, b_stage_bytes;
  int tmem_cols;
  int vec;                // 1: unit W stride and 16-bit input -> vectorised halo reads
  uint32_t off_a, off_b, off_halo, off_tab, off_bar;
};

struct TileCoord {
  int n, od, oh0, ow0, nt;
};

// Output-channel tile fastest, then the frame od, then the spatial blocks:
// tiles running concurrently share two of their three input frames in L2.
__device__ __forceinline__ TileCoord decode_tile(const FastParams& p, int64_t t) {
  TileCoord c;
  c.nt = static_cast<int>(t % p.n_ntiles); t /= p.n_ntiles;
  c.od = static_cast<int>(t % p.g.OD); t /= p.g.OD;
  const int owb = static_cast<int>(t % p.n_owb); t /= p.n_owb;
  const int ohb = static_cast<int>(t % p.n_ohb);
  c.n = static_cast<int>(t / p.n_ohb);
  c.oh0 = ohb * p.TH * p.n_mt;
  c.ow0 = owb * p.TW;
  return c;
}

__device__ __forceinline__ int floor_div(int a, int b) { return (a >= 0) ? a / b : -((-a + b - 1) / b); }

// First input column of a tile's halo: the leftmost tap rounded down to a
// 16-byte boundary (the TMA start-coordinate rule).
__device__ __forceinline__ int halo_w0(const FastParams& p, int ow0) {
  return floor_div(ow0 * p.g.sw - p.g.pw, p.align) * p.align;
}

// Lowest / highest halo slot holding a column of K slice s.
__device__ __forceinline__ int slot_lo(const FastParams& p, int s) { return ((kBlockK * s) / p.g.taps) / p.c_slot; }
__device__ __forceinline__ int slot_hi(const FastParams& p, int s) {
  return (min(kBlockK * s + kBlockK - 1, p.g.K - 1) / p.g.taps) / p.c_slot;
}

__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, unsigned int* err, unsigned int site,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, kQ3dSleepHintNs)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kQ3dWaitTimeoutNs) {
      if (err) atomicOr(err, site);
      *abort_flag = 1;
      return false;
    }
  }
}

// Incremental walk over the K columns (c, kd, kh, kw) of one thread's
// quantisation block, tracking the element offset of the tap inside the halo
// slot that holds channel c and the byte address of that slot.
struct TapWalker {
  int kw, kh, kd, cs;       // tap and channel-within-slot
  int q;                    // slot index within the tile
  int u;                    // element offset of the tap inside its slot (without the thread's own offset)
  uint32_t slot_addr;       // shared address of slot q

  __device__ __forceinline__ void init(const FastParams& p, int k, uint32_t halo_base, uint32_t slot_base) {
    const ConvGeom& g = p.g;
    const int c = k / g.taps;
    int r = k - c * g.taps;
    const int khw = g.KH * g.KW;
    kd = r / khw;
    r -= kd * khw;
    kh = r / g.KW;
    kw = r - kh * g.KW;
    q = c / p.c_slot;
    cs = c - q * p.c_slot;
    u = cs * p.chan_elems + kd * g.dd * p.h_ext * p.w_box + kh * g.dh * p.w_box + kw * g.dw;
    slot_addr = halo_base + ((slot_base + static_cast<uint32_t>(q)) % static_cast<uint32_t>(p.ring)) * p.slot_bytes;
  }

  __device__ __forceinline__ void step(const FastParams& p, uint32_t halo_base, uint32_t slot_base) {
    const ConvGeom& g = p.g;
    u += g.dw;
    if (++kw == g.KW) {
      kw = 0;
      u += g.dh * p.w_box - g.KW * g.dw;
      if (++kh == g.KH) {
        kh = 0;
        u += g.dd * p.h_ext * p.w_box - g.KH * g.dh * p.w_box;
        if (++kd == g.KD) {
          kd = 0;
          u += p.chan_elems - g.KD * g.dd * p.h_ext * p.w_box;
          if (++cs == p.c_slot) {
            cs = 0;
            u = 0;
            ++q;
            slot_addr = halo_base + ((slot_base + static_cast<uint32_t>(q)) % static_cast<uint32_t>(p.ring)) *
                                        p.slot_bytes;
          }
        }
      }
    }
  }
};

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ uint32_t max_abs_x2_bf16(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t max_abs_x2_f16(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

template <typename T>
struct Pair16;
template <>
struct Pair16<__nv_bfloat16> {
  static __device__ __forceinline__ float lo(uint32_t w) { return __uint_as_float(w << 16); }
  static __device__ __forceinline__ float hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
  static __device__ __forceinline__ uint32_t maxabs(uint32_t a, uint32_t b) { return max_abs_x2_bf16(a, b); }
  static __device__ __forceinline__ float abs_lo(uint32_t w) { return __uint_as_float((w << 16) & 0x7FFFFFFFu); }
  static __device__ __forceinline__ float abs_hi(uint32_t w) { return __uint_as_float(w & 0x7FFF0000u); }
  static __device__ __forceinline__ uint32_t to_bf16x2(uint32_t w) { return w; }
};
template <>
struct Pair16<__half> {
  static __device__ __forceinline__ float lo(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xFFFFu)));
  }
  static __device__ __forceinline__ float hi(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
  }
  static __device__ __forceinline__ uint32_t maxabs(uint32_t a, uint32_t b) { return max_abs_x2_f16(a, b); }
  static __device__ __forceinline__ float abs_lo(uint32_t w) { return fabsf(lo(w)); }
  static __device__ __forceinline__ float abs_hi(uint32_t w) { return fabsf(hi(w)); }
  static __device__ __forceinline__ uint32_t to_bf16x2(uint32_t w) { return pack_bf16x2(lo(w), hi(w)); }
};

// Fake-quantise a pair of values from two different rows (own scales).
__device__ __forceinline__ uint32_t quant_pair_bf16x2(float v0, float v1, float inv0, float inv1, float s0, float s1) {
  const float a0 = __fmul_rn(v0, inv0);
  const float a1 = __fmul_rn(v1, inv1);
  uint32_t h2;
  asm("{\n\t.reg .b8 q;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q, %1, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, q;\n\t}"
      : "=r"(h2)
      : "f"(a1), "f"(a0));
  const float q0 = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
  const float q1 = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
  return pack_bf16x2(__fmul_rn(q0, s0), __fmul_rn(q1, s1));
}

// Scales of two rows from their block maxima: the correctly rounded
// bmax / (6 g) clamped to 448, E4M3 rounding of both rows in one conversion,
// then (scale, 1/scale) from the per-CTA table indexed by the E4M3 code.
__device__ __forceinline__ void row_scales(float bmax0, float bmax1, const Nvfp4Global& G, uint32_t tab,
                                           float& s0, float& i0, float& s1, float& i1) {
  const float r0 = nvfp4_ratio(bmax0, G.t, G.rt);
  const float r1 = nvfp4_ratio(bmax1, G.t, G.rt);
  uint16_t codes;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(codes) : "f"(r1), "f"(r0));
  float2 e0, e1;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(e0.x), "=f"(e0.y) : "r"(tab + (codes & 0x7Fu) * 8u));
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(e1.x), "=f"(e1.y) : "r"(tab + ((codes >> 8) & 0x7Fu) * 8u));
  s0 = e0.x; i0 = e0.y;
  s1 = e1.x; i1 = e1.y;
}

// MN-major swizzled position of the 16-byte chunk holding 8 rows (chunk
// index rg8 within the subtile) of column kk of a subtile's K slice: atom
// (kk/8, rg8/8) of 1 KB, K-row kk%8, chunk rg8%8 stored at (rg8 ^ kk) % 8.
__device__ __forceinline__ uint32_t a_chunk_offset(int rg8, int kk) {
  const int kr = kk & 7;
  return static_cast<uint32_t>(((kk >> 3) * 2 + (rg8 >> 3)) * 1024 + kr * 128 + (((rg8 & 7) ^ kr) << 4));
}

__device__ __forceinline__ void lds128(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "r"(addr));
}
__device__ __forceinline__ void lds64(uint32_t addr, uint32_t& a, uint32_t& b) {
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(a), "=r"(b) : "r"(addr));
}
__device__ __forceinline__ void sts64(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}

// Read P consecutive 16-bit elements starting f elements (0 <= f < P) past a
// (P*2)-byte aligned shared address, as P/2 packed words.  f is the same for
// every lane of the warp, so the case split does not diverge.
template <int P>
__device__ __forceinline__ void load_rows(uint32_t addr, int f, uint32_t (&out)[P / 2]);

template <>
__device__ __forceinline__ void load_rows<8>(uint32_t addr, int f, uint32_t (&out)[4]) {
  uint32_t w[8];
  lds128(addr, w[0], w[1], w[2], w[3]);
  if (f == 0) {
    out[0] = w[0]; out[1] = w[1]; out[2] = w[2]; out[3] = w[3];
    return;
  }
  lds128(addr + 16, w[4], w[5], w[6], w[7]);
  const uint32_t sel = (f & 1) ? 0x5432u : 0x3210u;
  switch (f >> 1) {
    case 0:
#pragma unroll
      for (int j = 0; j < 4; ++j) out[j] = __byte_perm(w[j], w[j + 1], sel);
      break;
    case 1:
#pragma unroll
      for (int j = 0; j < 4; ++j) out[j] = __byte_perm(w[j + 1], w[j + 2], sel);
      break;
    case 2:
#pragma unroll
      for (int j = 0; j < 4; ++j) out[j] = __byte_perm(w[j + 2], w[j + 3], sel);
      break;
    default:
#pragma unroll
      for (int j = 0; j < 4; ++j) out[j] = __byte_perm(w[j + 3], w[j + 4], sel);
      break;
  }
}

template <>
__device__ __forceinline__ void load_rows<4>(uint32_t addr, int f, uint32_t (&out)[2]) {
  uint32_t w[4];
  lds64(addr, w[0], w[1]);
  if (f == 0) {
    out[0] = w[0]; out[1] = w[1];
    return;
  }
  lds64(addr + 8, w[2], w[3]);
  const uint32_t sel = (f & 1) ? 0x5432u : 0x3210u;
  if (f >> 1) {
    out[0] = __byte_perm(w[1], w[2], sel);
    out[1] = __byte_perm(w[2], w[3], sel);
  } else {
    out[0] = __byte_perm(w[0], w[1], sel);
    out[1] = __byte_perm(w[1], w[2], sel);
  }
}

// Store P rows (P/2 packed words) of column kk: a whole 16-byte chunk for
// P = 8, half of one for P = 4 (rg = row group of P rows).
template <int P>
__device__ __forceinline__ void store_rows(uint32_t a_sub, int rg, int kk, const uint32_t (&w)[P / 2]) {
  if constexpr (P == 8) {
    sts128(a_sub + a_chunk_offset(rg, kk), w[0], w[1], w[2], w[3]);
  } else {
    sts64(a_sub + a_chunk_offset(rg >> 1, kk) + 8u * static_cast<uint32_t>(rg & 1), w[0], w[1]);
  }
}

// ---------------------------------------------------------------------------
// transform: one task = P rows (row group rg of one subtile) x 16 columns
// ---------------------------------------------------------------------------
template <typename T, int P>
__device__ __forceinline__ void transform_task_vec(const FastParams& p, uint32_t a_sub, int rg, int kb,
                                                  uint32_t thr_addr, int delta, uint32_t halo_base,
                                                  uint32_t slot_base, const Nvfp4Global& G, uint32_t tab) {
  constexpr int NW = P / 2;
  uint32_t d[16][NW];
  TapWalker wk;
  wk.init(p, kb, halo_base, slot_base);
#pragma unroll
  for (int kk = 0; kk < 16; ++kk) {
    if (kb + kk < p.g.K) {
      const int e = wk.u + delta;           // warp-uniform element offset
      const int f = e & (P - 1);
      uint32_t out[NW];
      load_rows<P>(wk.slot_addr + thr_addr + static_cast<uint32_t>(e - f) * 2u, f, out);
#pragma unroll
      for (int j = 0; j < NW; ++j) d[kk][j] = out[j];
    } else {
#pragma unroll
      for (int j = 0; j < NW; ++j) d[kk][j] = 0u;
    }
    if (kk < 15) wk.step(p, halo_base, slot_base);
  }
  const int kl = kb & (kBlockK - 1);
  if (p.quant) {
    uint32_t mx[NW];
#pragma unroll
    for (int j = 0; j < NW; ++j) {
      mx[j] = Pair16<T>::maxabs(d[0][j], d[1][j]);
#pragma unroll
      for (int kk = 2; kk < 16; ++kk) mx[j] = Pair16<T>::maxabs(mx[j], d[kk][j]);
    }
    float sc[P], iv[P];
#pragma unroll
    for (int j = 0; j < NW; ++j)
      row_scales(Pair16<T>::abs_lo(mx[j]), Pair16<T>::abs_hi(mx[j]), G, tab, sc[2 * j], iv[2 * j], sc[2 * j + 1],
                 iv[2 * j + 1]);
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      uint32_t w[NW];
#pragma unroll
      for (int j = 0; j < NW; ++j)
        w[j] = quant_pair_bf16x2(Pair16<T>::lo(d[kk][j]), Pair16<T>::hi(d[kk][j]), iv[2 * j], iv[2 * j + 1],
                                 sc[2 * j], sc[2 * j + 1]);
      store_rows<P>(a_sub, rg, kl + kk, w);
    }
  } else {
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      uint32_t w[NW];
#pragma unroll
      for (int j = 0; j < NW; ++j) w[j] = Pair16<T>::to_bf16x2(d[kk][j]);
      store_rows<P>(a_sub, rg, kl + kk, w);
    }
  }
}

template <typename T>
__device__ __forceinline__ float lds_elem(uint32_t addr);
template <>
__device__ __forceinline__ float lds_elem<float>(uint32_t addr) { return __uint_as_float(lds32(addr)); }
template <>
__device__ __forceinline__ float lds_elem<__half>(uint32_t addr) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(lds16(addr))));
}
template <>
__device__ __forceinline__ float lds_elem<__nv_bfloat16>(uint32_t addr) { return __uint_as_float(lds16(addr) << 16); }

// General path (any W stride, any dtype): element loads, two passes (block
// maxima, then quantisation) so only one column is held at a time.
template <typename T, int P>
__device__ __forceinline__ void transform_task_gen(const FastParams& p, uint32_t a_sub, int rg, int kb,
                                                  const int (&roff)[8], uint32_t halo_base, uint32_t slot_base,
                                                  const Nvfp4Global& G, uint32_t tab) {
  constexpr uint32_t esz = sizeof(T);
  constexpr int NW = P / 2;
  float sc[P], iv[P];
  if (p.quant) {
    float bm[P];
#pragma unroll
    for (int r = 0; r < P; ++r) bm[r] = 0.0f;
    TapWalker wk;
    wk.init(p, kb, halo_base, slot_base);
#pragma unroll 1
    for (int kk = 0; kk < 16; ++kk) {
      if (kb + kk < p.g.K) {
#pragma unroll
        for (int r = 0; r < P; ++r)
          bm[r] = fmaxf(bm[r], fabsf(lds_elem<T>(wk.slot_addr + static_cast<uint32_t>(wk.u + roff[r]) * esz)));
      }
      if (kk < 15) wk.step(p, halo_base, slot_base);
    }
#pragma unroll
    for (int j = 0; j < NW; ++j)
      row_scales(bm[2 * j], bm[2 * j + 1], G, tab, sc[2 * j], iv[2 * j], sc[2 * j + 1], iv[2 * j + 1]);
  }
  TapWalker wk;
  wk.init(p, kb, halo_base, slot_base);
  const int kl = kb & (kBlockK - 1);
#pragma unroll 1
  for (int kk = 0; kk < 16; ++kk) {
    float v[P];
#pragma unroll
    for (int r = 0; r < P; ++r)
      v[r] = (kb + kk < p.g.K) ? lds_elem<T>(wk.slot_addr + static_cast<uint32_t>(wk.u + roff[r]) * esz) : 0.0f;
    uint32_t w[NW];
#pragma unroll
    for (int j = 0; j < NW; ++j)
      w[j] = p.quant ? quant_pair_bf16x2(v[2 * j], v[2 * j + 1], iv[2 * j], iv[2 * j + 1], sc[2 * j], sc[2 * j + 1])
                     : pack_bf16x2(v[2 * j], v[2 * j + 1]);
    store_rows<P>(a_sub, rg, kl + kk, w);
    if (kk < 15) wk.step(p, halo_base, slot_base);
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
    conv3d_igemm_fast_kernel(const __grid_constant__ FastParams p, const __grid_constant__ CUtensorMap tmap_x,
                             const __grid_constant__ CUtensorMap tmap_w) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);

  const uint32_t bar_halo_full = base + p.off_bar;
  const uint32_t bar_halo_empty = bar_halo_full + 8u * p.ring;
  const uint32_t bar_b_full = bar_halo_empty + 8u * p.ring;
  const uint32_t bar_b_empty = bar_b_full + 8u * p.sb;
  const uint32_t bar_a_full = bar_b_empty + 8u * p.sb;
  const uint32_t bar_a_empty = bar_a_full + 8u * p.sa;
  const uint32_t bar_acc_full = bar_a_empty + 8u * p.sa;
  const uint32_t bar_acc_empty = bar_acc_full + 8u * kMaxAcc;
  const uint32_t bar_drain = bar_acc_empty + 8u * kMaxAcc;
  const uint32_t bar_end = bar_drain + 8u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + (bar_end - base));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + (bar_end - base) + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const ConvGeom& g = p.g;
  const int xf_warps_per_group = kNumXfWarps / p.groups;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.ring; ++i) {
      mbar_init(bar_halo_full + 8u * i, 1);
      mbar_init(bar_halo_empty + 8u * i, 1);
    }
    for (int i = 0; i < p.sb; ++i) {
      mbar_init(bar_b_full + 8u * i, 1);
      mbar_init(bar_b_empty + 8u * i, 1);
    }
    for (int i = 0; i < p.sa; ++i) {
      mbar_init(bar_a_full + 8u * i, xf_warps_per_group);
      mbar_init(bar_a_empty + 8u * i, 1);
    }
    for (int i = 0; i < kMaxAcc; ++i) {
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

  if (warp == kWarpB) {
    // ------------------------------------------------------------ weight producer
    if (lane == 0) {
      uint32_t gb = 0;  // weight stages issued
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        const TileCoord tc = decode_tile(p, t);
        for (int s = 0; s < p.ks; ++s, ++gb) {
          const uint32_t e = gb % p.sb, u = gb / p.sb;
          if (u > 0 && !wait_or_abort(bar_b_empty + 8u * e, (u - 1u) & 1u, p.err, kSiteProducerEmpty, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar_b_full + 8u * e, p.b_stage_bytes);
          for (int i = 0; i < p.n_sub; ++i)
            tma_load_2d(base + p.off_b + e * p.b_stage_bytes + static_cast<uint32_t>(i * p.sub_n) * 128u, &tmap_w,
                        bar_b_full + 8u * e, kBlockK * s, tc.nt * p.n_tile + i * p.sub_n);
        }
      }
      if (!ok) drain_ring(bar_b_full, static_cast<uint32_t>(p.sb), gb, p.err, kSiteDrain);
    }
  } else if (warp == kWarpHalo) {
    // ------------------------------------------------------------ halo producer
    if (lane == 0) {
      uint32_t gs = 0;  // halo slots issued
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        const TileCoord tc = decode_tile(p, t);
        const int w0 = halo_w0(p, tc.ow0);
        const int h0 = tc.oh0 * g.sh - g.ph;
        const int d0 = tc.od * g.sd - g.pd;
        for (int q = 0; q < p.q_slots; ++q, ++gs) {
          const uint32_t e = gs % p.ring, u = gs / p.ring;
          if (u > 0 && !wait_or_abort(bar_halo_empty + 8u * e, (u - 1u) & 1u, p.err, kSiteHaloEmpty, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar_halo_full + 8u * e, p.slot_tx);
          tma_load_5d(base + p.off_halo + e * p.slot_bytes, &tmap_x, bar_halo_full + 8u * e, w0, h0, d0,
                      q * p.c_slot, tc.n);
        }
      }
      if (!ok) drain_ring(bar_halo_full, static_cast<uint32_t>(p.ring), gs, p.err, kSiteDrain);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16_f32_amn(128, static_cast<uint32_t>(p.sub_n));
      uint32_t ga = 0, gb = 0, it = 0, gs_base = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x, ++it) {
        int released = 0;
        for (int s = 0; ok && s < p.ks; ++s, ++ga, ++gb) {
          const uint32_t ea = ga % p.sa, eb = gb % p.sb;
          if (!wait_or_abort(bar_a_full + 8u * ea, (ga / p.sa) & 1u, p.err, kSiteAStageFull, abort_flag)) {
            ok = false;
            break;
          }
          // Slices are complete in order up to s, and no later slice reads a
          // halo slot below the first one slice s+1 needs: hand those back.
          const int keep = (s + 1 < p.ks) ? slot_lo(p, s + 1) : p.q_slots;
          for (; released < keep; ++released)
            mbar_arrive(bar_halo_empty + 8u * ((gs_base + static_cast<uint32_t>(released)) % p.ring));
          if (!wait_or_abort(bar_b_full + 8u * eb, (gb / p.sb) & 1u, p.err, kSiteTmaFull, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_stage = base + p.off_a + ea * p.a_stage_bytes;
          const uint64_t bdesc = umma_desc_kmajor_sw128(base + p.off_b + eb * p.b_stage_bytes);
          for (int i = 0; ok && i < p.n_mt; ++i) {
            const uint64_t adesc =
                umma_desc_mnmajor_sw128(a_stage + static_cast<uint32_t>(i) * kASubBytes, 1024u, 2048u);
            for (int ns = 0; ns < p.n_sub; ++ns) {
              const int acc = i * p.n_sub + ns;
              if (s == 0 && it > 0) {
                if (!wait_or_abort(bar_acc_empty + 8u * acc, (it - 1u) & 1u, p.err, kSiteAccEmpty, abort_flag)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
              }
              const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(i * p.n_tile + ns * p.sub_n);
#pragma unroll
              for (int j = 0; j < kBlockK / 16; ++j)
                umma_bf16(d_tmem, adesc + static_cast<uint64_t>(j * 256),
                          bdesc + static_cast<uint64_t>(ns * p.sub_n * 8 + 2 * j), idesc, (s > 0 || j > 0) ? 1u : 0u);
              if (s == p.ks - 1) umma_commit(bar_acc_full + 8u * acc);
            }
          }
          if (!ok) break;
          umma_commit(bar_a_empty + 8u * ea);
          umma_commit(bar_b_empty + 8u * eb);
        }
        gs_base += static_cast<uint32_t>(p.q_slots);
      }
      if (!ok) {
        umma_commit(bar_drain);
        mbar_wait(bar_drain, 0, p.err, kSiteDrain);
      }
    }
  } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + 4) {
    // ------------------------------------------------------------ epilogue
    const int qw = warp - kWarpEpi0;
    const int lr = qw * 32 + lane;  // row within a subtile
    const int th_l = lr / p.TW, tw_l = lr % p.TW;
    const int S_hw = g.OH * g.OW;
    const int64_t S = static_cast<int64_t>(g.OD) * S_hw;
    T* y = static_cast<T*>(p.y);
    const T* bias = static_cast<const T*>(p.bias);
    uint32_t it = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x, ++it) {
      const TileCoord tc = decode_tile(p, t);
      const int ow = tc.ow0 + tw_l;
      for (int i = 0; ok && i < p.n_mt; ++i) {
        const int oh = tc.oh0 + i * p.TH + th_l;
        const bool valid = oh < g.OH && ow < g.OW;
        const int64_t ybase = (static_cast<int64_t>(tc.n) * g.Cout) * S + static_cast<int64_t>(tc.od) * S_hw +
                              static_cast<int64_t>(oh) * g.OW + ow;
        for (int ns = 0; ns < p.n_sub; ++ns) {
          const int acc = i * p.n_sub + ns;
          if (!wait_or_abort(bar_acc_full + 8u * acc, it & 1u, p.err, kSiteAccFull, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int co0 = tc.nt * p.n_tile + ns * p.sub_n;
          const uint32_t taddr =
              tmem_base + (static_cast<uint32_t>(qw * 32) << 16) + static_cast<uint32_t>(i * p.n_tile + ns * p.sub_n);
          for (int c0 = 0; c0 < p.sub_n; c0 += 16) {
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
          if (lane == 0) mbar_arrive(bar_acc_empty + 8u * acc);
        }
      }
    }
  } else if (warp >= kWarpXf0) {
    // ------------------------------------------------------------ transform
    // A warp covers one 16-column block of a K slice for 32 row groups:
    // 8-row groups of two subtiles (n_mt >= 2) or 4-row groups of the single
    // subtile (n_mt == 1), so the taps it walks are the same in every lane.
    const int P = p.n_mt >= 2 ? 8 : 4;
    const int xw = warp - kWarpXf0;
    const int grp = xw / xf_warps_per_group;     // which K slices this warp works on
    const int lw = xw % xf_warps_per_group;
    const int blk = lw & 3;                      // 16-column block within the K slice
    const int sub = (P == 8) ? 2 * (lw >> 2) + (lane >> 4) : 0;
    const int rg = (P == 8) ? (lane & 15) : lane;
    const int lr0 = P * rg;                      // first row of the group within the subtile
    const int th = sub * p.TH + lr0 / p.TW;      // row of the tile
    const int tw0 = lr0 % p.TW;
    const uint32_t halo_base = base + p.off_halo;
    const uint32_t tab = base + p.off_tab;
    const int xf_tid = threadIdx.x - kWarpXf0 * 32;

    // per-CTA table of (scale, 1/scale) for every non-negative E4M3 code
    const Nvfp4Global G = p.quant ? nvfp4_global(__ldg(p.act_amax)) : Nvfp4Global{0.0f, 0.0f, 0.0f};
    {
      if (p.quant && xf_tid < 128) {
        uint32_t h2;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<unsigned short>(xf_tid & 0x7F)));
        const float s8 = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
        float s = __fmul_rn(s8, G.g);
        if (s < 1e-5f) s = 1.0f;
        float* e = reinterpret_cast<float*>(smem + p.off_tab + xf_tid * 8);
        e[0] = s;
        e[1] = __frcp_rn(s);
      }
      named_bar_sync(1, kNumXfWarps * 32);
    }

    int roff[8];
    uint32_t gs_base = 0;  // global slot counter at the start of the tile
    uint32_t ga = 0;       // global K-slice counter at the start of the tile
    bool ok = true;
    for (int64_t tt = blockIdx.x; ok && tt < p.num_tiles; tt += gridDim.x) {
      const TileCoord tc = decode_tile(p, tt);
      const int w0 = halo_w0(p, tc.ow0);
      const int delta = tc.ow0 * g.sw - g.pw - w0;
      const int thr_al = th * g.sh * p.w_box + tw0 * g.sw;
      const uint32_t thr_addr = static_cast<uint32_t>(thr_al) * 2u;
#pragma unroll
      for (int r = 0; r < 8; ++r) roff[r] = thr_al + r * g.sw + delta;
      // first K slice of this tile that belongs to this warp's group
      int s = static_cast<int>((static_cast<uint32_t>(grp) + static_cast<uint32_t>(p.groups) -
                                ga % static_cast<uint32_t>(p.groups)) % static_cast<uint32_t>(p.groups));
      for (; s < p.ks; s += p.groups) {
        const uint32_t gslice = ga + static_cast<uint32_t>(s);
        const uint32_t ea = gslice % p.sa, ua = gslice / p.sa;
        if (ua > 0 && !wait_or_abort(bar_a_empty + 8u * ea, (ua - 1u) & 1u, p.err, kSiteMmaDone, abort_flag)) {
          ok = false;
          break;
        }
        for (int q = slot_lo(p, s), qh = slot_hi(p, s); ok && q <= qh; ++q) {
          const uint32_t gsl = gs_base + static_cast<uint32_t>(q);
          ok = wait_or_abort(bar_halo_full + 8u * (gsl % p.ring), (gsl / p.ring) & 1u, p.err, kSiteHaloFull,
                             abort_flag);
        }
        if (!ok) break;
        const uint32_t a_sub = base + p.off_a + ea * p.a_stage_bytes + static_cast<uint32_t>(sub) * kASubBytes;
        const int kb = kBlockK * s + 16 * blk;
        if constexpr (sizeof(T) == 2) {
          if (p.vec) {
            if (P == 8)
              transform_task_vec<T, 8>(p, a_sub, rg, kb, thr_addr, delta, halo_base, gs_base, G, tab);
            else
              transform_task_vec<T, 4>(p, a_sub, rg, kb, thr_addr, delta, halo_base, gs_base, G, tab);
          } else if (P == 8) {
            transform_task_gen<T, 8>(p, a_sub, rg, kb, roff, halo_base, gs_base, G, tab);
          } else {
            transform_task_gen<T, 4>(p, a_sub, rg, kb, roff, halo_base, gs_base, G, tab);
          }
        } else if (P == 8) {
          transform_task_gen<T, 8>(p, a_sub, rg, kb, roff, halo_base, gs_base, G, tab);
        } else {
          transform_task_gen<T, 4>(p, a_sub, rg, kb, roff, halo_base, gs_base, G, tab);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_a_full + 8u * ea);
      }
      if (!ok) break;
      gs_base += static_cast<uint32_t>(p.q_slots);
      ga += static_cast<uint32_t>(p.ks);
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
  if (!v) return 0;
  if (!strcmp(v, "basic")) return 1;
  if (!strcmp(v, "fast")) return 2;
  return 0;
}

int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace

// Tiling and pipeline plan of the specialised kernel for one problem (pure
// host arithmetic).  Returns false when the kernel does not apply.
static bool plan_fast(const ConvGeom& g, int dtype, FastParams& p, size_t& smem) {
  const int esz = dtype == 0 ? 4 : 2;
  const int align = 16 / esz;
  if ((static_cast<int64_t>(g.W) * esz) % 16 != 0) return false;
  memset(&p, 0, sizeof(p));
  p.g = g;
  p.align = align;

  // output channels per tile: all of Cout up to 512, else tiles of 256
  int n_ntiles = 1, n_tile = (g.Cout + 15) / 16 * 16;
  if (n_tile > 512) {
    n_ntiles = ceil_div(g.Cout, 256);
    n_tile = (ceil_div(g.Cout, n_ntiles) + 15) / 16 * 16;
  }
  const int n_sub = ceil_div(n_tile, 256);
  const int sub_n = (ceil_div(n_tile, n_sub) + 15) / 16 * 16;
  n_tile = sub_n * n_sub;
  p.n_tile = n_tile; p.n_ntiles = n_ntiles; p.n_sub = n_sub; p.sub_n = sub_n;
  const int max_mt = std::min(4, 512 / n_tile);

  // tile shape: subtile TH x TW = 128, n_mt subtiles stacked along oh
  const int kd_ext = (g.KD - 1) * g.dd + 1;
  double best = 1e30;
  int bTW = 0, bMT = 0;
  for (int mt = max_mt; mt >= 1; mt /= 2) {
    if (mt == 3) continue;
    for (int TW = 128; TW >= 8; TW /= 2) {
      const int TH = 128 / TW, rows = TH * mt;
      const int h_ext = (rows - 1) * g.sh + (g.KH - 1) * g.dh + 1;
      const int w_ext = (TW - 1) * g.sw + (g.KW - 1) * g.dw + 1;
      const int w_box = (w_ext + 2 * (align - 1)) / align * align;
      if (w_box > 256 || h_ext > 256 || kd_ext > 256) continue;
      const double waste = (double)(ceil_div(g.OH, rows) * rows) * (ceil_div(g.OW, TW) * TW) / ((double)g.OH * g.OW);
      const double halo = (double)h_ext * w_box / (128.0 * mt);
      // fewer subtiles per tile cost weight bandwidth: about 8% per halving
      const double score = waste * (1.0 + 0.01 * halo) * (1.0 + 0.08 * (mt >= 4 ? 0 : mt == 2 ? 1 : 2));
      if (score < best - 1e-9) { best = score; bTW = TW; bMT = mt; }
    }
  }
  if (bTW == 0) return false;
  p.TW = bTW; p.TH = 128 / bTW; p.n_mt = bMT;
  p.groups = bMT >= 4 ? 1 : 2;  // 8 transform warps; a K slice needs 2*n_mt (n_mt >= 2) or 4 warps
  p.n_owb = ceil_div(g.OW, p.TW);
  p.n_ohb = ceil_div(g.OH, p.TH * p.n_mt);
  p.h_ext = (p.TH * p.n_mt - 1) * g.sh + (g.KH - 1) * g.dh + 1;
  const int w_ext = (p.TW - 1) * g.sw + (g.KW - 1) * g.dw + 1;
  p.w_box = (w_ext + 2 * (align - 1)) / align * align;
  p.kd_ext = kd_ext;
  p.chan_elems = p.kd_ext * p.h_ext * p.w_box;
  p.ks = ceil_div(g.K, kBlockK);
  p.num_tiles = static_cast<int64_t>(g.N) * g.OD * p.n_ohb * p.n_owb * n_ntiles;
  p.a_stage_bytes = static_cast<uint32_t>(p.n_mt) * kASubBytes;
  p.b_stage_bytes = static_cast<uint32_t>(n_tile) * 128u;
  p.vec = (esz == 2 && g.sw == 1) ? 1 : 0;
  int tmem = 32;
  while (tmem < p.n_mt * n_tile) tmem <<= 1;
  p.tmem_cols = tmem;

  const int chan_bytes = p.chan_elems * esz;
  // Halo ring: the MMA thread hands a slot back once every slice that reads
  // it is complete, while the transform may run up to sa slices ahead of the
  // MMA, so the ring must hold the slots of sa consecutive slices (+2 so the
  // producer can run ahead).  A stages must number at least the transform
  // groups (each group owns every groups-th slice), or a group could wait on
  // an A-stage barrier two phases ahead.
  for (int target = 10240; target >= 1; target = (target > chan_bytes ? target / 2 : 0)) {
    p.c_slot = std::max(1, std::min(std::min(256, g.C), target / chan_bytes));
    p.q_slots = ceil_div(g.C, p.c_slot);
    p.slot_tx = static_cast<uint32_t>(p.c_slot) * chan_bytes;
    p.slot_bytes = (p.slot_tx + 127u) / 128u * 128u;
    auto span_of = [&](int w) {
      int sp = 1;
      for (int s0 = 0; s0 < p.ks; ++s0) {
        const int lo = ((kBlockK * s0) / g.taps) / p.c_slot;
        const int hi = (std::min(kBlockK * (s0 + w) - 1, g.K - 1) / g.taps) / p.c_slot;
        sp = std::max(sp, hi - lo + 1);
      }
      return sp;
    };
    auto total = [&](int a, int b, int r) {
      const int nbar = 2 * r + 2 * b + 2 * a + 2 * kMaxAcc + 1;
      return 1024 + a * static_cast<int>(p.a_stage_bytes) + b * static_cast<int>(p.b_stage_bytes) +
             r * static_cast<int>(p.slot_bytes) + 64 /* pad after the halo ring */ + 1024 /* scale table */ +
             nbar * 8 + 16;
    };
    for (int a = 4; a >= 2; --a) {
      if (a < p.groups) continue;
      for (int b = 8; b >= 2; --b) {
        const int r = span_of(a) + 2;
        if (total(a, b, r) <= kMaxSmem) {
          p.sa = a; p.sb = b; p.ring = r;
          p.off_a = 0;
          p.off_b = p.off_a + a * p.a_stage_bytes;
          p.off_halo = p.off_b + b * p.b_stage_bytes;
          p.off_tab = (p.off_halo + r * p.slot_bytes + 64u + 15u) / 16u * 16u;
          p.off_bar = p.off_tab + 1024u;
          smem = static_cast<size_t>(total(a, b, r));
          // at most 512 / tmem_cols CTAs may share an SM, so tcgen05.alloc never waits
          const size_t max_ctas = 512 / static_cast<size_t>(p.tmem_cols);
          const size_t min_smem = 233472 / (max_ctas + 1) + 1;
          if (max_ctas < 4 && smem + 1024 < min_smem) smem = min_smem - 1024;
          return true;
        }
      }
    }
    if (p.c_slot == 1) break;
  }
  return false;
}

bool plan_conv3d_fast(const ConvGeom& g, int dtype, int32_t* out, int n_out) {
  FastParams p{};
  size_t smem = 0;
  const bool ok = plan_fast(g, dtype, p, smem);
  const int64_t v[] = {ok ? 1 : 0, p.TH, p.TW, p.n_mt, p.groups, p.n_tile, p.n_ntiles, p.n_sub, p.sub_n, p.ks,
                       p.c_slot, p.q_slots, p.ring, p.sa, p.sb, p.tmem_cols, static_cast<int64_t>(smem),
                       p.n_ohb, p.n_owb, p.vec, p.w_box, p.h_ext, p.kd_ext};
  const int nv = static_cast<int>(sizeof(v) / sizeof(v[0]));
  for (int i = 0; i < n_out; ++i) out[i] = i < nv ? static_cast<int32_t>(v[i]) : 0;
  return ok;
}

cudaError_t launch_conv3d_fast(const ConvGeom& g, const ConvLaunch& L, cudaStream_t s, const char** why,
                               bool* handled) {
  *handled = false;
  if (kernel_choice() == 1) return cudaSuccess;
  if (L.quant && !(L.qfmt == 1 && L.qblock == 16)) return cudaSuccess;  // NVFP4 blocks of 16 only
  const int esz = L.dtype == 0 ? 4 : 2;
  if (reinterpret_cast<uintptr_t>(L.x) % 16 != 0) return cudaSuccess;
  FastParams p{};
  size_t smem = 0;
  if (!plan_fast(g, L.dtype, p, smem)) return cudaSuccess;
  p.bias = L.bias; p.y = L.y; p.act_amax = L.act_amax; p.err = L.err; p.quant = L.quant;

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
