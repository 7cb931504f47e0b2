// conv3d_tmem_kernel.cuh -- the tensor-memory implicit-GEMM Conv3D kernel
// template, its host planner and launch helpers, shared by the translation
// units that instantiate it (conv3d_igemm_tmem.cu: BF16 operands, A in
// tensor memory; conv3d_igemm_tmem_sa.cu: BF16 operands, A in shared memory;
// conv3d_fp4.cu: NVFP4 operands for the block-scaled MMA).  The kernel
// parameters (TmemParams) have external linkage; everything else here is
// internal to each unit.
//
// GEMM view as in the Model-Optimizer "Conv3D Implicit GEMM CUDA kernel"
// article, sec. 5.1 (rows (n, od, oh, ow), columns (c, kd, kh, kw)), with the
// NVFP4 activation quantiser of sec. 6.3 fused into the A-operand producer.
//
// A tile is n_mt M-subtiles of 128 output positions (TH x TW rectangles of one
// (n, od) plane, stacked along oh) times n_tile output channels.  Per 64-wide
// K slice, the weights arrive in shared memory (TMA, K-major, 128B swizzle;
// prepacked NVFP4 images by bulk copy in the NVFP4 form) and the transform
// warps build the slice of A from the input halo: BF16 values straight into
// tensor memory with tcgen05.st (one 32-bit column per pair of consecutive K
// elements), or BF16 values / NVFP4 codes into a swizzled shared-memory stage.
// tcgen05.mma reads A from there and B from shared memory, accumulating in
// FP32 in tensor memory (one or two accumulator buffers).
//
// Roles (24 warps, one persistent CTA per SM):
//   warp 0      weight producer;
//   warp 1      TMEM owner and MMA issuer (tcgen05.mma, M = 128, N = n_tile
//               in <= 256-wide instructions; kind::f16 with K = 16 per
//               instruction = one quantisation block, or the block-scaled
//               kind::mxf4nvf4 with K = 64);
//   warp 2      halo producer: 5-D TMA boxes of x (zero fill outside the
//               input = the convolution padding) into a ring of slots;
//   warps 4-7   epilogue: tcgen05.ld, the NVFP4 form's global scales and the
//               bias in FP32, rounding to the output dtype, bounds-checked
//               NCDHW stores staged for 16-byte writes;
//   warps 8-23  transform, in two groups taking alternate K slices.  Warp w
//               owns lane quadrant w % 4 (the TMEM lanes its tcgen05.st may
//               reach) and two 16-column blocks of each of its slices; each
//               thread owns one output position (row) of every subtile.  Per
//               block it gathers its 16 halo values, takes the block maximum,
//               looks up the block's quantiser entry (E4M3 scale, 1/scale and
//               the dequantisation table) in per-CTA tables, and writes the
//               quantised values.
// All waits are bounded; a timeout in any role aborts all roles.
#pragma once
#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <cuda_runtime.h>
#include <utility>

#include "nvfp4.cuh"
#include "q3d_internal.h"
#include "sm100_ptx.cuh"

namespace q3d {

// Kernel parameters (external linkage, so the translation units that
// instantiate the kernel can hand a plan to each other).
struct TmemParams {
  ConvGeom g;
  const void* bias;
  void* y;
  const float* act_amax;
  unsigned int* err;
  int quant;
  // tiling
  int TH, TW, n_mt;
  int n_ohb, n_owb;
  int n_tile, n_ntiles, n_sub, sub_n;
  int64_t num_tiles;
  int ks;
  // halo staging
  int align;
  int w_box, h_ext, kd_ext, c_slot, q_slots, chan_elems;
  uint32_t chan_bytes, slot_bytes, slot_tx;
  int ring;
  // pipelines
  int sa, sb;
  uint32_t b_stage_bytes;
  int a_col0;             // first TMEM column of the A stages (accumulators start at column 0)
  int acc_bufs;           // accumulator buffers (2: tile t + 1 accumulates while tile t drains)
  int acc_cols;           // TMEM columns of one accumulator buffer (n_mt * n_tile)
  int dk2_c, dk2_phi;     // 128 = dk2_c * taps + dk2_phi (a transform warp's step: two slices)
  int dk16_c, dk16_phi;   // 16 = dk16_c * taps + dk16_phi (from one block to the next)
  int slot_aligned;       // c_slot * taps is a multiple of 16: no block straddles two halo slots
  uint32_t off_dq, off_b, off_halo, off_code, off_epi, off_phase, off_bar;
  int y_vec;  // y is 16-byte aligned and OW a multiple of 16 / sizeof(T): vector stores
  int withhold_arrive;  // test of the bounded waits only (0 otherwise): see the epilogue
  // NVFP4-operand variant only: the A stages live in shared memory (packed
  // E2M1 codes, 32-byte swizzle, and a scale-factor atom per subtile); the
  // weights arrive as prepacked images, one per N-part and K slice; the
  // scale factors of both operands are copied into tensor memory, a region
  // per A stage
  int fp4;                // aop == NVFP4 (kept for the host side)
  int aop;                // A operand mode: 0 BF16 in tensor memory, 1 BF16 in shared memory, 2 NVFP4
  int dtype_code;         // element type of x: 0 f32, 1 f16, 2 bf16
  uint32_t off_a, a_stage_bytes;
  uint32_t b_img_bytes;   // one N-part's image: sub_n rows x 32 bytes of codes, then n_atoms scale atoms
  int n_atoms;            // 512-byte scale-factor atoms per N-part (128 rows each)
  int n_parts;            // N-parts over all N-tiles (n_ntiles * n_sub)
  int sf_col0, sf_cols;   // scale-factor columns of A stage e: sf_col0 + e * sf_cols
  const uint8_t* wq;      // the first image (slice 0, part 0)
  const float* g_w;       // global scale of the weights (device scalar)
  // BF16 forms, when quant: the activation quantiser (kQMode*) and, for
  // MXFP4, the largest magnitude a group's maximum is scaled to (0: the
  // E2M1 rule floor(log2 amax) - 2)
  int qmode;
  float dst_max;
  // transform warps wait for each halo slot's fill before handing it back
  // (plans whose warps could otherwise hand back a slot a ring lap early)
  int hb_wait;
};

// The BF16 kernel with A in shared memory (instantiated in its own
// translation unit, conv3d_igemm_tmem_sa.cu).
cudaError_t launch_tmem_smem_a(const TmemParams& p, const CUtensorMap& tx, const CUtensorMap& tw, int grid,
                               size_t smem, cudaStream_t s);
// The BF16 kernel with the 32-column-group quantisers (p.qmode NVFP4 blocks
// of 32 or MXFP4), A in tensor or shared memory as p.aop says (instantiated
// in conv3d_igemm_tmem_g32.cu).
cudaError_t launch_tmem_groups(const TmemParams& p, const CUtensorMap& tx, const CUtensorMap& tw, int grid,
                               size_t smem, cudaStream_t s);

namespace {

constexpr int kThreads = 768;
constexpr int kWarpB = 0;
constexpr int kWarpMma = 1;
constexpr int kWarpHalo = 2;
constexpr int kWarpEpi0 = 4;
constexpr int kWarpXf0 = 8;
constexpr int kNumXfWarps = 16;
constexpr int kBlockK = 64;
constexpr int kMaxSmem = 232448;  // 227 KB dynamic shared memory per CTA
constexpr int kMaxAcc = 16;     // accumulator barriers: buffers x subtiles x N-parts
constexpr int kMaxTaps = 343;     // 7x7x7
constexpr uint32_t kTmemCols = 512;
// Where the transform warps put the A operand and in which format:
//   BF16 values in tensor memory (tcgen05.st; the MMA reads A from TMEM);
//   BF16 values in shared memory (128-byte-swizzled K-major, like B);
//   NVFP4 codes and scale bytes in shared memory (block-scaled MMA).
constexpr int kAOpBf16Tmem = 0, kAOpBf16Smem = 1, kAOpNvfp4 = 2;
// The activation quantiser of the BF16 forms: NVFP4 with blocks of 16 (the
// default), NVFP4 with blocks of 32 (an E4M3 scale per 32 columns), MXFP4
// (a power-of-two scale per 32 columns), NVFP4 with blocks of 64.  A warp's
// two adjacent 16-column blocks of a K slice (b0 even) are one 32-column
// group, so a group's maximum never leaves the thread that owns its row.  A
// 64-column block is a whole K slice: with A in shared memory the threads
// are then mapped so that lanes l and l + 16 of a warp hold the two halves
// of one row, and the block maximum is one shuffle away.
constexpr int kQModeNv16 = 0, kQModeNv32 = 1, kQModeMx = 2, kQModeNv64 = 3;


struct TileCoord {
  int n, od, oh0, ow0, nt;
};

// Output-channel tile fastest, then the frame od, then the spatial blocks:
// tiles running concurrently share two of their three input frames in L2.
__device__ __forceinline__ TileCoord decode_tile(const TmemParams& p, int64_t t) {
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
__device__ __forceinline__ int halo_w0(const TmemParams& p, int ow0) {
  return floor_div(ow0 * p.g.sw - p.g.pw, p.align) * p.align;
}

// Position in a ring of n pipeline entries: the entry, and the parity of the
// pass over the ring (the barrier phase that a use of the entry completes).
// Advanced by one compare per step, so no pipeline loop divides.
struct RingPos {
  uint32_t e, ph;
  __device__ __forceinline__ void next(uint32_t n) {
    if (++e == n) {
      e = 0;
      ph ^= 1u;
    }
  }
};
__device__ __forceinline__ RingPos ring_pos(uint32_t g, uint32_t n) { return RingPos{g % n, (g / n) & 1u}; }

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

__device__ __forceinline__ uint32_t ld_shared_u16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void ld_shared_v4(uint32_t addr, int& a, int& b, int& c, int& d) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "r"(addr));
}

// E2M1 codes (round to nearest even, saturating) of four non-negative
// values, one per nibble of the low 16 bits (a0 lowest).
__device__ __forceinline__ uint32_t e2m1_codes4(float a0, float a1, float a2, float a3) {
  uint32_t r;
  asm("{\n\t.reg .b8 q0, q1;\n\t.reg .b16 h;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "mov.b16 h, {q0, q1};\n\t"
      "cvt.u32.u16 %0, h;\n\t}"
      : "=r"(r)
      : "f"(a0), "f"(a1), "f"(a2), "f"(a3));
  return r;
}

__device__ __forceinline__ uint32_t cvt_bf16x2(float hi, float lo) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint32_t maxabs_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t maxabs_f16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Dequantisation table of one row's block: the BF16 bit patterns of q*scale
// for the eight E2M1 magnitudes q in code order {0, .5, 1, 1.5, 2, 3, 4, 6},
// split into low bytes (lo_a = codes 0-3, lo_b = codes 4-7) and high bytes.
// Each product is the binary32 product rounded to BF16; multiplying by a
// power of two commutes with both roundings, so every entry follows from
// BF16(scale) and BF16(binary32(1.5 * scale)) by adding to the exponent field.
struct DqTable {
  uint32_t lo_a, lo_b, hi_a, hi_b;
};
__device__ __forceinline__ DqTable dq_table(float scale) {
  const uint32_t p = cvt_bf16x2(__fmul_rn(1.5f, scale), scale);  // lo: BF16(s), hi: BF16(1.5 s)
  const uint32_t e01 = (p << 16) - 0x00800000u;                  // {0, s/2}
  const uint32_t e45 = p + 0x00800080u;                          // {2s, 3s}
  const uint32_t e67 = p + 0x01000100u;                          // {4s, 6s}
  DqTable t;
  t.lo_a = __byte_perm(e01, p, 0x6420);
  t.hi_a = __byte_perm(e01, p, 0x7531);
  t.lo_b = __byte_perm(e45, e67, 0x6420);
  t.hi_b = __byte_perm(e45, e67, 0x7531);
  return t;
}

// Four quantised BF16 values (two packed words) from four scaled magnitudes
// a = |v| / scale, with the signs of the inputs (sign bits at 15 and 31 of
// sgn01 and sgn23).
__device__ __forceinline__ void dq4(const DqTable& t, float a0, float a1, float a2, float a3, uint32_t sgn01,
                                    uint32_t sgn23, uint32_t& o01, uint32_t& o23) {
  const uint32_t sel = e2m1_codes4(a0, a1, a2, a3);
  const uint32_t lo = __byte_perm(t.lo_a, t.lo_b, sel);
  const uint32_t hi = __byte_perm(t.hi_a, t.hi_b, sel);
  o01 = __byte_perm(lo, hi, 0x5140) | (sgn01 & 0x80008000u);
  o23 = __byte_perm(lo, hi, 0x7362) | (sgn23 & 0x80008000u);
}

// Per-CTA quantiser tables in shared memory.
//  - Entry table: for every E4M3 code of a block scale (0..127), 32 bytes:
//    the block's DqTable (16 B) and 1/scale (binary32), where scale =
//    E4M3(code) * g, or 1.0 when that is below 1e-5.
//  - BF16 inputs only, code table: a block maximum of a BF16 input is itself
//    a BF16 value, and the scale step (ratio to 6 g, clamp to 448, E4M3
//    rounding) is a monotone function of it; the table maps each BF16 bit
//    pattern b in [lo, hi] to the byte offset of its code's entry.  The
//    window spans the 22 binades from 2^-11 t (every smaller maximum gives
//    code 0) up past 2^9 t (every larger one clamps to 448), so patterns
//    outside it take the entry of the nearer end.  The entries are computed
//    with the same device arithmetic as the direct path, so both give the
//    same code for every maximum.
constexpr int kDqEntryBytes = 32;
constexpr int kDqTableBytes = 128 * kDqEntryBytes;
constexpr int kCodeBinades = 22;
constexpr int kCodeEntries = kCodeBinades * 128;  // BF16 has 128 patterns per binade
constexpr int kCodeTableBytes = kCodeEntries * 2;

struct QCtx {
  Nvfp4Global G;
  uint32_t dq;      // shared address of the entry table
  uint32_t cb;      // shared address of the code table minus 2 * lo
  uint32_t lo, hi;  // BF16 bit patterns covered by the code table
};

__device__ __forceinline__ uint32_t e4m3_code(float r) {
  uint16_t code;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(code) : "f"(0.0f), "f"(r));
  return code & 0x7Fu;
}

// Shared address of the entry for a block maximum given as a binary32 value.
__device__ __forceinline__ uint32_t entry_of_max(float bmax, const QCtx& q) {
  return q.dq + e4m3_code(nvfp4_ratio(bmax, q.G.t, q.G.rt)) * kDqEntryBytes;
}

__device__ __forceinline__ void load_entry(uint32_t e, DqTable& t, float& inv) {
  int a, b, c, d;
  ld_shared_v4(e, a, b, c, d);
  t.lo_a = static_cast<uint32_t>(a);
  t.lo_b = static_cast<uint32_t>(b);
  t.hi_a = static_cast<uint32_t>(c);
  t.hi_b = static_cast<uint32_t>(d);
  inv = __uint_as_float(ld_shared_u32(e + 16u));
}

// Per-element views of a packed pair of 16-bit inputs.
template <typename T>
struct Half2;
template <>
struct Half2<__nv_bfloat16> {
  // |x| as an operand modifier of the consuming multiply or max
  static __device__ __forceinline__ float abs_lo(uint32_t w) { return fabsf(__uint_as_float(w << 16)); }
  static __device__ __forceinline__ float abs_hi(uint32_t w) { return fabsf(__uint_as_float(w & 0xFFFF0000u)); }
  static __device__ __forceinline__ float lo(uint32_t w) { return __uint_as_float(w << 16); }
  static __device__ __forceinline__ float hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
  static __device__ __forceinline__ uint32_t maxabs(uint32_t a, uint32_t b) { return maxabs_bf16x2(a, b); }
  static __device__ __forceinline__ uint32_t to_bf16x2(uint32_t w) { return w; }
  // entry of a block from the packed |v| maximum of its eight words: the
  // larger half's BF16 pattern indexes the code table (clamped to its window)
  static __device__ __forceinline__ uint32_t entry(uint32_t m, const QCtx& q) {
    const uint32_t m2 = maxabs_bf16x2(m, __byte_perm(m, 0u, 0x1032));
    const uint32_t b = min(max(m2 & 0x7FFFu, q.lo), q.hi);
    return q.dq + ld_shared_u16(q.cb + 2u * b);
  }
};
template <>
struct Half2<__half> {
  static __device__ __forceinline__ float abs_lo(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0x7FFFu)));
  }
  static __device__ __forceinline__ float abs_hi(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>((w >> 16) & 0x7FFFu)));
  }
  static __device__ __forceinline__ float lo(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xFFFFu)));
  }
  static __device__ __forceinline__ float hi(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
  }
  static __device__ __forceinline__ uint32_t maxabs(uint32_t a, uint32_t b) { return maxabs_f16x2(a, b); }
  static __device__ __forceinline__ uint32_t to_bf16x2(uint32_t w) {
    return cvt_bf16x2(__half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16))),
                      __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xFFFFu))));
  }
  static __device__ __forceinline__ uint32_t entry(uint32_t m, const QCtx& q) {
    return entry_of_max(fmaxf(abs_lo(m), abs_hi(m)), q);
  }
};

// |v| maximum of a block held as eight packed words.
template <typename T>
__device__ __forceinline__ uint32_t maxabs8(const uint32_t (&p)[8]) {
  using H = Half2<T>;
  return H::maxabs(H::maxabs(H::maxabs(p[0], p[1]), H::maxabs(p[2], p[3])),
                   H::maxabs(H::maxabs(p[4], p[5]), H::maxabs(p[6], p[7])));
}

// Quantise one block of a 16-bit input (eight packed words) with its entry.
template <typename T>
__device__ __forceinline__ void quant8(const uint32_t (&pk)[8], const DqTable& dt, float inv, uint32_t (&out)[8]) {
  using H = Half2<T>;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t w0 = pk[2 * i], w1 = pk[2 * i + 1];
    dq4(dt, __fmul_rn(H::abs_lo(w0), inv), __fmul_rn(H::abs_hi(w0), inv), __fmul_rn(H::abs_lo(w1), inv),
        __fmul_rn(H::abs_hi(w1), inv), w0, w1, out[2 * i], out[2 * i + 1]);
  }
}

// Two blocks of a 16-bit input (two rows, or two blocks of one row), each
// quantised with its own scale; the two chains are interleaved so each hides
// the other's latency.  Without quantisation the values are only converted.
template <typename T>
__device__ __forceinline__ void quant8_x2(const uint32_t (&pa)[8], const uint32_t (&pb)[8], bool quant, const QCtx& q,
                                          uint32_t (&out_a)[8], uint32_t (&out_b)[8]) {
  if (!quant) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      out_a[i] = Half2<T>::to_bf16x2(pa[i]);
      out_b[i] = Half2<T>::to_bf16x2(pb[i]);
    }
    return;
  }
  const uint32_t ma = maxabs8<T>(pa), mb = maxabs8<T>(pb);
  const uint32_t ea = Half2<T>::entry(ma, q), eb = Half2<T>::entry(mb, q);
  DqTable da, db;
  float ia, ib;
  load_entry(ea, da, ia);
  load_entry(eb, db, ib);
  quant8<T>(pa, da, ia, out_a);
  quant8<T>(pb, db, ib, out_b);
}

template <int OFF>
__device__ __forceinline__ uint32_t ld_shared_u16_at(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1+%2];" : "=h"(v) : "r"(addr), "n"(OFF));
  return v;
}

// Gathers of one row's 16 values of a block into eight packed words.
//  - By tap offsets: addr0 + off[j] for column j (columns past K read zero
//    when nvalid < 16).
//  - By rows (kernels three taps wide): the block's taps lie on six rows of
//    three columns DWB bytes apart; rb[r] is the address of row r's first
//    column and the block starts at column P3 of row 0, so every column step
//    is an immediate of the load.
template <typename T>
__device__ __forceinline__ void gather_taps(uint32_t addr0, const int (&off)[16], int nvalid, uint32_t (&pk)[8]) {
  static_assert(sizeof(T) == 2, "16-bit inputs only");
  uint32_t r[16];
  if (nvalid >= 16) {
#pragma unroll
    for (int j = 0; j < 16; ++j) r[j] = ld_shared_u16(addr0 + static_cast<uint32_t>(off[j]));
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) r[j] = j < nvalid ? ld_shared_u16(addr0 + static_cast<uint32_t>(off[j])) : 0u;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) pk[i] = __byte_perm(r[2 * i], r[2 * i + 1], 0x5410);
}

template <int P3, int DWB, int... J>
__device__ __forceinline__ void gather_rows_seq(const uint32_t (&rb)[6], uint32_t (&r)[16],
                                                std::integer_sequence<int, J...>) {
  ((r[J] = ld_shared_u16_at<((P3 + J) % 3) * DWB>(rb[(P3 + J) / 3])), ...);
}
template <int P3, int DWB>
__device__ __forceinline__ void gather_rows(const uint32_t (&rb)[6], uint32_t (&pk)[8]) {
  uint32_t r[16];
  gather_rows_seq<P3, DWB>(rb, r, std::make_integer_sequence<int, 16>{});
#pragma unroll
  for (int i = 0; i < 8; ++i) pk[i] = __byte_perm(r[2 * i], r[2 * i + 1], 0x5410);
}

// Row bases of a block from its phase-table row (six row offsets), with the
// rows from `split` on moved by `adj` (their channel opens the next slot).
__device__ __forceinline__ void row_bases(uint32_t org, uint32_t prow, int split, int adj, uint32_t (&rb)[6]) {
  int o[8];
  ld_shared_v4(prow, o[0], o[1], o[2], o[3]);
  ld_shared_v4(prow + 16u, o[4], o[5], o[6], o[7]);
#pragma unroll
  for (int r = 0; r < 6; ++r) rb[r] = org + static_cast<uint32_t>(o[r] + (r >= split ? adj : 0));
}

// The 16 tap offsets of a phase-table row.
__device__ __forceinline__ void load_taps(uint32_t prow, int (&off)[16]) {
#pragma unroll
  for (int j = 0; j < 16; j += 4) ld_shared_v4(prow + 4u * j, off[j], off[j + 1], off[j + 2], off[j + 3]);
}

// The 16 tap offsets of a block from a row-gather phase-table row: tap j is
// column (p3 + j) % 3 of row (p3 + j) / 3, p3 = phi % 3.
template <int DWB>
__device__ __forceinline__ void taps_from_rows(uint32_t prow, int p3, int (&off)[16]) {
  int o[8];
  ld_shared_v4(prow, o[0], o[1], o[2], o[3]);
  ld_shared_v4(prow + 16u, o[4], o[5], o[6], o[7]);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int a = j / 3, b = j % 3;  // p3 + j = 3a + b + p3
    const bool wrap = b + p3 >= 3;
    off[j] = (wrap ? o[a + 1 < 8 ? a + 1 : 7] : o[a]) + (b + p3 - (wrap ? 3 : 0)) * DWB;
  }
}

// Quantise (or only convert) one block of a 16-bit input.
template <typename T>
__device__ __forceinline__ void quant8_1(const uint32_t (&pk)[8], bool quant, const QCtx& q, uint32_t (&out)[8]) {
  if (!quant) {
#pragma unroll
    for (int i = 0; i < 8; ++i) out[i] = Half2<T>::to_bf16x2(pk[i]);
    return;
  }
  DqTable dt;
  float inv;
  load_entry(Half2<T>::entry(maxabs8<T>(pk), q), dt, inv);
  quant8<T>(pk, dt, inv, out);
}

// One row x one 16-column block of any input type: the 16 BF16 values of A as
// 8 packed words, gathered by tap offsets (nvalid < 16 only in a partial
// last block).
template <typename T>
__device__ __forceinline__ void row_block(uint32_t addr0, const int (&off)[16], int nvalid, bool quant, const QCtx& q,
                                          uint32_t (&out)[8]) {
  if constexpr (sizeof(T) == 2) {
    uint32_t pk[8];
    gather_taps<T>(addr0, off, nvalid, pk);
    if (!quant) {
#pragma unroll
      for (int i = 0; i < 8; ++i) out[i] = Half2<T>::to_bf16x2(pk[i]);
      return;
    }
    DqTable dt;
    float inv;
    load_entry(Half2<T>::entry(maxabs8<T>(pk), q), dt, inv);
    quant8<T>(pk, dt, inv, out);
  } else {
    float v[16];
    if (nvalid >= 16) {
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(ld_shared_u32(addr0 + static_cast<uint32_t>(off[j])));
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        v[j] = j < nvalid ? __uint_as_float(ld_shared_u32(addr0 + static_cast<uint32_t>(off[j]))) : 0.0f;
    }
    if (!quant) {
#pragma unroll
      for (int i = 0; i < 8; ++i) out[i] = cvt_bf16x2(v[2 * i + 1], v[2 * i]);
      return;
    }
    float bmax = fabsf(v[0]);
#pragma unroll
    for (int j = 1; j < 16; ++j) bmax = fmaxf(bmax, fabsf(v[j]));
    DqTable dt;
    float inv;
    load_entry(entry_of_max(bmax, q), dt, inv);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = 4 * i;
      // sign bits of (v[j], v[j+1]) and (v[j+2], v[j+3]) at bits 15 and 31
      const uint32_t s01 = __byte_perm(__float_as_uint(v[j]), __float_as_uint(v[j + 1]), 0x7632);
      const uint32_t s23 = __byte_perm(__float_as_uint(v[j + 2]), __float_as_uint(v[j + 3]), 0x7632);
      dq4(dt, __fmul_rn(fabsf(v[j]), inv), __fmul_rn(fabsf(v[j + 1]), inv), __fmul_rn(fabsf(v[j + 2]), inv),
          __fmul_rn(fabsf(v[j + 3]), inv), s01, s23, out[2 * i], out[2 * i + 1]);
    }
  }
}

// ---------------------------------------------------------------------------
// NVFP4 operands of the block-scaled MMA variant.  Per block: the E2M1 codes
// of v * (1/scale) (the sign travels through the conversion) and the E4M3
// scale byte, both from the block's quantiser entry (word 4: 1/scale, word 5:
// the scale byte, 0 when the block takes the 1.0 fallback scale, which is no
// E4M3 value times g: such a block contributes nothing).
// ---------------------------------------------------------------------------

__device__ __forceinline__ void st_shared_v2(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ void st_shared_u8(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u8 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(static_cast<unsigned short>(v)) : "memory");
}

// (v0 * s, v1 * s), each product rounded to nearest binary32, as one packed
// f32x2 multiply.
__device__ __forceinline__ void mul2_rn(float v0, float v1, float s, float& a0, float& a1) {
  asm("{\n\t.reg .b64 x, y, z;\n\t"
      "mov.b64 x, {%2, %3};\n\t"
      "mov.b64 y, {%4, %4};\n\t"
      "mul.rn.f32x2 z, x, y;\n\t"
      "mov.b64 {%0, %1}, z;\n\t}"
      : "=f"(a0), "=f"(a1)
      : "f"(v0), "f"(v1), "f"(s));
}

// E2M1 codes (round to nearest even, saturating) of eight scaled values,
// value i in nibble i.
__device__ __forceinline__ uint32_t e2m1_pack8(const float* a) {
  uint32_t r;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(r)
      : "f"(a[0]), "f"(a[1]), "f"(a[2]), "f"(a[3]), "f"(a[4]), "f"(a[5]), "f"(a[6]), "f"(a[7]));
  return r;
}

// Signed binary32 values of the two halves of a packed 16-bit pair.
template <typename T>
__device__ __forceinline__ float half_lo(uint32_t w);
template <typename T>
__device__ __forceinline__ float half_hi(uint32_t w);
template <>
__device__ __forceinline__ float half_lo<__nv_bfloat16>(uint32_t w) { return __uint_as_float(w << 16); }
template <>
__device__ __forceinline__ float half_hi<__nv_bfloat16>(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
template <>
__device__ __forceinline__ float half_lo<__half>(uint32_t w) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xFFFFu)));
}
template <>
__device__ __forceinline__ float half_hi<__half>(uint32_t w) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
}

__device__ __forceinline__ void load_fp4_entry(uint32_t e, float& inv, uint32_t& sbyte) {
  uint32_t a, b;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(a), "=r"(b) : "r"(e + 16u));
  inv = __uint_as_float(a);
  sbyte = b;
}

// Codes of one block of a 16-bit input held as eight packed words.
template <typename T>
__device__ __forceinline__ void fp4_codes16(const uint32_t (&pk)[8], float inv, uint32_t& c0, uint32_t& c1) {
  float a[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) mul2_rn(half_lo<T>(pk[i]), half_hi<T>(pk[i]), inv, a[2 * i], a[2 * i + 1]);
  c0 = e2m1_pack8(a);
  c1 = e2m1_pack8(a + 8);
}

template <typename T>
__device__ __forceinline__ void fp4_block(const uint32_t (&pk)[8], const QCtx& q, uint32_t& c0, uint32_t& c1,
                                          uint32_t& sbyte) {
  float inv;
  load_fp4_entry(Half2<T>::entry(maxabs8<T>(pk), q), inv, sbyte);
  fp4_codes16<T>(pk, inv, c0, c1);
}

// Two blocks (two rows, or two blocks of one row) with interleaved chains.
template <typename T>
__device__ __forceinline__ void fp4_block_x2(const uint32_t (&pa)[8], const uint32_t (&pb)[8], const QCtx& q,
                                             uint32_t& ca0, uint32_t& ca1, uint32_t& sa, uint32_t& cb0, uint32_t& cb1,
                                             uint32_t& sb) {
  const uint32_t ea = Half2<T>::entry(maxabs8<T>(pa), q), eb = Half2<T>::entry(maxabs8<T>(pb), q);
  float ia, ib;
  load_fp4_entry(ea, ia, sa);
  load_fp4_entry(eb, ib, sb);
  fp4_codes16<T>(pa, ia, ca0, ca1);
  fp4_codes16<T>(pb, ib, cb0, cb1);
}

// ---- 32-column groups (NVFP4 blocks of 32, MXFP4) ----
//
// The dequantisation table of a scale by direct products, each q * s
// rounded to binary32 and then to BF16 like every other entry.  An MXFP4
// scale 2^E reaches the subnormal and the overflow ends of binary32, where
// the exponent-field steps of dq_table do not hold.
__device__ __forceinline__ DqTable dq_table_direct(float s) {
  const uint32_t p01 = cvt_bf16x2(__fmul_rn(0.5f, s), __fmul_rn(0.0f, s));
  const uint32_t p23 = cvt_bf16x2(__fmul_rn(1.5f, s), s);
  const uint32_t p45 = cvt_bf16x2(__fmul_rn(3.0f, s), __fmul_rn(2.0f, s));
  const uint32_t p67 = cvt_bf16x2(__fmul_rn(6.0f, s), __fmul_rn(4.0f, s));
  DqTable t;
  t.lo_a = __byte_perm(p01, p23, 0x6420);
  t.hi_a = __byte_perm(p01, p23, 0x7531);
  t.lo_b = __byte_perm(p45, p67, 0x6420);
  t.hi_b = __byte_perm(p45, p67, 0x7531);
  return t;
}

// The MXFP4 scale 2^E of a group from its |v| maximum: its table and
// down = 2^-E (an all-zero group gets E = -127 and only zero codes).
__device__ __forceinline__ void mx_group_scale(float gmax, float dst_max, DqTable& dt, float& down) {
  const int e = mx_scale_exp(gmax, dst_max);
  down = mx_exp2i(-e);
  dt = dq_table_direct(mx_exp2i(e));
}

// Two 16-column blocks of one row (eight packed words each) that form one
// 32-column group: the joint maximum sets one scale for both.
template <typename T>
__device__ __forceinline__ void quant_group32(const uint32_t (&pa)[8], const uint32_t (&pb)[8], int qmode,
                                              float dst_max, const QCtx& q, uint32_t (&wa)[8], uint32_t (&wb)[8]) {
  using H = Half2<T>;
  uint32_t m = H::maxabs(maxabs8<T>(pa), maxabs8<T>(pb));
  // blocks of 64: the row's other 32 columns are held by lane ^ 16 (every
  // lane of the warp reaches this shuffle)
  if (qmode == kQModeNv64) m = H::maxabs(m, __shfl_xor_sync(0xffffffffu, m, 16));
  DqTable dt;
  float inv;
  if (qmode != kQModeMx)
    load_entry(H::entry(m, q), dt, inv);
  else
    mx_group_scale(fmaxf(H::abs_lo(m), H::abs_hi(m)), dst_max, dt, inv);
  quant8<T>(pa, dt, inv, wa);
  quant8<T>(pb, dt, inv, wb);
}

// The same for binary32 inputs (16 values per block).
__device__ __forceinline__ void quant_group32_f32(const float (&va)[16], const float (&vb)[16], int qmode,
                                                  float dst_max, const QCtx& q, uint32_t (&wa)[8],
                                                  uint32_t (&wb)[8]) {
  float gmax = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) gmax = fmaxf(gmax, fmaxf(fabsf(va[j]), fabsf(vb[j])));
  if (qmode == kQModeNv64) gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, 16));
  DqTable dt;
  float inv;
  if (qmode != kQModeMx)
    load_entry(entry_of_max(gmax, q), dt, inv);
  else
    mx_group_scale(gmax, dst_max, dt, inv);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = 4 * i;
    uint32_t s01 = __byte_perm(__float_as_uint(va[j]), __float_as_uint(va[j + 1]), 0x7632);
    uint32_t s23 = __byte_perm(__float_as_uint(va[j + 2]), __float_as_uint(va[j + 3]), 0x7632);
    dq4(dt, __fmul_rn(fabsf(va[j]), inv), __fmul_rn(fabsf(va[j + 1]), inv), __fmul_rn(fabsf(va[j + 2]), inv),
        __fmul_rn(fabsf(va[j + 3]), inv), s01, s23, wa[2 * i], wa[2 * i + 1]);
    s01 = __byte_perm(__float_as_uint(vb[j]), __float_as_uint(vb[j + 1]), 0x7632);
    s23 = __byte_perm(__float_as_uint(vb[j + 2]), __float_as_uint(vb[j + 3]), 0x7632);
    dq4(dt, __fmul_rn(fabsf(vb[j]), inv), __fmul_rn(fabsf(vb[j + 1]), inv), __fmul_rn(fabsf(vb[j + 2]), inv),
        __fmul_rn(fabsf(vb[j + 3]), inv), s01, s23, wb[2 * i], wb[2 * i + 1]);
  }
}

// One block's 16 tap offsets from its phase-table row, the columns from
// `split` on moved by `adj` (their channel opens the next halo slot).
template <int kDWB>
__device__ __forceinline__ void block_taps(uint32_t prow, int phi, int split, int adj, int (&off)[16]) {
  if constexpr (kDWB > 0)
    taps_from_rows<kDWB>(prow, phi % 3, off);
  else
    load_taps(prow, off);
  if (adj != 0) {
#pragma unroll
    for (int j = 0; j < 16; ++j) off[j] += (j >= split) ? adj : 0;
  }
}

// One row's 32-column group by tap offsets: block a at addr_a with nv_a
// valid columns, block b (the next 16 columns) at addr_b with nv_b (<= 0:
// past K, zeros).
template <typename T, int kDWB>
__device__ __forceinline__ void group32_taps(uint32_t addr_a, uint32_t prow_a, int phi_a, int split_a, int adj_a,
                                             int nv_a, uint32_t addr_b, uint32_t prow_b, int phi_b, int split_b,
                                             int adj_b, int nv_b, int qmode, float dst_max, const QCtx& q,
                                             uint32_t (&wa)[8], uint32_t (&wb)[8]) {
  int off[16];
  if constexpr (sizeof(T) == 2) {
    uint32_t pa[8], pb[8];
    block_taps<kDWB>(prow_a, phi_a, split_a, adj_a, off);
    gather_taps<T>(addr_a, off, nv_a, pa);
    if (nv_b > 0) {
      block_taps<kDWB>(prow_b, phi_b, split_b, adj_b, off);
      gather_taps<T>(addr_b, off, nv_b, pb);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) pb[i] = 0u;
    }
    quant_group32<T>(pa, pb, qmode, dst_max, q, wa, wb);
  } else {
    float va[16], vb[16];
    block_taps<kDWB>(prow_a, phi_a, split_a, adj_a, off);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      va[j] = j < nv_a ? __uint_as_float(ld_shared_u32(addr_a + static_cast<uint32_t>(off[j]))) : 0.0f;
    if (nv_b > 0) block_taps<kDWB>(prow_b, phi_b, split_b, adj_b, off);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      vb[j] = j < nv_b ? __uint_as_float(ld_shared_u32(addr_b + static_cast<uint32_t>(off[j]))) : 0.0f;
    quant_group32_f32(va, vb, qmode, dst_max, q, wa, wb);
  }
}

// One row x one 16-column block of any input type, gathered by tap offsets
// (nvalid < 16 only in a partial last block: the missing columns are zero).
template <typename T>
__device__ __forceinline__ void fp4_row_block(uint32_t addr0, const int (&off)[16], int nvalid, const QCtx& q,
                                              uint32_t& c0, uint32_t& c1, uint32_t& sbyte) {
  if constexpr (sizeof(T) == 2) {
    uint32_t pk[8];
    gather_taps<T>(addr0, off, nvalid, pk);
    fp4_block<T>(pk, q, c0, c1, sbyte);
  } else {
    float v[16];
    if (nvalid >= 16) {
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(ld_shared_u32(addr0 + static_cast<uint32_t>(off[j])));
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        v[j] = j < nvalid ? __uint_as_float(ld_shared_u32(addr0 + static_cast<uint32_t>(off[j]))) : 0.0f;
    }
    float bmax = fabsf(v[0]);
#pragma unroll
    for (int j = 1; j < 16; ++j) bmax = fmaxf(bmax, fabsf(v[j]));
    float inv;
    load_fp4_entry(entry_of_max(bmax, q), inv, sbyte);
    float a[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) mul2_rn(v[2 * i], v[2 * i + 1], inv, a[2 * i], a[2 * i + 1]);
    c0 = e2m1_pack8(a);
    c1 = e2m1_pack8(a + 8);
  }
}

// Store one row-block of the A stage: 8 bytes of codes and the scale byte.
__device__ __forceinline__ void fp4_put(uint32_t code_addr, uint32_t sf_addr, uint32_t c0, uint32_t c1,
                                        uint32_t sbyte) {
  st_shared_v2(code_addr, c0, c1);
  st_shared_u8(sf_addr, sbyte);
}

// Column step in bytes of the row gather (kernels three taps wide, 16-bit
// input, W dilation 1 or 2), or 0 where the tap-offset gather applies.
__host__ __device__ inline int row_gather_step(const ConvGeom& g, int esz) {
  return (esz == 2 && g.KW == 3 && (g.dw == 1 || g.dw == 2)) ? g.dw * esz : 0;
}

struct MmaBars {
  uint32_t a_full, b_full, a_empty, b_empty, acc_full, acc_empty, drain;
};

// The MMA issuer, run by a whole warp: per K slice, wait for the A stage and
// the weight stage, issue n_mt x n_sub x 4 tcgen05.mma (A from TMEM, B from
// shared memory, K = 16 each), commit the accumulators after the tile's last
// slice and the two stages after every slice.  Every lane computes the same
// operands and one elected lane issues, so the operands are warp-uniform;
// wait results are combined over the warp so all lanes take the same path.
// NMT / NSUB fix the subtile and N-part counts at compile time (0: taken from
// the plan), so the common shapes issue straight-line code.
// kSmemA: A is a 128B-swizzled K-major tile in shared memory (16 KB per
// subtile), read through a descriptor like B; otherwise A is in TMEM.
template <int NMT, int NSUB, bool kSmemA = false>
__device__ __forceinline__ void mma_issue_loop(const TmemParams& p, uint32_t base, uint32_t tmem_base,
                                               const MmaBars& b, volatile int* abort_flag) {
  const int n_mt = NMT ? NMT : p.n_mt;
  const int n_sub = NSUB ? NSUB : p.n_sub;
  const uint32_t idesc = umma_idesc_bf16_f32(128, static_cast<uint32_t>(p.sub_n));
  const uint32_t sub_cols = static_cast<uint32_t>(p.sub_n);
  const uint32_t tile_cols = static_cast<uint32_t>(p.n_tile);
  const uint64_t bsub_step = static_cast<uint64_t>(p.sub_n * 8);  // descriptor units of 16 B
  uint32_t it = 0;
  RingPos ap{0u, 0u}, bp{0u, 0u};
  bool ok = true;
  for (int64_t t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x, ++it) {
    // accumulator buffer of this tile and how many tiles used it before
    const uint32_t buf = p.acc_bufs == 2 ? (it & 1u) : 0u, use = p.acc_bufs == 2 ? (it >> 1) : it;
    const int abase = static_cast<int>(buf) * n_mt * n_sub;
    const uint32_t acc_base = tmem_base + buf * static_cast<uint32_t>(p.acc_cols);
    for (int s = 0; ok && s < p.ks; ++s, ap.next(static_cast<uint32_t>(p.sa)), bp.next(static_cast<uint32_t>(p.sb))) {
      const uint32_t ea = ap.e, eb = bp.e;
      ok = wait_or_abort(b.a_full + 8u * ea, ap.ph, p.err, kSiteAStageFull, abort_flag) &&
           wait_or_abort(b.b_full + 8u * eb, bp.ph, p.err, kSiteTmaFull, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t a_stage = kSmemA ? base + p.off_a + ea * p.a_stage_bytes
                                      : tmem_base + static_cast<uint32_t>(p.a_col0) + ea * static_cast<uint32_t>(n_mt * 32);
      const uint64_t bdesc = umma_desc_kmajor_sw128(base + p.off_b + eb * p.b_stage_bytes);
      const bool first = (s == 0), last = (s == p.ks - 1);
#pragma unroll
      for (int i = 0; i < (NMT ? NMT : 4); ++i) {
        if (!NMT && i >= n_mt) break;
#pragma unroll
        for (int ns = 0; ns < (NSUB ? NSUB : 2); ++ns) {
          if (!NSUB && ns >= n_sub) break;
          const int acc = abase + i * n_sub + ns;
          if (first && use > 0 && ok) {
            ok = __all_sync(0xffffffffu,
                            wait_or_abort(b.acc_empty + 8u * acc, (use - 1u) & 1u, p.err, kSiteAccEmpty, abort_flag));
            tc_fence_after();
          }
          if (ok) {
            const uint32_t d_tmem =
                acc_base + static_cast<uint32_t>(i) * tile_cols + static_cast<uint32_t>(ns) * sub_cols;
            const uint64_t bsub = bdesc + static_cast<uint64_t>(ns) * bsub_step;
            if constexpr (kSmemA) {
              // K advances 32 bytes (16 BF16) inside the 128-byte swizzle atom
              const uint64_t asub = umma_desc_kmajor_sw128(a_stage + static_cast<uint32_t>(i) * 16384u);
#pragma unroll
              for (int j = 0; j < kBlockK / 16; ++j)
                umma_bf16_ss_elect(d_tmem, asub + static_cast<uint64_t>(2 * j), bsub + static_cast<uint64_t>(2 * j),
                                   idesc, (first && j == 0) ? 0u : 1u);
            } else {
              const uint32_t a_sub = a_stage + static_cast<uint32_t>(i * 32);
#pragma unroll
              for (int j = 0; j < kBlockK / 16; ++j)
                umma_bf16_ts_elect(d_tmem, a_sub + 8u * j, bsub + static_cast<uint64_t>(2 * j), idesc,
                                   (first && j == 0) ? 0u : 1u);
            }
            if (last) umma_commit_elect(b.acc_full + 8u * acc);
          }
        }
      }
      if (!ok) break;
      umma_commit_elect(b.a_empty + 8u * ea);
      umma_commit_elect(b.b_empty + 8u * eb);
    }
  }
  if (!ok) {
    umma_commit_elect(b.drain);
    mbar_wait(b.drain, 0, p.err, kSiteDrain);
  }
}

// The MMA issuer of the NVFP4-operand variant.  Per K slice (one MMA of
// K = 64 per subtile and N-part): wait for the A stage and the weight stage,
// copy the slice's scale factors into the A stage's tensor-memory region
// (one 32-row atom per subtile, n_atoms per N-part; the copies execute in
// order with the MMAs issued after them), then issue the block-scaled MMAs
// with both operands in shared memory.  The accumulators, the waits on them
// and the commits are those of the BF16 loop.
template <int NMT, int NSUB>
__device__ __forceinline__ void mma_issue_loop_fp4(const TmemParams& p, uint32_t base, uint32_t tmem_base,
                                                   const MmaBars& b, volatile int* abort_flag) {
  const int n_mt = NMT ? NMT : p.n_mt;
  const int n_sub = NSUB ? NSUB : p.n_sub;
  const uint32_t idesc = umma_idesc_nvfp4(128, static_cast<uint32_t>(p.sub_n));
  const uint32_t sub_cols = static_cast<uint32_t>(p.sub_n);
  const uint32_t tile_cols = static_cast<uint32_t>(p.n_tile);
  const uint32_t codes_a = static_cast<uint32_t>(n_mt) * 4096u;  // the A stage's scale atoms follow its codes
  const uint32_t codes_b = static_cast<uint32_t>(p.sub_n) * 32u;  // an image's scale atoms follow its codes
  uint32_t it = 0;
  RingPos ap{0u, 0u}, bp{0u, 0u};
  bool ok = true;
  for (int64_t t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x, ++it) {
    // accumulator buffer of this tile and how many tiles used it before
    const uint32_t buf = p.acc_bufs == 2 ? (it & 1u) : 0u, use = p.acc_bufs == 2 ? (it >> 1) : it;
    const int abase = static_cast<int>(buf) * n_mt * n_sub;
    const uint32_t acc_base = tmem_base + buf * static_cast<uint32_t>(p.acc_cols);
    for (int s = 0; ok && s < p.ks; ++s, ap.next(static_cast<uint32_t>(p.sa)), bp.next(static_cast<uint32_t>(p.sb))) {
      const uint32_t ea = ap.e, eb = bp.e;
      ok = wait_or_abort(b.a_full + 8u * ea, ap.ph, p.err, kSiteAStageFull, abort_flag) &&
           wait_or_abort(b.b_full + 8u * eb, bp.ph, p.err, kSiteTmaFull, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t a_st = base + p.off_a + ea * p.a_stage_bytes;
      const uint32_t b_st = base + p.off_b + eb * p.b_stage_bytes;
      const uint32_t sfa = tmem_base + static_cast<uint32_t>(p.sf_col0) + ea * static_cast<uint32_t>(p.sf_cols);
      const uint32_t sfb = sfa + 4u * static_cast<uint32_t>(n_mt);
#pragma unroll
      for (int i = 0; i < (NMT ? NMT : 4); ++i) {
        if (!NMT && i >= n_mt) break;
        tmem_cp_sf_atom_elect(sfa + 4u * i, umma_desc_sf_atom(a_st + codes_a + 512u * i));
      }
      for (int ns = 0; ns < n_sub; ++ns)
        for (int a = 0; a < p.n_atoms; ++a)
          tmem_cp_sf_atom_elect(sfb + 4u * static_cast<uint32_t>(ns * p.n_atoms + a),
                                umma_desc_sf_atom(b_st + ns * p.b_img_bytes + codes_b + 512u * a));
      const bool first = (s == 0), last = (s == p.ks - 1);
#pragma unroll
      for (int i = 0; i < (NMT ? NMT : 4); ++i) {
        if (!NMT && i >= n_mt) break;
#pragma unroll
        for (int ns = 0; ns < (NSUB ? NSUB : 2); ++ns) {
          if (!NSUB && ns >= n_sub) break;
          const int acc = abase + i * n_sub + ns;
          if (first && use > 0 && ok) {
            ok = __all_sync(0xffffffffu,
                            wait_or_abort(b.acc_empty + 8u * acc, (use - 1u) & 1u, p.err, kSiteAccEmpty, abort_flag));
            tc_fence_after();
          }
          if (ok) {
            const uint32_t d_tmem =
                acc_base + static_cast<uint32_t>(i) * tile_cols + static_cast<uint32_t>(ns) * sub_cols;
            umma_nvfp4_ss_elect(d_tmem, umma_desc_kmajor_sw32(a_st + 4096u * i),
                                umma_desc_kmajor_sw32(b_st + ns * p.b_img_bytes), idesc, sfa + 4u * i,
                                sfb + 4u * static_cast<uint32_t>(ns * p.n_atoms), first ? 0u : 1u);
            if (last) umma_commit_elect(b.acc_full + 8u * acc);
          }
        }
      }
      if (!ok) break;
      umma_commit_elect(b.a_empty + 8u * ea);
      umma_commit_elect(b.b_empty + 8u * eb);
    }
  }
  if (!ok) {
    umma_commit_elect(b.drain);
    mbar_wait(b.drain, 0, p.err, kSiteDrain);
  }
}

// kPairs: the tile has at least two M-subtiles, built in interleaved pairs
// (a separate instantiation, so single-subtile tiles keep their register
// allocation).  kDWB > 0: 16-bit input and a kernel three taps wide whose
// taps along W are kDWB bytes apart (dilation * element size), gathered by
// rows with immediate column offsets; 0: gathered by tap offsets.  kFp4: the
// NVFP4-operand variant (A as E2M1 codes and scale bytes in shared memory,
// prepacked NVFP4 weights, block-scaled MMA, the two global scales applied
// in the epilogue); otherwise BF16 operands with A in tensor memory.  kQ = 1:
// the activation quantiser works on 32-column groups (NVFP4 blocks of 32 or
// MXFP4, p.qmode), a separate instantiation so the default quantiser's
// forms keep their code; 0: blocks of 16, or no quantisation.
template <typename T, bool kPairs, int kDWB, int kAOp, int kQ = 0>
__global__ void __launch_bounds__(kThreads, 1)
    conv3d_igemm_tmem_kernel(const __grid_constant__ TmemParams p, const __grid_constant__ CUtensorMap tmap_x,
                             const __grid_constant__ CUtensorMap tmap_w) {
  constexpr bool kFp4 = kAOp == kAOpNvfp4;
  constexpr bool kSmemA = kAOp != kAOpBf16Tmem;
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

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.ring; ++i) {
      mbar_init(bar_halo_full + 8u * i, 1);
      mbar_init(bar_halo_empty + 8u * i, kNumXfWarps);  // every transform warp hands the slot back
    }
    for (int i = 0; i < p.sb; ++i) {
      mbar_init(bar_b_full + 8u * i, 1);
      mbar_init(bar_b_empty + 8u * i, 1);
    }
    for (int i = 0; i < p.sa; ++i) {
      mbar_init(bar_a_full + 8u * i, kNumXfWarps / 2);  // the 8 warps of the slice's group
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
    if (!kFp4) tma_prefetch_desc(&tmap_w);
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kWarpB) {
    // ------------------------------------------------------------ weight producer
    if (lane == 0) {
      uint32_t gb = 0;  // weight stages issued
      RingPos bp{0u, 0u};
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        const TileCoord tc = decode_tile(p, t);
        for (int s = 0; s < p.ks; ++s, ++gb, bp.next(static_cast<uint32_t>(p.sb))) {
          const uint32_t e = bp.e;
          if (gb >= static_cast<uint32_t>(p.sb) &&
              !wait_or_abort(bar_b_empty + 8u * e, bp.ph ^ 1u, p.err, kSiteProducerEmpty, abort_flag)) {
            ok = false;
            break;
          }
          if constexpr (kFp4) {
            // the tile's n_sub images of this slice are adjacent: one bulk copy
            const uint32_t bytes = static_cast<uint32_t>(p.n_sub) * p.b_img_bytes;
            mbar_arrive_expect_tx(bar_b_full + 8u * e, bytes);
            bulk_load(base + p.off_b + e * p.b_stage_bytes,
                      p.wq + (static_cast<int64_t>(s) * p.n_parts + static_cast<int64_t>(tc.nt) * p.n_sub) * p.b_img_bytes,
                      bytes, bar_b_full + 8u * e);
          } else {
            mbar_arrive_expect_tx(bar_b_full + 8u * e, p.b_stage_bytes);
            for (int i = 0; i < p.n_sub; ++i)
              tma_load_2d(base + p.off_b + e * p.b_stage_bytes + static_cast<uint32_t>(i * p.sub_n) * 128u, &tmap_w,
                          bar_b_full + 8u * e, kBlockK * s, tc.nt * p.n_tile + i * p.sub_n);
          }
        }
      }
      if (!ok) drain_ring(bar_b_full, static_cast<uint32_t>(p.sb), gb, p.err, kSiteDrain);
    }
  } else if (warp == kWarpHalo) {
    // ------------------------------------------------------------ halo producer
    if (lane == 0) {
      uint32_t gs = 0;  // halo slots issued
      RingPos hp{0u, 0u};
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        const TileCoord tc = decode_tile(p, t);
        const int w0 = halo_w0(p, tc.ow0);
        const int h0 = tc.oh0 * g.sh - g.ph;
        const int d0 = tc.od * g.sd - g.pd;
        for (int q = 0; q < p.q_slots; ++q, ++gs, hp.next(static_cast<uint32_t>(p.ring))) {
          const uint32_t e = hp.e;
          if (gs >= static_cast<uint32_t>(p.ring) &&
              !wait_or_abort(bar_halo_empty + 8u * e, hp.ph ^ 1u, p.err, kSiteHaloEmpty, abort_flag)) {
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
    // ------------------------------------------------------------ MMA issuer (whole warp)
    {
      const MmaBars bars{bar_a_full, bar_b_full, bar_a_empty, bar_b_empty, bar_acc_full, bar_acc_empty, bar_drain};
      const uint32_t tb = __shfl_sync(0xffffffffu, tmem_base, 0);
      if constexpr (kFp4) {
        switch (p.n_mt * 4 + p.n_sub) {
          case 1 * 4 + 1: mma_issue_loop_fp4<1, 1>(p, base, tb, bars, abort_flag); break;
          case 2 * 4 + 1: mma_issue_loop_fp4<2, 1>(p, base, tb, bars, abort_flag); break;
          default: mma_issue_loop_fp4<0, 0>(p, base, tb, bars, abort_flag); break;
        }
      } else {
        switch (p.n_mt * 4 + p.n_sub) {  // straight-line issue for the common shapes
          case 1 * 4 + 1: mma_issue_loop<1, 1, kSmemA>(p, base, tb, bars, abort_flag); break;
          case 1 * 4 + 2: mma_issue_loop<1, 2, kSmemA>(p, base, tb, bars, abort_flag); break;
          case 2 * 4 + 1: mma_issue_loop<2, 1, kSmemA>(p, base, tb, bars, abort_flag); break;
          case 2 * 4 + 2: mma_issue_loop<2, 2, kSmemA>(p, base, tb, bars, abort_flag); break;
          case 4 * 4 + 1: mma_issue_loop<4, 1, kSmemA>(p, base, tb, bars, abort_flag); break;
          default: mma_issue_loop<0, 0, kSmemA>(p, base, tb, bars, abort_flag); break;
        }
      }
      __syncwarp();
    }
  } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + 4) {
    // ------------------------------------------------------------ epilogue
    // Warp qw drains TMEM lanes 32*qw.. (subtile rows = output positions), 16
    // channels per step: tcgen05.ld gives each lane its position's 16 FP32
    // accumulators, the bias is added in FP32 and the result rounded to the
    // output dtype, and the 32 positions x 16 channels pass through the
    // warp's shared staging rows (one row of 32 positions per channel), so
    // that each lane then writes kPer consecutive ow of one channel as one
    // 16-byte store.  A lane's store unit covers positions kPer*gq..+kPer-1 of
    // the warp (one row segment, since kPer divides TW), the same for every
    // step; units at the ragged edge of OW fall back to element stores.  When
    // OW is not a multiple of kPer (or y is not 16-byte aligned) no row start
    // is aligned, and each lane instead writes its own position for the 16
    // channels (consecutive lanes hold consecutive ow).  The accumulator is
    // handed back to the MMA as soon as its last step is in registers.
    constexpr int kEsz = static_cast<int>(sizeof(T));
    constexpr int kPer = 16 / kEsz;          // positions per 16-byte store
    constexpr int kGroups = 32 / kPer;       // store units per channel row
    constexpr int kUnits = kGroups / 2;      // store units per lane per step (16 channels x kGroups / 32)
    constexpr uint32_t kPitch = 32 * kEsz + 16;
    const int qw = warp - kWarpEpi0;  // == warp % 4: TMEM lanes 32*qw..
    const uint32_t stage = base + p.off_epi + static_cast<uint32_t>(qw) * 16u * kPitch;
    const int gq = lane % kGroups;           // this lane's position group
    const int r0 = qw * 32 + gq * kPer;      // its first row within a subtile
    const int th_u = r0 / p.TW, tw_u = r0 % p.TW;
    const int S_hw = g.OH * g.OW;
    const int64_t S = static_cast<int64_t>(g.OD) * S_hw;
    const bool vec_ok = p.y_vec != 0;
    T* y = static_cast<T*>(p.y);
    const T* bias = static_cast<const T*>(p.bias);
    // NVFP4 operands: the accumulator is in units of g_act * g_w
    float gg = 1.0f;
    if constexpr (kFp4) gg = __fmul_rn(nvfp4_global(__ldg(p.act_amax)).g, __ldg(p.g_w));
    uint32_t it = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x, ++it) {
      const TileCoord tc = decode_tile(p, t);
      const int ow = tc.ow0 + tw_u;
      const uint32_t buf = p.acc_bufs == 2 ? (it & 1u) : 0u, use = p.acc_bufs == 2 ? (it >> 1) : it;
      for (int i = 0; ok && i < p.n_mt; ++i) {
        const int oh = tc.oh0 + i * p.TH + th_u;
        const bool row_ok = oh < g.OH && ow < g.OW;
        const bool full = row_ok && ow + kPer <= g.OW;
        const int64_t ubase = (static_cast<int64_t>(tc.n) * g.Cout) * S + static_cast<int64_t>(tc.od) * S_hw +
                              static_cast<int64_t>(oh) * g.OW + ow;
        for (int ns = 0; ns < p.n_sub; ++ns) {
          const int acc = static_cast<int>(buf) * p.n_mt * p.n_sub + i * p.n_sub + ns;
          if (!wait_or_abort(bar_acc_full + 8u * acc, use & 1u, p.err, kSiteAccFull, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int co0 = tc.nt * p.n_tile + ns * p.sub_n;
          const uint32_t taddr = tmem_base + (static_cast<uint32_t>(qw * 32) << 16) + buf * static_cast<uint32_t>(p.acc_cols) +
                                 static_cast<uint32_t>(i * p.n_tile + ns * p.sub_n);
          if constexpr (kEsz == 2) {
            if (vec_ok) {
              // 16-bit outputs in 16-byte stores: the 16x256b TMEM shape gives
              // each thread channel pairs of two positions, which stmatrix
              // stores transposed straight into the staging rows (channel j:
              // 32 positions), two shared-memory stores per step instead of
              // one per channel.  Thread t's stmatrix row: channel
              // 8 (mi / 2) + t % 8, position group 2 hh + mi % 2, mi = t / 8.
              const int mi = lane >> 3;
              const uint32_t srow = stage + static_cast<uint32_t>(8 * (mi >> 1) + (lane & 7)) * kPitch +
                                    static_cast<uint32_t>(mi & 1) * 16u;
              const int cpair = 2 * (lane & 3);  // the thread's first channel in each 8-channel half
              uint32_t nv[16];
              tmem_ld_16x256b_x2(taddr, *reinterpret_cast<uint32_t(*)[8]>(&nv[0]));
              tmem_ld_16x256b_x2(taddr + (16u << 16), *reinterpret_cast<uint32_t(*)[8]>(&nv[8]));
              for (int c0 = 0; c0 < p.sub_n; c0 += 16) {
                uint32_t v[16];
                tmem_wait_ld_regs(nv);
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = nv[j];
                if (c0 + 16 < p.sub_n) {
                  const uint32_t tn = taddr + static_cast<uint32_t>(c0 + 16);
                  tmem_ld_16x256b_x2(tn, *reinterpret_cast<uint32_t(*)[8]>(&nv[0]));
                  tmem_ld_16x256b_x2(tn + (16u << 16), *reinterpret_cast<uint32_t(*)[8]>(&nv[8]));
                } else {  // the accumulator is in registers: hand it back
                  tc_fence_before();
                  __syncwarp();
                  const bool withhold = p.withhold_arrive && blockIdx.x == 0 && it == 0 && acc == 0 && qw == 0;
                  if (lane == 0 && !withhold) mbar_arrive(bar_acc_empty + 8u * acc);
                }
                // scale, bias, rounding to channel pairs: m[4 hh + 2 cc + bot]
                // is positions 16 hh + 8 bot + lane / 4, channels 8 cc + cpair + {0, 1}
                uint32_t m[8];
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                  const int co = co0 + c0 + 8 * cc + cpair;
                  float b0 = 0.0f, b1 = 0.0f;
                  if (bias) {
                    if (co < g.Cout) b0 = DTypeOps<T>::to_f32(__ldg(bias + co));
                    if (co + 1 < g.Cout) b1 = DTypeOps<T>::to_f32(__ldg(bias + co + 1));
                  }
#pragma unroll
                  for (int hb = 0; hb < 4; ++hb) {  // hb = 2 hh + bot
                    const int src = (hb >> 1) * 8 + cc * 4 + (hb & 1) * 2;
                    float f0 = __uint_as_float(v[src]), f1 = __uint_as_float(v[src + 1]);
                    if constexpr (kFp4) {
                      f0 = __fmul_rn(f0, gg);
                      f1 = __fmul_rn(f1, gg);
                    }
                    if (bias) {
                      f0 = __fadd_rn(f0, b0);
                      f1 = __fadd_rn(f1, b1);
                    }
                    uint32_t w;
                    if constexpr (std::is_same<T, __half>::value) {
                      const __half2 h = __floats2half2_rn(f0, f1);
                      memcpy(&w, &h, 4);
                    } else {
                      w = cvt_bf16x2(f1, f0);
                    }
                    m[(hb >> 1) * 4 + cc * 2 + (hb & 1)] = w;
                  }
                }
                stmatrix_x4_trans(srow, m[0], m[1], m[2], m[3]);
                stmatrix_x4_trans(srow + 32u, m[4], m[5], m[6], m[7]);
                __syncwarp();
#pragma unroll
                for (int k = 0; k < kUnits; ++k) {
                  const int j = lane / kGroups + k * (32 / kGroups);
                  const int co = co0 + c0 + j;
                  if (co < g.Cout && row_ok) {
                    const uint32_t a = stage + static_cast<uint32_t>(j) * kPitch + static_cast<uint32_t>(gq * 16);
                    int w0, w1, w2, w3;
                    ld_shared_v4(a, w0, w1, w2, w3);
                    T* dst = y + ubase + static_cast<int64_t>(co) * S;
                    if (full) {
                      __stcs(reinterpret_cast<int4*>(dst), make_int4(w0, w1, w2, w3));
                    } else {
                      const uint32_t ws[4] = {static_cast<uint32_t>(w0), static_cast<uint32_t>(w1),
                                              static_cast<uint32_t>(w2), static_cast<uint32_t>(w3)};
#pragma unroll
                      for (int e = 0; e < kPer; ++e) {
                        if (ow + e < g.OW) {
                          const unsigned short b = static_cast<unsigned short>(ws[e >> 1] >> (16 * (e & 1)));
                          memcpy(dst + e, &b, 2);
                        }
                      }
                    }
                  }
                }
                __syncwarp();
              }
              continue;
            }
          }
          // each step's 16 columns are loaded while the previous step's are
          // processed, so the accumulator is handed back one step earlier and
          // the loads' latency is hidden
          uint32_t nv[16];
          tmem_ld16(taddr, nv);
          for (int c0 = 0; c0 < p.sub_n; c0 += 16) {
            uint32_t v[16];
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = nv[j];
            if (c0 + 16 < p.sub_n) tmem_ld16(taddr + static_cast<uint32_t>(c0 + 16), nv);
            if (c0 + 16 >= p.sub_n) {  // the accumulator is in registers: hand it back
              tc_fence_before();
              __syncwarp();
              // a test of the bounded waits withholds one of the four arrivals of
              // CTA 0's first hand-back, so the MMA issuer's wait for it gives up
              const bool withhold = p.withhold_arrive && blockIdx.x == 0 && it == 0 && acc == 0 && qw == 0;
              if (lane == 0 && !withhold) mbar_arrive(bar_acc_empty + 8u * acc);
            }
            if (!vec_ok) {
              // rows whose length breaks 16-byte alignment: each lane writes its
              // own position for the 16 channels (consecutive lanes, consecutive ow)
              const int r = qw * 32 + lane;
              const int ohp = tc.oh0 + i * p.TH + r / p.TW, owp = tc.ow0 + r % p.TW;
              if (ohp < g.OH && owp < g.OW) {
                T* dst = y + (static_cast<int64_t>(tc.n) * g.Cout) * S + static_cast<int64_t>(tc.od) * S_hw +
                         static_cast<int64_t>(ohp) * g.OW + owp;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                  const int co = co0 + c0 + j;
                  if (co < g.Cout) {
                    float f = __uint_as_float(v[j]);
                    if constexpr (kFp4) f = __fmul_rn(f, gg);
                    if (bias) f = __fadd_rn(f, DTypeOps<T>::to_f32(__ldg(bias + co)));
                    dst[static_cast<int64_t>(co) * S] = DTypeOps<T>::from_f32(f);
                  }
                }
              }
              continue;
            }
            // bias, rounding, and the staging rows (row j = channel co0 + c0 + j)
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int co = co0 + c0 + j;
              float f = __uint_as_float(v[j]);
              if constexpr (kFp4) f = __fmul_rn(f, gg);
              if (bias && co < g.Cout) f = __fadd_rn(f, DTypeOps<T>::to_f32(__ldg(bias + co)));
              const T o = DTypeOps<T>::from_f32(f);
              const uint32_t a = stage + static_cast<uint32_t>(j) * kPitch + static_cast<uint32_t>(lane * kEsz);
              if constexpr (kEsz == 2) {
                unsigned short b;
                memcpy(&b, &o, 2);
                asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"(b) : "memory");
              } else {
                asm volatile("st.shared.b32 [%0], %1;" ::"r"(a), "r"(__float_as_uint(f)) : "memory");
              }
            }
            __syncwarp();
#pragma unroll
            for (int k = 0; k < kUnits; ++k) {
              const int j = lane / kGroups + k * (32 / kGroups);
              const int co = co0 + c0 + j;
              if (co < g.Cout && row_ok) {
                const uint32_t a = stage + static_cast<uint32_t>(j) * kPitch + static_cast<uint32_t>(gq * 16);
                int w0, w1, w2, w3;
                ld_shared_v4(a, w0, w1, w2, w3);
                T* dst = y + ubase + static_cast<int64_t>(co) * S;
                if (full) {
                  __stcs(reinterpret_cast<int4*>(dst), make_int4(w0, w1, w2, w3));
                } else {
                  const uint32_t ws[4] = {static_cast<uint32_t>(w0), static_cast<uint32_t>(w1),
                                          static_cast<uint32_t>(w2), static_cast<uint32_t>(w3)};
#pragma unroll
                  for (int e = 0; e < kPer; ++e) {
                    if (ow + e < g.OW) {
                      if constexpr (kEsz == 2) {
                        const unsigned short b = static_cast<unsigned short>(ws[e >> 1] >> (16 * (e & 1)));
                        memcpy(dst + e, &b, 2);
                      } else {
                        dst[e] = __uint_as_float(ws[e]);
                      }
                    }
                  }
                }
              }
            }
            __syncwarp();
          }
        }
      }
    }
  } else if (warp >= kWarpXf0) {
    // ------------------------------------------------------------ transform
    // Two groups of 8 warps take the K slices of alternate global index;
    // within a group, warp w owns TMEM lane quadrant w % 4 (the lanes its
    // tcgen05.st may reach) and two adjacent 16-column blocks b0, b0 + 1 of
    // each of its slices, for every subtile.
    constexpr uint32_t esz = sizeof(T);
    const int xw = warp - kWarpXf0;
    const int quad = warp & 3;                 // TMEM lanes 32*quad..+31
    const int grp = xw >> 3;                   // global slices of this parity
    // blocks of 64 (A in shared memory only): the quad's two warps take 16
    // rows each, lanes l and l + 16 the two halves of row l % 16 of them
    const bool blk64 = kQ == 1 && kSmemA && p.qmode == kQModeNv64;
    const int b0 = blk64 ? 2 * (lane >> 4) : ((xw >> 2) & 1) * 2;  // first of the thread's two blocks
    const int row = blk64 ? quad * 32 + ((xw >> 2) & 1) * 16 + (lane & 15)
                          : quad * 32 + lane;  // output position within a subtile
    const int th = row / p.TW, tw = row % p.TW;
    const uint32_t halo_base = base + p.off_halo;
    const uint32_t phase_tab = base + p.off_phase;
    const int xf_tid = threadIdx.x - kWarpXf0 * 32;

    // Per-CTA tables (quantiser tables as described at QCtx).  The phase
    // table holds, for every block phase phi (column of the block's first
    // element within its channel), 16 ints: with the row gather (kDWB > 0)
    // the byte offsets of the six tap rows the block touches (column 0 of
    // each), otherwise the byte offsets of the block's 16 taps, both from the
    // origin of the block's first channel, the columns past the channel end
    // taken in the next channel as if it followed contiguously (chan_bytes
    // further on).
    QCtx q{};
    // the NVFP4 tables (MXFP4 takes no global amax: act_amax may be null)
    const bool nv_tables = p.quant && (kQ == 0 || p.qmode != kQModeMx);
    q.G = nv_tables ? nvfp4_global(__ldg(p.act_amax)) : Nvfp4Global{0.0f, 0.0f, 0.0f};
    q.dq = base + p.off_dq;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
      // the window starts 11 binades below t's binade (pattern 0 if t is
      // that small)
      const int e_t = static_cast<int>((__float_as_uint(q.G.t) >> 23) & 0xFFu);
      q.lo = static_cast<uint32_t>(max(e_t - 11, 0)) << 7;
      q.hi = q.lo + static_cast<uint32_t>(kCodeEntries - 1);
      q.cb = base + p.off_code - 2u * q.lo;
    }
    {
      if (nv_tables) {
        if (xf_tid < 128) {
          uint32_t h2;
          asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<unsigned short>(xf_tid & 0x7F)));
          const float s8 = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
          float s = __fmul_rn(s8, q.G.g);
          const bool fallback = s < 1e-5f;
          if (fallback) s = 1.0f;
          const DqTable dt = dq_table(s);
          uint32_t* e = reinterpret_cast<uint32_t*>(smem + p.off_dq + xf_tid * kDqEntryBytes);
          e[0] = dt.lo_a;
          e[1] = dt.lo_b;
          e[2] = dt.hi_a;
          e[3] = dt.hi_b;
          e[4] = __float_as_uint(__frcp_rn(s));
          e[5] = fallback ? 0u : static_cast<uint32_t>(xf_tid & 0x7F);  // scale byte of the NVFP4 operand
        }
        if constexpr (std::is_same<T, __nv_bfloat16>::value) {
          uint16_t* ct = reinterpret_cast<uint16_t*>(smem + p.off_code);
          for (int i = xf_tid; i < kCodeEntries; i += kNumXfWarps * 32)
            ct[i] = static_cast<uint16_t>(entry_of_max(__uint_as_float((q.lo + static_cast<uint32_t>(i)) << 16), q) - q.dq);
        }
      }
      int* ph = reinterpret_cast<int*>(smem + p.off_phase);
      for (int i = xf_tid; i < g.taps * 16; i += kNumXfWarps * 32) {
        const int phi = i >> 4, j = i & 15;
        if (kDWB > 0 && j >= 6) {
          ph[i] = 0;
          continue;
        }
        // tap tt from the block's first channel's origin: the block's tap j,
        // or (row gather) column 0 of its row j
        const int tt = kDWB > 0 ? (phi / 3 + j) * 3 : phi + j;
        const int nch = tt / g.taps;  // channels past the block's first one
        const int t = tt - nch * g.taps;
        const int chan = nch * static_cast<int>(p.chan_bytes);
        const int kw = t % g.KW, r = t / g.KW;
        const int kh = r % g.KH, kd = r / g.KH;
        ph[i] = (kd * g.dd * p.h_ext * p.w_box + kh * g.dh * p.w_box + kw * g.dw) * static_cast<int>(esz) + chan;
      }
      named_bar_sync(1, kNumXfWarps * 32);
    }

    const uint32_t lane_field = static_cast<uint32_t>(quad * 32) << 16;
    // NVFP4 operands: this thread's row of an A stage (32 bytes of codes,
    // 16-byte chunk b0 / 2 holding its two blocks, at the 32-byte-swizzled
    // position) and its two scale bytes in the subtile's scale atom (row
    // r = 32 * quad + lane at byte 16 * lane + 4 * quad + block)
    const uint32_t a_code_off =
        static_cast<uint32_t>(row * 32 + ((((b0 >> 1) ^ (row >> 2)) & 1) << 4));
    const uint32_t a_sf_off = static_cast<uint32_t>(p.n_mt * 4096 + lane * 16 + quad * 4 + b0);
    // BF16 A in shared memory: this thread's row (128 bytes) of a subtile's
    // 128B-swizzled tile and the swizzled 16-byte chunks of its two blocks
    // (block b0 + bb holds K columns 16 (b0 + bb) .. +15: chunks 2 (b0 + bb)
    // and 2 (b0 + bb) + 1, chunk j stored at j ^ (row & 7))
    const uint32_t a_row16 = static_cast<uint32_t>(row) * 128u;
    const uint32_t sw7 = static_cast<uint32_t>(row & 7);
    const uint32_t ach0 = ((2u * b0) ^ sw7) << 4, ach1 = ((2u * b0 + 1u) ^ sw7) << 4;
    const uint32_t ach2 = ((2u * b0 + 2u) ^ sw7) << 4, ach3 = ((2u * b0 + 3u) ^ sw7) << 4;
    const uint32_t ring = static_cast<uint32_t>(p.ring);
    const int cb = static_cast<int>(p.chan_bytes);
    uint32_t gs_base = 0;                 // global halo slot counter at the start of the tile
    uint32_t ga = 0;                      // global K-slice counter at the start of the tile
    uint32_t gslice = static_cast<uint32_t>(grp);  // global index of this group's next slice
    RingPos as{static_cast<uint32_t>(grp) % static_cast<uint32_t>(p.sa), 0u};  // its A stage
    RingPos hr{0u, 0u};                   // next halo slot this warp hands back
    bool ok = true;
    for (int64_t tt = blockIdx.x; ok && tt < p.num_tiles; tt += gridDim.x) {
      const TileCoord tc = decode_tile(p, tt);
      const int w0 = halo_w0(p, tc.ow0);
      const int delta = tc.ow0 * g.sw - g.pw - w0;
      // byte offset of this thread's output position in subtile 0, and the
      // step to the same position in the next subtile (TH rows further down)
      const uint32_t thr0 = static_cast<uint32_t>((th * g.sh * p.w_box + tw * g.sw + delta) * static_cast<int>(esz));
      const uint32_t thr_step = static_cast<uint32_t>(p.TH * g.sh * p.w_box * static_cast<int>(esz));
      // first slice of this tile that belongs to the group, and the state of
      // block b0 there: first column k0, its channel c0 = (slot q0, cs0
      // within the slot), phase phi = k0 - c0 * taps, ring entry h0 of q0
      int s = static_cast<int>((gslice - ga) & 0x7FFFFFFFu);
      int k0 = kBlockK * s + 16 * b0;
      int c0 = k0 / g.taps;
      int phi = k0 - c0 * g.taps;
      int q0 = c0 / p.c_slot;
      int cs0 = c0 - q0 * p.c_slot;
      RingPos h0 = ring_pos(gs_base + static_cast<uint32_t>(q0), ring);
      int released = 0;  // halo slots of this tile this warp has handed back
      for (; s < p.ks; s += 2, gslice += 2, as.next(static_cast<uint32_t>(p.sa)), as.next(static_cast<uint32_t>(p.sa))) {
        const uint32_t ea = as.e;
        if (gslice >= static_cast<uint32_t>(p.sa) &&
            !wait_or_abort(bar_a_empty + 8u * ea, as.ph ^ 1u, p.err, kSiteMmaDone, abort_flag)) {
          ok = false;
          break;
        }
        // block b0 + 1 starts 16 columns on
        int phi1 = phi + p.dk16_phi, cs1 = cs0 + p.dk16_c, q1 = q0;
        RingPos h1 = h0;
        if (phi1 >= g.taps) {
          phi1 -= g.taps;
          ++cs1;
        }
        while (cs1 >= p.c_slot) {
          cs1 -= p.c_slot;
          ++q1;
          h1.next(ring);
        }
        const int nv0 = g.K - k0, nv1 = nv0 - 16;
        const int split0 = g.taps - phi, split1 = g.taps - phi1;  // columns j >= split are in the next channel
        // the block's second channel opens the next slot (never with slot-aligned blocks)
        const bool cross0 = !p.slot_aligned && split0 < min(16, nv0) && cs0 + 1 == p.c_slot;
        const bool cross1 = !p.slot_aligned && split1 < min(16, nv1) && cs1 + 1 == p.c_slot;
        // halo slots the two blocks read: q0 .. q_last
        if (nv0 > 0) {
          const int q_last = nv1 > 0 ? q1 + (cross1 ? 1 : 0) : q0 + (cross0 ? 1 : 0);
          RingPos hw = h0;
          for (int q = q0; ok && q <= q_last; ++q, hw.next(ring))
            ok = wait_or_abort(bar_halo_full + 8u * hw.e, hw.ph, p.err, kSiteHaloFull, abort_flag);
        }
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_col = tmem_base + lane_field + static_cast<uint32_t>(p.a_col0) +
                               ea * static_cast<uint32_t>(p.n_mt * 32) + static_cast<uint32_t>(b0 * 8);
        // NVFP4 operands: this slice's A stage in shared memory (subtile i
        // 4096 bytes further for the codes, 512 for the scale bytes)
        const uint32_t a_stage = base + p.off_a + ea * p.a_stage_bytes;
        const uint32_t a_code = a_stage + a_code_off, a_sf = a_stage + a_sf_off;
        // the 16 BF16 values of block b0 + bb of subtile i, into TMEM or the
        // shared-memory tile
        auto put = [&](int i, int bb, const uint32_t (&w)[8]) {
          if constexpr (kSmemA) {
            const uint32_t r = a_stage + static_cast<uint32_t>(i) * 16384u + a_row16;
            st_shared_v4(r + (bb ? ach2 : ach0), w[0], w[1], w[2], w[3]);
            st_shared_v4(r + (bb ? ach3 : ach1), w[4], w[5], w[6], w[7]);
          } else {
            tmem_st8(a_col + 8u * static_cast<uint32_t>(bb) + static_cast<uint32_t>(i * 32), w);
          }
        };
        const bool quant = p.quant != 0;
        bool pair_done = false;
        if constexpr (!kFp4 && kQ == 1) {
          {
            // NVFP4 blocks of 32 or MXFP4 (always quantised): the warp's
            // blocks b0, b0 + 1 of a row are one group; both are gathered
            // per subtile and share the scale of their joint maximum
            pair_done = true;
            // blocks of 64 keep every lane on one path: the block maximum is
            // exchanged by a shuffle in each subtile's quantisation
            if (nv0 <= 0 && !blk64) {
              uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
              for (int i = 0; i < p.n_mt; ++i) {
                put(i, 0, z);
                put(i, 1, z);
              }
            } else {
              const uint32_t org0 = halo_base + h0.e * p.slot_bytes + static_cast<uint32_t>(cs0 * cb);
              const uint32_t org1 = halo_base + h1.e * p.slot_bytes + static_cast<uint32_t>(cs1 * cb);
              const uint32_t prow0 = phase_tab + static_cast<uint32_t>(phi * 64);
              const uint32_t prow1 = phase_tab + static_cast<uint32_t>(phi1 * 64);
              // a block whose second channel opens the next slot: its columns there move by adj
              int adj0 = 0, adj1 = 0;
              if (cross0) {
                RingPos hn = h0;
                hn.next(ring);
                adj0 = static_cast<int>(halo_base + hn.e * p.slot_bytes) - static_cast<int>(org0) - cb;
              }
              if (cross1) {
                RingPos hn = h1;
                hn.next(ring);
                adj1 = static_cast<int>(halo_base + hn.e * p.slot_bytes) - static_cast<int>(org1) - cb;
              }
              bool rows_done = false;
              if constexpr (kDWB > 0 && sizeof(T) == 2) {
                if (blk64 ? g.K - kBlockK * s >= kBlockK : nv1 >= 16) {
                  // both blocks full: row gathers (block b0 + 1 starts one
                  // column further in the row pattern, taps being a multiple of 3)
                  const int p3 = phi % 3;
                  uint32_t r0[6], r1[6];
                  row_bases(org0 + thr0, prow0, cross0 ? (g.taps - phi + p3) / 3 : 6, adj0, r0);
                  row_bases(org1 + thr0, prow1, cross1 ? (g.taps - phi1 + phi1 % 3) / 3 : 6, adj1, r1);
                  for (int i = 0; i < p.n_mt; ++i) {
                    uint32_t pa[8], pb[8], wa[8], wb[8];
                    switch (p3) {
                      case 0: gather_rows<0, kDWB>(r0, pa); gather_rows<1, kDWB>(r1, pb); break;
                      case 1: gather_rows<1, kDWB>(r0, pa); gather_rows<2, kDWB>(r1, pb); break;
                      default: gather_rows<2, kDWB>(r0, pa); gather_rows<0, kDWB>(r1, pb); break;
                    }
                    quant_group32<T>(pa, pb, p.qmode, p.dst_max, q, wa, wb);
                    put(i, 0, wa);
                    put(i, 1, wb);
#pragma unroll
                    for (int r = 0; r < 6; ++r) {
                      r0[r] += thr_step;
                      r1[r] += thr_step;
                    }
                  }
                  rows_done = true;
                }
              }
              if (!rows_done) {
                uint32_t a0 = org0 + thr0, a1 = org1 + thr0;
#pragma unroll 1
                for (int i = 0; i < p.n_mt; ++i, a0 += thr_step, a1 += thr_step) {
                  uint32_t wa[8], wb[8];
                  group32_taps<T, kDWB>(a0, prow0, phi, split0, adj0, nv0, a1, prow1, phi1, split1, adj1, nv1, p.qmode,
                                        p.dst_max, q, wa, wb);
                  put(i, 0, wa);
                  put(i, 1, wb);
                }
              }
            }
          }
        }
        if constexpr (!kPairs && sizeof(T) == 2 && kQ == 0) {
          // single subtile, both blocks full and within their slots: one interleaved pass
          if (nv0 >= 32 && !cross0 && !cross1) {
            const uint32_t org0 = halo_base + h0.e * p.slot_bytes + static_cast<uint32_t>(cs0 * cb) + thr0;
            const uint32_t org1 = halo_base + h1.e * p.slot_bytes + static_cast<uint32_t>(cs1 * cb) + thr0;
            uint32_t pa[8], pb[8];
            if constexpr (kDWB > 0) {
              uint32_t ra[6], rb[6];
              row_bases(org0, phase_tab + static_cast<uint32_t>(phi * 64), 6, 0, ra);
              row_bases(org1, phase_tab + static_cast<uint32_t>(phi1 * 64), 6, 0, rb);
              // the second block starts 16 columns on, one column further in the row pattern
              switch (phi % 3) {
                case 0: gather_rows<0, kDWB>(ra, pa); gather_rows<1, kDWB>(rb, pb); break;
                case 1: gather_rows<1, kDWB>(ra, pa); gather_rows<2, kDWB>(rb, pb); break;
                default: gather_rows<2, kDWB>(ra, pa); gather_rows<0, kDWB>(rb, pb); break;
              }
            } else {
              int off[16];
              load_taps(phase_tab + static_cast<uint32_t>(phi * 64), off);
              gather_taps<T>(org0, off, 16, pa);
              load_taps(phase_tab + static_cast<uint32_t>(phi1 * 64), off);
              gather_taps<T>(org1, off, 16, pb);
            }
            if constexpr (kFp4) {
              // the warp's two blocks of this row are one 16-byte chunk
              uint32_t ca0, ca1, sa8, cb0, cb1, sb8;
              fp4_block_x2<T>(pa, pb, q, ca0, ca1, sa8, cb0, cb1, sb8);
              st_shared_v4(a_code, ca0, ca1, cb0, cb1);
              st_shared_u16(a_sf, sa8 | (sb8 << 8));
            } else {
              uint32_t wa[8], wb[8];
              quant8_x2<T>(pa, pb, quant, q, wa, wb);
              put(0, 0, wa);
              put(0, 1, wb);
            }
            pair_done = true;
          }
        }
#pragma unroll 1
        for (int bb = 0; bb < 2 && !pair_done; ++bb) {
          const int nv = bb ? nv1 : nv0;
          const uint32_t codeb = a_code + 8u * static_cast<uint32_t>(bb), sfb = a_sf + static_cast<uint32_t>(bb);
          if (nv <= 0) {
            // a block entirely past K: zeros (the weights there are zero-filled too)
            if constexpr (kFp4) {
              for (int i = 0; i < p.n_mt; ++i)
                fp4_put(codeb + static_cast<uint32_t>(i) * 4096u, sfb + static_cast<uint32_t>(i) * 512u, 0u, 0u, 0u);
            } else {
              uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
              for (int i = 0; i < p.n_mt; ++i) put(i, bb, z);
            }
            continue;
          }
          const int phb = bb ? phi1 : phi, csb = bb ? cs1 : cs0, splitb = bb ? split1 : split0;
          const RingPos hb = bb ? h1 : h0;
          const uint32_t org = halo_base + hb.e * p.slot_bytes + static_cast<uint32_t>(csb * cb);
          const uint32_t prow = phase_tab + static_cast<uint32_t>(phb * 64);
          // the block's second channel opens the next ring slot: its columns move by adj
          int adj = 0;
          const bool crossb = bb ? cross1 : cross0;
          if (crossb) {
            RingPos hn = hb;
            hn.next(ring);
            adj = static_cast<int>(halo_base + hn.e * p.slot_bytes) - static_cast<int>(org) - cb;
          }
          int i = 0;
          if constexpr (kDWB > 0) {
            if (nv >= 16) {
              // rows of three taps: the rows of the next channel start at
              // row (taps - phi + phi % 3) / 3 of the block
              const int p3 = phb % 3;
              uint32_t rb0[6];
              row_bases(org + thr0, prow, crossb ? (g.taps - phb + p3) / 3 : 6, adj, rb0);
              if constexpr (kPairs) {
                for (; i + 1 < p.n_mt; i += 2) {
                  uint32_t ra[6], rb[6], pa[8], pb[8], wa[8], wb[8];
#pragma unroll
                  for (int r = 0; r < 6; ++r) {
                    ra[r] = rb0[r] + static_cast<uint32_t>(i) * thr_step;
                    rb[r] = ra[r] + thr_step;
                  }
                  switch (p3) {
                    case 0: gather_rows<0, kDWB>(ra, pa); gather_rows<0, kDWB>(rb, pb); break;
                    case 1: gather_rows<1, kDWB>(ra, pa); gather_rows<1, kDWB>(rb, pb); break;
                    default: gather_rows<2, kDWB>(ra, pa); gather_rows<2, kDWB>(rb, pb); break;
                  }
                  if constexpr (kFp4) {
                    uint32_t ca0, ca1, sa8, cb0, cb1, sb8;
                    fp4_block_x2<T>(pa, pb, q, ca0, ca1, sa8, cb0, cb1, sb8);
                    fp4_put(codeb + static_cast<uint32_t>(i) * 4096u, sfb + static_cast<uint32_t>(i) * 512u, ca0, ca1, sa8);
                    fp4_put(codeb + static_cast<uint32_t>(i + 1) * 4096u, sfb + static_cast<uint32_t>(i + 1) * 512u, cb0,
                            cb1, sb8);
                  } else {
                    quant8_x2<T>(pa, pb, quant, q, wa, wb);
                    put(i, bb, wa);
                    put(i + 1, bb, wb);
                  }
                }
              }
              for (; i < p.n_mt; ++i) {
                uint32_t ra[6], pa[8], wa[8];
#pragma unroll
                for (int r = 0; r < 6; ++r) ra[r] = rb0[r] + static_cast<uint32_t>(i) * thr_step;
                switch (p3) {
                  case 0: gather_rows<0, kDWB>(ra, pa); break;
                  case 1: gather_rows<1, kDWB>(ra, pa); break;
                  default: gather_rows<2, kDWB>(ra, pa); break;
                }
                if constexpr (kFp4) {
                  uint32_t c0, c1, s8b;
                  fp4_block<T>(pa, q, c0, c1, s8b);
                  fp4_put(codeb + static_cast<uint32_t>(i) * 4096u, sfb + static_cast<uint32_t>(i) * 512u, c0, c1, s8b);
                } else {
                  quant8_1<T>(pa, quant, q, wa);
                  put(i, bb, wa);
                }
              }
              continue;
            }
          }
          // by tap offsets (the row-gather table is expanded to taps first)
          int off[16];
          if constexpr (kDWB > 0)
            taps_from_rows<kDWB>(prow, phb % 3, off);
          else
            load_taps(prow, off);
          if (crossb) {
#pragma unroll
            for (int j = 0; j < 16; ++j) off[j] += (j >= splitb) ? adj : 0;
          }
          if constexpr (kPairs && sizeof(T) == 2) {
            // full blocks, subtiles in pairs: interleaved chains
            if (nv >= 16)
              for (; i + 1 < p.n_mt; i += 2) {
                uint32_t pa[8], pb[8], wa[8], wb[8];
                const uint32_t ra = org + thr0 + static_cast<uint32_t>(i) * thr_step;
                gather_taps<T>(ra, off, 16, pa);
                gather_taps<T>(ra + thr_step, off, 16, pb);
                if constexpr (kFp4) {
                  uint32_t ca0, ca1, sa8, cb0, cb1, sb8;
                  fp4_block_x2<T>(pa, pb, q, ca0, ca1, sa8, cb0, cb1, sb8);
                  fp4_put(codeb + static_cast<uint32_t>(i) * 4096u, sfb + static_cast<uint32_t>(i) * 512u, ca0, ca1, sa8);
                  fp4_put(codeb + static_cast<uint32_t>(i + 1) * 4096u, sfb + static_cast<uint32_t>(i + 1) * 512u, cb0, cb1,
                          sb8);
                } else {
                  quant8_x2<T>(pa, pb, quant, q, wa, wb);
                  put(i, bb, wa);
                  put(i + 1, bb, wb);
                }
              }
          }
          for (; i < p.n_mt; ++i) {
            if constexpr (kFp4) {
              uint32_t c0, c1, s8b;
              fp4_row_block<T>(org + thr0 + static_cast<uint32_t>(i) * thr_step, off, nv, q, c0, c1, s8b);
              fp4_put(codeb + static_cast<uint32_t>(i) * 4096u, sfb + static_cast<uint32_t>(i) * 512u, c0, c1, s8b);
            } else {
              uint32_t w[8];
              row_block<T>(org + thr0 + static_cast<uint32_t>(i) * thr_step, off, nv, quant, q, w);
              put(i, bb, w);
            }
          }
        }
        if constexpr (kSmemA) {
          // the MMA reads the stage through the async proxy
          fence_proxy_async_smem();
        } else {
          tmem_wait_st();
          tc_fence_before();
        }
        __syncwarp();
        // this warp's next slice is two on: its blocks move 128 columns
        k0 += 2 * kBlockK;
        phi += p.dk2_phi;
        int dc = p.dk2_c;
        if (phi >= g.taps) {
          phi -= g.taps;
          ++dc;
        }
        cs0 += dc;
        while (cs0 >= p.c_slot) {
          cs0 -= p.c_slot;
          ++q0;
          h0.next(ring);
        }
        if (lane == 0) {
          mbar_arrive(bar_a_full + 8u * ea);
          // Later blocks of this warp start at slot q0 or above: hand the
          // slots below back (a slot is free once all transform warps have).
          // A warp also hands back slots it never read (the other group's
          // slices).  Where its lead over the slowest warp can reach a ring
          // lap (fewer K slices per tile than A stages: sa slices span
          // several tiles' slots; or a ring sized for another plan's
          // coupling) each hand-back waits for the slot's fill first, or it
          // could land in the previous use's phase (p.hb_wait, set by the
          // planner).  Otherwise the stage coupling keeps every warp within
          // a ring lap.
          const int keep = (s + 2 < p.ks) ? min(q0, p.q_slots) : p.q_slots;
          for (; ok && released < keep; ++released, hr.next(ring)) {
            if (p.hb_wait) ok = wait_or_abort(bar_halo_full + 8u * hr.e, hr.ph, p.err, kSiteHaloFull, abort_flag);
            mbar_arrive(bar_halo_empty + 8u * hr.e);
          }
        }
        if (p.hb_wait) {  // only a hand-back that waits for a fill can fail
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
        }
      }
      if (!ok) break;
      // Hand back the tile's remaining slots.  With fewer K slices than A
      // stages (all of them in a tile with no slice for this group, when
      // ks == 1) each waits for its fill first: a warp with nothing to
      // build would otherwise run a ring lap ahead of the others and arrive
      // in an earlier phase.
      if (lane == 0)
        for (; ok && released < p.q_slots; ++released, hr.next(ring)) {
          if (p.hb_wait) ok = wait_or_abort(bar_halo_full + 8u * hr.e, hr.ph, p.err, kSiteHaloFull, abort_flag);
          mbar_arrive(bar_halo_empty + 8u * hr.e);
        }
      if (p.hb_wait) ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      gs_base += static_cast<uint32_t>(p.q_slots);
      ga += static_cast<uint32_t>(p.ks);
    }
  }

  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <typename T, bool kPairs, int kDWB, int kAOp, int kQ>
cudaError_t launch_tmem_inst(const TmemParams& p, const CUtensorMap& tx, const CUtensorMap& tw, int grid, size_t smem,
                             cudaStream_t s) {
  auto kern = conv3d_igemm_tmem_kernel<T, kPairs, kDWB, kAOp, kQ>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, s>>>(p, tx, tw);
  return cudaGetLastError();
}

// Row gather for 16-bit inputs and kernels three taps wide with W dilation 1
// or 2; tap-offset gather otherwise.
template <typename T, int kAOp, int kQ = 0>
cudaError_t launch_tmem_typed(const TmemParams& p, const CUtensorMap& tx, const CUtensorMap& tw, int grid,
                              size_t smem, cudaStream_t s) {
  const int dwb = row_gather_step(p.g, sizeof(T));
  const bool pairs = p.n_mt >= 2;
  if constexpr (sizeof(T) == 2) {
    if (dwb == 2)
      return pairs ? launch_tmem_inst<T, true, 2, kAOp, kQ>(p, tx, tw, grid, smem, s)
                   : launch_tmem_inst<T, false, 2, kAOp, kQ>(p, tx, tw, grid, smem, s);
    if (dwb == 4)
      return pairs ? launch_tmem_inst<T, true, 4, kAOp, kQ>(p, tx, tw, grid, smem, s)
                   : launch_tmem_inst<T, false, 4, kAOp, kQ>(p, tx, tw, grid, smem, s);
  }
  return pairs ? launch_tmem_inst<T, true, 0, kAOp, kQ>(p, tx, tw, grid, smem, s)
               : launch_tmem_inst<T, false, 0, kAOp, kQ>(p, tx, tw, grid, smem, s);
}

// Output channels per tile: all of Cout up to 448 (448 + two 32-column A
// stages fill the 512 TMEM columns), else the fewest equal tiles of at most
// 448 (each N-tile rebuilds the A operand); each tile in n_sub N-parts of at
// most 256 (one MMA instruction's N), every size a multiple of 16.  Depends
// on Cout alone, so the packed NVFP4 weights can be laid out by it.
struct NPlan {
  int n_tile, n_ntiles, n_sub, sub_n;
};
inline NPlan n_plan(int Cout) {
  NPlan r;
  r.n_ntiles = 1;
  r.n_tile = (Cout + 15) / 16 * 16;
  if (r.n_tile > 448) {
    r.n_ntiles = (Cout + 447) / 448;
    r.n_tile = ((Cout + r.n_ntiles - 1) / r.n_ntiles + 15) / 16 * 16;
  }
  r.n_sub = (r.n_tile + 255) / 256;
  r.sub_n = ((r.n_tile + r.n_sub - 1) / r.n_sub + 15) / 16 * 16;
  r.n_tile = r.sub_n * r.n_sub;
  return r;
}

// The 5-D tensor map of x for the halo boxes of a plan (zero fill outside
// the input); false when the TMA unit cannot describe it.
inline bool encode_halo_map(const ConvGeom& g, const void* x, int dtype, const TmemParams& p, CUtensorMap* tmap) {
  EncodeTiledFn encode = get_encode_tiled();
  if (!encode) return false;
  const int esz = dtype == 0 ? 4 : 2;
  const CUtensorMapDataType dt = dtype == 0   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : dtype == 1 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                              : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const cuuint64_t dims[5] = {(cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.D, (cuuint64_t)g.C, (cuuint64_t)g.N};
  const cuuint64_t st[4] = {(cuuint64_t)g.W * esz, (cuuint64_t)g.H * g.W * esz, (cuuint64_t)g.D * g.H * g.W * esz,
                            (cuuint64_t)g.C * g.D * g.H * g.W * esz};
  const cuuint32_t box[5] = {(cuuint32_t)p.w_box, (cuuint32_t)p.h_ext, (cuuint32_t)p.kd_ext, (cuuint32_t)p.c_slot, 1};
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return encode(tmap, dt, 5, const_cast<void*>(x), dims, st, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Tiling and pipeline plan of the tensor-memory kernel (pure host
// arithmetic).  Returns false when the kernel does not apply: rows of x not
// a multiple of 16 bytes (TMA stride rule), more than 343 taps, or no plan
// that fits.
//
// aop: the A operand mode.  kAOpBf16Tmem: A stages of n_mt x 32 columns in
// tensor memory beside the accumulators.  kAOpBf16Smem: A stages of n_mt x
// 16 KB in shared memory, tensor memory only for the accumulators.
// kAOpNvfp4: A stages of n_mt x (4096 bytes of codes + a 512-byte scale
// atom) in shared memory, weight stages of n_sub prepacked images, and in
// tensor memory the accumulators and per A stage the scale factors (4
// columns per subtile and per 128 rows of an N-part).
bool plan_tmem(const ConvGeom& g, int dtype, TmemParams& p, size_t& smem, int aop = kAOpBf16Tmem) {
  const bool fp4 = aop == kAOpNvfp4, smem_a = aop != kAOpBf16Tmem;
  const int esz = dtype == 0 ? 4 : 2;
  const int align = 16 / esz;
  if ((static_cast<int64_t>(g.W) * esz) % 16 != 0) return false;
  if (g.taps > kMaxTaps) return false;
  memset(&p, 0, sizeof(p));
  p.g = g;
  p.align = align;

  const NPlan np = n_plan(g.Cout);
  const int n_tile = np.n_tile, n_ntiles = np.n_ntiles, n_sub = np.n_sub, sub_n = np.sub_n;
  p.n_tile = n_tile; p.n_ntiles = n_ntiles; p.n_sub = n_sub; p.sub_n = sub_n;
  p.fp4 = fp4 ? 1 : 0;
  p.aop = aop;
  p.dtype_code = dtype;
  p.n_atoms = (sub_n + 127) / 128;
  p.n_parts = n_ntiles * n_sub;
  p.b_img_bytes = static_cast<uint32_t>(sub_n * 32 + p.n_atoms * 512);
  // TMEM columns after the accumulators (32-aligned), and what one A stage
  // takes there: 32 BF16-pair columns per subtile (A in tensor memory), the
  // scale factors (NVFP4), or nothing (BF16 A in shared memory)
  auto a_col0_of = [&](int mt, int nb = 1) { return (nb * mt * n_tile + 31) / 32 * 32; };
  auto stage_cols = [&](int mt) { return fp4 ? 4 * mt + 4 * p.n_atoms * n_sub : smem_a ? 0 : mt * 32; };
  auto stages_of = [&](int mt, int nb = 1) {
    const int left = static_cast<int>(kTmemCols) - a_col0_of(mt, nb);
    if (left < 0) return 0;
    return stage_cols(mt) == 0 ? 4 : left / stage_cols(mt);
  };

  // tile shape: subtile TH x TW = 128, n_mt subtiles stacked along oh; at
  // least two A stages must fit next to the accumulators
  const int kd_ext = (g.KD - 1) * g.dd + 1;
  double best = 1e30;
  int bTW = 0, bMT = 0;
  for (int mt = 4; mt >= 1; mt /= 2) {
    if (2 * mt * n_sub > kMaxAcc || stages_of(mt) < 2) continue;
    // measured on the 96-channel edge layer with W dilation 2: four subtiles
    // 14.2 ms, two 11.3 ms with NVFP4 operands (undilated: 7.6 vs 9.6), and
    // 12.3 vs 11.9 ms with BF16 ones
    if (smem_a && g.dw > 1 && mt > 2) continue;
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
  // two accumulator buffers where two A stages still fit beside them: the
  // MMAs of the next tile then overlap the epilogue's drain of this one
  p.acc_bufs = stages_of(bMT, 2) >= 2 ? 2 : 1;
  p.acc_cols = bMT * n_tile;
  p.a_col0 = smem_a ? 0 : a_col0_of(bMT, p.acc_bufs);
  p.sf_col0 = fp4 ? a_col0_of(bMT, p.acc_bufs) : 0;
  p.sf_cols = fp4 ? stage_cols(bMT) : 0;
  p.a_stage_bytes = fp4      ? static_cast<uint32_t>((bMT * (4096 + 512) + 1023) / 1024 * 1024)
                    : smem_a ? static_cast<uint32_t>(bMT) * 16384u
                             : 0u;
  p.sa = std::min(4, stages_of(bMT, p.acc_bufs));
  p.n_owb = ceil_div(g.OW, p.TW);
  p.n_ohb = ceil_div(g.OH, p.TH * p.n_mt);
  p.h_ext = (p.TH * p.n_mt - 1) * g.sh + (g.KH - 1) * g.dh + 1;
  const int w_ext = (p.TW - 1) * g.sw + (g.KW - 1) * g.dw + 1;
  p.w_box = (w_ext + 2 * (align - 1)) / align * align;
  p.kd_ext = kd_ext;
  p.chan_elems = p.kd_ext * p.h_ext * p.w_box;
  p.chan_bytes = static_cast<uint32_t>(p.chan_elems * esz);
  p.ks = ceil_div(g.K, kBlockK);
  p.num_tiles = static_cast<int64_t>(g.N) * g.OD * p.n_ohb * p.n_owb * n_ntiles;
  p.b_stage_bytes = fp4 ? (static_cast<uint32_t>(n_sub) * p.b_img_bytes + 1023u) / 1024u * 1024u
                        : static_cast<uint32_t>(n_tile) * 128u;
  p.dk2_c = 2 * kBlockK / g.taps;
  p.dk2_phi = 2 * kBlockK - p.dk2_c * g.taps;
  p.dk16_c = 16 / g.taps;
  p.dk16_phi = 16 - p.dk16_c * g.taps;
  // Fewer than 16 taps: a block spans several channels, so slots hold a
  // multiple of cm channels (c_slot * taps a multiple of 16) and no block
  // straddles two slots.  From 16 taps on a block spans at most two
  // channels and may straddle; the transform then moves the second
  // channel's columns to the next slot.
  int cm = 1;
  if (g.taps < 16) {
    int a = g.taps, b = 16;
    while (b) { const int r = a % b; a = b; b = r; }
    cm = 16 / a;
  }

  const int chan_bytes = static_cast<int>(p.chan_bytes);
  const int phase_bytes = g.taps * 64;
  // quantiser tables: the per-code entries, and for BF16 inputs the code
  // table of the block maxima
  const int code_bytes = dtype == 2 ? kCodeTableBytes : 0;
  // epilogue staging: 4 warps x 16 channel rows x (32 positions + 16 bytes)
  const int epi_bytes = 4 * 16 * (32 * esz + 16);
  // Halo ring: the transform warps hand a slot back as soon as they are past
  // it, so the ring only has to hold one slice's slots for progress; it is
  // sized for sa slices plus two, and any shared memory left after the
  // weight stages buys further slots (more halo loads in flight).
  for (int target = 10240; target >= 1; target = (target > chan_bytes ? target / 2 : 0)) {
    p.c_slot = std::max(1, std::min(std::min(256, g.C), target / chan_bytes));
    if (cm > 1) p.c_slot = std::min(256 / cm * cm, (p.c_slot + cm - 1) / cm * cm);
    p.slot_aligned = (p.c_slot * g.taps) % 16 == 0 ? 1 : 0;
    p.q_slots = ceil_div(g.C, p.c_slot);
    p.slot_tx = static_cast<uint32_t>(p.c_slot) * p.chan_bytes;
    p.slot_bytes = (p.slot_tx + 127u) / 128u * 128u;
    // fewer A stages shrink the halo window the ring must cover
    const int sa_max = std::min(4, stages_of(bMT, p.acc_bufs));
    for (int a = sa_max; a >= 2; --a) {
      int span = 1;
      for (int s0 = 0; s0 < p.ks; ++s0) {
        const int lo = ((kBlockK * s0) / g.taps) / p.c_slot;
        const int hi = (std::min(kBlockK * (s0 + a) - 1, g.K - 1) / g.taps) / p.c_slot;
        span = std::max(span, hi - lo + 1);
      }
      for (int b = 8; b >= 2; --b) {
        int r = span + 2;
        const int nbar = 2 * r + 2 * b + 2 * a + 2 * kMaxAcc + 1;
        const int a_bytes = a * static_cast<int>(p.a_stage_bytes);  // A stages in shared memory only
        int total = 1024 + kDqTableBytes + b * static_cast<int>(p.b_stage_bytes) + a_bytes +
                    r * static_cast<int>(p.slot_bytes) + 64 /* pad after the halo ring */ + code_bytes + epi_bytes +
                    phase_bytes + nbar * 8 + 16;
        if (total <= kMaxSmem) {
          const int extra = std::min(32 - r, (kMaxSmem - total) / (static_cast<int>(p.slot_bytes) + 16));
          if (extra > 0) {
            r += extra;
            total += extra * (static_cast<int>(p.slot_bytes) + 16);
          }
          p.sa = a; p.sb = b; p.ring = r;
          p.hb_wait = p.ks < p.sa ? 1 : 0;
          p.off_dq = 0;
          p.off_b = kDqTableBytes;  // a multiple of 1024, as the swizzled weight stages need
          p.off_a = p.off_b + b * p.b_stage_bytes;  // A stages in shared memory (1024-aligned)
          p.off_halo = p.off_a + static_cast<uint32_t>(a_bytes);
          p.off_code = (p.off_halo + r * p.slot_bytes + 64u + 15u) / 16u * 16u;
          p.off_epi = p.off_code + static_cast<uint32_t>(code_bytes);
          p.off_phase = p.off_epi + static_cast<uint32_t>(epi_bytes);
          p.off_bar = p.off_phase + static_cast<uint32_t>(phase_bytes);
          smem = static_cast<size_t>(total);
          return true;
        }
      }
    }
    if (p.c_slot == 1) break;
  }
  return false;
}

}  // namespace

}  // namespace q3d
