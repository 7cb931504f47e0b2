// sm100_ptx.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a)
// features the kernels use: mbarriers with bounded waits, TMA tiled loads,
// tcgen05 tensor-memory allocation, MMA, commit and loads.
//
// Every wait is bounded: it gives up after kQ3dWaitTimeoutNs of global time,
// records a site code in the device error word and returns false, so no
// kernel of this library can spin forever.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace q3d {

// Maximum time a single mbarrier wait may take before the kernel reports
// Q3D_ERR_DEVICE_TIMEOUT (2 s; a full tile of the largest layer takes well
// under 1 ms).
constexpr unsigned long long kQ3dWaitTimeoutNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, but the thread may be suspended for up to hint_ns while
// the phase is incomplete (it resumes as soon as the phase completes), so a
// waiting warp does not take issue slots from the warps doing the work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Suspend hint for bounded waits: long enough that waiting threads sleep
// instead of spinning, short enough that timeouts and aborts are noticed.
constexpr uint32_t kQ3dSleepHintNs = 200000u;

// Wait for the phase with the given parity to complete.  Returns false (and
// sets bit `site` of *err) if it has not completed within the time limit.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned int* err, unsigned int site) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, kQ3dSleepHintNs)) return true;
    if (global_timer_ns() - t0 > kQ3dWaitTimeoutNs) {
      if (err) atomicOr(err, site);
      return false;
    }
  }
}

// After an abort, wait (bounded) for every copy a producer may still have in
// flight in a ring of n entries whose full barriers count its issues: issue i
// went to entry i % n and completes that entry's phase of parity (i / n) & 1.
// Only the last min(issued, n) issues can be outstanding (each earlier entry
// was handed back empty, hence landed, before its reuse); waiting on an
// already completed phase returns at once.  A CTA must not exit while a bulk
// copy into its shared memory is still running.
__device__ __forceinline__ void drain_ring(uint32_t full_bar0, uint32_t n, uint32_t issued, unsigned int* err,
                                           unsigned int site) {
  const uint32_t first = issued > n ? issued - n : 0u;
  for (uint32_t i = first; i < issued; ++i) mbar_wait(full_bar0 + 8u * (i % n), (i / n) & 1u, err, site);
}

// ---------------------------------------------------------------------------
// proxy fences
// ---------------------------------------------------------------------------
// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor core / TMA) before signalling a barrier.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMA (tiled, no multicast)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, uint32_t bar, int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_5d(uint32_t dst, const void* tmap, uint32_t bar, int32_t c0, int32_t c1,
                                            int32_t c2, int32_t c3, int32_t c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6, %7}], [%2];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory
// ---------------------------------------------------------------------------
// Allocate ncols (power of two, 32..512) TMEM columns; the base address is
// written to shared memory at dst.  Executed by one full warp.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, BF16 x BF16 -> FP32, one CTA.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D (TMEM, FP32) (+)= A (TMEM, BF16) * B (shared memory, BF16), M = 128.
// A occupies 128 lanes (one row each) x K/2 columns, each 32-bit column
// holding two consecutive K elements (the lower K index in the low half).
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Store 8 consecutive 32-bit columns of this thread's TMEM lane (the warp
// covers lanes 32*(warp%4)..+31, given in the address's lane field).
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
// Wait until this thread's earlier tcgen05.st have completed.
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Arrive once on the mbarrier when every tcgen05.mma issued so far by this
// thread has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// Warp-wide forms of the two calls above: every lane of the (converged) warp
// makes the call with the same operands and elect.sync picks the one lane
// that issues, so the operands stay warp-uniform.
__device__ __forceinline__ void umma_bf16_ts_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                   uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_bf16_ss_elect(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                   uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit_elect(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
      : "memory");
}

// 32 lanes x 32 bits, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// 16 TMEM lanes x 16 columns (the 16x256b shape, two 8-column repetitions):
// thread t holds lanes t/4 and t/4 + 8 of the 16 and, in each 8-column half
// h, columns 2 (t % 4) and 2 (t % 4) + 1:
//   r[4h + 0], r[4h + 1]: lane t/4,     columns 8h + 2 (t % 4) + {0, 1}
//   r[4h + 2], r[4h + 3]: lane t/4 + 8, the same columns
// (the layout of an m16n8 accumulator fragment).
__device__ __forceinline__ void tmem_ld_16x256b_x2(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
// tcgen05.wait::ld that also orders every later use of the 16 loaded
// registers after the wait.
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}
// Four 8x8 matrices of 16-bit elements, each stored transposed: thread i
// gives the shared address of stored row i % 8 of matrix i / 8; register m
// holds the thread's element pair (row t / 4, columns 2 (t % 4) + {0, 1}) of
// matrix m, and stored row k of a matrix is its column k.
__device__ __forceinline__ void stmatrix_x4_trans(uint32_t addr, uint32_t m0, uint32_t m1, uint32_t m2, uint32_t m3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(m0), "r"(m1),
               "r"(m2), "r"(m3)
               : "memory");
}

// ---------------------------------------------------------------------------
// UMMA descriptors
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor for a K-major operand stored in the
// canonical 128-byte-swizzled layout: rows of 64 BF16 (128 B), groups of 8
// rows 1024 B apart, 16-byte chunk j of row r stored at chunk (j ^ (r & 7)).
// The tile must start on a 1024-byte boundary.  Advancing K by 16 elements
// inside the 64-wide atom adds 32 bytes to the start address.
__device__ __forceinline__ uint64_t umma_desc_kmajor_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);        // start address, 16-B units
  d |= (uint64_t)(1u) << 16;                          // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;                  // stride byte offset: 8-row group pitch
  d |= (uint64_t)1u << 46;                            // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                            // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor for kind::f16 with BF16 A/B, FP32 accumulator,
// both operands K-major, M x N tile.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32(uint32_t M, uint32_t N) {
  return (1u << 4)            // D format: F32
         | (1u << 7)          // A format: BF16
         | (1u << 10)         // B format: BF16
         | ((N >> 3) << 17)   // N / 8
         | ((M >> 4) << 24);  // M / 16
}

// Shared-memory matrix descriptor for an MN-major operand in the canonical
// 128-byte-swizzled layout: atoms of 64 MN elements (one 128-byte row) x 8 K
// rows (1024 bytes); in K-row r of an atom, 16-byte chunk j (8 MN elements)
// is stored at chunk (j ^ (r & 7)).  Atoms adjacent along MN are lbo bytes
// apart, atoms adjacent along K are sbo bytes apart.  Atoms start on
// 1024-byte boundaries.
__device__ __forceinline__ uint64_t umma_desc_mnmajor_sw128(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// kind::f16 instruction descriptor with an MN-major A operand and a K-major
// B operand (BF16 x BF16 -> FP32, M x N).
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32_amn(uint32_t M, uint32_t N) {
  return umma_idesc_bf16_f32(M, N) | (1u << 15);
}

// ---------------------------------------------------------------------------
// Block-scaled FP4 MMA (kind::mxf4nvf4, NVFP4: E2M1 operands packed two per
// byte, element 2i in the low nibble; unsigned E4M3 scale factors, one per 16
// consecutive K elements of a row, held in tensor memory)
// ---------------------------------------------------------------------------

// Shared-memory matrix descriptor for a K-major operand in the canonical
// 32-byte-swizzled layout: rows of 32 bytes (64 E2M1 values, one MMA's K),
// groups of 8 rows 256 bytes apart, 16-byte chunk j of row r stored at chunk
// (j ^ ((r >> 2) & 1)).  The tile must start on a 256-byte boundary.
__device__ __forceinline__ uint64_t umma_desc_kmajor_sw32(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);  // start address, 16-B units
  d |= (uint64_t)(1u) << 16;                    // leading byte offset (unused: one atom along K)
  d |= (uint64_t)(256u >> 4) << 32;             // stride byte offset: 8-row group pitch
  d |= (uint64_t)1u << 46;                      // descriptor version (sm_100)
  d |= (uint64_t)6u << 61;                      // layout: 32-byte swizzle
  return d;
}

// Shared-memory descriptor of a scale-factor atom, the source of
// tcgen05.cp.32x128b: 32 rows of 16 bytes stored contiguously (no swizzle;
// core matrices of 8 rows x 16 bytes, 128 bytes apart).
__device__ __forceinline__ uint64_t umma_desc_sf_atom(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)(128u >> 4) << 16;
  d |= (uint64_t)(128u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  return d;  // layout type 0: no swizzle
}

// Instruction descriptor for kind::mxf4nvf4 with E2M1 A and B (both K-major),
// UE4M3 scale factors (scale-factor ids 0), FP32 accumulator, M x N, K = 64.
__host__ __device__ constexpr uint32_t umma_idesc_nvfp4(uint32_t M, uint32_t N) {
  return (1u << 7)            // A format: E2M1
         | (1u << 10)         // B format: E2M1
         | ((N >> 3) << 17)   // N / 8
         | ((M >> 4) << 24);  // M / 16  (bit 23 = 0: UE4M3 scale factors)
}

// D (+)= (A x SFA) * (B x SFB) over K = 64, A and B from shared memory, the
// scale factors at tensor-memory addresses sfa / sfb; the whole (converged)
// warp calls it and elect.sync picks the issuing lane.
__device__ __forceinline__ void umma_nvfp4_ss_elect(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                    uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Copy a 32-row x 16-byte shared-memory atom into tensor memory, replicated
// into all four lane quadrants: row r lands in lanes r, 32 + r, 64 + r and
// 96 + r, bytes 4j..4j+3 of it in column taddr + j.  Issued like the MMA and
// executed in order with the MMAs this thread issues after it.
__device__ __forceinline__ void tmem_cp_sf_atom_elect(uint32_t taddr, uint64_t s_desc) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n\t}" ::"r"(taddr), "l"(s_desc)
      : "memory");
}

// Bulk copy of `bytes` contiguous bytes (both addresses 16-byte aligned, size
// a multiple of 16) from global into this CTA's shared memory, completing as
// transaction bytes on the mbarrier.  No multicast.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// Named barrier over `nthreads` threads (a multiple of 32) with id 1..15.
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Byte offset of the 16-byte chunk `chunk` (0..7) of row `row` inside a
// 128B-swizzled K-major tile (rows of 128 bytes).
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

}  // namespace q3d
