/*
 * q3d_testing.h -- test hooks exported by libq3d.so beside the C ABI of
 * q3d.h.  None of them is part of the convolution path: they expose the
 * device format conversions, the block-scale quotient and the host-side
 * tiling plans so that tests can check them in isolation.  Same conventions
 * as q3d.h (device pointers, asynchronous on `stream`, q3d_status results).
 */
#ifndef Q3D_TESTING_H_
#define Q3D_TESTING_H_

#include "q3d.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * q3d_selftest_formats -- TEST HOOK, not part of the convolution path.
 * Applies the device format conversions of the quantiser to n binary32
 * inputs: e2m1[i] = E2M1 RNE-saturating value of in[i] (sign kept),
 * e4m3[i] = E4M3 RNE-saturating value of |in[i]|.  All pointers are device
 * pointers; enqueued on `stream`.
 */
Q3D_API q3d_status q3d_selftest_formats(const float* in, int64_t n, float* e2m1, float* e4m3, q3d_stream_t stream);

/*
 * q3d_selftest_ratio -- TEST HOOK, not part of the convolution path.
 * Applies the device step that feeds the E4M3 block-scale rounding
 * (Model-Optimizer "Conv3D Implicit GEMM CUDA kernel", sec. 6.2: the block
 * maximum over 6 g, clamped to 448) to n pairs: out[i] = min(RN(bmax[i] /
 * t[i]), 448), a NaN quotient giving 448.  The device computes it as every
 * quantiser in this library does.  All pointers are device pointers of n
 * binary32 values; enqueued on `stream`.  Q3D_ERR_NULLPTR / _INVALID_ARG
 * (n < 0) before anything is enqueued.
 */
Q3D_API q3d_status q3d_selftest_ratio(const float* bmax, const float* t, int64_t n, float* out, q3d_stream_t stream);

/*
 * q3d_plan_conv -- TEST HOOK (host only, no CUDA call): the tiling and
 * pipeline plan the specialised sm_100a kernel would use for a convolution of
 * this geometry and dtype.  plan[0..plan_len) receives, in order: applicable
 * (0/1), TH, TW, n_mt, groups, n_tile, n_ntiles, n_sub, sub_n, K slices per
 * tile, channels per halo slot, halo slots per tile, halo ring entries,
 * A stages, B stages, TMEM columns, shared-memory bytes, tiles along OH,
 * tiles along OW, vectorised halo reads (0/1), halo box W, H and D extents;
 * further entries are 0.
 */
Q3D_API q3d_status q3d_plan_conv(const int64_t x_shape[5], const int64_t w_shape[5], const int32_t stride[3],
                                 const int32_t pad_lo[3], const int32_t pad_hi[3], const int32_t dil[3],
                                 int32_t dtype, int32_t* plan, int32_t plan_len);

/*
 * q3d_plan_conv_tmem -- TEST HOOK (host only, no CUDA call): as
 * q3d_plan_conv, for the kernel that builds the A operand in tensor memory.
 * Same field order; groups (transform warp groups, each taking the K
 * slices of one parity) is always 2, TMEM columns 512, vectorised reads 0,
 * and more entries follow the halo box extents: the first TMEM column of
 * the A stages, the A operand's place (0 tensor memory, 1 shared memory: the
 * launcher's choice), the number of accumulator buffers and whether the
 * transform warps wait for a halo slot's fill before handing it back (1 where
 * the ring does not by itself keep every hand-back in its phase).
 * applicable = 0 where that kernel does not apply (x rows
 * not a multiple of 16 bytes, more than 343 taps, or no plan that fits).
 */
Q3D_API q3d_status q3d_plan_conv_tmem(const int64_t x_shape[5], const int64_t w_shape[5], const int32_t stride[3],
                                      const int32_t pad_lo[3], const int32_t pad_hi[3], const int32_t dil[3],
                                      int32_t dtype, int32_t* plan, int32_t plan_len);

/*
 * q3d_plan_conv_fp4 -- TEST HOOK: the plan conv3d_implicit_gemm_fp4 would
 * use (host arithmetic only).  The fields of q3d_plan_conv_tmem up to the
 * halo box extents, then: the first TMEM column of the scale factors, the
 * TMEM columns per A stage, the bytes of one A stage in shared memory and of
 * one weight stage, the number of accumulator buffers and the hand-back
 * fill-wait flag (as for q3d_plan_conv_tmem).
 */
Q3D_API q3d_status q3d_plan_conv_fp4(const int64_t x_shape[5], const int64_t w_shape[5], const int32_t stride[3],
                                     const int32_t pad_lo[3], const int32_t pad_hi[3], const int32_t dil[3],
                                     int32_t dtype, int32_t* plan, int32_t plan_len);

/*
 * q3d_selftest_withheld_arrive -- TEST HOOK of the bounded waits, not part
 * of the convolution path.  Enqueues conv3d_implicit_gemm_pad2 (no bias, no
 * quantisation) on the tensor-memory kernel, except that in CTA 0 one of the
 * four epilogue warps withholds its arrival on the first hand-back of
 * accumulator 0: the MMA issuer's wait for that accumulator when CTA 0 next
 * uses it (its second tile, or its third where the plan double-buffers the
 * accumulators) never completes, nor do the waits that depend on it (the transform
 * warps' waits for a free A stage, the producers' for a free stage or slot,
 * the epilogue's for the next accumulator).  The first of them to reach the
 * library's wait limit (2 s) gives up, sets its site bit in the device error
 * word (e.g. 1 << 5 for the accumulator, 1 << 3 for an A stage) and raises
 * the CTA's abort flag; every role of CTA 0 then stops, after waiting for the
 * bulk copies and tensor-core operations it has in flight, and the launch
 * ends normally.  The other CTAs complete; out is unspecified.  The next
 * q3d_check_device_error returns Q3D_ERR_DEVICE_TIMEOUT with the site bits
 * and clears them; later calls are unaffected.
 *   x, w  BF16, contiguous, K % 8 == 0, w 16-byte aligned; the problem must
 *         run on the tensor-memory kernel with more tiles than CTAs times
 *         accumulator buffers (Q3D_ERR_INVALID_ARG otherwise, nothing
 *         enqueued).
 */
Q3D_API q3d_status q3d_selftest_withheld_arrive(const q3d_tensor* x, const q3d_tensor* w, const int32_t stride[3],
                                                const int32_t pad_lo[3], const int32_t pad_hi[3],
                                                const int32_t dil[3], q3d_tensor* out, q3d_stream_t stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* Q3D_TESTING_H_ */
