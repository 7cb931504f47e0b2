/*
 * q3d.h -- C ABI of the B200 (sm_100a) Conv3D implicit-GEMM library with
 * fused NVFP4 activation fake-quantisation.
 *
 * The operations follow the Model-Optimizer "Conv3D Implicit GEMM CUDA kernel"
 * article (lpqz.cn/news/178135):
 *   - conv3d_implicit_gemm*: sec. 5.1 (convolution as a GEMM with
 *     M = N*OD*OH*OW, Ngemm = Cout, K = Cin*kD*kH*kW, rows decomposed as
 *     (n, od, oh, ow), columns as (c, kd, kh, kw), no materialised im2col),
 *     sec. 3 (FP32/FP16/BF16 in and out, BF16 tensor-core arithmetic with
 *     FP32 accumulation) and sec. 7.1 (arguments, asymmetric padding, output
 *     shape of torch.nn.functional.conv3d, groups == 1);
 *   - fused activation quantisation: sec. 6.1-6.3 (E2M1 values, E4M3 block
 *     scales, blocks of 16 consecutive K elements of one A row, global scale
 *     act_amax / (6*448), tiny-scale fallback 1.0), rounding to nearest even;
 *   - fp4_fake_quant: sec. 6.4 and 7.3 (the same quantiser on a flat tensor
 *     viewed as [numel/16, 16]), fp4_fake_quant_bs the block sizes 32..256
 *     of sec. 7.1.
 * mxfp4_quantize follows a second page, the CANN aclnnFlatQuantV2 article
 * (MXFP4: E2M1 with a power-of-two scale per 32 elements).
 *
 * Conventions for every call:
 *   - All tensor data pointers are DEVICE pointers to contiguous row-major
 *     storage on the current CUDA device.  The caller owns every buffer; the
 *     library never retains or frees a caller pointer.
 *   - Calls enqueue work on `stream` (NULL = legacy default stream) and
 *     return without synchronising.  Arguments are validated on the host
 *     before anything is enqueued; on any non-OK status nothing has been
 *     enqueued, except for Q3D_ERR_CUDA from a failed launch.
 *   - Every device-side wait of the library is bounded; a wait that gives
 *     up sets a device error word, which q3d_check_device_error() reports as
 *     Q3D_ERR_DEVICE_TIMEOUT (the output is then unspecified).
 *   - Errors are returned as q3d_status; q3d_last_error() gives a message
 *     for the last non-OK status on the calling host thread.
 *   - Requires a compute-capability 10.x device (B200); otherwise
 *     Q3D_ERR_ARCH.
 *   - Per-device state (the device error word's address, the staging area
 *     of conv3d_implicit_gemm_noalloc, a memory pool) is looked up on the
 *     first call on each device and kept for the life of the process.  Do
 *     not keep using the library on a device after cudaDeviceReset() on it:
 *     the addresses it cached belong to the destroyed context.
 *   - Host-side test hooks (not part of the convolution path) are declared
 *     separately in q3d_testing.h.
 */
#ifndef Q3D_H_
#define Q3D_H_

#include <stdint.h>

#if defined(__GNUC__)
#define Q3D_API __attribute__((visibility("default")))
#else
#define Q3D_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* q3d_stream_t;

typedef enum {
  Q3D_F32 = 0,
  Q3D_F16 = 1,
  Q3D_BF16 = 2
} q3d_dtype;

/* A contiguous tensor: `ndim` leading entries of `shape` are used. */
typedef struct {
  void* data;       /* device pointer */
  int32_t dtype;    /* q3d_dtype */
  int32_t ndim;
  int64_t shape[5];
} q3d_tensor;

typedef enum {
  Q3D_OK = 0,
  Q3D_ERR_NULLPTR = 1,            /* a required pointer is NULL */
  Q3D_ERR_INVALID_ARG = 2,        /* rank, shape, groups != 1, stride/dilation < 1, pad < 0,
                                     empty output extent, aliasing, numel % 16 != 0 */
  Q3D_ERR_UNSUPPORTED_DTYPE = 3,  /* dtype not F32/F16/BF16, or w/bias/out dtype != x dtype */
  Q3D_ERR_ARCH = 4,               /* current device is not compute capability 10.x */
  Q3D_ERR_CUDA = 5,               /* a CUDA runtime call or launch failed */
  Q3D_ERR_DEVICE_TIMEOUT = 6,     /* a bounded device wait gave up (see q3d_check_device_error) */
  Q3D_ERR_UNSUPPORTED_SHAPE = 7   /* valid convolution outside the library's limits (e.g. 32-bit index range) */
} q3d_status;

/*
 * conv3d_implicit_gemm -- y = conv3d(x, w) + bias with symmetric padding,
 * optionally fake-quantising the activation operand to NVFP4 on the fly.
 *
 *   x        [N, Cin, D, H, W], dtype F32/F16/BF16.
 *   w        [Cout, Cin, kD, kH, kW], same dtype as x (groups == 1: the
 *            Cin of w must equal the Cin of x).  Rounded to BF16 for the
 *            tensor cores.
 *   bias     [Cout] in x's dtype, or NULL.  Added in FP32 to the FP32
 *            accumulator.
 *   act_amax device pointer to one float: the tensor-wide max|x| that sets
 *            the NVFP4 global scale; must be finite and >= 0.  Read on the
 *            device (no host sync).  Required iff quant_act != 0.
 *   stride, pad, dil  (d, h, w); stride >= 1, dil >= 1, pad >= 0.
 *   quant_act  nonzero: every element of the implicit im2col matrix A is
 *            fake-quantised (blocks of 16 consecutive K columns of one row, K
 *            ordered (c, kd, kh, kw), zeros of the padding included) before
 *            its BF16 rounding.
 *   out      [N, Cout, OD, OH, OW] in x's dtype, preallocated, must not
 *            overlap x or w.  OD = floor((D + 2*pad_d - dil_d*(kD-1) - 1) /
 *            stride_d) + 1, likewise OH, OW.
 * Returns Q3D_OK or an error status (see above).  N == 0 or Cout == 0 is a
 * valid no-op.
 */
Q3D_API q3d_status conv3d_implicit_gemm(const q3d_tensor* x, const q3d_tensor* w, const q3d_tensor* bias,
                                const float* act_amax, const int32_t stride[3], const int32_t pad[3],
                                const int32_t dil[3], int32_t quant_act, q3d_tensor* out,
                                q3d_stream_t stream);

/*
 * conv3d_implicit_gemm_pad2 -- as conv3d_implicit_gemm, with separate
 * leading and trailing padding per dimension (d, h, w), e.g. causal temporal
 * padding (2, 0).  The article applies such asymmetric (6-tuple) padding on
 * the host before the kernel (sec. 7.1); here the padding is never
 * materialised: out-of-range taps read as zero.
 * OD = floor((D + pad_lo_d + pad_hi_d - dil_d*(kD-1) - 1) / stride_d) + 1.
 */
Q3D_API q3d_status conv3d_implicit_gemm_pad2(const q3d_tensor* x, const q3d_tensor* w, const q3d_tensor* bias,
                                     const float* act_amax, const int32_t stride[3],
                                     const int32_t pad_lo[3], const int32_t pad_hi[3],
                                     const int32_t dil[3], int32_t quant_act, q3d_tensor* out,
                                     q3d_stream_t stream);

/* Activation quantiser formats of conv3d_implicit_gemm_ex. */
typedef enum {
  Q3D_QUANT_NONE = 0,
  Q3D_QUANT_NVFP4 = 1,   /* E2M1 values, E4M3 block scales, global scale act_amax / (6*448) */
  Q3D_QUANT_MXFP4 = 2    /* E2M1 values, power-of-two E8M0 group scales */
} q3d_quant_format;

/*
 * conv3d_implicit_gemm_ex -- conv3d_implicit_gemm_pad2 with the activation
 * quantiser chosen explicitly (same x, w, bias, stride, pad_lo, pad_hi,
 * dil, out and stream).  Each row of the implicit im2col matrix A is split
 * into blocks of block_size consecutive K columns (K ordered (c, kd, kh,
 * kw); a short last block acts as zero-filled), every element is rounded to
 * E2M1 with its block's scale and dequantised, then rounded to BF16:
 *   quant_format Q3D_QUANT_NONE   no quantisation (block_size ignored).
 *   quant_format Q3D_QUANT_NVFP4  the article's quantiser (sec. 6.1-6.3)
 *       with its call's fp4_block_size (sec. 7.1): block_size 16, 32, 64,
 *       128 or 256; act_amax required as for conv3d_implicit_gemm.
 *   quant_format Q3D_QUANT_MXFP4  the CANN aclnnFlatQuantV2 page's per-group
 *       route: block_size 32, scale 2^E with E = floor(log2(block max)) - 2
 *       (dst_type_max 0) or the exponent of block max / dst_type_max rounded
 *       up (dst_type_max in [6, 12]), as in mxfp4_quantize; act_amax unused.
 * NVFP4 with block_size 16 runs the same kernels as
 * conv3d_implicit_gemm_pad2 (bit-identical results).  NVFP4 blocks of 32
 * and 64 and MXFP4 run the tensor-memory kernel where its tensor maps apply
 * (rows of x a multiple of 16 bytes; blocks of 64 also need its plan with A
 * in shared memory), with each group's maximum taken inside the thread or
 * thread pair that builds the row; blocks of 128 and 256, and every setting
 * the tensor-memory kernel does not take, run the general kernel, which
 * takes each block's maximum in a separate gather pass.  All kernels build
 * the same quantised operand, bit for bit.  Q3D_ERR_INVALID_ARG for another format, block size or
 * dst_type_max, before anything is enqueued.
 */
Q3D_API q3d_status conv3d_implicit_gemm_ex(const q3d_tensor* x, const q3d_tensor* w, const q3d_tensor* bias,
                                           const float* act_amax, const int32_t stride[3],
                                           const int32_t pad_lo[3], const int32_t pad_hi[3],
                                           const int32_t dil[3], int32_t quant_format, int32_t block_size,
                                           float dst_type_max, q3d_tensor* out, q3d_stream_t stream);

/*
 * conv3d_implicit_gemm_noalloc -- as conv3d_implicit_gemm_pad2 (same
 * arguments, same kernels, same result), for callers that may not allocate
 * device memory during the call.  The article has no counterpart to this
 * entry point.
 *
 * Weights that cannot be read in place (dtype other than BF16, K not a
 * multiple of 8, or a base that is not 16-byte aligned) are converted to
 * BF16 [Cout, ld], ld = K rounded up to a multiple of 8, into a fixed
 * staging area compiled into the library (16 MiB per device, reserved when
 * the library module holding it first loads on that device), instead of a
 * stream-ordered allocation.  Nothing there needs to start at zero: the
 * staging kernel writes every byte the convolution reads, padding columns
 * included.
 *   - Limit: Cout * ld * 2 <= 16 MiB (e.g. Cout 384 with Cin 384 and a
 *     3x3x3 kernel, or Cout 512 with Cin 512); larger staged weights are
 *     rejected with Q3D_ERR_UNSUPPORTED_SHAPE before anything is enqueued.
 *     BF16 weights usable in place have no limit.
 *   - The first call on each device looks up the staging area's address
 *     (cudaGetSymbolAddress) with that device current; make that first
 *     call before any stream capture begins.  A failed lookup returns
 *     Q3D_ERR_CUDA.
 *   - There is one staging area per device: two calls that stage weights
 *     and may run at the same time on one device (different streams, or
 *     different host threads) race on it and may read each other's
 *     weights.  Calls ordered on one stream are safe.
 */
Q3D_API q3d_status conv3d_implicit_gemm_noalloc(const q3d_tensor* x, const q3d_tensor* w, const q3d_tensor* bias,
                                        const float* act_amax, const int32_t stride[3],
                                        const int32_t pad_lo[3], const int32_t pad_hi[3],
                                        const int32_t dil[3], int32_t quant_act, q3d_tensor* out,
                                        q3d_stream_t stream);

/*
 * The true-FP4 convolution: both operands quantised to NVFP4 and multiplied
 * by the block-scaled tensor core (tcgen05.mma kind::mxf4nvf4).  The formats
 * and codes are those of the article's quantiser (sec. 6.1-6.3: E2M1 values,
 * an E4M3 scale E4M3(min(bmax / (6 g), 448)) per block of 16 consecutive K
 * elements of a row, g = amax / (6 * 448)), applied to the activations with
 * act_amax and, along their reduction axis K (sec. 7.2), to the weights with
 * their own w_amax; the tensor core multiplies the codes and scales exactly
 * and accumulates in FP32, and the epilogue multiplies by
 * RN(g_act * g_w) and adds the bias.  The article dequantises to BF16
 * instead, so the result differs from conv3d_implicit_gemm by the BF16
 * rounding of both operands (and the weights are quantised here).  A block
 * whose scale would take the article's 1.0 fallback (E4M3 code times g below
 * 1e-5) contributes zero: 1.0 is no E4M3 scale times g.
 *
 * q3d_fp4_weight_bytes -- size in bytes of the packed weights of a
 * [Cout, Cin, kd, kh, kw] weight tensor; -1 for a non-positive extent.
 *
 * conv3d_fp4_pack_weights -- quantise w into `packed`, once per set of
 * weights (the convolution reads nothing else of w).
 *   w        [Cout, Cin, kd, kh, kw] F32/F16/BF16, contiguous, on the device.
 *   w_amax   device pointer to one float: the weights' global amax, e.g.
 *            from q3d_act_amax(w).
 *   packed   device buffer of packed_bytes >= q3d_fp4_weight_bytes(w.shape)
 *            bytes, 256-byte aligned, not overlapping w; owned by the
 *            caller.  Layout (opaque to callers, stated for the record): a
 *            256-byte header whose first word is g_w, then per K slice of
 *            64 and per N-part of the tile plan an image of the codes in
 *            the layout the MMA reads and the scale bytes.
 * Enqueues a memset of the buffer and one kernel on `stream`.
 *
 * conv3d_implicit_gemm_fp4 -- the convolution over packed weights.
 *   x, bias, stride, pad_lo, pad_hi, dil, out, stream  as for
 *            conv3d_implicit_gemm_pad2 (quant_act implied).
 *   packed_w the buffer written by conv3d_fp4_pack_weights for weights of
 *            shape w_shape (not checked against it on the host).
 *   act_amax device pointer to one float: the activations' global amax.
 * Runs on the tensor-memory kernel only: x 16-byte aligned with rows of W a
 * multiple of 16 bytes and at most 343 taps, else
 * Q3D_ERR_UNSUPPORTED_SHAPE.  Q3D_ERR_NULLPTR / _INVALID_ARG /
 * _UNSUPPORTED_DTYPE as for conv3d_implicit_gemm_pad2, before anything is
 * enqueued.
 */
Q3D_API int64_t q3d_fp4_weight_bytes(const int64_t w_shape[5]);
Q3D_API q3d_status conv3d_fp4_pack_weights(const q3d_tensor* w, const float* w_amax, void* packed, int64_t packed_bytes,
                                           q3d_stream_t stream);
Q3D_API q3d_status conv3d_implicit_gemm_fp4(const q3d_tensor* x, const void* packed_w, const int64_t w_shape[5],
                                            const q3d_tensor* bias, const float* act_amax, const int32_t stride[3],
                                            const int32_t pad_lo[3], const int32_t pad_hi[3], const int32_t dil[3],
                                            q3d_tensor* out, q3d_stream_t stream);

/*
 * fp4_fake_quant -- out = NVFP4 fake-quantisation of x (sec. 6.4, 7.3).
 *   x     any rank 1..5, dtype F32/F16/BF16, numel % 16 == 0; consecutive
 *         groups of 16 elements in memory order form the blocks.
 *   amax  device pointer to one float (finite, >= 0): the global amax.
 *   out   same shape and dtype as x; may be the same buffer as x (in place)
 *         but must not partially overlap it.
 * Each output is the binary32 result sign * E2M1(|v|/s) * s rounded (RNE) to
 * the dtype; bit-exact with the CPU oracle.
 */
Q3D_API q3d_status fp4_fake_quant(const q3d_tensor* x, const float* amax, q3d_tensor* out, q3d_stream_t stream);

/*
 * fp4_fake_quant_bs -- fp4_fake_quant with the other block sizes the
 * article's call accepts (sec. 7.1: fp4_block_size 16, 32, 64, 128 or 256;
 * sec. 7.3: the flat tensor viewed as [numel / block_size, block_size]).
 *   block_size  16, 32, 64, 128 or 256; numel % block_size == 0.
 *   x, amax, out  as for fp4_fake_quant (block_size 16 is that call).
 * Each block of block_size consecutive elements takes one E4M3 scale from
 * its own |v| maximum; the quantiser is otherwise the same.  Bit-exact with
 * the CPU oracle.  Q3D_ERR_INVALID_ARG for another block size or a numel
 * that is not a multiple of it, before anything is enqueued.
 */
Q3D_API q3d_status fp4_fake_quant_bs(const q3d_tensor* x, const float* amax, int32_t block_size, q3d_tensor* out,
                                     q3d_stream_t stream);

/*
 * mxfp4_quantize -- MXFP4 quantisation of x: groups of 32 consecutive
 * elements (memory order) share one power-of-two scale 2^E, stored as an
 * E8M0 byte E + 127, and every element becomes an E2M1 value (round to
 * nearest, ties to even, saturating at 6).  Follows the CANN
 * aclnnFlatQuantV2 page, its per-group route with FLOAT4_E2M1 output
 * (step 3) and the dstTypeMax rule (step 4):
 *   dst_type_max == 0:  E = floor(log2(group max |x|)) - 2;
 *   dst_type_max in [6, 12]:  E = exponent of S = group max / dst_type_max
 *       (binary32 division), plus one when S is normal, below the top binade
 *       and not a power of two (the scale rounds up);
 *   E is clamped to [-127, 127] (a zero or subnormal maximum or S gives -127).
 * Arguments (device pointers, caller-owned):
 *   x       rank 1..5, F32/F16/BF16, numel % 32 == 0.
 *   out     NULL, or the dequantised tensor E2M1 * 2^E in x's shape and
 *           dtype (may be x itself, not a partial overlap).
 *   scales  NULL, or numel / 32 bytes: the E8M0 byte of each group in order.
 *   codes   NULL, or numel / 2 bytes of packed E2M1 codes (sign in bit 3 of
 *           each nibble; element 2i in the low nibble of byte i).
 * At least one of out, scales, codes; none may overlap x or each other.
 * Bit-exact with the CPU oracle.  Q3D_ERR_NULLPTR / _INVALID_ARG (numel,
 * dst_type_max, shape, overlap) / _UNSUPPORTED_DTYPE before anything is
 * enqueued.
 */
Q3D_API q3d_status mxfp4_quantize(const q3d_tensor* x, float dst_type_max, q3d_tensor* out, uint8_t* scales,
                                  uint8_t* codes, q3d_stream_t stream);

/*
 * q3d_act_amax -- *amax = max |x| over every element of x, the global amax
 * that conv3d_implicit_gemm(quant_act) and fp4_fake_quant take.  The article
 * feeds its quantiser this scalar: its usage example (sec. 7.2) passes
 * x.abs().max(), and the quantised inference path (sec. 8.3) gets it from
 * the input quantizer.
 *   x     any rank 1..5, dtype F32/F16/BF16, numel >= 0, any alignment.
 *   amax  device pointer to one float (4-byte aligned, not inside x),
 *         written with the binary32 value of the largest |x[i]| (exact: the
 *         value of an input element, widened to binary32); 0 when x is
 *         empty.  It can be passed straight on as act_amax / amax.
 * Enqueues a 4-byte memset of *amax and one streaming kernel on `stream`.
 * NaN in x: the result is unspecified (a NaN).  Q3D_ERR_NULLPTR /
 * _INVALID_ARG / _UNSUPPORTED_DTYPE before anything is enqueued.
 */
Q3D_API q3d_status q3d_act_amax(const q3d_tensor* x, float* amax, q3d_stream_t stream);

/* Message for the last non-OK status returned on this host thread ("" if
 * none).  The pointer stays valid until the next call on this thread. */
Q3D_API const char* q3d_last_error(void);

/* Synchronise `stream`, then read and clear the device error word set by
 * bounded waits that gave up.  Returns Q3D_OK, Q3D_ERR_DEVICE_TIMEOUT or
 * Q3D_ERR_CUDA.  *site_bits (if not NULL) receives the bit mask of the
 * waits that gave up. */
Q3D_API q3d_status q3d_check_device_error(q3d_stream_t stream, uint32_t* site_bits);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
Q3D_API int32_t q3d_version(void);

/*
 * q3d_conv_out_shape -- out_shape = [N, Cout, OD, OH, OW] of a convolution
 * of x [N, Cin, D, H, W] with w [Cout, Cin, kD, kH, kW] (host only, no CUDA
 * call, no device needed): the output extents of
 * torch.nn.functional.conv3d, which the article's call promises (sec. 7.1),
 * with separate leading and trailing padding:
 *   OD = floor((D + pad_lo_d + pad_hi_d - dil_d*(kD-1) - 1) / stride_d) + 1,
 * likewise OH, OW.  All arrays are host arrays.  Q3D_ERR_NULLPTR,
 * Q3D_ERR_INVALID_ARG (Cin mismatch, N or Cout < 0, stride or dilation < 1,
 * pad < 0, kernel extent < 1, or an empty output extent).
 */
Q3D_API q3d_status q3d_conv_out_shape(const int64_t x_shape[5], const int64_t w_shape[5], const int32_t stride[3],
                                      const int32_t pad_lo[3], const int32_t pad_hi[3], const int32_t dil[3],
                                      int64_t out_shape[5]);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* Q3D_H_ */
