// q3d_api.cu -- the C ABI declared in include/q3d.h: host-side argument
// validation, output-extent arithmetic, dispatch, and the device error word.
//
// Argument rules follow the Model-Optimizer "Conv3D Implicit GEMM CUDA
// kernel" article, sec. 7.1 and 7.3 (5-D tensors, the Cin of w equal to the
// Cin of x since groups must be 1, numel divisible by the block size for the
// standalone call, output dtype equal to the input dtype) and sec. 5.4 (the
// device architecture is checked before dispatch; here compute capability
// 10.x, the only target this library is built for).
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include <cuda.h>
#include <cuda_runtime.h>

#include "q3d.h"
#include "q3d_testing.h"
#include "q3d_internal.h"

namespace q3d {
cudaError_t launch_conv3d_basic(const ConvGeom& g, const ConvLaunch& L, cudaStream_t s, const char** why);
cudaError_t launch_conv3d_fast(const ConvGeom& g, const ConvLaunch& L, cudaStream_t s, const char** why,
                               bool* handled);
cudaError_t launch_conv3d_tmem(const ConvGeom& g, const ConvLaunch& L, cudaStream_t s, const char** why,
                               bool* handled);
}  // namespace q3d

namespace {

thread_local std::string g_last_error;

// One word per device; bounded waits that give up OR their site bit into it.
__device__ unsigned int g_device_error_word;

q3d_status fail(q3d_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
q3d_status fail(q3d_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

q3d_status cuda_fail(cudaError_t e, const char* what) {
  return fail(Q3D_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

struct DeviceInfo {
  bool init = false;
  int major = 0, minor = 0, sm_count = 0;
  unsigned int* err_word = nullptr;
  // the library's own stream-ordered pool for per-call scratch (the BF16
  // copy of weights that cannot be read in place): freed blocks stay cached up to
  // kPoolKeepBytes across synchronisations, so a call after a synchronise
  // does not map fresh memory while the GPU waits; the process's default
  // pool is left as it is
  cudaMemPool_t pool = nullptr;
};
constexpr uint64_t kPoolKeepBytes = uint64_t{1} << 30;
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Resolve the current device, check its architecture, and fetch the device
// address of its error word (once per device).
q3d_status current_device(DeviceInfo** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(Q3D_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
    d.major = prop.major;
    d.minor = prop.minor;
    d.sm_count = prop.multiProcessorCount;
    if (d.major == 10) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_device_error_word);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error word)");
      d.err_word = static_cast<unsigned int*>(p);
      cudaMemPoolProps props = {};
      props.allocType = cudaMemAllocationTypePinned;
      props.handleTypes = cudaMemHandleTypeNone;
      props.location.type = cudaMemLocationTypeDevice;
      props.location.id = dev;
      // without a pool of its own the library uses the default stream-ordered
      // allocator (correct, only slower after a synchronise)
      if (cudaMemPoolCreate(&d.pool, &props) == cudaSuccess) {
        uint64_t keep = kPoolKeepBytes;
        if (cudaMemPoolSetAttribute(d.pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess)
          cudaGetLastError();  // the pool still works, only without the kept blocks
      } else {
        d.pool = nullptr;
        cudaGetLastError();  // not an error of the caller's call
      }
    }
    d.init = true;
  }
  if (d.major != 10)
    return fail(Q3D_ERR_ARCH, "device %d has compute capability %d.%d; this library needs 10.x (sm_100a)", dev,
                d.major, d.minor);
  *out = &d;
  return Q3D_OK;
}

bool dtype_ok(int32_t dt) { return dt == Q3D_F32 || dt == Q3D_F16 || dt == Q3D_BF16; }

// Output extents of a convolution (torch.nn.functional.conv3d's formula with
// separate leading and trailing padding); Q3D_OK or an argument error.
q3d_status conv_out_dims(const int64_t in_dims[3], const int64_t k_dims[3], const int32_t stride[3],
                         const int32_t pad_lo[3], const int32_t pad_hi[3], const int32_t dil[3], int64_t o_dims[3]) {
  for (int i = 0; i < 3; ++i) {
    if (stride[i] < 1) return fail(Q3D_ERR_INVALID_ARG, "stride[%d] = %d must be >= 1", i, stride[i]);
    if (dil[i] < 1) return fail(Q3D_ERR_INVALID_ARG, "dilation[%d] = %d must be >= 1", i, dil[i]);
    if (pad_lo[i] < 0 || pad_hi[i] < 0) return fail(Q3D_ERR_INVALID_ARG, "padding[%d] must be >= 0", i);
    if (k_dims[i] < 1 || in_dims[i] < 0) return fail(Q3D_ERR_INVALID_ARG, "extents along dim %d must be >= 0", i);
    const int64_t span = in_dims[i] + pad_lo[i] + pad_hi[i] - static_cast<int64_t>(dil[i]) * (k_dims[i] - 1) - 1;
    if (span < 0)
      return fail(Q3D_ERR_INVALID_ARG, "kernel extent exceeds the padded input along dim %d (empty output)", i);
    o_dims[i] = span / stride[i] + 1;
  }
  return Q3D_OK;
}

int64_t dtype_size(int32_t dt) { return dt == Q3D_F32 ? 4 : 2; }

int64_t numel(const q3d_tensor* t) {
  int64_t n = 1;
  for (int i = 0; i < t->ndim; ++i) n *= t->shape[i];
  return n;
}

bool overlaps(const q3d_tensor* a, const q3d_tensor* b) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a->data), b0 = reinterpret_cast<uintptr_t>(b->data);
  const uintptr_t a1 = a0 + static_cast<uintptr_t>(numel(a) * dtype_size(a->dtype));
  const uintptr_t b1 = b0 + static_cast<uintptr_t>(numel(b) * dtype_size(b->dtype));
  return a0 < b1 && b0 < a1 && a1 > a0 && b1 > b0;
}

q3d_status check_tensor(const q3d_tensor* t, const char* name, int ndim) {
  if (!t) return fail(Q3D_ERR_NULLPTR, "%s is NULL", name);
  if (t->ndim != ndim) return fail(Q3D_ERR_INVALID_ARG, "%s must have rank %d (got %d)", name, ndim, t->ndim);
  for (int i = 0; i < ndim; ++i)
    if (t->shape[i] < 0) return fail(Q3D_ERR_INVALID_ARG, "%s.shape[%d] is negative", name, i);
  if (!dtype_ok(t->dtype)) return fail(Q3D_ERR_UNSUPPORTED_DTYPE, "%s dtype %d is not F32/F16/BF16", name, t->dtype);
  if (!t->data && numel(t) > 0) return fail(Q3D_ERR_NULLPTR, "%s.data is NULL", name);
  return Q3D_OK;
}

// Host-side checks and geometry shared by the convolution entry points.
// Returns Q3D_OK with *noop set for an empty batch or Cout == 0 (nothing to
// enqueue); otherwise fills *g and *L (weights not yet staged).  With
// w_is_tensor false, w only describes the weights' shape (its data is a
// packed buffer whose overlap the caller checks).
q3d_status prepare_conv(const q3d_tensor* x, const q3d_tensor* w, const q3d_tensor* bias, const float* act_amax,
                        const int32_t stride[3], const int32_t pad_lo[3], const int32_t pad_hi[3],
                        const int32_t dil[3], int32_t quant_act, q3d_tensor* out, q3d::ConvGeom* gp,
                        q3d::ConvLaunch* Lp, bool* noop, bool w_is_tensor = true) {
  *noop = false;
  q3d_status st;
  if ((st = check_tensor(x, "x", 5)) != Q3D_OK) return st;
  if ((st = check_tensor(w, "w", 5)) != Q3D_OK) return st;
  if ((st = check_tensor(out, "out", 5)) != Q3D_OK) return st;
  if (bias && (st = check_tensor(bias, "bias", 1)) != Q3D_OK) return st;
  if (!stride || !pad_lo || !pad_hi || !dil) return fail(Q3D_ERR_NULLPTR, "stride/pad/dil array is NULL");
  if (quant_act && !act_amax) return fail(Q3D_ERR_NULLPTR, "quant_act requires act_amax");
  if (w->dtype != x->dtype || out->dtype != x->dtype || (bias && bias->dtype != x->dtype))
    return fail(Q3D_ERR_UNSUPPORTED_DTYPE, "w, bias and out must have the dtype of x");
  const int64_t N = x->shape[0], C = x->shape[1], D = x->shape[2], H = x->shape[3], W = x->shape[4];
  const int64_t Cout = w->shape[0], KD = w->shape[2], KH = w->shape[3], KW = w->shape[4];
  if (w->shape[1] != C)
    return fail(Q3D_ERR_INVALID_ARG, "w has %lld input channels but x has %lld (groups != 1 is not supported)",
                (long long)w->shape[1], (long long)C);
  if (C < 1 || KD < 1 || KH < 1 || KW < 1)
    return fail(Q3D_ERR_INVALID_ARG, "Cin and kernel extents must be >= 1");
  if (bias && bias->shape[0] != Cout) return fail(Q3D_ERR_INVALID_ARG, "bias must have shape [Cout]");
  const int64_t in_dims[3] = {D, H, W}, k_dims[3] = {KD, KH, KW};
  int64_t o_dims[3];
  if ((st = conv_out_dims(in_dims, k_dims, stride, pad_lo, pad_hi, dil, o_dims)) != Q3D_OK) return st;
  if (out->shape[0] != N || out->shape[1] != Cout || out->shape[2] != o_dims[0] || out->shape[3] != o_dims[1] ||
      out->shape[4] != o_dims[2])
    return fail(Q3D_ERR_INVALID_ARG, "out must have shape [%lld, %lld, %lld, %lld, %lld]", (long long)N,
                (long long)Cout, (long long)o_dims[0], (long long)o_dims[1], (long long)o_dims[2]);
  if (N == 0 || Cout == 0) {  // empty batch or no output channels: nothing to compute
    *noop = true;
    return Q3D_OK;
  }
  if (overlaps(out, x) || (w_is_tensor && overlaps(out, w)) || (bias && overlaps(out, bias)))
    return fail(Q3D_ERR_INVALID_ARG, "out overlaps an input tensor");
  const int64_t K = C * KD * KH * KW;
  const int64_t M = N * o_dims[0] * o_dims[1] * o_dims[2];
  if (K > 0x7FFFFFFFll / 2 || Cout > 0x7FFFFFFFll || numel(x) > 0x7FFFFFFFll || numel(out) > (1ll << 40) ||
      C * D * H * W > 0x7FFFFFFFll)
    return fail(Q3D_ERR_UNSUPPORTED_SHAPE, "problem exceeds the 32-bit per-sample index range of the kernels");

  DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != Q3D_OK) return st;

  q3d::ConvGeom& g = *gp;
  g.N = (int32_t)N; g.C = (int32_t)C; g.D = (int32_t)D; g.H = (int32_t)H; g.W = (int32_t)W;
  g.Cout = (int32_t)Cout; g.KD = (int32_t)KD; g.KH = (int32_t)KH; g.KW = (int32_t)KW;
  g.sd = stride[0]; g.sh = stride[1]; g.sw = stride[2];
  g.pd = pad_lo[0]; g.ph = pad_lo[1]; g.pw = pad_lo[2];
  g.dd = dil[0]; g.dh = dil[1]; g.dw = dil[2];
  g.OD = (int32_t)o_dims[0]; g.OH = (int32_t)o_dims[1]; g.OW = (int32_t)o_dims[2];
  g.M = M; g.K = (int32_t)K; g.taps = (int32_t)(KD * KH * KW);

  q3d::ConvLaunch& L = *Lp;
  L.x = x->data; L.bias = bias ? bias->data : nullptr; L.y = out->data;
  L.act_amax = quant_act ? act_amax : nullptr;
  L.dtype = x->dtype; L.quant = quant_act ? 1 : 0; L.err = dev->err_word; L.sm_count = dev->sm_count;
  L.pool = dev->pool;
  return Q3D_OK;
}

// The convolution kernels proper, once the BF16 weights are in place: the
// tensor-memory kernel where it applies, else the shared-memory specialised
// kernel, else the general one.  Each declines what it does not cover: the
// tensor-memory kernel takes NVFP4 blocks of 16 or 32 and MXFP4, the
// specialised one NVFP4 blocks of 16 only, the general one every format.  Q3D_KERNEL=tmem|fast|basic starts the chain
// at that kernel, and Q3D_KERNEL=smem_a runs the tensor-memory kernel with
// its A operand in shared memory wherever that form applies (all compute the
// same result).
cudaError_t launch_conv(const q3d::ConvGeom& g, const q3d::ConvLaunch& L, cudaStream_t s, const char** why) {
  const char* kc = getenv("Q3D_KERNEL");
  const int first = (kc && !strcmp(kc, "basic")) ? 2 : (kc && !strcmp(kc, "fast")) ? 1 : 0;
  bool handled = false;
  cudaError_t e = cudaSuccess;
  if (first <= 0) {
    e = q3d::launch_conv3d_tmem(g, L, s, why, &handled);
    if (e != cudaSuccess || handled) return e;
  }
  if (first <= 1) {
    e = q3d::launch_conv3d_fast(g, L, s, why, &handled);
    if (e != cudaSuccess || handled) return e;
  }
  return q3d::launch_conv3d_basic(g, L, s, why);
}

}  // namespace

namespace q3d {

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace q3d

extern "C" {

const char* q3d_last_error(void) { return g_last_error.c_str(); }

int32_t q3d_version(void) { return 100; }

}  // extern "C"

namespace {

// Weight staging and the kernel chain for a prepared convolution.
q3d_status run_conv(const q3d::ConvGeom& g, q3d::ConvLaunch& L, const q3d_tensor* w, int32_t dtype,
                    q3d_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t K = g.K, Cout = g.Cout;

  // B operand: BF16 [Cout, ld] with a 16-byte row pitch.  BF16 weights with
  // K % 8 == 0 and a 16-byte aligned base are used in place; otherwise a
  // stream-ordered scratch copy is made.
  void* scratch = nullptr;
  cudaError_t e;
  if (dtype == Q3D_BF16 && K % 8 == 0 && reinterpret_cast<uintptr_t>(w->data) % 16 == 0) {
    L.w_bf16 = w->data;
    L.w_ld = K;
  } else {
    const int64_t ld = (K + 7) / 8 * 8;
    e = L.pool ? cudaMallocFromPoolAsync(&scratch, static_cast<size_t>(Cout * ld * 2), L.pool, s)
               : cudaMallocAsync(&scratch, static_cast<size_t>(Cout * ld * 2), s);
    if (e != cudaSuccess) return cuda_fail(e, "stream-ordered allocation (weight staging)");
    e = q3d::launch_stage_weights(w->data, dtype, (int32_t)Cout, (int32_t)K, ld, scratch, s);
    if (e != cudaSuccess) { cudaFreeAsync(scratch, s); return cuda_fail(e, "weight staging launch"); }
    L.w_bf16 = scratch;
    L.w_ld = ld;
  }

  const char* why = nullptr;
  e = launch_conv(g, L, s, &why);
  if (scratch) cudaFreeAsync(scratch, s);
  if (e != cudaSuccess) {
    if (why) return fail(Q3D_ERR_CUDA, "conv3d launch: %s (%s)", why, cudaGetErrorString(e));
    return cuda_fail(e, "conv3d launch");
  }
  return Q3D_OK;
}

}  // namespace

extern "C" {

q3d_status conv3d_implicit_gemm_pad2(const q3d_tensor* x, const q3d_tensor* w, const q3d_tensor* bias,
                                     const float* act_amax, const int32_t stride[3], const int32_t pad_lo[3],
                                     const int32_t pad_hi[3], const int32_t dil[3], int32_t quant_act,
                                     q3d_tensor* out, q3d_stream_t stream) {
  q3d::ConvGeom g;
  q3d::ConvLaunch L;
  bool noop = false;
  q3d_status st = prepare_conv(x, w, bias, act_amax, stride, pad_lo, pad_hi, dil, quant_act, out, &g, &L, &noop);
  if (st != Q3D_OK || noop) return st;
  return run_conv(g, L, w, x->dtype, stream);
}

q3d_status conv3d_implicit_gemm_ex(const q3d_tensor* x, const q3d_tensor* w, const q3d_tensor* bias,
                                   const float* act_amax, const int32_t stride[3], const int32_t pad_lo[3],
                                   const int32_t pad_hi[3], const int32_t dil[3], int32_t quant_format,
                                   int32_t block_size, float dst_type_max, q3d_tensor* out, q3d_stream_t stream) {
  if (quant_format != Q3D_QUANT_NONE && quant_format != Q3D_QUANT_NVFP4 && quant_format != Q3D_QUANT_MXFP4)
    return fail(Q3D_ERR_INVALID_ARG, "quant_format %d is not NONE, NVFP4 or MXFP4", quant_format);
  if (quant_format == Q3D_QUANT_NVFP4 && block_size != 16 && block_size != 32 && block_size != 64 &&
      block_size != 128 && block_size != 256)
    return fail(Q3D_ERR_INVALID_ARG, "NVFP4 block_size %d is not 16, 32, 64, 128 or 256", block_size);
  if (quant_format == Q3D_QUANT_MXFP4) {
    if (block_size != 32) return fail(Q3D_ERR_INVALID_ARG, "MXFP4 block_size %d is not 32", block_size);
    if (!(dst_type_max == 0.0f || (dst_type_max >= 6.0f && dst_type_max <= 12.0f)))
      return fail(Q3D_ERR_INVALID_ARG, "dst_type_max must be 0 or in [6, 12]");
  }
  q3d::ConvGeom g;
  q3d::ConvLaunch L;
  bool noop = false;
  // NVFP4 needs the global amax; MXFP4 scales come from each group alone
  q3d_status st = prepare_conv(x, w, bias, quant_format == Q3D_QUANT_NVFP4 ? act_amax : nullptr, stride, pad_lo,
                               pad_hi, dil, quant_format == Q3D_QUANT_NVFP4 ? 1 : 0, out, &g, &L, &noop);
  if (st != Q3D_OK || noop) return st;
  L.quant = quant_format != Q3D_QUANT_NONE ? 1 : 0;
  L.qfmt = quant_format == Q3D_QUANT_MXFP4 ? 2 : 1;
  L.qblock = quant_format == Q3D_QUANT_NONE ? 16 : block_size;
  L.dst_max = dst_type_max;
  return run_conv(g, L, w, x->dtype, stream);
}

int64_t q3d_fp4_weight_bytes(const int64_t w_shape[5]) {
  if (!w_shape) return -1;
  for (int i = 0; i < 5; ++i)
    if (w_shape[i] < 1) return -1;
  const int64_t K = w_shape[1] * w_shape[2] * w_shape[3] * w_shape[4];
  q3d::Fp4WeightLayout lay;
  if (!q3d::fp4_weight_layout(w_shape[0], K, &lay)) return -1;
  return lay.bytes;
}

q3d_status conv3d_fp4_pack_weights(const q3d_tensor* w, const float* w_amax, void* packed, int64_t packed_bytes,
                                   q3d_stream_t stream) {
  q3d_status st;
  if ((st = check_tensor(w, "w", 5)) != Q3D_OK) return st;
  if (!w_amax) return fail(Q3D_ERR_NULLPTR, "w_amax is NULL");
  if (!packed) return fail(Q3D_ERR_NULLPTR, "packed is NULL");
  const int64_t need = q3d_fp4_weight_bytes(w->shape);
  if (need < 0) return fail(Q3D_ERR_INVALID_ARG, "w must have positive extents (and at most 2^20 output channels)");
  if (packed_bytes < need)
    return fail(Q3D_ERR_INVALID_ARG, "packed holds %lld bytes; these weights need %lld", (long long)packed_bytes,
                (long long)need);
  if (reinterpret_cast<uintptr_t>(packed) % 256 != 0) return fail(Q3D_ERR_INVALID_ARG, "packed must be 256-byte aligned");
  const uintptr_t p0 = reinterpret_cast<uintptr_t>(packed), w0 = reinterpret_cast<uintptr_t>(w->data);
  const uintptr_t w1 = w0 + static_cast<uintptr_t>(numel(w) * dtype_size(w->dtype));
  if (p0 < w1 && w0 < p0 + static_cast<uintptr_t>(need)) return fail(Q3D_ERR_INVALID_ARG, "packed overlaps w");
  const int64_t K = w->shape[1] * w->shape[2] * w->shape[3] * w->shape[4];
  if (K > 0x7FFFFFFFll / 2) return fail(Q3D_ERR_UNSUPPORTED_SHAPE, "K exceeds the 32-bit index range");
  DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != Q3D_OK) return st;
  q3d::Fp4WeightLayout lay;
  q3d::fp4_weight_layout(w->shape[0], K, &lay);
  const cudaError_t e = q3d::launch_fp4_pack_weights(w->data, w->dtype, static_cast<int32_t>(w->shape[0]),
                                                     static_cast<int32_t>(K), w_amax, packed, lay,
                                                     reinterpret_cast<cudaStream_t>(stream), dev->sm_count);
  if (e != cudaSuccess) return cuda_fail(e, "NVFP4 weight packing");
  return Q3D_OK;
}

q3d_status conv3d_implicit_gemm_fp4(const q3d_tensor* x, const void* packed_w, const int64_t w_shape[5],
                                    const q3d_tensor* bias, const float* act_amax, const int32_t stride[3],
                                    const int32_t pad_lo[3], const int32_t pad_hi[3], const int32_t dil[3],
                                    q3d_tensor* out, q3d_stream_t stream) {
  if (!x) return fail(Q3D_ERR_NULLPTR, "x is NULL");
  if (!packed_w) return fail(Q3D_ERR_NULLPTR, "packed_w is NULL");
  if (!w_shape) return fail(Q3D_ERR_NULLPTR, "w_shape is NULL");
  if (!act_amax) return fail(Q3D_ERR_NULLPTR, "act_amax is NULL");
  const int64_t need = q3d_fp4_weight_bytes(w_shape);
  if (need < 0) return fail(Q3D_ERR_INVALID_ARG, "w_shape must have positive extents");
  if (reinterpret_cast<uintptr_t>(packed_w) % 256 != 0)
    return fail(Q3D_ERR_INVALID_ARG, "packed_w must be 256-byte aligned");
  // the weights' shape, for the shared checks (their data is the packed buffer)
  q3d_tensor wd;
  wd.data = const_cast<void*>(packed_w);
  wd.dtype = x->dtype;
  wd.ndim = 5;
  for (int i = 0; i < 5; ++i) wd.shape[i] = w_shape[i];
  if (out && out->ndim == 5 && dtype_ok(out->dtype)) {
    const uintptr_t o0 = reinterpret_cast<uintptr_t>(out->data), p0 = reinterpret_cast<uintptr_t>(packed_w);
    if (o0 < p0 + static_cast<uintptr_t>(need) && p0 < o0 + static_cast<uintptr_t>(numel(out) * dtype_size(out->dtype)))
      return fail(Q3D_ERR_INVALID_ARG, "out overlaps packed_w");
  }
  q3d::ConvGeom g;
  q3d::ConvLaunch L;
  bool noop = false;
  q3d_status st = prepare_conv(x, &wd, bias, act_amax, stride, pad_lo, pad_hi, dil, 1, out, &g, &L, &noop,
                               /*w_is_tensor=*/false);
  if (st != Q3D_OK || noop) return st;
  const char* why = nullptr;
  bool handled = false;
  const cudaError_t e = q3d::launch_conv3d_fp4(g, L, packed_w, reinterpret_cast<cudaStream_t>(stream), &why, &handled);
  if (e != cudaSuccess) {
    if (why) return fail(Q3D_ERR_CUDA, "NVFP4 conv3d launch: %s (%s)", why, cudaGetErrorString(e));
    return cuda_fail(e, "NVFP4 conv3d launch");
  }
  if (!handled)
    return fail(Q3D_ERR_UNSUPPORTED_SHAPE,
                "the NVFP4-operand convolution needs a 16-byte aligned x whose rows are a multiple of 16 bytes, at "
                "most 343 taps, and a tile plan that fits");
  return Q3D_OK;
}

q3d_status conv3d_implicit_gemm(const q3d_tensor* x, const q3d_tensor* w, const q3d_tensor* bias,
                                const float* act_amax, const int32_t stride[3], const int32_t pad[3],
                                const int32_t dil[3], int32_t quant_act, q3d_tensor* out, q3d_stream_t stream) {
  if (!pad) return fail(Q3D_ERR_NULLPTR, "pad is NULL");
  return conv3d_implicit_gemm_pad2(x, w, bias, act_amax, stride, pad, pad, dil, quant_act, out, stream);
}

q3d_status conv3d_implicit_gemm_noalloc(const q3d_tensor* x, const q3d_tensor* w, const q3d_tensor* bias,
                                        const float* act_amax, const int32_t stride[3], const int32_t pad_lo[3],
                                        const int32_t pad_hi[3], const int32_t dil[3], int32_t quant_act,
                                        q3d_tensor* out, q3d_stream_t stream) {
  q3d::ConvGeom g;
  q3d::ConvLaunch L;
  bool noop = false;
  q3d_status st = prepare_conv(x, w, bias, act_amax, stride, pad_lo, pad_hi, dil, quant_act, out, &g, &L, &noop);
  if (st != Q3D_OK || noop) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (x->dtype == Q3D_BF16 && g.K % 8 == 0 && reinterpret_cast<uintptr_t>(w->data) % 16 == 0) {
    L.w_bf16 = w->data;  // usable in place, as in conv3d_implicit_gemm_pad2
    L.w_ld = g.K;
  } else {
    const int64_t ld = (static_cast<int64_t>(g.K) + 7) / 8 * 8;
    const int64_t bytes = static_cast<int64_t>(g.Cout) * ld * 2;
    if (bytes > static_cast<int64_t>(q3d::kNoAllocStagingBytes))
      return fail(Q3D_ERR_UNSUPPORTED_SHAPE,
                  "staged BF16 weights need %lld bytes (Cout %d x %lld x 2) but the fixed staging area of "
                  "conv3d_implicit_gemm_noalloc holds %lld; use conv3d_implicit_gemm_pad2",
                  (long long)bytes, g.Cout, (long long)ld, (long long)q3d::kNoAllocStagingBytes);
    void* area = nullptr;
    e = q3d::noalloc_staging_area(&area);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc staging area)");
    e = q3d::launch_stage_weights(w->data, x->dtype, g.Cout, g.K, ld, area, s);
    if (e != cudaSuccess) return cuda_fail(e, "weight staging launch");
    L.w_bf16 = area;
    L.w_ld = ld;
  }
  const char* why = nullptr;
  e = launch_conv(g, L, s, &why);
  if (e != cudaSuccess) {
    if (why) return fail(Q3D_ERR_CUDA, "conv3d launch: %s (%s)", why, cudaGetErrorString(e));
    return cuda_fail(e, "conv3d launch");
  }
  return Q3D_OK;
}

}  // extern "C"

namespace {

q3d_status fake_quant_blocks(const q3d_tensor* x, const float* amax, int32_t block, q3d_tensor* out,
                             q3d_stream_t stream) {
  if (!x || !out) return fail(Q3D_ERR_NULLPTR, "x or out is NULL");
  if (!amax) return fail(Q3D_ERR_NULLPTR, "amax is NULL");
  if (block != 16 && block != 32 && block != 64 && block != 128 && block != 256)
    return fail(Q3D_ERR_INVALID_ARG, "block_size %d is not 16, 32, 64, 128 or 256", block);
  if (x->ndim < 1 || x->ndim > 5) return fail(Q3D_ERR_INVALID_ARG, "x must have rank 1..5");
  q3d_status st;
  if ((st = check_tensor(x, "x", x->ndim)) != Q3D_OK) return st;
  if ((st = check_tensor(out, "out", x->ndim)) != Q3D_OK) return st;
  if (out->dtype != x->dtype) return fail(Q3D_ERR_UNSUPPORTED_DTYPE, "out must have the dtype of x");
  for (int i = 0; i < x->ndim; ++i)
    if (out->shape[i] != x->shape[i]) return fail(Q3D_ERR_INVALID_ARG, "out must have the shape of x");
  const int64_t n = numel(x);
  if (n % block != 0)
    return fail(Q3D_ERR_INVALID_ARG, "numel (%lld) must be a multiple of the block size %d", (long long)n, block);
  if (n == 0) return Q3D_OK;
  if (out->data != x->data && overlaps(out, x))
    return fail(Q3D_ERR_INVALID_ARG, "out partially overlaps x");
  DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != Q3D_OK) return st;
  cudaError_t e = q3d::launch_fp4_fake_quant(x->data, out->data, x->dtype, n, block, amax,
                                             reinterpret_cast<cudaStream_t>(stream), dev->sm_count);
  if (e != cudaSuccess) return cuda_fail(e, "fp4_fake_quant launch");
  return Q3D_OK;
}

}  // namespace

extern "C" {

q3d_status fp4_fake_quant(const q3d_tensor* x, const float* amax, q3d_tensor* out, q3d_stream_t stream) {
  return fake_quant_blocks(x, amax, 16, out, stream);
}

q3d_status fp4_fake_quant_bs(const q3d_tensor* x, const float* amax, int32_t block_size, q3d_tensor* out,
                             q3d_stream_t stream) {
  return fake_quant_blocks(x, amax, block_size, out, stream);
}

q3d_status mxfp4_quantize(const q3d_tensor* x, float dst_type_max, q3d_tensor* out, uint8_t* scales, uint8_t* codes,
                          q3d_stream_t stream) {
  if (!x) return fail(Q3D_ERR_NULLPTR, "x is NULL");
  if (!out && !scales && !codes) return fail(Q3D_ERR_NULLPTR, "out, scales and codes are all NULL");
  if (!(dst_type_max == 0.0f || (dst_type_max >= 6.0f && dst_type_max <= 12.0f)))
    return fail(Q3D_ERR_INVALID_ARG, "dst_type_max must be 0 or in [6, 12]");
  if (x->ndim < 1 || x->ndim > 5) return fail(Q3D_ERR_INVALID_ARG, "x must have rank 1..5");
  q3d_status st;
  if ((st = check_tensor(x, "x", x->ndim)) != Q3D_OK) return st;
  if (out) {
    if ((st = check_tensor(out, "out", x->ndim)) != Q3D_OK) return st;
    if (out->dtype != x->dtype) return fail(Q3D_ERR_UNSUPPORTED_DTYPE, "out must have the dtype of x");
    for (int i = 0; i < x->ndim; ++i)
      if (out->shape[i] != x->shape[i]) return fail(Q3D_ERR_INVALID_ARG, "out must have the shape of x");
  }
  const int64_t n = numel(x);
  if (n % 32 != 0) return fail(Q3D_ERR_INVALID_ARG, "numel (%lld) must be a multiple of 32", (long long)n);
  if (n == 0) return Q3D_OK;
  const uintptr_t x0 = reinterpret_cast<uintptr_t>(x->data), x1 = x0 + static_cast<uintptr_t>(n * dtype_size(x->dtype));
  if (out && out->data != x->data && overlaps(out, x)) return fail(Q3D_ERR_INVALID_ARG, "out partially overlaps x");
  const struct { const uint8_t* p; int64_t bytes; const char* name; } side[2] = {{scales, n / 32, "scales"},
                                                                                 {codes, n / 2, "codes"}};
  for (const auto& b : side) {
    if (!b.p) continue;
    const uintptr_t b0 = reinterpret_cast<uintptr_t>(b.p), b1 = b0 + static_cast<uintptr_t>(b.bytes);
    if (b0 < x1 && x0 < b1) return fail(Q3D_ERR_INVALID_ARG, "%s overlaps x", b.name);
    if (out) {
      const uintptr_t o0 = reinterpret_cast<uintptr_t>(out->data), o1 = o0 + (x1 - x0);
      if (b0 < o1 && o0 < b1) return fail(Q3D_ERR_INVALID_ARG, "%s overlaps out", b.name);
    }
  }
  if (scales && codes) {
    const uintptr_t s0 = reinterpret_cast<uintptr_t>(scales), c0 = reinterpret_cast<uintptr_t>(codes);
    if (s0 < c0 + static_cast<uintptr_t>(n / 2) && c0 < s0 + static_cast<uintptr_t>(n / 32))
      return fail(Q3D_ERR_INVALID_ARG, "scales overlaps codes");
  }
  DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != Q3D_OK) return st;
  cudaError_t e = q3d::launch_mxfp4(x->data, out ? out->data : nullptr, scales, codes, x->dtype, n, dst_type_max,
                                    reinterpret_cast<cudaStream_t>(stream), dev->sm_count);
  if (e != cudaSuccess) return cuda_fail(e, "mxfp4 launch");
  return Q3D_OK;
}

q3d_status q3d_act_amax(const q3d_tensor* x, float* amax, q3d_stream_t stream) {
  if (!x) return fail(Q3D_ERR_NULLPTR, "x is NULL");
  if (!amax) return fail(Q3D_ERR_NULLPTR, "amax is NULL");
  if (x->ndim < 1 || x->ndim > 5) return fail(Q3D_ERR_INVALID_ARG, "x must have rank 1..5");
  q3d_status st;
  if ((st = check_tensor(x, "x", x->ndim)) != Q3D_OK) return st;
  const int64_t n = numel(x);
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(amax), x0 = reinterpret_cast<uintptr_t>(x->data);
  const uintptr_t x1 = x0 + static_cast<uintptr_t>(n * dtype_size(x->dtype));
  if (a0 + sizeof(float) > x0 && a0 < x1) return fail(Q3D_ERR_INVALID_ARG, "amax lies inside x");
  if (a0 % sizeof(float) != 0) return fail(Q3D_ERR_INVALID_ARG, "amax is not 4-byte aligned");
  DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != Q3D_OK) return st;
  cudaError_t e = q3d::launch_act_amax(x->data, x->dtype, n, amax, reinterpret_cast<cudaStream_t>(stream),
                                       dev->sm_count);
  if (e != cudaSuccess) return cuda_fail(e, "act_amax launch");
  return Q3D_OK;
}

q3d_status q3d_check_device_error(q3d_stream_t stream, uint32_t* site_bits) {
  DeviceInfo* dev = nullptr;
  q3d_status st;
  if ((st = current_device(&dev)) != Q3D_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int v = 0;
  e = cudaMemcpy(&v, dev->err_word, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (site_bits) *site_bits = v;
  if (v) {
    const unsigned int zero = 0;
    e = cudaMemcpy(dev->err_word, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
    return fail(Q3D_ERR_DEVICE_TIMEOUT, "a bounded device wait gave up (site bits 0x%x)", v);
  }
  return Q3D_OK;
}

q3d_status q3d_conv_out_shape(const int64_t x_shape[5], const int64_t w_shape[5], const int32_t stride[3],
                              const int32_t pad_lo[3], const int32_t pad_hi[3], const int32_t dil[3],
                              int64_t out_shape[5]) {
  if (!x_shape || !w_shape || !stride || !pad_lo || !pad_hi || !dil || !out_shape)
    return fail(Q3D_ERR_NULLPTR, "NULL pointer");
  if (w_shape[1] != x_shape[1])
    return fail(Q3D_ERR_INVALID_ARG, "w has %lld input channels but x has %lld (groups != 1 is not supported)",
                (long long)w_shape[1], (long long)x_shape[1]);
  if (x_shape[0] < 0 || w_shape[0] < 0) return fail(Q3D_ERR_INVALID_ARG, "N and Cout must be >= 0");
  const int64_t in_dims[3] = {x_shape[2], x_shape[3], x_shape[4]}, k_dims[3] = {w_shape[2], w_shape[3], w_shape[4]};
  int64_t o_dims[3];
  const q3d_status st = conv_out_dims(in_dims, k_dims, stride, pad_lo, pad_hi, dil, o_dims);
  if (st != Q3D_OK) return st;
  out_shape[0] = x_shape[0];
  out_shape[1] = w_shape[0];
  for (int i = 0; i < 3; ++i) out_shape[2 + i] = o_dims[i];
  return Q3D_OK;
}

q3d_status q3d_selftest_withheld_arrive(const q3d_tensor* x, const q3d_tensor* w, const int32_t stride[3],
                                        const int32_t pad_lo[3], const int32_t pad_hi[3], const int32_t dil[3],
                                        q3d_tensor* out, q3d_stream_t stream) {
  q3d::ConvGeom g;
  q3d::ConvLaunch L;
  bool noop = false;
  q3d_status st = prepare_conv(x, w, nullptr, nullptr, stride, pad_lo, pad_hi, dil, 0, out, &g, &L, &noop);
  if (st != Q3D_OK) return st;
  if (noop || x->dtype != Q3D_BF16 || g.K % 8 != 0 || reinterpret_cast<uintptr_t>(w->data) % 16 != 0)
    return fail(Q3D_ERR_INVALID_ARG, "the bounded-wait test takes BF16 weights usable in place and a non-empty output");
  L.w_bf16 = w->data;
  L.w_ld = g.K;
  L.withhold_arrive = 1;
  const char* why = nullptr;
  bool handled = false;
  cudaError_t e = q3d::launch_conv3d_tmem(g, L, reinterpret_cast<cudaStream_t>(stream), &why, &handled);
  if (e != cudaSuccess)
    return why ? fail(Q3D_ERR_INVALID_ARG, "%s", why) : cuda_fail(e, "bounded-wait test launch");
  if (!handled) return fail(Q3D_ERR_INVALID_ARG, "the tensor-memory kernel does not take this problem");
  return Q3D_OK;
}

q3d_status q3d_selftest_formats(const float* in, int64_t n, float* e2m1, float* e4m3, q3d_stream_t stream) {
  if (!in || !e2m1 || !e4m3) return fail(Q3D_ERR_NULLPTR, "NULL pointer");
  if (n < 0) return fail(Q3D_ERR_INVALID_ARG, "n < 0");
  DeviceInfo* dev = nullptr;
  q3d_status st;
  if ((st = current_device(&dev)) != Q3D_OK) return st;
  cudaError_t e = q3d::launch_selftest_formats(in, n, e2m1, e4m3, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return Q3D_OK;
}

q3d_status q3d_selftest_ratio(const float* bmax, const float* t, int64_t n, float* out, q3d_stream_t stream) {
  if (!bmax || !t || !out) return fail(Q3D_ERR_NULLPTR, "NULL pointer");
  if (n < 0) return fail(Q3D_ERR_INVALID_ARG, "n < 0");
  DeviceInfo* dev = nullptr;
  q3d_status st;
  if ((st = current_device(&dev)) != Q3D_OK) return st;
  cudaError_t e = q3d::launch_selftest_ratio(bmax, t, n, out, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return Q3D_OK;
}

// Geometry of a planning request (host only); Q3D_OK or an argument error.
static q3d_status plan_geom(const int64_t x_shape[5], const int64_t w_shape[5], const int32_t stride[3],
                            const int32_t pad_lo[3], const int32_t pad_hi[3], const int32_t dil[3], int32_t dtype,
                            int32_t* plan, q3d::ConvGeom* gp) {
  if (!x_shape || !w_shape || !stride || !pad_lo || !pad_hi || !dil || !plan)
    return fail(Q3D_ERR_NULLPTR, "NULL pointer");
  if (!dtype_ok(dtype)) return fail(Q3D_ERR_UNSUPPORTED_DTYPE, "dtype");
  q3d::ConvGeom& g = *gp;
  const int64_t k_dims[3] = {w_shape[2], w_shape[3], w_shape[4]};
  const int64_t in_dims[3] = {x_shape[2], x_shape[3], x_shape[4]};
  int64_t o_dims[3];
  const q3d_status st = conv_out_dims(in_dims, k_dims, stride, pad_lo, pad_hi, dil, o_dims);
  if (st != Q3D_OK) return st;
  if (w_shape[1] != x_shape[1]) return fail(Q3D_ERR_INVALID_ARG, "groups != 1");
  g.N = (int32_t)x_shape[0]; g.C = (int32_t)x_shape[1]; g.D = (int32_t)x_shape[2]; g.H = (int32_t)x_shape[3];
  g.W = (int32_t)x_shape[4];
  g.Cout = (int32_t)w_shape[0]; g.KD = (int32_t)k_dims[0]; g.KH = (int32_t)k_dims[1]; g.KW = (int32_t)k_dims[2];
  g.sd = stride[0]; g.sh = stride[1]; g.sw = stride[2];
  g.pd = pad_lo[0]; g.ph = pad_lo[1]; g.pw = pad_lo[2];
  g.dd = dil[0]; g.dh = dil[1]; g.dw = dil[2];
  g.OD = (int32_t)o_dims[0]; g.OH = (int32_t)o_dims[1]; g.OW = (int32_t)o_dims[2];
  g.M = x_shape[0] * o_dims[0] * o_dims[1] * o_dims[2];
  g.K = (int32_t)(x_shape[1] * k_dims[0] * k_dims[1] * k_dims[2]);
  g.taps = (int32_t)(k_dims[0] * k_dims[1] * k_dims[2]);
  return Q3D_OK;
}

q3d_status q3d_plan_conv(const int64_t x_shape[5], const int64_t w_shape[5], const int32_t stride[3],
                         const int32_t pad_lo[3], const int32_t pad_hi[3], const int32_t dil[3], int32_t dtype,
                         int32_t* plan, int32_t plan_len) {
  q3d::ConvGeom g;
  const q3d_status st = plan_geom(x_shape, w_shape, stride, pad_lo, pad_hi, dil, dtype, plan, &g);
  if (st != Q3D_OK) return st;
  q3d::plan_conv3d_fast(g, dtype, plan, plan_len);
  return Q3D_OK;
}

q3d_status q3d_plan_conv_fp4(const int64_t x_shape[5], const int64_t w_shape[5], const int32_t stride[3],
                             const int32_t pad_lo[3], const int32_t pad_hi[3], const int32_t dil[3], int32_t dtype,
                             int32_t* plan, int32_t plan_len) {
  q3d::ConvGeom g;
  const q3d_status st = plan_geom(x_shape, w_shape, stride, pad_lo, pad_hi, dil, dtype, plan, &g);
  if (st != Q3D_OK) return st;
  q3d::plan_conv3d_fp4(g, dtype, plan, plan_len);
  return Q3D_OK;
}

q3d_status q3d_plan_conv_tmem(const int64_t x_shape[5], const int64_t w_shape[5], const int32_t stride[3],
                              const int32_t pad_lo[3], const int32_t pad_hi[3], const int32_t dil[3], int32_t dtype,
                              int32_t* plan, int32_t plan_len) {
  q3d::ConvGeom g;
  const q3d_status st = plan_geom(x_shape, w_shape, stride, pad_lo, pad_hi, dil, dtype, plan, &g);
  if (st != Q3D_OK) return st;
  q3d::plan_conv3d_tmem(g, dtype, plan, plan_len);
  return Q3D_OK;
}

}  // extern "C"

