// q3d_internal.h -- declarations shared between the C-ABI layer and the
// kernel translation units (not installed, not part of the ABI).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace q3d {

// Site bits recorded in the device error word when a bounded wait gives up.
enum WaitSite : unsigned int {
  kSiteProducerEmpty = 1u << 0,   // producer waiting for a free pipeline stage
  kSiteTmaFull = 1u << 1,         // consumer waiting for a TMA stage to land
  kSiteAStageFull = 1u << 2,      // MMA issuer waiting for the transformed A stage
  kSiteMmaDone = 1u << 3,         // waiting for tensor-core completion of a stage
  kSiteAccFull = 1u << 4,         // epilogue waiting for an accumulator
  kSiteAccEmpty = 1u << 5,        // MMA issuer waiting for the epilogue to drain TMEM
  kSiteHaloFull = 1u << 6,        // transform waiting for an input halo slot
  kSiteHaloEmpty = 1u << 7,       // producer waiting for a free halo slot
  kSiteDrain = 1u << 8,           // final drain of in-flight copies after an abort
};

// Geometry of one convolution, all in elements.  pd/ph/pw are the leading
// (low-side) paddings; the trailing ones only enter through OD/OH/OW.
struct ConvGeom {
  int32_t N, C, D, H, W;
  int32_t Cout, KD, KH, KW;
  int32_t sd, sh, sw;
  int32_t pd, ph, pw;
  int32_t dd, dh, dw;
  int32_t OD, OH, OW;
  int64_t M;      // N*OD*OH*OW
  int32_t K;      // C*KD*KH*KW
  int32_t taps;   // KD*KH*KW
};

struct ConvLaunch {
  const void* x;            // [N, C, D, H, W] in dtype
  const void* bias;         // [Cout] in dtype or nullptr
  void* y;                  // [N, Cout, OD, OH, OW] in dtype
  const float* act_amax;    // device scalar or nullptr
  const void* w_bf16;       // [Cout, w_ld] bf16, K-major (w_ld >= K, w_ld % 8 == 0)
  int64_t w_ld;             // row pitch of w_bf16 in elements
  int dtype;                // 0 f32, 1 f16, 2 bf16
  int quant;
  int qfmt = 1;             // quantiser when quant: 1 NVFP4 (blocks of qblock), 2 MXFP4 (groups of 32)
  int qblock = 16;
  float dst_max = 0.0f;     // MXFP4 only
  int withhold_arrive = 0;  // test of the bounded waits (tensor-memory kernel only)
  unsigned int* err;        // device error word
  int sm_count;
  // stream-ordered pool of the device for the staged BF16 weights (kept
  // cached across synchronisations), or nullptr (then the default
  // stream-ordered allocator); the kernels never read it
  cudaMemPool_t pool = nullptr;
};

// Driver entry point for cuTensorMapEncodeTiled (resolved once through the
// runtime, so the library does not link libcuda directly).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();

// block: elements per quantisation block (16, 32, 64, 128 or 256; numel a multiple of it)
cudaError_t launch_fp4_fake_quant(const void* x, void* y, int dtype, int64_t numel, int block, const float* amax,
                                  cudaStream_t s, int sm_count);
// MXFP4 over numel elements (numel % 32 == 0): any of y (dequantised, dtype),
// scales (E8M0 byte per group of 32) and codes (packed E2M1, 2 per byte) may be null.
cudaError_t launch_mxfp4(const void* x, void* y, uint8_t* scales, uint8_t* codes, int dtype, int64_t numel,
                         float dst_max, cudaStream_t s, int sm_count);
cudaError_t launch_selftest_formats(const float* in, int64_t n, float* e2m1, float* e4m3, cudaStream_t s);
cudaError_t launch_selftest_ratio(const float* bmax, const float* t, int64_t n, float* out, cudaStream_t s);
// *amax = max |x| over n elements of dtype (0 when n == 0); zeroes *amax on s first.
cudaError_t launch_act_amax(const void* x, int dtype, int64_t n, float* amax, cudaStream_t s, int sm_count);

// Convert w [Cout, K] (dtype) to bf16 [Cout, ld] with zero columns K..ld-1.
cudaError_t launch_stage_weights(const void* w, int dtype, int32_t Cout, int32_t K, int64_t ld, void* w_bf16,
                                 cudaStream_t s);

// Fixed device-resident staging area used by conv3d_implicit_gemm_noalloc
// for BF16 weights (one per device, reserved when its module loads).
constexpr size_t kNoAllocStagingBytes = static_cast<size_t>(16) << 20;
// Device address of the current device's staging area (looked up once per
// device with cudaGetSymbolAddress; the lookup's error is returned).
cudaError_t noalloc_staging_area(void** out);

// Plan of the specialised kernel (test hook): out[0] = applicable, then the
// tiling and pipeline parameters in a fixed order (see q3d.h).
bool plan_conv3d_fast(const ConvGeom& g, int dtype, int32_t* out, int n_out);
// The same for the tensor-memory kernel (groups = 1, TMEM columns = 512,
// vectorised reads = 0; one more entry: the first TMEM column of A).
bool plan_conv3d_tmem(const ConvGeom& g, int dtype, int32_t* out, int n_out);

// Packed NVFP4 weights of the block-scaled convolution variant: a 256-byte
// header (word 0: the weights' global scale g_w = w_amax / 2688, binary32),
// then one image per (K slice of 64, N-part) in slice-major order.  An image
// is sub_n rows x 32 bytes of E2M1 codes (two per byte, element 2i in the low
// nibble) in the 32-byte-swizzled K-major layout the MMA reads, then n_atoms
// 512-byte scale atoms (row n of the part at byte 16 * (n % 32) +
// 4 * ((n / 32) % 4) + block of atom n / 128; unsigned E4M3, 0 for a block
// that takes the 1.0 fallback).  Rows past Cout and columns past K are zero.
struct Fp4WeightLayout {
  int32_t n_tile, n_ntiles, n_sub, sub_n, ks, n_atoms, n_parts;
  int64_t img_bytes, bytes;
};
constexpr int64_t kFp4WeightHeaderBytes = 256;
bool fp4_weight_layout(int64_t Cout, int64_t K, Fp4WeightLayout* out);
// Quantise w [Cout, K] (dtype) into `packed` (zeroed first, on s).
cudaError_t launch_fp4_pack_weights(const void* w, int dtype, int32_t Cout, int32_t K, const float* w_amax,
                                    void* packed, const Fp4WeightLayout& lay, cudaStream_t s, int sm_count);
// The NVFP4-operand convolution over packed weights (*handled false when the
// tensor-memory kernel does not apply to the problem).
cudaError_t launch_conv3d_fp4(const ConvGeom& g, const ConvLaunch& L, const void* packed, cudaStream_t s,
                              const char** why, bool* handled);
// The plan of that variant (test hook; the fields of plan_conv3d_tmem).
bool plan_conv3d_fp4(const ConvGeom& g, int dtype, int32_t* out, int n_out);

// The implicit-GEMM convolution; returns a CUDA error or cudaSuccess, and a
// short reason in *why when it rejects the problem before launching.
cudaError_t launch_conv3d_igemm(const ConvGeom& g, const ConvLaunch& L, cudaStream_t s, const char** why);

}  // namespace q3d
