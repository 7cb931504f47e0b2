// conv3d_fp4.cu -- the true-FP4 variant of the tensor-memory Conv3D: both
// operands quantised to NVFP4 (E2M1 values, an unsigned E4M3 scale per 16
// consecutive K elements of a row, a global scale per tensor) and multiplied
// by the block-scaled tensor-core MMA (tcgen05.mma kind::mxf4nvf4, K = 64 per
// instruction), the two global scales applied in the epilogue.
//
// The codes and block scales are those of the fake-quantiser of the
// Model-Optimizer "Conv3D Implicit GEMM CUDA kernel" article (sec. 6.1-6.3:
// g = amax / (6 * 448), scale E4M3(min(bmax / (6 g), 448)), E2M1 of
// v * (1 / (scale * g))); the weights are quantised the same way along their
// reduction axis with their own amax (sec. 7.2 quantises weights along K).
// The article dequantises to BF16 before a BF16 MMA; here the tensor core
// takes the codes and scales themselves, so each product is exact and only
// the FP32 accumulation rounds.  A block whose scale would fall back to 1.0
// has no E4M3 representation relative to g and contributes zero.
//
// This file holds the weight packing kernel and the launcher; the kernel
// template (its NVFP4-operand instantiation) is in conv3d_tmem_kernel.cuh.
#include "conv3d_tmem_kernel.cuh"

namespace q3d {

namespace {

// One thread per (output channel, block of 16 K elements): the block's codes
// and scale byte at their places in the packed images (see
// Fp4WeightLayout); thread 0 also writes the global scale.
template <typename T>
__global__ void __launch_bounds__(256) fp4_pack_weights_kernel(const T* w, int32_t Cout, int32_t K,
                                                               const float* w_amax, uint8_t* packed,
                                                               Fp4WeightLayout lay) {
  const int32_t nkb = (K + 15) / 16;
  const int64_t total = static_cast<int64_t>(Cout) * nkb;
  const Nvfp4Global G = nvfp4_global(__ldg(w_amax));
  if (blockIdx.x == 0 && threadIdx.x == 0) *reinterpret_cast<float*>(packed) = G.g;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total; t += stride) {
    const int32_t co = static_cast<int32_t>(t / nkb), kb = static_cast<int32_t>(t % nkb);
    const T* src = w + static_cast<int64_t>(co) * K + static_cast<int64_t>(kb) * 16;
    const int nv = min(16, K - kb * 16);
    float v[16];
    float bmax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      v[j] = j < nv ? DTypeOps<T>::to_f32(src[j]) : 0.0f;
      bmax = fmaxf(bmax, fabsf(v[j]));
    }
    const float r = nvfp4_ratio(bmax, G.t, G.rt);
    const uint32_t code = e4m3_code(r);
    float sc = __fmul_rn(e4m3_round_trip(r), G.g);
    const bool fallback = sc < 1e-5f;
    if (fallback) sc = 1.0f;
    const float inv = __frcp_rn(sc);
    float a[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) mul2_rn(v[2 * i], v[2 * i + 1], inv, a[2 * i], a[2 * i + 1]);
    const uint32_t c0 = e2m1_pack8(a), c1 = e2m1_pack8(a + 8);
    const int part = co / lay.sub_n, row = co % lay.sub_n, slice = kb / 4, bb = kb % 4;
    uint8_t* img = packed + kFp4WeightHeaderBytes +
                   (static_cast<int64_t>(slice) * lay.n_parts + part) * lay.img_bytes;
    *reinterpret_cast<uint2*>(img + row * 32 + ((((bb >> 1) ^ (row >> 2)) & 1) << 4) + (bb & 1) * 8) =
        make_uint2(c0, c1);
    img[lay.sub_n * 32 + (row / 128) * 512 + (row % 32) * 16 + ((row / 32) % 4) * 4 + bb] =
        static_cast<uint8_t>(fallback ? 0u : code);
  }
}

}  // namespace

bool fp4_weight_layout(int64_t Cout, int64_t K, Fp4WeightLayout* out) {
  if (Cout < 1 || K < 1 || Cout > (1 << 20) || K > (1 << 26)) return false;
  const NPlan np = n_plan(static_cast<int>(Cout));
  Fp4WeightLayout l;
  l.n_tile = np.n_tile; l.n_ntiles = np.n_ntiles; l.n_sub = np.n_sub; l.sub_n = np.sub_n;
  l.ks = static_cast<int32_t>((K + kBlockK - 1) / kBlockK);
  l.n_atoms = (np.sub_n + 127) / 128;
  l.n_parts = np.n_ntiles * np.n_sub;
  l.img_bytes = static_cast<int64_t>(np.sub_n) * 32 + static_cast<int64_t>(l.n_atoms) * 512;
  l.bytes = kFp4WeightHeaderBytes + static_cast<int64_t>(l.ks) * l.n_parts * l.img_bytes;
  *out = l;
  return true;
}

cudaError_t launch_fp4_pack_weights(const void* w, int dtype, int32_t Cout, int32_t K, const float* w_amax,
                                    void* packed, const Fp4WeightLayout& lay, cudaStream_t s, int sm_count) {
  cudaError_t e = cudaMemsetAsync(packed, 0, static_cast<size_t>(lay.bytes), s);
  if (e != cudaSuccess) return e;
  const int64_t total = static_cast<int64_t>(Cout) * ((K + 15) / 16);
  const int64_t want = (total + 255) / 256;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, static_cast<int64_t>(sm_count) * 8)));
  uint8_t* pk = static_cast<uint8_t*>(packed);
  switch (dtype) {
    case 0: fp4_pack_weights_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(w), Cout, K, w_amax, pk, lay); break;
    case 1: fp4_pack_weights_kernel<__half><<<grid, 256, 0, s>>>(static_cast<const __half*>(w), Cout, K, w_amax, pk, lay); break;
    default:
      fp4_pack_weights_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w), Cout, K,
                                                                  w_amax, pk, lay);
      break;
  }
  return cudaGetLastError();
}

bool plan_conv3d_fp4(const ConvGeom& g, int dtype, int32_t* out, int n_out) {
  TmemParams p{};
  size_t smem = 0;
  const bool ok = plan_tmem(g, dtype, p, smem, kAOpNvfp4);
  const int64_t v[] = {ok ? 1 : 0, p.TH, p.TW, p.n_mt, 2, p.n_tile, p.n_ntiles, p.n_sub, p.sub_n, p.ks,
                       p.c_slot, p.q_slots, p.ring, p.sa, p.sb, static_cast<int64_t>(kTmemCols),
                       static_cast<int64_t>(smem), p.n_ohb, p.n_owb, 0, p.w_box, p.h_ext, p.kd_ext, p.sf_col0,
                       p.sf_cols, static_cast<int64_t>(p.a_stage_bytes), static_cast<int64_t>(p.b_stage_bytes),
                       p.acc_bufs, p.hb_wait};
  const int nv = static_cast<int>(sizeof(v) / sizeof(v[0]));
  for (int i = 0; i < n_out; ++i) out[i] = i < nv ? static_cast<int32_t>(v[i]) : 0;
  return ok;
}

cudaError_t launch_conv3d_fp4(const ConvGeom& g, const ConvLaunch& L, const void* packed, cudaStream_t s,
                              const char** why, bool* handled) {
  *handled = false;
  const int esz = L.dtype == 0 ? 4 : 2;
  if (reinterpret_cast<uintptr_t>(L.x) % 16 != 0) return cudaSuccess;
  TmemParams p{};
  size_t smem = 0;
  if (!plan_tmem(g, L.dtype, p, smem, kAOpNvfp4)) return cudaSuccess;
  p.bias = L.bias; p.y = L.y; p.act_amax = L.act_amax; p.err = L.err; p.quant = 1;
  p.y_vec = (reinterpret_cast<uintptr_t>(L.y) % 16 == 0 && g.OW % (16 / esz) == 0) ? 1 : 0;
  p.g_w = static_cast<const float*>(packed);
  p.wq = static_cast<const uint8_t*>(packed) + kFp4WeightHeaderBytes;
  if (!get_encode_tiled()) { *why = "cuTensorMapEncodeTiled unavailable"; return cudaErrorNotSupported; }
  CUtensorMap tmap_x, tmap_w;
  memset(&tmap_w, 0, sizeof(tmap_w));  // the weights arrive by bulk copies; no tensor map
  if (!encode_halo_map(g, L.x, L.dtype, p, &tmap_x)) return cudaSuccess;
  const int grid = static_cast<int>(std::min<int64_t>(p.num_tiles, L.sm_count));
  *handled = true;
  switch (L.dtype) {
    case 0: return launch_tmem_typed<float, kAOpNvfp4>(p, tmap_x, tmap_w, grid, smem, s);
    case 1: return launch_tmem_typed<__half, kAOpNvfp4>(p, tmap_x, tmap_w, grid, smem, s);
    default: return launch_tmem_typed<__nv_bfloat16, kAOpNvfp4>(p, tmap_x, tmap_w, grid, smem, s);
  }
}

}  // namespace q3d
