// conv3d_igemm_tmem.cu -- the tensor-memory Conv3D kernel with BF16
// tensor-core operands (the A operand fake-quantised to NVFP4 values and
// rounded to BF16 in the transform warps, or only converted): its plan query
// and launcher.  The kernel template, the planner and the role descriptions
// are in conv3d_tmem_kernel.cuh.
#include "conv3d_tmem_kernel.cuh"

namespace q3d {

// The plan the launcher runs: A in tensor memory, or A in shared memory when
// that frees tensor memory for more subtiles per tile, a second accumulator
// buffer or more A stages (measured: edge 96 channels 11.8 -> 10.7 ms with
// four subtiles, wan_hi 3.45 -> 3.27 ms with four A stages instead of two;
// the 384- and 1024-channel layers, which gain nothing, were 8 % slower with
// A in shared memory).  Q3D_KERNEL=smem_a takes the shared-memory form
// wherever it applies (the tests run every shape through it too).
//
// The shared-memory form's halo ring is sized for the plans this rule picks
// (checked against a model of the barrier protocol on the CPU); where the
// form is taken otherwise (forced, or required by blocks of 64) its
// transform warps wait for each slot's fill before handing it back, which
// keeps every hand-back in its own phase whatever the ring.
static bool choose_plan(const ConvGeom& g, int dtype, TmemParams& p, size_t& smem, bool need_smem_a = false) {
  const bool tmem_ok = plan_tmem(g, dtype, p, smem);
  const char* kc = getenv("Q3D_KERNEL");
  const bool force = need_smem_a || (kc && !strcmp(kc, "smem_a"));
  TmemParams q{};
  size_t qsmem = 0;
  if (!plan_tmem(g, dtype, q, qsmem, kAOpBf16Smem)) return tmem_ok && !need_smem_a;
  const bool better =
      tmem_ok && (q.n_mt > p.n_mt || (q.n_mt == p.n_mt && (q.acc_bufs > p.acc_bufs || q.sa > p.sa)));
  if (better || force) {
    if (!better) q.hb_wait = 1;
    p = q;
    smem = qsmem;
    return true;
  }
  return tmem_ok;
}

bool plan_conv3d_tmem(const ConvGeom& g, int dtype, int32_t* out, int n_out) {
  TmemParams p{};
  size_t smem = 0;
  const bool ok = choose_plan(g, dtype, p, smem);
  const int64_t v[] = {ok ? 1 : 0, p.TH, p.TW, p.n_mt, 2, p.n_tile, p.n_ntiles, p.n_sub, p.sub_n, p.ks,
                       p.c_slot, p.q_slots, p.ring, p.sa, p.sb, static_cast<int64_t>(kTmemCols),
                       static_cast<int64_t>(smem), p.n_ohb, p.n_owb, 0, p.w_box, p.h_ext, p.kd_ext, p.a_col0,
                       p.aop, p.acc_bufs, p.hb_wait};
  const int nv = static_cast<int>(sizeof(v) / sizeof(v[0]));
  for (int i = 0; i < n_out; ++i) out[i] = i < nv ? static_cast<int32_t>(v[i]) : 0;
  return ok;
}

cudaError_t launch_conv3d_tmem(const ConvGeom& g, const ConvLaunch& L, cudaStream_t s, const char** why,
                               bool* handled) {
  *handled = false;
  // quantisers: NVFP4 blocks of 16, 32 or 64, MXFP4 (blocks of 128 and 256
  // span the two transform groups' K slices: the general kernel)
  int qmode = kQModeNv16;
  if (L.quant) {
    if (L.qfmt == 2)
      qmode = kQModeMx;
    else if (L.qblock == 32)
      qmode = kQModeNv32;
    else if (L.qblock == 64)
      qmode = kQModeNv64;
    else if (L.qblock != 16)
      return cudaSuccess;
  }
  const int esz = L.dtype == 0 ? 4 : 2;
  if (reinterpret_cast<uintptr_t>(L.x) % 16 != 0) return cudaSuccess;
  TmemParams p{};
  size_t smem = 0;
  // blocks of 64 pair two lanes per row, which only A in shared memory allows
  if (!choose_plan(g, L.dtype, p, smem, qmode == kQModeNv64)) return cudaSuccess;
  p.bias = L.bias; p.y = L.y; p.act_amax = L.act_amax; p.err = L.err; p.quant = L.quant;
  p.qmode = qmode; p.dst_max = L.dst_max;
  p.y_vec = (reinterpret_cast<uintptr_t>(L.y) % 16 == 0 && g.OW % (16 / esz) == 0) ? 1 : 0;

  EncodeTiledFn encode = get_encode_tiled();
  if (!encode) { *why = "cuTensorMapEncodeTiled unavailable"; return cudaErrorNotSupported; }
  CUtensorMap tmap_x, tmap_w;
  // a shape the TMA unit cannot describe goes to another kernel
  if (!encode_halo_map(g, L.x, L.dtype, p, &tmap_x)) return cudaSuccess;
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
  if (L.withhold_arrive) {
    // the withheld hand-back is only waited for when CTA 0 reuses accumulator
    // buffer 0, at its tile acc_bufs (counting from 0)
    if (p.num_tiles <= static_cast<int64_t>(p.acc_bufs) * grid64) {
      *why = "the bounded-wait test needs more tiles per CTA than accumulator buffers";
      return cudaErrorInvalidValue;
    }
    p.withhold_arrive = 1;
  }
  *handled = true;
  if (L.quant && qmode != kQModeNv16) return launch_tmem_groups(p, tmap_x, tmap_w, static_cast<int>(grid64), smem, s);
  if (p.aop == kAOpBf16Smem) return launch_tmem_smem_a(p, tmap_x, tmap_w, static_cast<int>(grid64), smem, s);
  switch (L.dtype) {
    case 0: return launch_tmem_typed<float, kAOpBf16Tmem>(p, tmap_x, tmap_w, static_cast<int>(grid64), smem, s);
    case 1: return launch_tmem_typed<__half, kAOpBf16Tmem>(p, tmap_x, tmap_w, static_cast<int>(grid64), smem, s);
    default: return launch_tmem_typed<__nv_bfloat16, kAOpBf16Tmem>(p, tmap_x, tmap_w, static_cast<int>(grid64), smem, s);
  }
}

}  // namespace q3d
