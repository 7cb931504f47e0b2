// conv3d_igemm_tmem_g32.cu -- the tensor-memory Conv3D kernel with BF16
// tensor-core operands and an activation quantiser over 32-column groups:
// NVFP4 with blocks of 32 (an E4M3 scale per group, the article's
// fp4_block_size = 32) or MXFP4 (a power-of-two scale per group, the CANN
// aclnnFlatQuantV2 page).  A warp's two adjacent 16-column blocks of a K
// slice form one group, so the group maximum stays in the thread that owns
// the row.  Its own instantiations (kQ = 1), A in tensor memory or in shared
// memory as the plan says; the kernel template is in conv3d_tmem_kernel.cuh.
#include "conv3d_tmem_kernel.cuh"

namespace q3d {

cudaError_t launch_tmem_groups(const TmemParams& p, const CUtensorMap& tx, const CUtensorMap& tw, int grid,
                               size_t smem, cudaStream_t s) {
  // blocks of 64 pair two lanes per row, a mapping only the shared-memory
  // A placement has (with A in tensor memory a lane writes its own row)
  if (p.qmode == kQModeNv64 && p.aop != kAOpBf16Smem) return cudaErrorInvalidValue;
  if (p.aop == kAOpBf16Smem) {
    switch (p.dtype_code) {
      case 0: return launch_tmem_typed<float, kAOpBf16Smem, 1>(p, tx, tw, grid, smem, s);
      case 1: return launch_tmem_typed<__half, kAOpBf16Smem, 1>(p, tx, tw, grid, smem, s);
      default: return launch_tmem_typed<__nv_bfloat16, kAOpBf16Smem, 1>(p, tx, tw, grid, smem, s);
    }
  }
  switch (p.dtype_code) {
    case 0: return launch_tmem_typed<float, kAOpBf16Tmem, 1>(p, tx, tw, grid, smem, s);
    case 1: return launch_tmem_typed<__half, kAOpBf16Tmem, 1>(p, tx, tw, grid, smem, s);
    default: return launch_tmem_typed<__nv_bfloat16, kAOpBf16Tmem, 1>(p, tx, tw, grid, smem, s);
  }
}

}  // namespace q3d
