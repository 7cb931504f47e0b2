// conv3d_igemm_tmem_sa.cu -- the tensor-memory Conv3D kernel with BF16
// tensor-core operands and the A operand in shared memory (128-byte-swizzled
// K-major stages of 16 KB per subtile, read by the MMA through a descriptor
// like the weights).  Tensor memory then holds only the accumulators, so a
// tile can take four subtiles, or two accumulator buffers, where A stages in
// tensor memory leave no room.  The planner in conv3d_igemm_tmem.cu chooses
// this form; the kernel template is in conv3d_tmem_kernel.cuh.
#include "conv3d_tmem_kernel.cuh"

namespace q3d {

cudaError_t launch_tmem_smem_a(const TmemParams& p, const CUtensorMap& tx, const CUtensorMap& tw, int grid,
                               size_t smem, cudaStream_t s) {
  switch (p.dtype_code) {
    case 0: return launch_tmem_typed<float, kAOpBf16Smem>(p, tx, tw, grid, smem, s);
    case 1: return launch_tmem_typed<__half, kAOpBf16Smem>(p, tx, tw, grid, smem, s);
    default: return launch_tmem_typed<__nv_bfloat16, kAOpBf16Smem>(p, tx, tw, grid, smem, s);
  }
}

}  // namespace q3d
