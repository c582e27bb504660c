// fused_k6.cu -- single-launch decode instantiations for 6-bit K codes.
#include "fused_launch.cuh"

namespace lkv {
cudaError_t launch_fused_k6(const FusedArgs& a, int D, int H, int vb0, int vb1, size_t smem, int grid,
                             cudaStream_t s) {
  return fused::launch_kb<6, false>(a, D, H, vb0, vb1, smem, grid, s);
}
}  // namespace lkv
