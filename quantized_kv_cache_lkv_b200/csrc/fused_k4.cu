// fused_k4.cu -- single-launch decode instantiations for 4-bit K codes.
#include "fused_launch.cuh"

namespace lkv {
cudaError_t launch_fused_k4(const FusedArgs& a, int D, int H, int vb0, int vb1, size_t smem, int grid,
                             cudaStream_t s) {
  return fused::launch_kb<4, false>(a, D, H, vb0, vb1, smem, grid, s);
}
}  // namespace lkv
