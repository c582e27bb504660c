// fused_paged_k6.cu -- single-launch decode over a paged cache, 6-bit K codes.
#include "fused_launch.cuh"

namespace lkv {
cudaError_t launch_fused_paged_k6(const FusedArgs& a, int D, int H, int vb, size_t smem, int grid,
                                   cudaStream_t s) {
  return fused::launch_kb<6, true>(a, D, H, vb, vb, smem, grid, s);
}
}  // namespace lkv
