// fused_k16.cu -- single-launch decode instantiations for K at the 16-bit
// passthrough width (bf16 K rows, no (scale, zero)).
#include "fused_launch.cuh"

namespace lkv {
cudaError_t launch_fused_k16(const FusedArgs& a, int D, int H, int vb0, int vb1, size_t smem, int grid,
                              cudaStream_t s) {
  return fused::launch_kb<16, false>(a, D, H, vb0, vb1, smem, grid, s);
}
}  // namespace lkv
