// fused_launch.cuh -- cooperative launch of one instantiation of the
// single-launch decode kernel (included by the per-K-width .cu files).
#pragma once
#include "fused_impl.cuh"

namespace lkv {
namespace fused {

template <int D, int H, int KB, int VB0, int VB1, bool PAGED>
cudaError_t launch_one(const FusedArgs& a, size_t smem, int grid, cudaStream_t s) {
  auto kern = fused_decode_kernel<D, H, KB, VB0, VB1, PAGED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  FusedArgs args = a;
  void* params[] = {&args};
  return cudaLaunchCooperativeKernel((const void*)kern, dim3(grid), dim3(kThreads), params, smem, s);
}

// PAGED instantiations exist for plain decode only (one V width, not the
// 16-bit passthrough width).
template <int D, int H, int KB, bool PAGED>
cudaError_t launch_v(const FusedArgs& a, int vb0, int vb1, size_t smem, int grid, cudaStream_t s) {
  if (vb0 == vb1) {
    switch (vb0) {
      case 2: return launch_one<D, H, KB, 2, 2, PAGED>(a, smem, grid, s);
      case 4: return launch_one<D, H, KB, 4, 4, PAGED>(a, smem, grid, s);
      case 6: return launch_one<D, H, KB, 6, 6, PAGED>(a, smem, grid, s);
      case 8: return launch_one<D, H, KB, 8, 8, PAGED>(a, smem, grid, s);
      case 16:
        if constexpr (!PAGED) return launch_one<D, H, KB, 16, 16, false>(a, smem, grid, s);
        break;
    }
  }
  if constexpr (KB == 6 && !PAGED) {
    if (vb0 == 6 && vb1 == 4) return launch_one<D, H, KB, 6, 4, false>(a, smem, grid, s);
  }
  return cudaErrorInvalidValue;
}

template <int KB, bool PAGED>
cudaError_t launch_kb(const FusedArgs& a, int D, int H, int vb0, int vb1, size_t smem, int grid, cudaStream_t s) {
  if (D == 128) {
    if (H == 4) return launch_v<128, 4, KB, PAGED>(a, vb0, vb1, smem, grid, s);
    if (H == 2) return launch_v<128, 2, KB, PAGED>(a, vb0, vb1, smem, grid, s);
    if (H == 1) return launch_v<128, 1, KB, PAGED>(a, vb0, vb1, smem, grid, s);
  } else if (D == 64) {
    if (H == 4) return launch_v<64, 4, KB, PAGED>(a, vb0, vb1, smem, grid, s);
    if (H == 2) return launch_v<64, 2, KB, PAGED>(a, vb0, vb1, smem, grid, s);
    if (H == 1) return launch_v<64, 1, KB, PAGED>(a, vb0, vb1, smem, grid, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace fused
}  // namespace lkv
