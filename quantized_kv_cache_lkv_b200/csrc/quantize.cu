// quantize.cu -- bf16 K/V rows to packed low-bit codes plus (scale, zero).
//
// Asymmetric min-max quantization per group of G head_dim channels
// ("Super KV Compression", §第一层：自适应非对称量化; "TurboQuant",
// §TurboQuant的核心创新: asymmetric and group-wise).  The kernel is bound by
// HBM traffic (2*D bytes in, D*bits/8 + 8*D/G bytes out per row and tensor),
// so it streams rows with 32-byte vector loads and keeps everything else in
// registers: one lane quantizes 16 channels, the G/16 lanes of a group share
// their min/max by warp shuffles, and the lane packs its 16 codes into
// 2*BITS bytes that it stores itself.
#include "lkv_kernels.cuh"

namespace lkv {

// One row (token) of one tensor: lane j of the row's D/16 lanes.
template <int D, int BITS>
__device__ __forceinline__ void quantize_row_lane(const uint16_t* __restrict__ src, uint8_t* __restrict__ codes,
                                                  float* __restrict__ sz, int j, int G) {
  constexpr int LPR = D / kDimsPerLane;
  const unsigned mask = row_lane_mask<LPR>(threadIdx.x & 31);
  float x[16];
  load16_bf16(src + j * kDimsPerLane, x);
  uint32_t c[16];
  float scale, zero;
  const int lpg = G / kDimsPerLane;
  quantize16<BITS>(x, lpg, mask, c, scale, zero);
  LaneWords<BITS> lw;
  pack16<BITS>(c, lw);
  store_lane_words<BITS>(codes + j * (2 * BITS), lw);
  if (j % lpg == 0) *reinterpret_cast<float2*>(sz + 2 * (j / lpg)) = make_float2(scale, zero);
}

// Grid-stride over row slots of [B][Hkv][T_cap]; a warp covers 32/(D/16) rows.
template <int D, int KB, int VB>
__global__ void __launch_bounds__(256) quantize_kv_kernel(QuantizeArgs a) {
  constexpr int LPR = D / kDimsPerLane;
  constexpr int RPW = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const int j = lane % LPR;
  const int ng = D / a.G;
  const long long n_rows = (long long)a.B * a.Hkv * a.T_cap;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const long long n_warps = (long long)gridDim.x * blockDim.x / 32;
  for (long long base = warp0 * RPW; base < n_rows; base += n_warps * RPW) {
    const long long row = base + lane / LPR;
    if (row >= n_rows) continue;
    const long long bg = row / a.T_cap;
    const int t = (int)(row - bg * a.T_cap);
    const int b = (int)(bg / a.Hkv);
    if (t >= clamp_len(a.seq_lens[b], a.T_cap)) continue;
    // The lanes of one row take this path together, so the group shuffles
    // inside quantize16 only ever pair lanes that are both active.
    quantize_row_lane<D, KB>(a.k + row * D, a.k_codes + row * (D * KB / 8), a.k_sz + row * ng * 2, j, a.G);
    quantize_row_lane<D, VB>(a.v + row * D, a.v_codes + row * (D * VB / 8), a.v_sz + row * ng * 2, j, a.G);
  }
}

// Tier repack: row i of segment A (tier 2) or B (tier 1) of (b, g) is the
// token at pos[b][g][i], quantized from bf16 with K at 6 bits and V at 6 (A)
// or 4 (B) bits ("Super KV Compression", §第二层 items 1-2).
template <int D>
__global__ void __launch_bounds__(256) tier_repack_kernel(RepackArgs a) {
  constexpr int LPR = D / kDimsPerLane;
  constexpr int RPW = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const int j = lane % LPR;
  const int ng = D / a.G;
  const long long n_slots = (long long)a.B * a.Hkv * a.T_cap;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const long long n_warps = (long long)gridDim.x * blockDim.x / 32;
  const int seg = blockIdx.y;  // 0: segment A, 1: segment B
  const int32_t* pos = seg == 0 ? a.pos_a : a.pos_b;
  for (long long base = warp0 * RPW; base < n_slots; base += n_warps * RPW) {
    const long long slot = base + lane / LPR;
    if (slot >= n_slots) continue;
    const long long bg = slot / a.T_cap;
    const int i = (int)(slot - bg * a.T_cap);
    const int n = clamp_len(a.counts[2 * bg + seg], a.T_cap);
    if (i >= n) continue;
    int t = pos[slot];
    t = t < 0 ? 0 : (t >= a.T_cap ? a.T_cap - 1 : t);
    const long long src = bg * a.T_cap + t;
    if (seg == 0) {
      quantize_row_lane<D, 6>(a.k + src * D, a.a_kc + slot * (D * 6 / 8), a.a_ksz + slot * ng * 2, j, a.G);
      quantize_row_lane<D, 6>(a.v + src * D, a.a_vc + slot * (D * 6 / 8), a.a_vsz + slot * ng * 2, j, a.G);
    } else {
      quantize_row_lane<D, 6>(a.k + src * D, a.b_kc + slot * (D * 6 / 8), a.b_ksz + slot * ng * 2, j, a.G);
      quantize_row_lane<D, 4>(a.v + src * D, a.b_vc + slot * (D * 4 / 8), a.b_vsz + slot * ng * 2, j, a.G);
    }
  }
}

static int grid_for_rows(long long n_rows, int rows_per_block, int sms) {
  long long blocks = (n_rows + rows_per_block - 1) / rows_per_block;
  const long long cap = (long long)sms * 8;
  if (blocks > cap) blocks = cap;
  return (int)(blocks < 1 ? 1 : blocks);
}

template <int D, int KB>
static cudaError_t launch_quantize_vb(const QuantizeArgs& a, int vb, int grid, cudaStream_t s) {
  switch (vb) {
    case 2: quantize_kv_kernel<D, KB, 2><<<grid, 256, 0, s>>>(a); break;
    case 4: quantize_kv_kernel<D, KB, 4><<<grid, 256, 0, s>>>(a); break;
    case 6: quantize_kv_kernel<D, KB, 6><<<grid, 256, 0, s>>>(a); break;
    case 8: quantize_kv_kernel<D, KB, 8><<<grid, 256, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_quantize_d(const QuantizeArgs& a, int kb, int vb, int grid, cudaStream_t s) {
  switch (kb) {
    case 2: return launch_quantize_vb<D, 2>(a, vb, grid, s);
    case 4: return launch_quantize_vb<D, 4>(a, vb, grid, s);
    case 6: return launch_quantize_vb<D, 6>(a, vb, grid, s);
    case 8: return launch_quantize_vb<D, 8>(a, vb, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_quantize_kv(const QuantizeArgs& a, int kb, int vb, int D, cudaStream_t s) {
  const long long n_rows = (long long)a.B * a.Hkv * a.T_cap;
  if (n_rows == 0) return cudaSuccess;
  const int rows_per_block = 8 * (32 / (D / kDimsPerLane));
  const int grid = grid_for_rows(n_rows, rows_per_block, num_sms());
  if (D == 64) return launch_quantize_d<64>(a, kb, vb, grid, s);
  if (D == 128) return launch_quantize_d<128>(a, kb, vb, grid, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_tier_repack(const RepackArgs& a, int D, cudaStream_t s) {
  const long long n_slots = (long long)a.B * a.Hkv * a.T_cap;
  if (n_slots == 0) return cudaSuccess;
  const int rows_per_block = 8 * (32 / (D / kDimsPerLane));
  dim3 grid(grid_for_rows(n_slots, rows_per_block, num_sms()), 2);
  if (D == 64) tier_repack_kernel<64><<<grid, 256, 0, s>>>(a);
  else if (D == 128) tier_repack_kernel<128><<<grid, 256, 0, s>>>(a);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace lkv
