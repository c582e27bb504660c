// tier.cu -- attention-aware tier classification and stable compaction
// ("Super KV Compression", §第二层：注意力感知的Token淘汰机制: high-attention
// tokens keep a 6-bit V, medium ones a 4-bit V, low ones are evicted).
//
// One block per (b, kv head) walks the T_cap positions in tiles of
// kThreads * kPerThread; each thread classifies kPerThread consecutive
// positions, a block-wide exclusive scan of the per-thread (n2, n1) counts
// gives every kept token its output slot, and a running base carries the
// counts across tiles, so positions come out in ascending order.  The mass
// array is read once (4 bytes per token) and the tier array written once.
#include "lkv_kernels.cuh"

namespace lkv {

namespace {

constexpr int kThreads = 1024;
constexpr int kPerThread = 8;
constexpr int kTile = kThreads * kPerThread;

// Exclusive scan of two counters packed in one 32-bit word (16 bits each;
// a tile holds at most 8192 positions, so neither overflows).
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t x, uint32_t* warp_tot, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < kThreads / 32 ? warp_tot[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, wi, off);
      if (lane >= off) wi += y;
    }
    if (lane < kThreads / 32) warp_tot[lane] = wi - w;  // exclusive warp offsets
    if (lane == kThreads / 32 - 1) warp_tot[kThreads / 32] = wi;
  }
  __syncthreads();
  const uint32_t excl = warp_tot[warp] + incl - x;
  total = warp_tot[kThreads / 32];
  __syncthreads();  // warp_tot is reused by the next tile
  return excl;
}

__global__ void __launch_bounds__(kThreads) tier_classify_kernel(ClassifyArgs a) {
  __shared__ uint32_t warp_tot[kThreads / 32 + 1];
  const long long bg = blockIdx.x;
  const int b = (int)(bg / a.Hkv);
  const int T = clamp_len(a.seq_lens[b], a.T_cap);
  const float* mass = a.mass + bg * a.T_cap;
  int8_t* tier = a.tier + bg * a.T_cap;
  int32_t* pos_a = a.pos_a + bg * a.T_cap;
  int32_t* pos_b = a.pos_b + bg * a.T_cap;
  int base2 = 0, base1 = 0;
  // rows start 32-byte aligned for the masses and 8-byte aligned for the tiers
  const bool vec = (a.T_cap % 8) == 0 && (reinterpret_cast<uintptr_t>(a.mass) & 31u) == 0 &&
                   (reinterpret_cast<uintptr_t>(a.tier) & 7u) == 0;
  for (int t0 = 0; t0 < a.T_cap; t0 += kTile) {
    const int tb = t0 + threadIdx.x * kPerThread;
    // the thread's 8 masses: two 16-byte loads when the rows are aligned,
    // issued before the length test so they do not wait for it
    float m8[kPerThread];
    if (vec && tb + kPerThread <= a.T_cap) {
      const float4 x0 = __ldg(reinterpret_cast<const float4*>(mass + tb));
      const float4 x1 = __ldg(reinterpret_cast<const float4*>(mass + tb + 4));
      m8[0] = x0.x; m8[1] = x0.y; m8[2] = x0.z; m8[3] = x0.w;
      m8[4] = x1.x; m8[5] = x1.y; m8[6] = x1.z; m8[7] = x1.w;
    } else {
#pragma unroll
      for (int i = 0; i < kPerThread; ++i) m8[i] = tb + i < a.T_cap ? __ldg(mass + tb + i) : 0.0f;
    }
    int8_t c[kPerThread];
    uint32_t n2 = 0, n1 = 0;
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
      const float m = m8[i];
      int8_t ci = 0;
      if (tb + i < T) {
        if (m > a.tau_high) ci = 2;
        else if (m >= a.tau_low && m <= a.tau_high) ci = 1;
      }
      c[i] = ci;
      n2 += ci == 2;
      n1 += ci == 1;
    }
    if (vec && tb + kPerThread <= a.T_cap) {
      uint2 w;
      w.x = (uint32_t)(uint8_t)c[0] | ((uint32_t)(uint8_t)c[1] << 8) | ((uint32_t)(uint8_t)c[2] << 16) |
            ((uint32_t)(uint8_t)c[3] << 24);
      w.y = (uint32_t)(uint8_t)c[4] | ((uint32_t)(uint8_t)c[5] << 8) | ((uint32_t)(uint8_t)c[6] << 16) |
            ((uint32_t)(uint8_t)c[7] << 24);
      *reinterpret_cast<uint2*>(tier + tb) = w;
    } else {
#pragma unroll
      for (int i = 0; i < kPerThread; ++i)
        if (tb + i < a.T_cap) tier[tb + i] = c[i];
    }
    uint32_t total;
    const uint32_t excl = block_exclusive_scan(n2 | (n1 << 16), warp_tot, total);
    int o2 = base2 + (int)(excl & 0xFFFFu), o1 = base1 + (int)(excl >> 16);
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
      if (c[i] == 2) pos_a[o2++] = tb + i;
      else if (c[i] == 1) pos_b[o1++] = tb + i;
    }
    base2 += (int)(total & 0xFFFFu);
    base1 += (int)(total >> 16);
  }
  if (threadIdx.x == 0) {
    a.counts[2 * bg] = base2;
    a.counts[2 * bg + 1] = base1;
  }
}

}  // namespace

cudaError_t launch_tier_classify(const ClassifyArgs& a, cudaStream_t s) {
  const long long units = (long long)a.B * a.Hkv;
  if (units == 0) return cudaSuccess;
  tier_classify_kernel<<<(unsigned)units, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace lkv
