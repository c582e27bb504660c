// tier.cu -- attention-aware tier classification and stable compaction
// ("Super KV Compression", §第二层：注意力感知的Token淘汰机制: high-attention
// tokens keep a 6-bit V, medium ones a 4-bit V, low ones are evicted).
//
// Each (b, kv head) unit is split into P contiguous parts (P <= 8), one CTA
// per part, and the P CTAs of a unit form one thread-block cluster.  Pass 1:
// a CTA classifies its part (the mass of positions inside the sequence read
// once, 16 bytes per thread-load),
// writes the tier bytes and counts its tier-2 and tier-1 tokens.  The CTAs
// then exchange their counts through distributed shared memory across one
// cluster barrier, so each knows how many kept tokens precede its part.
// Pass 2: the CTA reads its tier bytes back (from L2) and a block-wide
// exclusive scan gives every kept token its output slot, so positions come
// out in ascending order.
#include <algorithm>

#include "lkv_kernels.cuh"

namespace lkv {

namespace {

constexpr int kThreads = 256;
constexpr int kPerThread = 8;
constexpr int kTile = kThreads * kPerThread;  // positions one pass of a CTA covers
constexpr int kMaxParts = 8;                  // CTAs per unit (portable cluster size)

// Exclusive scan of two counters packed in one 32-bit word (16 bits each; a
// tile holds at most 2048 positions, so neither overflows).
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

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Barrier of all threads of the cluster, ordering shared-memory writes before
// the reads that follow it (release / acquire).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// A 32-bit word of the shared memory of CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t ld_dsmem(const uint32_t* local, uint32_t rank) {
  uint32_t addr = static_cast<uint32_t>(__cvta_generic_to_shared(local)), remote, v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(addr), "r"(rank));
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
  return v;
}

// Classification of position t with mass m (t beyond the sequence: tier 0).
__device__ __forceinline__ int8_t classify(float m, bool valid, float lo, float hi) {
  if (!valid) return 0;
  if (m > hi) return 2;
  if (m >= lo && m <= hi) return 1;
  return 0;  // below tau_low, or NaN
}

// Grid: units * P CTAs, clusters of P along x; CTA rank p of unit u covers
// positions [p * L, min((p + 1) * L, T_cap)), L a multiple of kPerThread.
__global__ void __launch_bounds__(kThreads) tier_classify_kernel(ClassifyArgs a, int P, int L) {
  __shared__ uint32_t warp_tot[kThreads / 32 + 1];
  __shared__ uint32_t part_n[2];  // this CTA's tier-2 and tier-1 counts
  __shared__ int base[2];         // kept tokens of the unit's earlier parts
  const int p = (int)cluster_rank();
  const long long bg = blockIdx.x / P;
  const int b = (int)(bg / a.Hkv);
  const int T = clamp_len(a.seq_lens[b], a.T_cap);
  const float* mass = a.mass + bg * a.T_cap;
  int8_t* tier = a.tier + bg * a.T_cap;
  const int t_lo = min(a.T_cap, p * L), t_hi = min(a.T_cap, t_lo + L);
  // rows start 32-byte aligned for the masses and 8-byte aligned for the tiers
  const bool vec = (a.T_cap % 8) == 0 && (reinterpret_cast<uintptr_t>(a.mass) & 31u) == 0 &&
                   (reinterpret_cast<uintptr_t>(a.tier) & 7u) == 0;

  // pass 1: classify, write the tier bytes, count
  uint32_t n2 = 0, n1 = 0;
  for (int t0 = t_lo; t0 < t_hi; t0 += kTile) {
    const int tb = t0 + threadIdx.x * kPerThread;
    // masses are read for positions inside the sequence only (t >= T_b is tier 0)
    float m8[kPerThread];
    const bool full = vec && tb + kPerThread <= t_hi;
    if (full && tb + kPerThread <= T) {
      const float4 x0 = __ldg(reinterpret_cast<const float4*>(mass + tb));
      const float4 x1 = __ldg(reinterpret_cast<const float4*>(mass + tb + 4));
      m8[0] = x0.x; m8[1] = x0.y; m8[2] = x0.z; m8[3] = x0.w;
      m8[4] = x1.x; m8[5] = x1.y; m8[6] = x1.z; m8[7] = x1.w;
    } else {
#pragma unroll
      for (int i = 0; i < kPerThread; ++i) m8[i] = (tb + i < t_hi && tb + i < T) ? __ldg(mass + tb + i) : 0.0f;
    }
    int8_t c[kPerThread];
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
      c[i] = classify(m8[i], tb + i < T && tb + i < t_hi, a.tau_low, a.tau_high);
      n2 += c[i] == 2;
      n1 += c[i] == 1;
    }
    if (full) {
      uint2 w;
      w.x = (uint32_t)(uint8_t)c[0] | ((uint32_t)(uint8_t)c[1] << 8) | ((uint32_t)(uint8_t)c[2] << 16) |
            ((uint32_t)(uint8_t)c[3] << 24);
      w.y = (uint32_t)(uint8_t)c[4] | ((uint32_t)(uint8_t)c[5] << 8) | ((uint32_t)(uint8_t)c[6] << 16) |
            ((uint32_t)(uint8_t)c[7] << 24);
      *reinterpret_cast<uint2*>(tier + tb) = w;
    } else {
#pragma unroll
      for (int i = 0; i < kPerThread; ++i)
        if (tb + i < t_hi) tier[tb + i] = c[i];
    }
  }
  // the part's counts (a part may exceed 65535 kept tokens: two words)
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    n2 += __shfl_xor_sync(0xFFFFFFFFu, n2, off);
    n1 += __shfl_xor_sync(0xFFFFFFFFu, n1, off);
  }
  if (threadIdx.x == 0) { part_n[0] = 0u; part_n[1] = 0u; }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) { atomicAdd(&part_n[0], n2); atomicAdd(&part_n[1], n1); }
  // exchange: every CTA of the unit reads the counts of the parts before it
  cluster_sync();
  if (threadIdx.x < 2) {
    uint32_t s = 0, all = 0;
    for (int q = 0; q < P; ++q) {
      const uint32_t v = ld_dsmem(&part_n[threadIdx.x], (uint32_t)q);
      if (q < p) s += v;
      all += v;
    }
    base[threadIdx.x] = (int)s;
    if (p == P - 1) a.counts[2 * bg + threadIdx.x] = (int)all;
  }
  // no CTA leaves while another may still read its counts
  cluster_sync();

  // pass 2: the tier bytes back (this CTA wrote them; visible after the
  // barriers above), a scan per tile, the positions
  int32_t* pos_a = a.pos_a + bg * a.T_cap;
  int32_t* pos_b = a.pos_b + bg * a.T_cap;
  int base2 = base[0], base1 = base[1];
  for (int t0 = t_lo; t0 < t_hi; t0 += kTile) {
    const int tb = t0 + threadIdx.x * kPerThread;
    int8_t c[kPerThread];
    if (vec && tb + kPerThread <= t_hi) {
      const uint2 w = *reinterpret_cast<const uint2*>(tier + tb);
#pragma unroll
      for (int i = 0; i < 4; ++i) { c[i] = (int8_t)(w.x >> (8 * i)); c[4 + i] = (int8_t)(w.y >> (8 * i)); }
    } else {
#pragma unroll
      for (int i = 0; i < kPerThread; ++i) c[i] = tb + i < t_hi ? tier[tb + i] : 0;
    }
    uint32_t m2 = 0, m1 = 0;
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) { m2 += c[i] == 2; m1 += c[i] == 1; }
    uint32_t total;
    const uint32_t excl = block_exclusive_scan(m2 | (m1 << 16), warp_tot, total);
    int o2 = base2 + (int)(excl & 0xFFFFu), o1 = base1 + (int)(excl >> 16);
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
      if (c[i] == 2) pos_a[o2++] = tb + i;
      else if (c[i] == 1) pos_b[o1++] = tb + i;
    }
    base2 += (int)(total & 0xFFFFu);
    base1 += (int)(total >> 16);
  }
}

}  // namespace

cudaError_t launch_tier_classify(const ClassifyArgs& a, cudaStream_t s) {
  const long long units = (long long)a.B * a.Hkv;
  if (units == 0 || a.T_cap == 0) {
    if (units > 0) return cudaMemsetAsync(a.counts, 0, (size_t)units * 2 * sizeof(int32_t), s);
    return cudaSuccess;
  }
  // parts of at least one tile each, at most kMaxParts per unit
  const int P = (int)std::min<long long>(kMaxParts, ((long long)a.T_cap + kTile - 1) / kTile);
  const long long per = ((long long)a.T_cap + P - 1) / P;
  const int L = (int)((per + kPerThread - 1) / kPerThread * kPerThread);
  if (units * P >= (1ll << 31)) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(units * P));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)P;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tier_classify_kernel, a, P, L);
}

}  // namespace lkv
