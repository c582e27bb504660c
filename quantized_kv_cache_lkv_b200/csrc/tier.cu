// tier.cu -- attention-aware tier classification and stable compaction
// ("Super KV Compression", §第二层：注意力感知的Token淘汰机制: high-attention
// tokens keep a 6-bit V, medium ones a 4-bit V, low ones are evicted).
//
// Each (b, kv head) unit is split into P contiguous parts (P <= 8), one CTA
// of 256 threads per part, each thread taking 32 consecutive positions; the
// P CTAs of a unit form one thread-block cluster.  Pass 1: a CTA classifies
// its part (the mass of positions inside the sequence read once, 16 bytes
// per load), writes every tier byte of the part and counts its tier-2 and
// tier-1 tokens.  The CTAs then exchange their counts through distributed
// shared memory across one cluster barrier, so each knows how many kept
// tokens precede its part.  Pass 2: a block-wide exclusive scan of the
// threads' counts gives every kept token its output slot, so positions come
// out in ascending order.  A part of one tile (8192 positions, the usual
// case) keeps its tiers in registers between the passes; longer parts read
// their tier bytes back.
#include <algorithm>

#include "lkv_kernels.cuh"

namespace lkv {

namespace {

constexpr int kThreads = 256;
constexpr int kPerThread = 32;                // consecutive positions of one thread
constexpr int kTile = kThreads * kPerThread;  // positions one pass of a CTA covers
constexpr int kMaxParts = 8;                  // CTAs per unit (portable cluster size)

// Exclusive scan of two counters packed in one 32-bit word (16 bits each; a
// tile holds at most 8192 positions, so neither overflows).
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

// Tiers of the thread's kPerThread positions [tb, tb + 32) as two bit masks
// (bit i: position tb + i is tier 2, resp. tier 1); positions at or beyond
// `lim` (the end of the part or of the sequence) are tier 0 and their mass
// is not read.  NaN masses are tier 0.
__device__ __forceinline__ void classify32(const float* mass, int tb, int lim, bool vec, float lo, float hi,
                                           uint32_t& is2, uint32_t& is1) {
  float m[kPerThread];
  if (vec && tb + kPerThread <= lim) {
#pragma unroll
    for (int q = 0; q < kPerThread / 4; ++q) {
      const float4 x = __ldg(reinterpret_cast<const float4*>(mass + tb) + q);
      m[4 * q] = x.x; m[4 * q + 1] = x.y; m[4 * q + 2] = x.z; m[4 * q + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) m[i] = tb + i < lim ? __ldg(mass + tb + i) : 0.0f;
  }
  is2 = 0u;
  is1 = 0u;
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const bool in = tb + i < lim;
    is2 |= (in && m[i] > hi) ? (1u << i) : 0u;
    is1 |= (in && m[i] >= lo && m[i] <= hi) ? (1u << i) : 0u;
  }
}

// Tier bytes of 4 consecutive positions starting at bit i of the masks.
__device__ __forceinline__ uint32_t tier_word(uint32_t is2, uint32_t is1, int i) {
  uint32_t w = 0u;
#pragma unroll
  for (int k = 0; k < 4; ++k) w |= ((((is2 >> (i + k)) & 1u) << 1) | ((is1 >> (i + k)) & 1u)) << (8 * k);
  return w;
}

// Grid: units * P CTAs, clusters of P along x; CTA rank p of unit u covers
// positions [p * L, min((p + 1) * L, T_cap)), L a multiple of kPerThread.
__global__ void __launch_bounds__(kThreads) tier_classify_kernel(ClassifyArgs a, int P, int L) {
  __shared__ uint32_t warp_tot[kThreads / 32 + 1];
  __shared__ uint32_t part_n[2];  // this CTA's tier-2 and tier-1 counts
  __shared__ int base[2];         // kept tokens of the unit's earlier parts
  const int p = P > 1 ? (int)cluster_rank() : 0;
  const long long bg = blockIdx.x / P;
  const int b = (int)(bg / a.Hkv);
  const int T = clamp_len(a.seq_lens[b], a.T_cap);
  const float* mass = a.mass + bg * a.T_cap;
  int8_t* tier = a.tier + bg * a.T_cap;
  const int t_lo = min(a.T_cap, p * L), t_hi = min(a.T_cap, t_lo + L);
  const int lim = min(t_hi, T);  // positions of the part inside the sequence
  // rows start 32-byte aligned for the masses and 16-byte aligned for the tiers
  const bool vec = (a.T_cap % 16) == 0 && (reinterpret_cast<uintptr_t>(a.mass) & 31u) == 0 &&
                   (reinterpret_cast<uintptr_t>(a.tier) & 15u) == 0;
  const bool one_tile = t_hi - t_lo <= kTile;

  // pass 1: classify (masses read once), write every tier byte of the part, count
  uint32_t n2 = 0, n1 = 0, keep2 = 0, keep1 = 0;
  for (int t0 = t_lo; t0 < t_hi; t0 += kTile) {
    const int tb = t0 + threadIdx.x * kPerThread;
    uint32_t is2 = 0, is1 = 0;
    if (tb < t_hi) classify32(mass, tb, lim, vec, a.tau_low, a.tau_high, is2, is1);
    n2 += __popc(is2);
    n1 += __popc(is1);
    keep2 = is2;  // the part's only tile stays in registers for pass 2
    keep1 = is1;
    if (vec && tb + kPerThread <= t_hi) {
#pragma unroll
      for (int q = 0; q < kPerThread / 16; ++q)
        *reinterpret_cast<uint4*>(tier + tb + 16 * q) =
            make_uint4(tier_word(is2, is1, 16 * q), tier_word(is2, is1, 16 * q + 4), tier_word(is2, is1, 16 * q + 8),
                       tier_word(is2, is1, 16 * q + 12));
    } else {
      for (int i = 0; i < kPerThread && tb + i < t_hi; ++i)
        tier[tb + i] = (int8_t)((((is2 >> i) & 1u) << 1) | ((is1 >> i) & 1u));
    }
  }
  // the part's counts
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    n2 += __shfl_xor_sync(0xFFFFFFFFu, n2, off);
    n1 += __shfl_xor_sync(0xFFFFFFFFu, n1, off);
  }
  if (threadIdx.x == 0) { part_n[0] = 0u; part_n[1] = 0u; }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) { atomicAdd(&part_n[0], n2); atomicAdd(&part_n[1], n1); }
  if (P > 1) {
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
  } else {
    __syncthreads();
    if (threadIdx.x < 2) {
      base[threadIdx.x] = 0;
      a.counts[2 * bg + threadIdx.x] = (int)part_n[threadIdx.x];
    }
    __syncthreads();
  }

  // pass 2: per tile a scan of the threads' counts gives every kept token
  // its slot; a part of more than one tile reads its tier bytes back (this
  // CTA wrote them, each thread its own)
  int32_t* pos_a = a.pos_a + bg * a.T_cap;
  int32_t* pos_b = a.pos_b + bg * a.T_cap;
  int base2 = base[0], base1 = base[1];
  for (int t0 = t_lo; t0 < t_hi; t0 += kTile) {
    const int tb = t0 + threadIdx.x * kPerThread;
    uint32_t is2 = keep2, is1 = keep1;
    if (!one_tile) {
      is2 = 0u;
      is1 = 0u;
      for (int i = 0; i < kPerThread && tb + i < t_hi; ++i) {
        const int c = tier[tb + i];
        is2 |= (c == 2) ? (1u << i) : 0u;
        is1 |= (c == 1) ? (1u << i) : 0u;
      }
    }
    uint32_t total;
    const uint32_t excl = block_exclusive_scan((uint32_t)__popc(is2) | ((uint32_t)__popc(is1) << 16), warp_tot, total);
    int o2 = base2 + (int)(excl & 0xFFFFu), o1 = base1 + (int)(excl >> 16);
    while (is2) { const int i = __ffs(is2) - 1; pos_a[o2++] = tb + i; is2 &= is2 - 1u; }
    while (is1) { const int i = __ffs(is1) - 1; pos_b[o1++] = tb + i; is1 &= is1 - 1u; }
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
  // parts of at most one tile each while kMaxParts suffice
  const int P = (int)std::min<long long>(kMaxParts, ((long long)a.T_cap + kTile - 1) / kTile);
  const long long per = ((long long)a.T_cap + P - 1) / P;
  const int L = (int)((per + kPerThread - 1) / kPerThread * kPerThread);
  if (units * P >= (1ll << 31)) return cudaErrorInvalidValue;
  if (P == 1) {
    tier_classify_kernel<<<(unsigned)units, kThreads, 0, s>>>(a, 1, L);
    return cudaGetLastError();
  }
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
