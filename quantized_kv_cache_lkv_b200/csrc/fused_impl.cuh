// fused_impl.cuh -- single-launch decode attention over the packed KV cache
// with the sparse-V skip ("Super KV Compression" §第三层), for GQA groups of
// up to four query heads.  The same kernel reads the attention-tiered cache
// (§第二层) as two segments per (batch, KV head) with their own V widths.
//
// One persistent CTA per SM (cooperative launch, so all CTAs are resident).
// Work = the list of chunks (kChunk consecutive tokens of one segment of one
// (b, kv head) "unit"); every CTA takes an equal contiguous range of chunks.
// A unit's rows are numbered segment 0 first, padded to whole chunks, then
// segment 1, so a chunk never straddles the two segments.
//
//  phase 1  a producer warp streams the K rows of the CTA's chunks, tile by
//           tile, with 1-D bulk copies (TMA, evict-first in L2) into a
//           two-deep ring of shared-memory stages per consumer warp.  A
//           consumer lane computes whole rows (two per tile), so the 512
//           multiply-adds of a row need no cross-lane reduction; q is read
//           as warp-uniform broadcasts.  Each tile's per-head maximum and sum
//           of exp2 are reduced in the warp, and e = exp2(s - max_tile) is
//           written to an L2-resident workspace.
//  stats    per unit piece: the merged tile statistics.  A unit owned by one
//           CTA needs nothing else; a unit shared by neighbouring CTAs
//           exchanges piece statistics through the workspace (bounded wait
//           on a per-unit arrival counter).
//  phase 2  p = e * exp2(max_tile - max) / sum.  A (b, h, t) with p < tau is
//           skipped; the V rows some head keeps are listed per warp in row
//           order, gathered from HBM and accumulated as p * vhat.  Shared
//           units publish partial outputs; the last CTA to arrive adds them.
//
// Dequantization is folded into the dot products: codes become exact
// integers (unpack) and, with the group's (scale, zero),
//   sum_d q_d * (scale * c_d + zero) = scale * sum_d q_d c_d + zero * sum_d q_d.
#pragma once
#include <type_traits>
#include <cfloat>

#include "lkv_kernels.cuh"

namespace lkv {
namespace fused {

constexpr int kChunk = 256;    // tokens per chunk (work-partition granularity)
static_assert(kChunk == kPageTokens, "a chunk of a paged cache is one page");
constexpr int kSlotsPerWarp = 2;
constexpr int kMaxConsumerWarps = 12;
constexpr int kListCap = 512;  // V-row list entries per warp per batch
constexpr int kBatchBlocks = kListCap / 32;
constexpr int kRec = 16;       // ints per unit-list record
constexpr int kGatherUnroll = 4;
constexpr int kScanBlocks = 4;  // 32-row blocks whose logits one warp loads at once
constexpr int kTsCap = 128;    // tile statistics kept in shared memory up to this many tiles
constexpr int kQSlots = 4;     // units whose prescaled q is staged in shared memory
// Dense V pass (tau <= 0): per warp two buffers of one 32-row block each:
// V codes (up to 6 bits), (scale, zero) of 34 rows and the block's logits.
constexpr int kDenseCodes = 32 * 96;
constexpr int kDenseSz = 34 * 4 * 8;
constexpr int kDenseLogits = 32 * 4 * 4;
constexpr int kDenseBuf = (kDenseCodes + kDenseSz + kDenseLogits + 127) / 128 * 128;
constexpr int kDenseStaging = kMaxConsumerWarps * 2 * kDenseBuf;
constexpr int kDenseBar = 32;  // first mbarrier of the dense buffers
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kBarCons = 1;    // named barrier of the consumer warps
// Shared header (bytes): barriers [0, 512), per-group q sums of up to
// kQSlots units [512, 1536), misc ints [1536, 2048), tile statistics [2048, 8192), q of up to kQSlots
// units [8192, 16384).
constexpr int kQgOff = 512;
constexpr int kMiscOff = 1536;
constexpr int kTsOff = 2048;
constexpr int kQOff = 8192;
constexpr int kHeader = 16384;

// Compile-time geometry of one instantiation.
template <int D, int KB>
struct Geo {
  static constexpr int RB = D * KB / 8;                       // packed K row bytes
  static constexpr int RW = RB / 4;                           // ... in 32-bit words
  static constexpr int RPL = RW <= 24 ? 2 : 1;                // rows per lane in a tile
  static constexpr int kTileRows = 32 * RPL;
  static constexpr int kTilesPerChunk = kChunk / kTileRows;
  static constexpr int kCW = RPL == 2 ? 12 : 8;               // consumer warps
  static constexpr int kConsumers = kCW * 32;
  static constexpr int kThreads = kConsumers;                 // every warp streams its own tiles
  static constexpr int kStages = kCW * kSlotsPerWarp;
  static constexpr int kStageCodes = kTileRows * RB;
  static constexpr int kStageSz = (kTileRows + 2) * (D / 32) * 8;  // ng <= D/32, plus alignment rows
  static constexpr int kStageBytes = (kStageCodes + kStageSz + 127) / 128 * 128;
  static constexpr int kDimsPerWord = 32 / KB;                // not used for 6-bit
};

// Host-side view of the geometry (the same formulas as Geo).
struct GeoHost {
  int threads, stages, stage_bytes, tile_rows, consumer_warps;
};
inline GeoHost geo_host(int D, int KB) {
  const int rb = D * KB / 8, rw = rb / 4;
  const int rpl = rw <= 24 ? 2 : 1;
  GeoHost g;
  g.tile_rows = 32 * rpl;
  g.consumer_warps = rpl == 2 ? 12 : 8;
  g.threads = g.consumer_warps * 32;
  g.stages = g.consumer_warps * kSlotsPerWarp;
  g.stage_bytes = (g.tile_rows * rb + (g.tile_rows + 2) * (D / 32) * 8 + 127) / 128 * 128;
  return g;
}

// Unit-list record (ints): u, first chunk, chunks, n0, n1, owned, chunks of
// segment 0, -, then (max, sum) of the CTA's piece for up to 4 heads as floats.
struct Unit {
  int u, cb, nc, n0, n1, owned, nc0;
};

__device__ __forceinline__ Unit load_unit(const int* rec) {
  Unit x;
  x.u = rec[0]; x.cb = rec[1]; x.nc = rec[2]; x.n0 = rec[3]; x.n1 = rec[4]; x.owned = rec[5]; x.nc0 = rec[6];
  return x;
}

__device__ __forceinline__ void unit_lens(const DecodeArgs& d, int u, int& n0, int& n1) {
  if (d.len_mode == 0) {
    n0 = clamp_len(d.lens[u / d.Hkv], d.T_cap);
    n1 = 0;
  } else {
    n0 = clamp_len(d.lens[2 * u], d.T_cap);
    n1 = clamp_len(d.lens[2 * u + 1], d.T_cap - n0);
  }
}

__device__ __forceinline__ int chunks_of(int n) { return (n + kChunk - 1) / kChunk; }

__device__ __forceinline__ void merge_ml(float& m, float& l, float m2, float l2) {
  const float M = fmaxf(m, m2);
  if (M == -INFINITY) return;
  l = l * exp2f(m - M) + l2 * exp2f(m2 - M);
  m = M;
}

// Rows of chunk c (unit coordinates) and where they live.
struct ChunkRows {
  int seg, row0, rows;  // segment, first row inside the segment, valid rows
};

__device__ __forceinline__ ChunkRows chunk_rows(const Unit& x, int c) {
  ChunkRows r;
  r.seg = c >= x.nc0 ? 1 : 0;
  const int cs = r.seg ? c - x.nc0 : c;
  const int n = r.seg ? x.n1 : x.n0;
  r.row0 = cs * kChunk;
  r.rows = min(kChunk, n - r.row0);
  return r;
}

// Physical cache row of row `row` of unit u: contiguous, or (PAGED) the
// unit's slot in the page the block table names; a page id outside the pool
// is read as page 0 and reported in the status word.
template <bool PAGED>
__device__ __forceinline__ long long unit_row(const FusedArgs& a, int u, int row) {
  const DecodeArgs& d = a.d;
  if constexpr (!PAGED) {
    return (long long)u * d.T_cap + row;
  } else {
    const int b = u / d.Hkv, g = u - b * d.Hkv;
    int page = __ldg(a.block_table + (long long)b * a.pages_per_seq + row / kPageTokens);
    if (page < 0 || page >= a.num_pages) {
      atomicExch(d.status, kStatusInvalidArg);
      page = 0;
    }
    return ((long long)page * d.Hkv + g) * kPageTokens + row % kPageTokens;
  }
}

// Bounded spin on a counter written by other CTAs.
__device__ __forceinline__ bool wait_counter(const int* p, int target, uint64_t limit_ns) {
  if (ld_acquire(p) >= target) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    __nanosleep(128);
    if (ld_acquire(p) >= target) return true;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

template <int H>
__device__ __forceinline__ void load_heads(const float* p, float (&x)[H]) {
  if constexpr (H == 4) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  } else if constexpr (H == 2) {
    const float2 v = *reinterpret_cast<const float2*>(p);
    x[0] = v.x; x[1] = v.y;
  } else {
    x[0] = p[0];
  }
}

template <int H>
__device__ __forceinline__ void ldcg_heads(const float* p, float (&x)[H]) {
  if constexpr (H == 4) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(p));
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  } else if constexpr (H == 2) {
    const float2 v = __ldcg(reinterpret_cast<const float2*>(p));
    x[0] = v.x; x[1] = v.y;
  } else {
    x[0] = __ldcg(p);
  }
}

template <int H>
__device__ __forceinline__ void lds_heads(const float* p, float (&x)[H]) {
  if constexpr (H == 4) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  } else if constexpr (H == 2) {
    const float2 v = *reinterpret_cast<const float2*>(p);
    x[0] = v.x; x[1] = v.y;
  } else {
    x[0] = p[0];
  }
}

template <int H>
__device__ __forceinline__ void store_heads(float* p, const float (&x)[H]) {
  if constexpr (H == 4) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  } else if constexpr (H == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
  } else {
    p[0] = x[0];
  }
}

// Exponent fields of the unpack's magic floats, kept in registers so that a
// code costs a single AND-OR (an immediate mask plus this register).
template <int BITS>
struct Magic {
  uint32_t m[24];
  __device__ __forceinline__ void load(const int* src) {
#pragma unroll
    for (int k = 0; k < 24 - BITS; ++k) m[k] = (uint32_t)src[k];
  }
};

// Code I of a 16-code lane slice, plus its magic constant 2^(23-kk).
template <int BITS, int I>
__device__ __forceinline__ float code_plus_magic_r(const LaneWords<BITS>& lw, const Magic<BITS>& mg) {
  constexpr int s = copy_shift<BITS>(I);
  constexpr int kk = I * BITS - s;
  constexpr uint32_t mask = ((1u << BITS) - 1u) << kk;
  return __uint_as_float((stream_bits<BITS>(lw, s) & mask) | mg.m[kk]);
}

// Codes (2P, 2P+1) of the slice as exact floats.
template <int BITS, int P>
__device__ __forceinline__ float2 code_pair_r(const LaneWords<BITS>& lw, const Magic<BITS>& mg) {
  const float2 m = make_float2(code_plus_magic_r<BITS, 2 * P>(lw, mg), code_plus_magic_r<BITS, 2 * P + 1>(lw, mg));
  return __fadd2_rn(m, make_float2(-magic_value<BITS, 2 * P>(), -magic_value<BITS, 2 * P + 1>()));
}

template <int BITS>
__device__ __forceinline__ void unpack16_int_r(const LaneWords<BITS>& lw, const Magic<BITS>& mg, float2 (&c)[8]) {
  c[0] = code_pair_r<BITS, 0>(lw, mg);
  c[1] = code_pair_r<BITS, 1>(lw, mg);
  c[2] = code_pair_r<BITS, 2>(lw, mg);
  c[3] = code_pair_r<BITS, 3>(lw, mg);
  c[4] = code_pair_r<BITS, 4>(lw, mg);
  c[5] = code_pair_r<BITS, 5>(lw, mg);
  c[6] = code_pair_r<BITS, 6>(lw, mg);
  c[7] = code_pair_r<BITS, 7>(lw, mg);
}

// Global V-row load for the gather (lane's codes + its group's (scale, zero)).
template <int VB>
__device__ __forceinline__ void ldg_v(const uint8_t* codes_row, const float* sz_row, int j, int gi,
                                      LaneWords<VB>& lw, float2& sz) {
  load_lane_words<VB>(codes_row + j * (2 * VB), lw);
  sz = __ldg(reinterpret_cast<const float2*>(sz_row + gi * 2));
}

template <int H, int VB>
__device__ __forceinline__ void accumulate_v(const LaneWords<VB>& lw, const Magic<VB>& mg, float2 sz,
                                             const float (&w)[H], float2 (&acc)[H][8], float (&Z)[H]) {
  float2 c[8];
  unpack16_int_r<VB>(lw, mg, c);
#pragma unroll
  for (int h = 0; h < H; ++h) {
    const float ws = w[h] * sz.x;
    const float2 w2 = make_float2(ws, ws);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[h][i] = __ffma2_rn(w2, c[i], acc[h][i]);
    Z[h] = fmaf(w[h], sz.y, Z[h]);
  }
}

struct TileDesc {
  int slot, seg, row0, rows, entry, u;
};

// Pair P (0..7) of a 16-code slice; P is a constant once loops are unrolled.
template <int BITS>
__device__ __forceinline__ float2 code_pair_at(const LaneWords<BITS>& lw, const Magic<BITS>& mg, int P) {
  switch (P) {
    case 0: return code_pair_r<BITS, 0>(lw, mg);
    case 1: return code_pair_r<BITS, 1>(lw, mg);
    case 2: return code_pair_r<BITS, 2>(lw, mg);
    case 3: return code_pair_r<BITS, 3>(lw, mg);
    case 4: return code_pair_r<BITS, 4>(lw, mg);
    case 5: return code_pair_r<BITS, 5>(lw, mg);
    case 6: return code_pair_r<BITS, 6>(lw, mg);
    default: return code_pair_r<BITS, 7>(lw, mg);
  }
}

// ------------------------------------------------------------------ kernel

template <int D, int H, int KB, int VB0, int VB1, bool PAGED>
__global__ void __launch_bounds__(Geo<D, KB>::kThreads, 1) fused_decode_kernel(FusedArgs a) {
  using Gk = Geo<D, KB>;
  constexpr int CW = Gk::kCW, NCONS = Gk::kConsumers, NTHR = Gk::kThreads;
  constexpr int RPL = Gk::RPL, TR = Gk::kTileRows, TPC = Gk::kTilesPerChunk;
  constexpr int LPR = D / kDimsPerLane, RPW = 32 / LPR;  // phase-2 lane mapping (16 channels per lane)
  constexpr int NW = KB / 2;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cta = blockIdx.x, grid = gridDim.x;
  const DecodeArgs& d = a.d;
  const int units = d.B * d.Hkv;
  const int ng = D / d.G;
  const uint64_t limit_ns = (a.timeout_ns && *a.timeout_ns) ? *a.timeout_ns : 2000000000ull;
  const int j = lane % LPR;                 // phase 2: lane's 16-channel slice of a row
  const int gi = (j * kDimsPerLane) / d.G;  // its quantization group

  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw);
  int* misc = reinterpret_cast<int*>(smem_raw + kMiscOff);  // 128 ints
  uint8_t* ring = smem_raw + kHeader;

  int& s_total = misc[0];
  int& s_e0 = misc[1];
  int& s_nent = misc[2];
  int& s_abort = misc[3];
  int& s_carry_c = misc[4];
  int& s_carry_n = misc[5];
  int& s_last = misc[6];
  float* s_glob = reinterpret_cast<float*>(misc + 8);  // (max, 1/sum) x 4 heads
  int* s_wsum = misc + 16;                            // 2 x 12 warp partials
  int* s_magic = misc + 48;                           // 24 magic exponent fields
  int* s_nw = misc + 96;                              // kept rows per warp in a phase-2 batch

  if (tid == 0) {
    for (int s = 0; s < Gk::kStages; ++s) mbar_init(&full[s], 1);
    for (int s = 0; s < 2 * kMaxConsumerWarps; ++s) mbar_init(&full[kDenseBar + s], 1);
    fence_mbar_init();
    s_total = 0; s_e0 = 0; s_nent = 0; s_abort = 0; s_carry_c = 0; s_carry_n = 0; s_last = 0;
  }
  if (tid < 24) s_magic[tid] = (150 - tid) << 23;
  __syncthreads();

  // ------------------------------------------------------------ unit list
  const bool consumer = warp < CW;
  if (consumer) {
    int part = 0;
    for (int u = tid; u < units; u += NCONS) {
      int n0, n1;
      unit_lens(d, u, n0, n1);
      part += chunks_of(n0) + chunks_of(n1);
      if (n0 + n1 == 0 && (u % grid) == cta) {  // empty unit: its outputs are zero
        const int b = u / d.Hkv, g = u % d.Hkv;
        for (int e = 0; e < H * D; ++e) d.out[((long long)b * d.Hq + g * H + e / D) * D + e % D] = 0.0f;
      }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) part += __shfl_xor_sync(kFull, part, off);
    if (lane == 0) atomicAdd(&s_total, part);
    if (cta == 0) {  // length checks, spread over the CTA's threads (a serial loop here delays CTA 0)
      for (int u = tid; u < (d.len_mode == 0 ? d.B : units); u += NCONS) {
        bool bad;
        if (d.len_mode == 0) {
          bad = d.lens[u] < 0 || d.lens[u] > d.T_cap;
        } else {
          const int r0 = d.lens[2 * u], r1 = d.lens[2 * u + 1];
          bad = r0 < 0 || r1 < 0 || (long long)r0 + r1 > d.T_cap;
        }
        if (bad) atomicExch(d.status, kStatusInvalidArg);
      }
    }
  }
  __syncthreads();
  const int total = s_total;
  const int cpc = (total + grid - 1) / grid;
  const int k0 = min(cta * cpc, total), k1 = min(k0 + cpc, total);
  const int nck = k1 - k0;
  const int ntile = nck * TPC;
  int* ulist = a.ulist + (long long)cta * a.cpc_max * kRec;
  if (consumer) {
    for (int base = 0; base < units; base += NCONS) {
      const int u = base + tid;
      int n0 = 0, n1 = 0;
      if (u < units) unit_lens(d, u, n0, n1);
      const int nc0 = chunks_of(n0);
      const int nc = nc0 + chunks_of(n1);
      const int ne = nc > 0 ? 1 : 0;
      int sc = nc, sn = ne;  // warp inclusive scans
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(kFull, sc, off), z = __shfl_up_sync(kFull, sn, off);
        if (lane >= off) { sc += y; sn += z; }
      }
      if (lane == 31) { s_wsum[warp] = sc; s_wsum[16 + warp] = sn; }
      named_barrier(kBarCons, NCONS);
      int wc = 0, wn = 0, tc = 0, tn = 0;
      for (int w = 0; w < CW; ++w) {
        if (w < warp) { wc += s_wsum[w]; wn += s_wsum[16 + w]; }
        tc += s_wsum[w]; tn += s_wsum[16 + w];
      }
      const int cb = s_carry_c + wc + sc - nc;
      const int ne_idx = s_carry_n + wn + sn - ne;
      if (ne && cb <= k0 && k0 < cb + nc) s_e0 = ne_idx;
      named_barrier(kBarCons, NCONS);
      if (ne && cb < k1 && cb + nc > k0) {
        const int idx = ne_idx - s_e0;
        int* rec = ulist + (long long)idx * kRec;
        rec[0] = u; rec[1] = cb; rec[2] = nc; rec[3] = n0; rec[4] = n1;
        rec[5] = (cb >= k0 && cb + nc <= k1) ? 1 : 0;
        rec[6] = nc0;
        atomicMax(&s_nent, idx + 1);
      }
      named_barrier(kBarCons, NCONS);
      if (tid == 0) { s_carry_c += tc; s_carry_n += tn; }
      named_barrier(kBarCons, NCONS);
    }
  }
  // tile statistics (max, sum, factor per head): shared memory unless many tiles
  float* tsm;
  float* tsl;
  float* tsf;
  if (ntile <= kTsCap) {
    tsm = reinterpret_cast<float*>(smem_raw + kTsOff);
    tsl = tsm + kTsCap * 4;
    tsf = tsl + kTsCap * 4;
  } else {
    tsm = a.gstats + (long long)cta * a.cpc_max * 8 * 12;
    tsl = tsm + a.cpc_max * 8 * 4;
    tsf = tsl + a.cpc_max * 8 * 4;
  }
  for (int i = tid; i < ntile * H; i += NTHR) { tsm[i] = -INFINITY; tsl[i] = 0.0f; }
  __syncthreads();  // list complete
  const int nent = s_nent;
  // prescaled q of the CTA's units and its per-group sums (one warp per (unit, head))
  if (consumer) {
    constexpr int DPL = D / 32;  // channels per lane
    for (int task = warp; task < nent * H; task += CW) {
      const int e = task / H, h = task % H;
      const Unit x = load_unit(ulist + (long long)e * kRec);
      const int b = x.u / d.Hkv, g = x.u % d.Hkv;
      const uint16_t* qs = d.q + ((long long)b * d.Hq + g * H + h) * D + lane * DPL;
      float* qd = (e < kQSlots ? reinterpret_cast<float*>(smem_raw + kQOff) + e * H * D
                               : a.qbuf + (long long)x.u * H * D) + h * D + lane * DPL;
      float s = 0.0f;
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        const float v = __uint_as_float(((uint32_t)qs[i]) << 16) * d.q_scale;
        qd[i] = v;
        s += v;
      }
      const int lpg = d.G / DPL;  // lanes per quantization group
      for (int off = 1; off < lpg; off <<= 1) s += __shfl_xor_sync(kFull, s, off);
      if (lane % lpg == 0) {
        a.qgsum[((long long)x.u * H + h) * 4 + lane / lpg] = s;
        if (e < kQSlots) reinterpret_cast<float*>(smem_raw + kQgOff)[(e * H + h) * 4 + lane / lpg] = s;
      }
    }
  }
  __syncthreads();  // q ready; phase 1 starts

  float* lg = a.glogits + (long long)cta * a.cpc_max * kChunk * H;  // [slot][H], slot = kk * kChunk + row

  // ------------------------------------------------------------ phase 1
  // Warp w takes tiles w, w + CW, ... of the CTA (tile t = chunk t / TPC,
  // rows (t % TPC) * TR ...) and keeps two of them in flight in its own two
  // ring stages, issuing each bulk copy itself.
  {
    Magic<KB> mg;
    mg.load(s_magic);
    const uint64_t pol = policy_evict_first();
    volatile int* abort_flag = &s_abort;
    int nt = warp, ent = 0;
    // next non-empty tile of this warp, or false
    auto next_tile = [&](TileDesc& td) -> bool {
      while (nt < ntile) {
        const int t = nt;
        nt += CW;
        const int g = k0 + t / TPC, sub = t % TPC;
        while (ent + 1 < nent && ulist[(long long)(ent + 1) * kRec + 1] <= g) ++ent;
        const Unit x = load_unit(ulist + (long long)ent * kRec);
        const ChunkRows cr = chunk_rows(x, g - x.cb);
        const int rows = min(TR, cr.rows - sub * TR);
        if (rows > 0) {
          td.slot = t; td.seg = cr.seg; td.row0 = cr.row0 + sub * TR; td.rows = rows; td.entry = ent;
          td.u = x.u;
          return true;
        }
      }
      return false;
    };
    auto issue = [&](const TileDesc& td, int stage) {
      if (lane == 0) {
        const long long ubase = (long long)td.u * d.T_cap;
        const int row = td.row0, rows = td.rows;
        const int r0 = (ng == 1) ? (row & ~1) : row;
        const int r1 = (ng == 1) ? ((row + rows + 1) & ~1) : row + rows;
        const uint32_t cbytes = (uint32_t)rows * Gk::RB;
        const uint32_t sbytes = (uint32_t)(r1 - r0) * ng * 8;
        uint8_t* dst = ring + (size_t)stage * Gk::kStageBytes;
        mbar_arrive_expect_tx(&full[stage], cbytes + sbytes);
        // a tile lies in one chunk, which is one page of a paged cache
        const long long pr = PAGED ? unit_row<PAGED>(a, td.u, row) : ubase + row;
        const long long pr0 = PAGED ? unit_row<PAGED>(a, td.u, r0) : ubase + r0;
        bulk_g2s(dst, d.kc[td.seg] + pr * Gk::RB, cbytes, &full[stage], pol);
        bulk_g2s(dst + Gk::kStageCodes, d.ksz[td.seg] + pr0 * ng * 2, sbytes, &full[stage], pol);
      }
    };
    TileDesc p0, p1;
    int issued = 0, consumed = 0;
    if (next_tile(p0)) { issue(p0, warp * kSlotsPerWarp + 0); ++issued; }
    if (issued == 1 && next_tile(p1)) { issue(p1, warp * kSlotsPerWarp + 1); ++issued; }
    while (consumed < issued) {
      const int slotw = consumed % kSlotsPerWarp;
      const int stage = warp * kSlotsPerWarp + slotw;
      if (*abort_flag) break;
      if (!mbar_wait(&full[stage], (consumed / kSlotsPerWarp) & 1, limit_ns)) {
        atomicExch(d.status, kStatusTimeout);
        atomicExch(&s_abort, 1);
        break;
      }
      const TileDesc td = slotw ? p1 : p0;
      const uint8_t* codes = ring + (size_t)stage * Gk::kStageBytes;
      const float* szs = reinterpret_cast<const float*>(codes + Gk::kStageCodes) +
                         ((ng == 1) ? (td.row0 & 1) : 0) * ng * 2;
      bool valid[RPL];
      const uint4* src[RPL];
#pragma unroll
      for (int r = 0; r < RPL; ++r) {
        const int i = lane + 32 * r;
        valid[r] = i < td.rows;
        src[r] = reinterpret_cast<const uint4*>(codes + (valid[r] ? i : 0) * Gk::RB);
      }
      float dot[RPL][H];
      // The dot products of the tile's rows with the unit's prescaled q (qv)
      // and its per-group sums (qg).  Called with shared-memory pointers for
      // the CTA's first kQSlots units (shared loads) and with global ones
      // otherwise.
      // SPG (16-channel slices per quantization group) is G / 16 when known at
      // compile time, so the group folds sit at fixed places in the unrolled
      // loop, or 0 to read G at run time.
      auto k_rows = [&](auto spg, const float* __restrict__ qv, const float* __restrict__ qg) {
      constexpr int SPG = decltype(spg)::value;
      float2 acc[RPL][H];
#pragma unroll
      for (int r = 0; r < RPL; ++r)
#pragma unroll
        for (int h = 0; h < H; ++h) { dot[r][h] = 0.0f; acc[r][h] = make_float2(0.0f, 0.0f); }
      // q of the next 4-channel block, fetched one block ahead
      float4 qn[H];
#pragma unroll
      for (int h = 0; h < H; ++h) qn[h] = *reinterpret_cast<const float4*>(qv + h * D);
      constexpr int SW = 2 * KB;  // words of 64 channels of a row
#pragma unroll
      for (int sgm = 0; sgm < D / 64; ++sgm) {
        uint32_t w[RPL][SW];
#pragma unroll
        for (int r = 0; r < RPL; ++r)
#pragma unroll
          for (int q4 = 0; q4 < SW / 4; ++q4) {
            const uint4 v = src[r][sgm * (SW / 4) + q4];
            w[r][4 * q4] = v.x; w[r][4 * q4 + 1] = v.y; w[r][4 * q4 + 2] = v.z; w[r][4 * q4 + 3] = v.w;
          }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int c = sgm * 4 + cc;
          LaneWords<KB> lw[RPL];
#pragma unroll
          for (int r = 0; r < RPL; ++r)
#pragma unroll
            for (int k2 = 0; k2 < NW; ++k2) lw[r].w[k2] = w[r][cc * NW + k2];
#pragma unroll
          for (int b4 = 0; b4 < 4; ++b4) {
            const int blk = c * 4 + b4;
            float4 qc[H];
#pragma unroll
            for (int h = 0; h < H; ++h) qc[h] = qn[h];
            if (blk + 1 < D / 4) {
#pragma unroll
              for (int h = 0; h < H; ++h) qn[h] = *reinterpret_cast<const float4*>(qv + h * D + (blk + 1) * 4);
            }
            float2 cp[RPL][2];
#pragma unroll
            for (int r = 0; r < RPL; ++r) {
              cp[r][0] = code_pair_at<KB>(lw[r], mg, 2 * b4);
              cp[r][1] = code_pair_at<KB>(lw[r], mg, 2 * b4 + 1);
            }
#pragma unroll
            for (int h = 0; h < H; ++h)
#pragma unroll
              for (int r = 0; r < RPL; ++r) {
                acc[r][h] = __ffma2_rn(make_float2(qc[h].x, qc[h].y), cp[r][0], acc[r][h]);
                acc[r][h] = __ffma2_rn(make_float2(qc[h].z, qc[h].w), cp[r][1], acc[r][h]);
              }
          }
          if (SPG ? ((c + 1) % SPG == 0) : (((c + 1) * 16) % d.G == 0)) {  // end of a group: fold (scale, zero)
            const int gidx = SPG ? c / SPG : (c * 16) / d.G;
            float qsum[H];
#pragma unroll
            for (int h = 0; h < H; ++h) qsum[h] = qg[h * 4 + gidx];
#pragma unroll
            for (int r = 0; r < RPL; ++r) {
              const int i = valid[r] ? lane + 32 * r : 0;
              const float2 sz = *reinterpret_cast<const float2*>(szs + (i * ng + gidx) * 2);
#pragma unroll
              for (int h = 0; h < H; ++h) {
                dot[r][h] = fmaf(sz.x, acc[r][h].x + acc[r][h].y, fmaf(sz.y, qsum[h], dot[r][h]));
                acc[r][h] = make_float2(0.0f, 0.0f);
              }
            }
          }
        }
      }
      };
      if (td.entry < kQSlots) {
        const float* qv_s = reinterpret_cast<const float*>(smem_raw + kQOff) + td.entry * H * D;
        const float* qg_s = reinterpret_cast<const float*>(smem_raw + kQgOff) + td.entry * H * 4;
        if (d.G == 32) k_rows(std::integral_constant<int, 2>{}, qv_s, qg_s);
        else if (d.G == 64) k_rows(std::integral_constant<int, 4>{}, qv_s, qg_s);
        else k_rows(std::integral_constant<int, 8>{}, qv_s, qg_s);
      } else {
        k_rows(std::integral_constant<int, 0>{}, a.qbuf + (long long)td.u * H * D, a.qgsum + (long long)td.u * H * 4);
      }
      // The stage's data is in registers now: refill it with this warp's next tile.
      ++consumed;
      fence_proxy_async_smem();
      __syncwarp();
      {
        TileDesc tn;
        if (next_tile(tn)) {
          if (slotw) p1 = tn; else p0 = tn;
          issue(tn, stage);
          ++issued;
        }
      }
      // tile statistics: per-head maximum and sum of exp2 over the tile's rows
      float tm[H], tl[H];
#pragma unroll
      for (int h = 0; h < H; ++h) {
        float m = -INFINITY;
#pragma unroll
        for (int r = 0; r < RPL; ++r) m = valid[r] ? fmaxf(m, dot[r][h]) : m;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
        tm[h] = m;
        float l = 0.0f;
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
          dot[r][h] = exp2f(dot[r][h] - m);
          l += valid[r] ? dot[r][h] : 0.0f;
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) l += __shfl_xor_sync(kFull, l, off);
        tl[h] = l;
      }
#pragma unroll
      for (int r = 0; r < RPL; ++r)
        if (valid[r]) store_heads<H>(lg + ((long long)td.slot * TR + lane + 32 * r) * H, dot[r]);
      if (lane < H) {
        float mv = tm[0], lv = tl[0];
#pragma unroll
        for (int h = 1; h < H; ++h) if (lane == h) { mv = tm[h]; lv = tl[h]; }
        tsm[td.slot * H + lane] = mv;
        tsl[td.slot * H + lane] = lv;
      }
    }
    // Never leave copies in flight (only after an abort can any be pending).
    for (; consumed < issued; ++consumed)
      mbar_wait(&full[warp * kSlotsPerWarp + consumed % kSlotsPerWarp], (consumed / kSlotsPerWarp) & 1, limit_ns);
  }
  named_barrier(kBarCons, NCONS);
  // After a timed-out wait a bulk copy may still land in the ring, which
  // phase 2 reuses: skip straight to the end (the status word says why).
  const bool aborted = *static_cast<volatile int*>(&s_abort) != 0;
  const int n_work = aborted ? 0 : nent;

  // ------------------------------------------------------------ piece statistics
  for (int e = warp; e < n_work; e += CW) {
    int* rec = ulist + (long long)e * kRec;
    const Unit x = load_unit(rec);
    const int ta = (max(x.cb, k0) - k0) * TPC, tb = (min(x.cb + x.nc, k1) - k0) * TPC;
#pragma unroll 1
    for (int h = 0; h < H; ++h) {
      float m = -INFINITY, l = 0.0f;
      for (int t2 = ta + lane; t2 < tb; t2 += 32) merge_ml(m, l, tsm[t2 * H + h], tsl[t2 * H + h]);
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) {
        const float m2 = __shfl_xor_sync(kFull, m, off), l2 = __shfl_xor_sync(kFull, l, off);
        merge_ml(m, l, m2, l2);
      }
      if (lane == 0) {
        reinterpret_cast<float*>(rec + 8)[2 * h] = m;
        reinterpret_cast<float*>(rec + 8)[2 * h + 1] = l;
        if (!x.owned) {
          if (e == 0) {
            a.pstats[((long long)cta * 2 + 0) * H * 2 + 2 * h] = m;
            a.pstats[((long long)cta * 2 + 0) * H * 2 + 2 * h + 1] = l;
          }
          if (e == nent - 1) {
            a.pstats[((long long)cta * 2 + 1) * H * 2 + 2 * h] = m;
            a.pstats[((long long)cta * 2 + 1) * H * 2 + 2 * h + 1] = l;
          }
        }
      }
    }
  }
  named_barrier(kBarCons, NCONS);
  if (tid == 0 && n_work > 0) {
    __threadfence();  // orders every consumer's statistics before the arrivals
    const Unit x0 = load_unit(ulist);
    if (!x0.owned) atomicAdd(a.arrive1 + x0.u, 1);
    if (nent > 1) {
      const Unit x1 = load_unit(ulist + (long long)(nent - 1) * kRec);
      if (!x1.owned) atomicAdd(a.arrive1 + x1.u, 1);
    }
  }

  // ------------------------------------------------------------ phase 2
  // phase-2 shared memory (in the ring): kept-row lists [CW][kListCap], their
  // per-head weights [CW][kListCap][H] and the warps' partial outputs [CW][H][D]
  int* lists = reinterpret_cast<int*>(ring);
  float* wts = reinterpret_cast<float*>(ring + kMaxConsumerWarps * kListCap * 4);
  constexpr int kListsBytes = kMaxConsumerWarps * kListCap * 4 * (1 + H);
  float* red = reinterpret_cast<float*>(ring + (kListsBytes > kDenseStaging ? kListsBytes : kDenseStaging));
  // the dense V pass applies when every row is kept and the V rows fit its buffers
  const bool dense = d.tau <= 0.0f && VB0 <= 6 && VB1 <= 6;
  int dense_uses[2] = {0, 0};
  Magic<VB0> mg0;
  mg0.load(s_magic);
  Magic<VB1> mg1;
  mg1.load(s_magic);
  unsigned long long cnt_heads = 0, cnt_rows = 0;
  uint8_t* const smask = d.skip_mask;
  float* const mass_out = d.mass;
  for (int pass = 0; pass < 2; ++pass) {
    for (int e = 0; e < n_work; ++e) {
      int* rec = ulist + (long long)e * kRec;
      const Unit x = load_unit(rec);
      if ((pass == 0) != (x.owned != 0)) continue;  // owned pieces first, shared ones after
      const int b = x.u / d.Hkv, g = x.u % d.Hkv;
      const int i_first = x.cb / cpc, i_last = (x.cb + x.nc - 1) / cpc;
      // global statistics of the unit
      if (x.owned) {
        if (tid < H) {
          const float m = reinterpret_cast<float*>(rec + 8)[2 * tid];
          const float l = reinterpret_cast<float*>(rec + 8)[2 * tid + 1];
          s_glob[2 * tid] = m;
          s_glob[2 * tid + 1] = l > 0.0f ? 1.0f / l : 0.0f;
        }
      } else if (warp == 0) {
        bool ok = true;
        if (lane == 0) ok = wait_counter(a.arrive1 + x.u, i_last - i_first + 1, limit_ns);
        ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
        if (!ok) {
          if (lane == 0) atomicExch(d.status, kStatusTimeout);
          if (lane < H) { s_glob[2 * lane] = -INFINITY; s_glob[2 * lane + 1] = 0.0f; }
        } else if (lane < H) {
          __threadfence();
          float m = -INFINITY, l = 0.0f;
          for (int i = i_first; i <= i_last; ++i) {
            const int slot = (i == i_first) ? 1 : 0;
            const float* ps = a.pstats + ((long long)i * 2 + slot) * H * 2;
            merge_ml(m, l, __ldcg(ps + 2 * lane), __ldcg(ps + 2 * lane + 1));
          }
          s_glob[2 * lane] = m;
          s_glob[2 * lane + 1] = l > 0.0f ? 1.0f / l : 0.0f;
        }
      }
      named_barrier(kBarCons, NCONS);
      const int ga = max(x.cb, k0), gb = min(x.cb + x.nc, k1);
      // per-tile factors exp2(max_tile - max) / sum
      for (int q = tid; q < (gb - ga) * TPC * H; q += NCONS) {
        const int t2 = (ga - k0) * TPC + q / H, h = q % H;
        const float M = s_glob[2 * h], il = s_glob[2 * h + 1];
        const float mt = tsm[t2 * H + h];
        tsf[t2 * H + h] = (il > 0.0f && mt > -INFINITY) ? exp2f(mt - M) * il : 0.0f;
      }
      named_barrier(kBarCons, NCONS);

      const float* lgu = lg + (long long)(x.cb - k0) * kChunk * H;   // row v of the unit at lgu[v * H]
      const float* tfu = tsf + (x.cb - k0) * TPC * H;                 // tile v / TR at tfu[(v / TR) * H]
      const long long ubase = (long long)x.u * d.T_cap;
      const int v_lo = (ga - x.cb) * kChunk, v_hi = (gb - x.cb) * kChunk;  // chunk-aligned (padded) rows
      float2 acc[H][8];
      float Z[H];
#pragma unroll
      for (int h = 0; h < H; ++h) {
        Z[h] = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[h][i] = make_float2(0.0f, 0.0f);
      }
      if (dense) {
        // Dense V pass: every valid row is kept, so the warp streams its
        // 32-row blocks (round robin over warps) into shared memory with bulk
        // copies, two blocks in flight, and accumulates them from there.
        uint8_t* stg = ring + (size_t)warp * 2 * kDenseBuf;
        const int nblk = (v_hi - v_lo) / 32;
        const uint64_t pol = policy_evict_first();
        int rows_of[2] = {0, 0};
        auto issue = [&](int k, int buf) {
          rows_of[buf] = 0;
          const int blk = warp + k * CW;
          if (blk >= nblk) return;
          const int v0 = v_lo + blk * 32;
          const ChunkRows cr = chunk_rows(x, v0 / kChunk);
          const int rows = min(32, cr.rows - v0 % kChunk);
          if (rows <= 0) return;
          rows_of[buf] = rows;
          if (lane == 0) {
            const int seg = cr.seg, row = cr.row0 + v0 % kChunk;
            const int rbv = seg ? D * VB1 / 8 : D * VB0 / 8;
            const int r0 = (ng == 1) ? (row & ~1) : row;
            const int r1 = (ng == 1) ? ((row + rows + 1) & ~1) : row + rows;
            const uint32_t cbytes = (uint32_t)rows * rbv, sbytes = (uint32_t)(r1 - r0) * ng * 8;
            const uint32_t lbytes = 32u * H * 4u;
            uint8_t* dst = stg + buf * kDenseBuf;
            uint64_t* bar = &full[kDenseBar + warp * 2 + buf];
            mbar_arrive_expect_tx(bar, cbytes + sbytes + lbytes);
            const long long pr = PAGED ? unit_row<PAGED>(a, x.u, row) : ubase + row;
            const long long pr0 = PAGED ? unit_row<PAGED>(a, x.u, r0) : ubase + r0;
            bulk_g2s(dst, d.vc[seg] + pr * rbv, cbytes, bar, pol);
            bulk_g2s(dst + kDenseCodes, d.vsz[seg] + pr0 * ng * 2, sbytes, bar, pol);
            bulk_g2s(dst + kDenseCodes + kDenseSz, lgu + (long long)v0 * H, lbytes, bar, pol);
          }
        };
        issue(0, 0);
        issue(1, 1);
        bool stalled = false;
        for (int k = 0; warp + k * CW < nblk && !stalled; ++k) {
          const int buf = k & 1;
          const int rows = rows_of[buf];
          if (rows > 0) {
            if (!mbar_wait(&full[kDenseBar + warp * 2 + buf], dense_uses[buf] & 1, limit_ns)) {
              atomicExch(d.status, kStatusTimeout);
              stalled = true;  // leave the copy pending: it is drained below
              break;
            }
            ++dense_uses[buf];
            rows_of[buf] = 0;
            {
              const int v0 = v_lo + (warp + k * CW) * 32;
              const ChunkRows cr = chunk_rows(x, v0 / kChunk);
              const int row = cr.row0 + v0 % kChunk;
              const int sz_skip = (ng == 1) ? (row & 1) : 0;
              const uint8_t* src = stg + buf * kDenseBuf;
              const float* lgs = reinterpret_cast<const float*>(src + kDenseCodes + kDenseSz);
              const float* szs = reinterpret_cast<const float*>(src + kDenseCodes);
              float f[H];
              lds_heads<H>(tfu + (v0 / TR) * H, f);
              for (int s2 = 0; s2 < 32 / RPW; ++s2) {
                const int i = s2 * RPW + lane / LPR;
                if (i >= rows) continue;  // the lanes of a row agree
                float e[H], wgt[H];
                lds_heads<H>(lgs + i * H, e);
                float ms = 0.0f;
#pragma unroll
                for (int h = 0; h < H; ++h) { wgt[h] = e[h] * f[h]; ms += wgt[h]; }
                if (j == 0) {
                  if (smask) {
#pragma unroll
                    for (int h = 0; h < H; ++h) smask[((long long)b * d.Hq + g * H + h) * d.T_cap + v0 + i] = 0;
                  }
                  if (mass_out) mass_out[((long long)b * d.Hkv + g) * d.T_cap + v0 + i] = ms * (1.0f / H);
                }
                const float2 sz = *reinterpret_cast<const float2*>(szs + ((sz_skip + i) * ng + gi) * 2);
                if (cr.seg == 0) {
                  LaneWords<VB0> lw;
                  lds_lane_words<VB0>(src + i * (D * VB0 / 8) + j * 2 * VB0, lw);
                  accumulate_v<H, VB0>(lw, mg0, sz, wgt, acc, Z);
                } else {
                  LaneWords<VB1> lw;
                  lds_lane_words<VB1>(src + i * (D * VB1 / 8) + j * 2 * VB1, lw);
                  accumulate_v<H, VB1>(lw, mg1, sz, wgt, acc, Z);
                }
              }
            }
          }
          // the buffer's data is in registers: refill it
          fence_proxy_async_smem();
          __syncwarp();
          issue(k + 2, buf);
        }
        // never leave copies in flight (only a timed-out wait leaves one)
        for (int buf = 0; buf < 2; ++buf)
          if (rows_of[buf] > 0) {
            mbar_wait(&full[kDenseBar + warp * 2 + buf], dense_uses[buf] & 1, limit_ns);
            ++dense_uses[buf];
          }
      } else
      for (int vb = v_lo; vb < v_hi; vb += NCONS * kBatchBlocks) {
        // scan: 32-row blocks round robin over warps, row order kept per warp;
        // the logits of kScanBlocks blocks are loaded before any is used.  A
        // block lies in one chunk and one tile, so its valid-row count and
        // its tile factors are the same for the whole warp.
        int* list = lists + warp * kListCap;
        float* lwt = wts + warp * kListCap * H;
        int n_w = 0;
        uint32_t my_skip = 0, my_rows = 0;
        for (int blk0 = warp; blk0 < CW * kBatchBlocks; blk0 += kScanBlocks * CW) {
          if (vb + blk0 * 32 >= v_hi) break;
          float ev[kScanBlocks][H];
          int nvalid[kScanBlocks];
#pragma unroll
          for (int u = 0; u < kScanBlocks; ++u) {
            const int blk = blk0 + u * CW;
            const int v0 = vb + blk * 32;
            nvalid[u] = 0;
            if (blk < CW * kBatchBlocks && v0 < v_hi) nvalid[u] = chunk_rows(x, v0 / kChunk).rows - v0 % kChunk;
            if (lane < nvalid[u]) ldcg_heads<H>(lgu + (long long)(v0 + lane) * H, ev[u]);
          }
#pragma unroll
          for (int u = 0; u < kScanBlocks; ++u) {
            const int blk = blk0 + u * CW;
            const int v0 = vb + blk * 32;
            if (blk >= CW * kBatchBlocks || v0 >= v_hi) break;  // the same for the whole warp
            float f[H], wgt[H];
            lds_heads<H>(tfu + (v0 / TR) * H, f);
            bool need = false;
            if (lane < nvalid[u]) {
#pragma unroll
              for (int h = 0; h < H; ++h) {
                const float p = ev[u][h] * f[h];
                const bool keep = !(p < d.tau);
                wgt[h] = keep ? p : 0.0f;
                need |= keep;
                my_skip += keep ? 0u : 1u;
              }
              my_rows += need ? 0u : 1u;
              if (mass_out) {  // the group's mean attention to the row
                float ms = 0.0f;
#pragma unroll
                for (int h = 0; h < H; ++h) ms += ev[u][h] * f[h];
                mass_out[((long long)b * d.Hkv + g) * d.T_cap + v0 + lane] = ms * (1.0f / H);
              }
              if (smask) {
#pragma unroll
                for (int h = 0; h < H; ++h)
                  smask[((long long)b * d.Hq + g * H + h) * d.T_cap + v0 + lane] = (ev[u][h] * f[h] < d.tau) ? 1 : 0;
              }
            }
            const unsigned bal = __ballot_sync(kFull, need);
            if (need) {
              const int idx = n_w + __popc(bal & ((1u << lane) - 1u));
              list[idx] = v0 + lane;
              store_heads<H>(lwt + idx * H, wgt);
            }
            n_w += __popc(bal);
          }
        }
        cnt_heads += my_skip;
        cnt_rows += my_rows;
        __syncwarp();
        // gather: the CTA's kept rows (warp 0's list, then warp 1's, ...) are
        // split evenly over the warps, in order, so every warp waits for about
        // the same number of HBM round trips
        if (lane == 0) s_nw[warp] = n_w;
        named_barrier(kBarCons, NCONS);
        int n_all = 0;
#pragma unroll
        for (int w2 = 0; w2 < CW; ++w2) n_all += s_nw[w2];
        const int per = ((n_all + CW - 1) / CW + RPW - 1) / RPW * RPW;
        const int g_lo = min(n_all, warp * per), g_hi = min(n_all, g_lo + per);
        int sw = 0, sbase = 0;  // list holding the lane's next entry, entries before it
        for (int i0 = g_lo; i0 < g_hi; i0 += kGatherUnroll * RPW) {
          constexpr bool kOneWidth = (VB0 == VB1);
          LaneWords<VB0> w0[kGatherUnroll];
          LaneWords<kOneWidth ? 2 : VB1> w1[kOneWidth ? 1 : kGatherUnroll];
          float2 szv[kGatherUnroll];
          int vv[kGatherUnroll], li[kGatherUnroll];
#pragma unroll
          for (int s2 = 0; s2 < kGatherUnroll; ++s2) {
            const int gidx = i0 + s2 * RPW + lane / LPR;
            li[s2] = -1;
            if (gidx < g_hi) {
              while (gidx >= sbase + s_nw[sw]) { sbase += s_nw[sw]; ++sw; }
              li[s2] = sw * kListCap + gidx - sbase;
            }
            vv[s2] = li[s2] >= 0 ? lists[li[s2]] : -1;
            if (vv[s2] >= 0) {
              const int v = vv[s2];
              const ChunkRows cr = chunk_rows(x, v / kChunk);
              const long long row = PAGED ? unit_row<PAGED>(a, x.u, cr.row0 + v % kChunk) : ubase + cr.row0 + v % kChunk;
              if constexpr (kOneWidth) {
                ldg_v<VB0>(d.vc[cr.seg] + row * (D * VB0 / 8), d.vsz[cr.seg] + row * ng * 2, j, gi, w0[s2], szv[s2]);
              } else if (cr.seg == 0) {
                ldg_v<VB0>(d.vc[0] + row * (D * VB0 / 8), d.vsz[0] + row * ng * 2, j, gi, w0[s2], szv[s2]);
              } else {
                ldg_v<VB1>(d.vc[1] + row * (D * VB1 / 8), d.vsz[1] + row * ng * 2, j, gi, w1[s2], szv[s2]);
              }
            }
          }
#pragma unroll
          for (int s2 = 0; s2 < kGatherUnroll; ++s2) {
            const int v = vv[s2];
            if (v < 0) continue;
            float wgt[H];
            lds_heads<H>(wts + li[s2] * H, wgt);
            if constexpr (kOneWidth) {
              accumulate_v<H, VB0>(w0[s2], mg0, szv[s2], wgt, acc, Z);
            } else {
              if (v / kChunk < x.nc0) accumulate_v<H, VB0>(w0[s2], mg0, szv[s2], wgt, acc, Z);
              else accumulate_v<H, VB1>(w1[s2], mg1, szv[s2], wgt, acc, Z);
            }
          }
        }
        named_barrier(kBarCons, NCONS);  // other warps read this batch's lists
      }
      // fold the per-group constant, reduce the row slots of the warp
      // (code that runs once per piece is kept short: loops stay rolled)
#pragma unroll
      for (int h = 0; h < H; ++h)
#pragma unroll
        for (int i = 0; i < 8; ++i) { acc[h][i].x += Z[h]; acc[h][i].y += Z[h]; }
      if (lane < LPR) {
#pragma unroll
        for (int h = 0; h < H; ++h)
#pragma unroll
          for (int i = 0; i < 8; ++i)
            *reinterpret_cast<float2*>(red + (warp * H + h) * D + j * kDimsPerLane + 2 * i) = make_float2(0.0f, 0.0f);
      }
      __syncwarp();
      // the RPW row slots of the warp add their partial sums in shared memory
#pragma unroll 1
      for (int slot = 0; slot < RPW; ++slot) {
        if (lane / LPR == slot) {
#pragma unroll
          for (int h = 0; h < H; ++h)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float2* o = reinterpret_cast<float2*>(red + (warp * H + h) * D + j * kDimsPerLane + 2 * i);
              const float2 pv = *o;
              *o = make_float2(pv.x + acc[h][i].x, pv.y + acc[h][i].y);
            }
        }
        __syncwarp();
      }
      named_barrier(kBarCons, NCONS);
      for (int o = tid; o < H * D; o += NCONS) {
        float s2 = 0.0f;
#pragma unroll
        for (int w2 = 0; w2 < CW; ++w2) s2 += red[w2 * H * D + o];
        const int h = o / D, dd = o % D;
        if (x.owned) {
          d.out[((long long)b * d.Hq + g * H + h) * D + dd] = s2;
        } else {
          if (e == 0) a.ppart[(((long long)cta * 2 + 0) * H + h) * D + dd] = s2;
          if (e == nent - 1) a.ppart[(((long long)cta * 2 + 1) * H + h) * D + dd] = s2;
        }
      }
      if (!x.owned) {
        named_barrier(kBarCons, NCONS);
        if (tid == 0) {
          __threadfence();  // every thread's partial before the arrival
          const int old = atomicAdd(a.arrive2 + x.u, 1);
          s_last = (old == i_last - i_first) ? 1 : 0;
        }
        named_barrier(kBarCons, NCONS);
        if (s_last) {
          __threadfence();
          for (int o = tid; o < H * D; o += NCONS) {
            float s2 = 0.0f;
            for (int i = i_first; i <= i_last; ++i) {
              const int slot = (i == i_first) ? 1 : 0;
              s2 += __ldcg(a.ppart + (((long long)i * 2 + slot) * H) * D + o);
            }
            const int h = o / D, dd = o % D;
            d.out[((long long)b * d.Hq + g * H + h) * D + dd] = s2;
          }
          if (tid == 0) {
            a.arrive1[x.u] = 0;
            a.arrive2[x.u] = 0;
          }
        }
      }
      named_barrier(kBarCons, NCONS);
    }
  }

  // ------------------------------------------------------------ skip counts
  if (d.skip_counts) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      cnt_heads += __shfl_xor_sync(kFull, cnt_heads, off);
      cnt_rows += __shfl_xor_sync(kFull, cnt_rows, off);
    }
    if (lane == 0 && (cnt_heads | cnt_rows)) {
      atomicAdd(a.wcounts, cnt_heads);
      atomicAdd(a.wcounts + 1, cnt_rows);
    }
  }
  named_barrier(kBarCons, NCONS);
  if (tid == 0) {
    __threadfence();
    const int old = atomicAdd(a.done, 1);
    if (old == grid - 1) {
      __threadfence();
      const unsigned long long h = atomicExch(a.wcounts, 0ull);
      const unsigned long long rr = atomicExch(a.wcounts + 1, 0ull);
      if (d.skip_counts) {
        d.skip_counts[0] = h;
        d.skip_counts[1] = rr;
      }
      atomicExch(a.done, 0);
    }
  }
}

}  // namespace fused
}  // namespace lkv
