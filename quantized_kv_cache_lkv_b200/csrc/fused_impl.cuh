// fused_impl.cuh -- single-launch decode attention over the packed KV cache
// with the sparse-V skip ("Super KV Compression" §第三层), for GQA groups of
// up to four query heads.  The same kernel reads the attention-tiered cache
// (§第二层) as two segments per (batch, KV head) with their own V widths.
//
// One persistent CTA of sixteen warps per SM (cooperative launch, so all
// CTAs are resident).  Work = the list of chunks (kChunk consecutive tokens
// of one segment of one (b, kv head) "unit"); every CTA takes an equal
// contiguous range of chunks.  A unit's rows are numbered segment 0 first,
// padded to whole chunks, then segment 1, so a chunk never straddles the
// two segments.
//
//  phase 1  a producer warp streams the CTA's 64-row K tiles in order into a
//           ring of shared-memory stages with 1-D bulk copies (evict-first
//           in L2); fifteen consumer warps take the tiles round robin and
//           compute their logits on the tensor cores (mma_k.cuh): codes
//           become exact fp16 integers, q the head's exact fp16 value times
//           a power of two, and the (scale, zero) of each group is folded
//           after the MMA.  Each tile's per-head maximum and sum of exp2 are
//           reduced in the warp; e = exp2(s - max_tile) is written to an
//           L2-resident workspace.
//  stats    per unit piece: the merged tile statistics.  A unit owned by one
//           CTA needs nothing else; a unit shared by neighbouring CTAs
//           exchanges piece statistics through the workspace (bounded wait
//           on a per-unit arrival counter).  Every tile then gets its factor
//           exp2(max_tile - max) / sum.
//  phase 2  p = e * factor; (b, h, t) with p < tau is skipped.  Sparse mode
//           (tau > 0): one pass over the CTA's rows takes every decision,
//           writes the optional skip mask and attention mass, and lists the
//           rows some head keeps with their weights; their V rows are
//           brought into shared memory with 16-byte asynchronous copies and
//           accumulated piece by piece.  Dense mode (tau <= 0): every V row
//           is streamed.  (Lists that overflow shared memory fall back to a
//           per-piece scan and gather.)  Shared units publish partial
//           outputs; the last CTA to arrive adds them.
#pragma once
#include <type_traits>
#include <cfloat>

#include "lkv_kernels.cuh"
#include "mma_k.cuh"

namespace lkv {
namespace fused {

constexpr int kChunk = 256;    // tokens per chunk (work-partition granularity)
static_assert(kChunk == kPageTokens, "a chunk of a paged cache is one page");
constexpr int kTileRows = 64;  // rows of a K tile: four 16-row MMA tiles
constexpr int kTilesPerChunk = kChunk / kTileRows;
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kConsumers = 15;   // warps 0..14 compute, warp 15 streams
constexpr int kProducer = 15;
constexpr int kMaxStages = 24;   // ring stages, one chunk each
constexpr int kListCap = 256;  // fallback scan: V-row list entries per warp per batch
constexpr int kBatchBlocks = kListCap / 32;
constexpr int kRec = 16;       // ints per unit-list record
constexpr int kGatherUnroll = 2;
constexpr int kScanBlocks = 4;  // 32-row blocks whose logits one warp loads at once
constexpr int kTsCap = 128;    // tile statistics kept in shared memory up to this many tiles
constexpr int kQSlots = 4;     // units whose q is staged in shared memory
constexpr int kCandRowBits = 20;  // kept-row entry: CTA-local row | unit entry << 20
constexpr int kScanTiles = 1;      // tiles whose e-values one warp loads at once in the sparse scan
// Dense V pass (tau <= 0): per warp two buffers of one 32-row block each:
// V codes (up to 6 bits), (scale, zero) of 34 rows and the block's logits.
constexpr int kDenseCodes = 32 * 96;
constexpr int kDenseSz = 34 * 4 * 8;
constexpr int kDenseLogits = 32 * 4 * 4;
constexpr int kDenseBuf = (kDenseCodes + kDenseSz + kDenseLogits + 127) / 128 * 128;
constexpr int kDenseStaging = kWarps * 2 * kDenseBuf;
constexpr unsigned kFull = 0xFFFFFFFFu;
// Shared header (bytes): mbarriers [0, 1024) (full and empty per stage, two
// per warp for the dense pass), per q slot and head A and Z[4] [1024, 1536),
// misc ints [1536, 2560), tile statistics [2560, 8704), fp16 q of up to
// kQSlots units [8704, 12800), unit list [12800, 16896), stage descriptors
// [16896, 17664), tile descriptors [17664, 18688), spare [18688, 19200).
constexpr int kBarOff = 0;
constexpr int kAzOff = 1024;
constexpr int kMiscOff = 1536;
constexpr int kTsOff = 2560;
constexpr int kQOff = 8704;
constexpr int kUlOff = 12800;
constexpr int kUlCap = 64;
constexpr int kDescOff = 16896;
constexpr int kTinfoOff = 17664;  // per tile (valid rows | segment << 7 | unit entry << 8, first row)
constexpr int kHeader = 19200;
static_assert(2 * kMaxStages + 2 * kWarps <= 128, "barriers fit their 1024 bytes");
static_assert(kDescOff + kMaxStages * 32 <= kTinfoOff, "stage descriptors fit");
static_assert(kTinfoOff + kTsCap * 8 <= kHeader, "tile table fits");
static_assert(kHeader % 128 == 0, "the ring starts 128-byte aligned");

// Compile-time geometry of one instantiation.
template <int D, int KB>
struct Geo {
  static constexpr int RB = D * KB / 8;            // packed K row bytes
  static constexpr int SW = D * KB / 128;          // words of a lane's slice (D/4 codes)
  static constexpr int SWB = SW * 4;
  static constexpr int KS = D / 16;                // MMA k-steps per row
  static constexpr int kStageCodes = kChunk * RB;             // a stage holds one chunk
  // (scale, zero) rows: ng <= D/32, plus alignment rows; none at the 16-bit width
  static constexpr int kStageSz = KB == 16 ? 0 : (kChunk + 2) * (D / 32) * 8;
  static constexpr int kStageBytes = (kStageCodes + kStageSz + 127) / 128 * 128;
};

// Host-side view of the geometry (the same formulas as Geo).
inline int stage_bytes_host(int D, int KB) {
  const int rb = D * KB / 8;
  return (kChunk * rb + (KB == 16 ? 0 : (kChunk + 2) * (D / 32) * 8) + 127) / 128 * 128;
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

// 2^x with the hardware approximation (relative error about 2^-22; flushes
// subnormal results to zero, which only ever meets weights of 2^-126 or less).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Bounded wait until the producer has issued `target` chunks (or the CTA
// aborted); false after a timeout.
__device__ __forceinline__ bool wait_issued(const int* issued, int target, const volatile int* abort_flag,
                                            uint64_t limit_ns) {
  const volatile int* p = issued;
  if (*p >= target) { __threadfence_block(); return true; }
  const uint64_t t0 = global_ns();
  while (true) {
    __nanosleep(64);
    if (*p >= target) { __threadfence_block(); return true; }
    if (*abort_flag) return false;
    if (global_ns() - t0 > limit_ns) return false;
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

// Code I of a 16-code lane slice, plus its magic constant 2^(23-kk): the
// code sits at bit kk of a (shifted) word and the exponent field 150 - kk
// makes the float 2^(23-kk) + code exactly.
template <int BITS, int I>
__device__ __forceinline__ float code_plus_magic_r(const LaneWords<BITS>& lw) {
  constexpr int s = copy_shift<BITS>(I);
  constexpr int kk = I * BITS - s;
  constexpr uint32_t mask = ((1u << BITS) - 1u) << kk;
  constexpr uint32_t magic = (uint32_t)(150 - kk) << 23;
  return __uint_as_float((stream_bits<BITS>(lw, s) & mask) | magic);
}

// Codes (2P, 2P+1) of the slice as exact floats.
template <int BITS, int P>
__device__ __forceinline__ float2 code_pair_r(const LaneWords<BITS>& lw) {
  const float2 m = make_float2(code_plus_magic_r<BITS, 2 * P>(lw), code_plus_magic_r<BITS, 2 * P + 1>(lw));
  return __fadd2_rn(m, make_float2(-magic_value<BITS, 2 * P>(), -magic_value<BITS, 2 * P + 1>()));
}

template <int BITS>
__device__ __forceinline__ void unpack16_int_r(const LaneWords<BITS>& lw, float2 (&c)[8]) {
  c[0] = code_pair_r<BITS, 0>(lw);
  c[1] = code_pair_r<BITS, 1>(lw);
  c[2] = code_pair_r<BITS, 2>(lw);
  c[3] = code_pair_r<BITS, 3>(lw);
  c[4] = code_pair_r<BITS, 4>(lw);
  c[5] = code_pair_r<BITS, 5>(lw);
  c[6] = code_pair_r<BITS, 6>(lw);
  c[7] = code_pair_r<BITS, 7>(lw);
}

// Global V-row load for the gather (lane's codes + its group's (scale, zero)).
template <int VB>
__device__ __forceinline__ void ldg_v(const uint8_t* codes_row, const float* sz_row, int j, int gi,
                                      LaneWords<VB>& lw, float2& sz) {
  load_lane_words<VB>(codes_row + j * (2 * VB), lw);
  if constexpr (VB == 16) sz = make_float2(0.0f, 0.0f);  // passthrough width: no (scale, zero)
  else sz = __ldg(reinterpret_cast<const float2*>(sz_row + gi * 2));
}

template <int H, int VB>
__device__ __forceinline__ void accumulate_v(const LaneWords<VB>& lw, float2 sz, const float (&w)[H],
                                             float2 (&acc)[H][8], float (&Z)[H]) {
  float2 c[8];
  if constexpr (VB == 16) {
    // passthrough width: the lane's 16 bf16 values, weighted as they are
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = make_float2(__uint_as_float(lw.w[i] << 16), __uint_as_float(lw.w[i] & 0xFFFF0000u));
#pragma unroll
    for (int h = 0; h < H; ++h) {
      const float2 w2 = make_float2(w[h], w[h]);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[h][i] = __ffma2_rn(w2, c[i], acc[h][i]);
    }
  } else {
    unpack16_int_r<VB>(lw, c);
#pragma unroll
    for (int h = 0; h < H; ++h) {
      const float ws = w[h] * sz.x;
      const float2 w2 = make_float2(ws, ws);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[h][i] = __ffma2_rn(w2, c[i], acc[h][i]);
      Z[h] = fmaf(w[h], sz.y, Z[h]);
    }
  }
}

struct TileDesc {
  int slot, seg, row0, rows, entry, u;
};

// Lane slice words of row `r` of a staged tile (D/4 codes at tig * SWB).
template <int D, int KB>
__device__ __forceinline__ void lds_slice(const uint8_t* codes, int r, int tig, int gid,
                                          uint32_t (&w)[Geo<D, KB>::SW]) {
  using G = Geo<D, KB>;
  const uint8_t* p = codes + r * G::RB + tig * G::SWB;
  if constexpr (G::SWB % 16 == 0) {
#pragma unroll
    for (int q = 0; q < G::SW / 4; ++q) {
      // stagger the two 16-byte halves of 32-byte slices over odd rows (bank spread)
      const int qq = (G::SW / 4 == 2) ? (q ^ (gid & 1)) : q;
      const uint4 v = *reinterpret_cast<const uint4*>(p + 16 * qq);
      w[4 * qq] = v.x; w[4 * qq + 1] = v.y; w[4 * qq + 2] = v.z; w[4 * qq + 3] = v.w;
    }
  } else if constexpr (G::SWB % 8 == 0) {
#pragma unroll
    for (int q = 0; q < G::SW / 2; ++q) {
      const uint2 v = *reinterpret_cast<const uint2*>(p + 8 * q);
      w[2 * q] = v.x; w[2 * q + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int q = 0; q < G::SW; ++q) w[q] = reinterpret_cast<const uint32_t*>(p)[q];
  }
}

// Two 16-row MMA tiles (rows 16 mt + {gid, gid + 8} for mt = MT0, MT0 + 1)
// of a staged 64-row K tile: acc[m][nt] = C fragment of tile MT0 + m and
// n-tile nt.  The k-steps are the outer loop so that consecutive MMAs belong
// to different row tiles and do not wait on one another.
template <int D, int KB, int NT, int MT0>
__device__ __forceinline__ void mma_pair(const uint8_t* codes, int tig, int gid, const uint32_t (&bf)[2][D / 8],
                                         float (&acc)[2][2][4]) {
  using G = Geo<D, KB>;
  uint32_t w[2][2][G::SW];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) lds_slice<D, KB>(codes, 16 * (MT0 + m) + gid + 8 * hf, tig, gid, w[m][hf]);
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[m][nt][i] = 0.0f;
  auto step = [&](auto sc) {
    constexpr int s = decltype(sc)::value;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const uint32_t a0 = a_reg<KB, 2 * s>(w[m][0]), a1 = a_reg<KB, 2 * s>(w[m][1]);
      const uint32_t a2 = a_reg<KB, 2 * s + 1>(w[m][0]), a3 = a_reg<KB, 2 * s + 1>(w[m][1]);
      if constexpr (KB == 16) {
        hmma16816_bf16(acc[m][0], a0, a1, a2, a3, bf[0][2 * s], bf[0][2 * s + 1]);
        if constexpr (NT == 2) hmma16816_bf16(acc[m][1], a0, a1, a2, a3, bf[1][2 * s], bf[1][2 * s + 1]);
      } else {
        hmma16816(acc[m][0], a0, a1, a2, a3, bf[0][2 * s], bf[0][2 * s + 1]);
        if constexpr (NT == 2) hmma16816(acc[m][1], a0, a1, a2, a3, bf[1][2 * s], bf[1][2 * s + 1]);
      }
    }
  };
  step(std::integral_constant<int, 0>{});
  step(std::integral_constant<int, 1>{});
  step(std::integral_constant<int, 2>{});
  step(std::integral_constant<int, 3>{});
  if constexpr (D == 128) {
    step(std::integral_constant<int, 4>{});
    step(std::integral_constant<int, 5>{});
    step(std::integral_constant<int, 6>{});
    step(std::integral_constant<int, 7>{});
  }
}

// B fragments of the unit for this lane (see mma_k.cuh): column n = 8 nt +
// gid is (head n / ng, group n % ng); q16 holds the unit's scaled fp16 q
// [H][D].
template <int D, int KB, int H>
__device__ __forceinline__ void build_bfrags(const __half* q16, int ng, int G, int tig, int gid,
                                             uint32_t (&bf)[2][D / 8]) {
  const int lane_group = (tig * (D / 4)) / G;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const int n = 8 * nt + gid;
    const int h = n / ng, g = n - h * ng;
    const bool on = h < H && g == lane_group;
    const __half* qh = q16 + (on ? h : 0) * D;
    bfrag_one<KB, D, 0>(qh, tig * (D / 4), on, bf[nt]);
  }
}

// ------------------------------------------------------------------ kernel

template <int D, int H, int KB, int VB0, int VB1, bool PAGED>
__global__ void __launch_bounds__(kThreads, 1) fused_decode_kernel(FusedArgs a) {
  using Gk = Geo<D, KB>;
  constexpr int CW = kWarps, NTHR = kThreads;
  constexpr int TR = kTileRows, TPC = kTilesPerChunk;
  constexpr int LPR = D / kDimsPerLane, RPW = 32 / LPR;  // phase-2 lane mapping (16 channels per lane)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int cta = blockIdx.x, grid = gridDim.x;
  const DecodeArgs& d = a.d;
  const int units = d.B * d.Hkv;
  const int ng = D / d.G;
  const int S = a.stages;
  const uint64_t limit_ns = (a.timeout_ns && *a.timeout_ns) ? *a.timeout_ns : 2000000000ull;
  const int j = lane % LPR;                 // phase 2: lane's 16-channel slice of a row
  const int gi = (j * kDimsPerLane) / d.G;  // its quantization group

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + kBarOff);
  uint64_t* full = bars;                    // [kMaxStages] stage holds its tile
  uint64_t* empty = bars + kMaxStages;      // [kMaxStages] stage read by its consumer
  uint64_t* dbar = bars + 2 * kMaxStages;   // [2 * kWarps] dense V buffers
  int* misc = reinterpret_cast<int*>(smem_raw + kMiscOff);  // 256 ints
  int* desc = reinterpret_cast<int*>(smem_raw + kDescOff);  // [kMaxStages][8] tile descriptors
  uint8_t* ring = smem_raw + kHeader;

  int& s_total = misc[0];
  int& s_e0 = misc[1];
  int& s_nent = misc[2];
  int& s_abort = misc[3];
  int& s_carry_c = misc[4];
  int& s_carry_n = misc[5];
  int& s_last = misc[6];
  int& s_ovf = misc[7];
  int& s_issued = misc[8];                            // chunks the producer has issued
  int& s_valid = misc[9];                             // sparse mode: valid rows the scan saw
  int* s_kept = misc + 10;                            // sparse mode: kept (row, head) pairs, kept rows
  int* s_lastu = misc + 12;                           // sparse mode: shared pieces this CTA combines
  int* s_spiece = misc + 128;                         // sparse mode: piece in each warp's two slots
  int* s_pdone = misc + 160;                          // sparse mode: pieces written straight out (kUlCap)
  int* s_pref = misc + 224;                           // sparse mode: first list position of each warp (17)
  int* s_wsum = misc + 16;                            // 2 x 16 warp partials
  int* s_nw = misc + 88;                              // sparse mode: list length per warp

  if (tid == 0) {
    for (int s = 0; s < kMaxStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], kTilesPerChunk); }
    for (int s = 0; s < 2 * kWarps; ++s) mbar_init(&dbar[s], 1);
    fence_mbar_init();
    s_total = 0; s_e0 = 0; s_nent = 0; s_abort = 0; s_carry_c = 0; s_carry_n = 0; s_last = 0; s_ovf = 0;
    s_issued = 0; s_valid = 0; s_kept[0] = 0; s_kept[1] = 0;
  }
  for (int i = tid; i < kUlCap; i += kThreads) s_pdone[i] = 0;
  __syncthreads();

  // ------------------------------------------------------------ unit list
  // Every CTA derives the chunk ranges of all units (prefix sums of their
  // chunk counts), takes an equal contiguous range [k0, k1) of chunks, and
  // lists the units it touches.  Up to one unit per thread this is one pass
  // (lengths read once, one block scan); more units take two.
  if (cta == 0) {  // length checks, spread over the CTA's threads (a serial loop here delays CTA 0)
    for (int u = tid; u < (d.len_mode == 0 ? d.B : units); u += NTHR) {
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
  int total = 0, cpc = 0, k0 = 0, k1 = 0;
  int* ulist_g = a.ulist + (long long)cta * a.cpc_max * kRec;
  int* ulist_s = reinterpret_cast<int*>(smem_raw + kUlOff);
  // unit u's record, when its chunks [cb, cb + nc) meet [k0, k1)
  auto put_unit = [&](int u, int cb, int nc, int n0, int n1, int nc0, int idx) {
    // the list lives in shared memory when it fits, else in the workspace
    int* recs[2] = {ulist_g + (long long)idx * kRec, idx < kUlCap ? ulist_s + idx * kRec : nullptr};
    for (int c = 0; c < 2; ++c) {
      int* rec = recs[c];
      if (rec == nullptr) continue;
      rec[0] = u; rec[1] = cb; rec[2] = nc; rec[3] = n0; rec[4] = n1;
      rec[5] = (cb >= k0 && cb + nc <= k1) ? 1 : 0;
      rec[6] = nc0;
    }
    atomicMax(&s_nent, idx + 1);
  };
  auto zero_empty = [&](int u) {  // an empty unit: its outputs are zero
    const int b = u / d.Hkv, g = u % d.Hkv;
    for (int e = 0; e < H * D; ++e) d.out[((long long)b * d.Hq + g * H + e / D) * D + e % D] = 0.0f;
  };
  if (units <= NTHR) {
    const int u = tid;
    int n0 = 0, n1 = 0;
    if (u < units) unit_lens(d, u, n0, n1);
    if (u < units && n0 + n1 == 0 && (u % grid) == cta) zero_empty(u);
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
    __syncthreads();
    int wc = 0, wn = 0;
    for (int w = 0; w < CW; ++w) {
      if (w < warp) { wc += s_wsum[w]; wn += s_wsum[16 + w]; }
      total += s_wsum[w];
    }
    cpc = (total + grid - 1) / grid;
    k0 = min(cta * cpc, total);
    k1 = min(k0 + cpc, total);
    const int cb = wc + sc - nc;
    const int ne_idx = wn + sn - ne;
    if (ne && cb <= k0 && k0 < cb + nc) s_e0 = ne_idx;
    __syncthreads();
    if (ne && cb < k1 && cb + nc > k0) put_unit(u, cb, nc, n0, n1, nc0, ne_idx - s_e0);
  } else {
    int part = 0;
    for (int u = tid; u < units; u += NTHR) {
      int n0, n1;
      unit_lens(d, u, n0, n1);
      part += chunks_of(n0) + chunks_of(n1);
      if (n0 + n1 == 0 && (u % grid) == cta) zero_empty(u);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) part += __shfl_xor_sync(kFull, part, off);
    if (lane == 0) atomicAdd(&s_total, part);
    __syncthreads();
    total = s_total;
    cpc = (total + grid - 1) / grid;
    k0 = min(cta * cpc, total);
    k1 = min(k0 + cpc, total);
    for (int base = 0; base < units; base += NTHR) {
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
      __syncthreads();
      int wc = 0, wn = 0, tc = 0, tn = 0;
      for (int w = 0; w < CW; ++w) {
        if (w < warp) { wc += s_wsum[w]; wn += s_wsum[16 + w]; }
        tc += s_wsum[w]; tn += s_wsum[16 + w];
      }
      const int cb = s_carry_c + wc + sc - nc;
      const int ne_idx = s_carry_n + wn + sn - ne;
      if (ne && cb <= k0 && k0 < cb + nc) s_e0 = ne_idx;
      __syncthreads();
      if (ne && cb < k1 && cb + nc > k0) put_unit(u, cb, nc, n0, n1, nc0, ne_idx - s_e0);
      __syncthreads();
      if (tid == 0) { s_carry_c += tc; s_carry_n += tn; }
      __syncthreads();
    }
  }
  const int nck = k1 - k0;
  const int ntile = nck * TPC;
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
  int2* const tinfo = reinterpret_cast<int2*>(smem_raw + kTinfoOff);  // when ntile <= kTsCap
  for (int i = tid; i < min(ntile, kTsCap); i += NTHR) tinfo[i] = make_int2(0, 0);
  __syncthreads();  // list complete
  const int nent = s_nent;
  int* const ulist = nent <= kUlCap ? ulist_s : ulist_g;
  // q of the CTA's units (one consumer warp per (unit, head)): scaled by
  // 2^E so that its largest magnitude lies in [2^14, 2^15), stored as fp16
  // (exact for the bf16 inputs), with A = q_scale * 2^-E and Z[g] = q_scale
  // * sum of the group's q for the fold after the MMA.  The producer warp
  // does not take part: it starts streaming K meanwhile, and the consumers
  // meet at a barrier of their own before the first tile.
  if (warp != kProducer) {
    constexpr int DPL = D / 32;  // channels per lane
    for (int task = warp; task < nent * H; task += kConsumers) {
      const int e = task / H, h = task % H;
      const Unit x = load_unit(ulist + e * kRec);
      const int b = x.u / d.Hkv, g = x.u % d.Hkv;
      const uint16_t* qs = d.q + ((long long)b * d.Hq + g * H + h) * D + lane * DPL;
      float v[DPL];
      float amax = 0.0f, s = 0.0f;
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        v[i] = __uint_as_float(((uint32_t)qs[i]) << 16);
        amax = fmaxf(amax, fabsf(v[i]));
        s += v[i];
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, off));
      int ex = 0;
      const bool fin = amax > 0.0f && amax <= FLT_MAX;
      if (fin) frexpf(amax, &ex);
      // 16-bit K meets q in a bf16 MMA: q stays as it is (E = 0)
      const int E = (fin && KB != 16) ? 15 - ex : 0;
      __half* qd = (e < kQSlots ? reinterpret_cast<__half*>(smem_raw + kQOff) + e * H * D
                                : reinterpret_cast<__half*>(a.qbuf) + (long long)x.u * H * D) +
                   h * D + lane * DPL;
      if constexpr (KB == 16) {
#pragma unroll
        for (int i = 0; i < DPL; ++i) reinterpret_cast<uint16_t*>(qd)[i] = qs[i];
      } else {
#pragma unroll
        for (int i = 0; i < DPL; ++i) qd[i] = __float2half_rn(ldexpf(v[i], E));
      }
      const int lpg = d.G / DPL;  // lanes per quantization group
      for (int off = 1; off < lpg; off <<= 1) s += __shfl_xor_sync(kFull, s, off);
      float* az = e < kQSlots ? reinterpret_cast<float*>(smem_raw + kAzOff) + (e * H + h) * 8
                              : a.qgsum + ((long long)x.u * H + h) * 8;
      if (lane % lpg == 0) az[lane / lpg] = d.q_scale * s;
      if (lane == 0) az[4] = ldexpf(d.q_scale, -E);
    }
  }
  if (warp != kProducer) named_barrier(1, kConsumers * 32);  // q ready; the producer is already streaming

  float* lg = a.glogits + (long long)cta * a.cpc_max * kChunk * H;  // [tile * TR + row][H]

  // ------------------------------------------------------------ phase 1
  // The producer warp streams the CTA's chunks in order into a ring of S
  // stages (chunk c -> stage c % S) with two 1-D bulk copies each; consumer
  // warp w takes tiles w, w + kConsumers, ... (tile t = quarter t % 4 of
  // chunk t / 4).  "full" completes when a chunk has landed, "empty" when
  // the consumers of its four tiles have read it.
  volatile int* abort_flag = &s_abort;
  if (warp == kProducer) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int ent = 0, c = 0, s = 0, k = 0;
      for (; c < nck; ++c, s = (s + 1 == S) ? 0 : s + 1, k += (s == 0) ? 1 : 0) {
        if (k > 0 && !mbar_wait(&empty[s], (k - 1) & 1, limit_ns)) {
          atomicExch(d.status, kStatusTimeout);
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        const int g = k0 + c;
        while (ent + 1 < nent && ulist[(ent + 1) * kRec + 1] <= g) ++ent;
        const Unit x = load_unit(ulist + ent * kRec);
        const ChunkRows cr = chunk_rows(x, g - x.cb);
        const int row = cr.row0, rows = max(0, cr.rows);
        int* dd = desc + s * 8;
        dd[0] = cr.seg; dd[1] = row; dd[2] = rows; dd[3] = ent; dd[4] = x.u;
        if (rows > 0) {
          const int r0 = (ng == 1) ? (row & ~1) : row;
          const int r1 = (ng == 1) ? ((row + rows + 1) & ~1) : row + rows;
          const uint32_t cbytes = (uint32_t)rows * Gk::RB;
          const uint32_t sbytes = KB == 16 ? 0u : (uint32_t)(r1 - r0) * ng * 8;  // none at the 16-bit width
          uint8_t* dst = ring + (size_t)s * Gk::kStageBytes;
          mbar_arrive_expect_tx(&full[s], cbytes + sbytes);
          // a chunk is one page of a paged cache
          const long long ubase = (long long)x.u * d.T_cap;
          const long long pr = PAGED ? unit_row<PAGED>(a, x.u, row) : ubase + row;
          const long long pr0 = PAGED ? unit_row<PAGED>(a, x.u, r0) : ubase + r0;
          bulk_g2s(dst, d.kc[cr.seg] + pr * Gk::RB, cbytes, &full[s], pol);
          if (sbytes > 0) bulk_g2s(dst + Gk::kStageCodes, d.ksz[cr.seg] + pr0 * ng * 2, sbytes, &full[s], pol);
        } else {
          mbar_arrive(&full[s]);
        }
        // chunk c's phase of full[s] is now the current one; a consumer that
        // waited on the parity before this could match an older phase
        __threadfence_block();
        *static_cast<volatile int*>(&s_issued) = c + 1;
      }
      // never leave copies in flight: the last use of every stage has landed
      for (int s = 0; s < S && s < c; ++s) mbar_wait(&full[s], ((c - 1 - s) / S) & 1, limit_ns);
    }
  } else {
    // consumer warps, specialised on the number of quantization groups per
    // row (NG): tile t = quarter t % 4 of chunk t / 4, stage (t / 4) % S
    auto consume = [&](auto ngc) {
      constexpr int NG = decltype(ngc)::value;
      constexpr int NTC = (H * NG > 8) ? 2 : 1;
      int bf_ent = -1;               // unit entry whose B fragments are loaded
      uint32_t bf[2][D / 8];
      // fold constants of the head(s) whose C columns this lane holds:
      // NG 2: head tig (groups 0, 1); NG 1: heads 2 tig, 2 tig + 1;
      // NG 4: heads tig / 2 and 2 + tig / 2 (groups 2 (tig & 1), + 1)
      float fA[2] = {0.0f, 0.0f}, fZ[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};
      int t = warp, c = warp / TPC;
      int s = c % S, k = c / S;
      while (t < ntile) {
        const int sub = t % TPC;
        if (*abort_flag) break;
        if (!wait_issued(&s_issued, c + 1, abort_flag, limit_ns) || !mbar_wait(&full[s], k & 1, limit_ns)) {
          if (!*abort_flag) atomicExch(d.status, kStatusTimeout);
          *abort_flag = 1;
          break;
        }
        const int* dd = desc + s * 8;
        const int rows = max(0, min(TR, dd[2] - sub * TR));
        const int dseg = dd[0], drow = dd[1];  // read before the stage is handed back
        if (rows > 0) {
          const int entry = dd[3];
          if (entry != bf_ent) {
            // B fragments and fold constants of the tile's unit
            bf_ent = entry;
            const int u = dd[4];
            const __half* q16 = entry < kQSlots ? reinterpret_cast<const __half*>(smem_raw + kQOff) + entry * H * D
                                                : reinterpret_cast<const __half*>(a.qbuf) + (long long)u * H * D;
            const float* azb = entry < kQSlots ? reinterpret_cast<const float*>(smem_raw + kAzOff) + entry * H * 8
                                               : a.qgsum + (long long)u * H * 8;
            build_bfrags<D, KB, H>(q16, NG, KB == 16 ? D : d.G, tig, gid, bf);
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
              const int hh = NG == 2 ? tig : (NG == 1 ? 2 * tig + c2 : 2 * c2 + tig / 2);
              const int h = hh < H ? hh : 0;
              const int g0 = NG == 4 ? 2 * (tig & 1) : 0;
              fA[c2] = hh < H ? azb[h * 8 + 4] : 0.0f;
              fZ[c2][0] = azb[h * 8 + g0];
              fZ[c2][1] = azb[h * 8 + g0 + 1];
            }
          }
          const uint8_t* stg = ring + (size_t)s * Gk::kStageBytes;
          const uint8_t* codes = stg + sub * TR * Gk::RB;
          const float* szs = reinterpret_cast<const float*>(stg + Gk::kStageCodes) +
                             (((NG == 1) ? (drow & 1) : 0) + sub * TR) * NG * 2;
          // logits of head tig (base 2) for rows 16 mt + gid + 8 hf
          float sv[4][2];
          auto fold_pair = [&](auto mc) {
            constexpr int MT0 = decltype(mc)::value;
            float acc[2][2][4];
            mma_pair<D, KB, NTC, MT0>(codes, tig, gid, bf, acc);
#pragma unroll
            for (int m = 0; m < 2; ++m)
#pragma unroll
              for (int hf = 0; hf < 2; ++hf) {
                const int r = 16 * (MT0 + m) + gid + 8 * hf;
                float val;
                if constexpr (NG == 2) {
                  const float c0 = acc[m][0][2 * hf], c1 = acc[m][0][2 * hf + 1];
                  const float4 s4 = *reinterpret_cast<const float4*>(szs + r * 4);
                  val = fmaf(fA[0], fmaf(s4.z, c1, s4.x * c0), fmaf(s4.w, fZ[0][1], s4.y * fZ[0][0]));
                } else if constexpr (NG == 1) {
                  const float c0 = acc[m][0][2 * hf], c1 = acc[m][0][2 * hf + 1];
                  float v0, v1;
                  if constexpr (KB == 16) {  // bf16 K: no (scale, zero) to fold
                    v0 = fA[0] * c0;
                    v1 = fA[1] * c1;
                  } else {
                    const float2 s2 = *reinterpret_cast<const float2*>(szs + r * 2);
                    v0 = fmaf(fA[0] * s2.x, c0, s2.y * fZ[0][0]);
                    v1 = fmaf(fA[1] * s2.x, c1, s2.y * fZ[1][0]);
                  }
                  const int src = (lane & ~3) | (tig >> 1);
                  const float u0 = __shfl_sync(kFull, v0, src), u1 = __shfl_sync(kFull, v1, src);
                  val = (tig & 1) ? u1 : u0;
                } else {
                  const float4 s4 = *reinterpret_cast<const float4*>(szs + r * NG * 2 + 4 * (tig & 1));
                  float f[2];
#pragma unroll
                  for (int n2 = 0; n2 < 2; ++n2) {
                    const float e0 = acc[m][n2][2 * hf], e1 = acc[m][n2][2 * hf + 1];
                    float pv = fmaf(fA[n2], fmaf(s4.z, e1, s4.x * e0), fmaf(s4.w, fZ[n2][1], s4.y * fZ[n2][0]));
                    pv += __shfl_xor_sync(kFull, pv, 1);
                    f[n2] = pv;
                  }
                  const int src = (lane & ~3) | (2 * (tig & 1));
                  const float u0 = __shfl_sync(kFull, f[0], src), u1 = __shfl_sync(kFull, f[1], src);
                  val = (tig >> 1) ? u1 : u0;
                }
                sv[MT0 + m][hf] = val;
              }
          };
          fold_pair(std::integral_constant<int, 0>{});
          fold_pair(std::integral_constant<int, 2>{});
          // the stage's data is in registers: hand it back to the producer
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[s]);
          // tile statistics of head tig: maximum and sum of exp2 over the valid rows
          float m = -INFINITY, l = 0.0f;
          if (rows == TR) {
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) m = fmaxf(m, fmaxf(sv[mt][0], sv[mt][1]));
          } else {
#pragma unroll
            for (int mt = 0; mt < 4; ++mt)
#pragma unroll
              for (int hf = 0; hf < 2; ++hf)
                if (16 * mt + gid + 8 * hf < rows) m = fmaxf(m, sv[mt][hf]);
          }
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
#pragma unroll
          for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const float e = fast_exp2(sv[mt][hf] - m);
              sv[mt][hf] = (rows == TR || 16 * mt + gid + 8 * hf < rows) ? e : 0.0f;
              l += sv[mt][hf];
            }
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) l += __shfl_xor_sync(kFull, l, off);
          if (tig < H) {
            float* lgt = lg + (size_t)t * TR * H + gid * H + tig;
            if (rows == TR) {
#pragma unroll
              for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) lgt[(16 * mt + 8 * hf) * H] = sv[mt][hf];
            } else {
#pragma unroll
              for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
                  if (16 * mt + gid + 8 * hf < rows) lgt[(16 * mt + 8 * hf) * H] = sv[mt][hf];
            }
            if (gid == 0) {
              tsm[t * H + tig] = m;
              tsl[t * H + tig] = l;
            }
          }
          if (lane == 0 && t < kTsCap) tinfo[t] = make_int2(rows | (dseg << 7) | (entry << 8), drow + sub * TR);
        } else {
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[s]);
        }
        // this warp's next tile: the chunk index advances by 3 or 4
        t += kConsumers;
        const int c2 = t / TPC;
        s += c2 - c;
        while (s >= S) { s -= S; ++k; }
        c = c2;
      }
    };
    if constexpr (KB == 16) consume(std::integral_constant<int, 1>{});  // one "group": the whole row
    else if (ng == 2) consume(std::integral_constant<int, 2>{});
    else if (ng == 1) consume(std::integral_constant<int, 1>{});
    else if constexpr (D == 128) consume(std::integral_constant<int, 4>{});
  }
  __syncthreads();
  // After a timed-out wait a bulk copy may still land in the ring, which
  // phase 2 reuses: skip straight to the end (the status word says why).
  const bool aborted = *abort_flag != 0;
  const int n_work = aborted ? 0 : nent;
  // the dense V pass applies when every row is kept and the V rows fit its buffers
  const bool dense = d.tau <= 0.0f && VB0 <= 6 && VB1 <= 6;
  const int lcap = a.cand_cap;
  const bool sparse_try = !dense && lcap > 0 && n_work > 0 && nent <= kUlCap;
  // sparse mode layout in the ring: the CTA's kept-row list [lcap] rows and
  // [lcap][H] weights first; behind it the e-values of a round of tiles
  // during the scan, then the warps' last-piece partial outputs [CW][H][D]
  // and the V staging slots during the accumulation (a warp's first piece,
  // when its share holds more than one, goes to its workspace slot)
  const int lists_bytes = (lcap * (1 + H) * 4 + 127) / 128 * 128;
  float* const ebuf = reinterpret_cast<float*>(ring + lists_bytes);
  const int round_tiles = sparse_try ? (a.ring_bytes - lists_bytes) / (TR * H * 4) : 0;
  // The first round's e-values (each warp's contiguous run of tiles, one
  // bulk copy per warp on its first dense-pass barrier, unused in sparse
  // mode) land while the statistics below are merged.
  const int e_t1 = sparse_try ? min(ntile, round_tiles) : 0;
  const int e_lo = (e_t1 * warp) / CW, e_hi = (e_t1 * (warp + 1)) / CW;
  if (sparse_try && lane == 0 && e_hi > e_lo) {
    fence_proxy_async_global();  // the e-values were written by plain stores in phase 1
    const uint32_t eb = (uint32_t)(e_hi - e_lo) * TR * H * 4;
    mbar_arrive_expect_tx(&dbar[warp * 2], eb);
    bulk_g2s(ebuf + (size_t)e_lo * TR * H, lg + (long long)e_lo * TR * H, eb, &dbar[warp * 2], policy_evict_first());
  }

  // ------------------------------------------------------------ statistics
  // piece statistics: the CTA's tiles of each unit, merged -- one warp per
  // (piece, head): the maximum first, then the rescaled sum
  for (int task = warp; task < n_work * H; task += CW) {
    const int e = task / H, h = task % H;
    int* rec = ulist + e * kRec;
    const Unit x = load_unit(rec);
    const int ta = (max(x.cb, k0) - k0) * TPC, tb = (min(x.cb + x.nc, k1) - k0) * TPC;
    {
      float m = -INFINITY, l = 0.0f;
      for (int t2 = ta + lane; t2 < tb; t2 += 32) m = fmaxf(m, tsm[t2 * H + h]);
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
      if (m > -INFINITY) {
        for (int t2 = ta + lane; t2 < tb; t2 += 32) {
          const float mt = tsm[t2 * H + h];
          if (mt > -INFINITY) l = fmaf(tsl[t2 * H + h], exp2f(mt - m), l);
        }
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) l += __shfl_xor_sync(kFull, l, off);
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
  __syncthreads();
  if (tid == 0 && n_work > 0) {
    __threadfence();  // orders every warp's statistics before the arrivals
    const Unit x0 = load_unit(ulist);
    if (!x0.owned) atomicAdd(a.arrive1 + x0.u, 1);
    if (nent > 1) {
      const Unit x1 = load_unit(ulist + (nent - 1) * kRec);
      if (!x1.owned) atomicAdd(a.arrive1 + x1.u, 1);
    }
  }
  // global statistics of every piece's unit: (max, 1 / sum) per head replace
  // the piece's own in its record; a unit shared with other CTAs waits
  // (bounded) for their pieces
  for (int e = warp; e < n_work; e += CW) {
    int* rec = ulist + e * kRec;
    const Unit x = load_unit(rec);
    float* st = reinterpret_cast<float*>(rec + 8);
    if (x.owned) {
      if (lane < H) {
        const float l = st[2 * lane + 1];
        st[2 * lane + 1] = l > 0.0f ? 1.0f / l : 0.0f;
      }
    } else {
      const int i_first = x.cb / cpc, i_last = (x.cb + x.nc - 1) / cpc;
      bool ok = true;
      if (lane == 0) ok = wait_counter(a.arrive1 + x.u, i_last - i_first + 1, limit_ns);
      ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
      if (!ok) {
        if (lane == 0) atomicExch(d.status, kStatusTimeout);
        if (lane < H) { st[2 * lane] = -INFINITY; st[2 * lane + 1] = 0.0f; }
      } else if (lane < H) {
        __threadfence();
        float m = -INFINITY, l = 0.0f;
        for (int i = i_first; i <= i_last; ++i) {
          const int slot = (i == i_first) ? 1 : 0;
          const float* ps = a.pstats + ((long long)i * 2 + slot) * H * 2;
          merge_ml(m, l, __ldcg(ps + 2 * lane), __ldcg(ps + 2 * lane + 1));
        }
        st[2 * lane] = m;
        st[2 * lane + 1] = l > 0.0f ? 1.0f / l : 0.0f;
      }
    }
  }
  __syncthreads();
  // per-tile factors exp2(max_tile - max) / sum (the sparse scan computes
  // its own as it goes; a sparse pass that falls back computes them later)
  auto tile_factors = [&]() {
    for (int q = tid; q < (n_work > 0 ? ntile * H : 0); q += NTHR) {
      const int t2 = q / H, h = q % H;
      const int g = k0 + t2 / TPC;
      int lo = 0, hi = nent - 1;  // entry holding chunk g
      while (lo < hi) { const int mid = (lo + hi + 1) >> 1; if (ulist[mid * kRec + 1] <= g) lo = mid; else hi = mid - 1; }
      const float* st = reinterpret_cast<const float*>(ulist + lo * kRec + 8);
      const float M = st[2 * h], il = st[2 * h + 1];
      const float mt = tsm[t2 * H + h];
      tsf[t2 * H + h] = (il > 0.0f && mt > -INFINITY) ? exp2f(mt - M) * il : 0.0f;
    }
  };
  if (!sparse_try) tile_factors();
  __syncthreads();

  // ------------------------------------------------------------ phase 2
  // phase-2 shared memory (in the ring).  Sparse mode: the kept rows
  // [lcap] and their weights [lcap][H]; the warps' partial outputs
  // [CW][H][D]; then one staging slot per kept V row.  Scan mode: kept-row lists [CW][kListCap] and weights; dense mode:
  // the V staging buffers; for both, the warps' partial outputs [CW][H][D]
  // are last.
  const int red_off = a.ring_bytes - CW * H * D * 4;
  float* red = reinterpret_cast<float*>(ring + red_off);
  unsigned long long cnt_heads = 0, cnt_rows = 0;
  uint8_t* const smask = d.skip_mask;
  float* const mass_out = d.mass;
  constexpr int kSzSlot = 8 * ((D / 32) > 2 ? (D / 32) : 2);
  constexpr int kVRowMax = D * (VB0 > VB1 ? VB0 : VB1) / 8;
  constexpr int kSlotBytes = kVRowMax + kSzSlot;
  int* const krow = reinterpret_cast<int*>(ring);             // CTA-local row | unit entry << 20
  float* const kw = reinterpret_cast<float*>(krow + lcap);    // weights p (0 for a skipping head)
  float* const red2 = reinterpret_cast<float*>(ring + lists_bytes);      // [CW][H][D]
  const int red2_bytes = CW * H * D * 4;
  uint8_t* const stage0 = ring + lists_bytes + red2_bytes;
  const int stage_slots = sparse_try ? max(0, (a.ring_bytes - lists_bytes - red2_bytes) / kSlotBytes) : 0;
  uint32_t kh_lane = 0, kr_lane = 0, kv_lane = 0;  // kept (row, head) pairs, kept rows and valid rows seen by this lane
  if (sparse_try) {
    // 1. every row of the CTA, in rounds of round_tiles tiles: the round's
    //    e-values come into shared memory in one go (each warp copies its
    //    own contiguous run of tiles); pass A takes every skip decision,
    //    writes the skip mask and attention mass and counts the kept rows;
    //    pass B lists them, in row order, in the CTA-wide list at offsets
    //    from the counts, with their weights, and starts bringing their V
    //    rows into L2.
    int kbase = 0;
    const int wcap = lcap / CW;  // list entries of one warp
    int n_w = 0;                 // this warp's kept rows so far
    for (int T0 = 0; T0 < ntile; T0 += round_tiles) {
      const int T1 = min(ntile, T0 + round_tiles);
      const int t_lo = T0 + ((T1 - T0) * warp) / CW, t_hi = T0 + ((T1 - T0) * (warp + 1)) / CW;
      // tile t: valid rows, entry, segment, position
      auto tile_info = [&](int t, int& nrow, int& ent, int& seg, int& pos) {
        if (t < kTsCap) {
          const int2 ti = tinfo[t];
          nrow = ti.x & 127; seg = (ti.x >> 7) & 1; ent = ti.x >> 8; pos = ti.y;
        } else {
          const int g = k0 + t / TPC;
          int lo2 = 0, hi2 = nent - 1;
          while (lo2 < hi2) { const int mid = (lo2 + hi2 + 1) >> 1; if (ulist[mid * kRec + 1] <= g) lo2 = mid; else hi2 = mid - 1; }
          const Unit x = load_unit(ulist + lo2 * kRec);
          const ChunkRows cr = chunk_rows(x, g - x.cb);
          nrow = max(0, min(TR, cr.rows - (t % TPC) * TR)); ent = lo2; seg = cr.seg; pos = cr.row0 + (t % TPC) * TR;
        }
      };
      if (T0 == 0) {
        // the first round's bulk copy, issued after phase 1 (same tiles)
        if (t_hi > t_lo && !mbar_wait(&dbar[warp * 2], 0, limit_ns)) {
          atomicExch(d.status, kStatusTimeout);
          mbar_wait(&dbar[warp * 2], 0, limit_ns);  // never leave the copy in flight
        }
      } else {
        // copy: the e-values of this warp's tiles (a tile's rows are one run
        // of nrow * H floats in the workspace, 16-byte aligned)
#pragma unroll 1
        for (int t = t_lo; t < t_hi; ++t) {
          int nrow, ent, seg, pos;
          tile_info(t, nrow, ent, seg, pos);
          const int nchk = (nrow * H * 4 + 15) / 16;
          const uint8_t* src = reinterpret_cast<const uint8_t*>(lg + (long long)t * TR * H);
          uint8_t* dst = reinterpret_cast<uint8_t*>(ebuf + (t - T0) * TR * H);
          for (int q = lane; q < nchk; q += 32) cp_async16(dst + q * 16, src + q * 16);
        }
        cp_async_wait_all();
      }
      __syncwarp();
      // one pass: the skip decisions; kept rows (with their weights p, 0 for
      // a head that skips) go to the warp's list, in row order
      const float tau = d.tau;
#pragma unroll 1
      for (int t = t_lo; t < t_hi; ++t) {
        int nrow, ent, seg, pos;
        tile_info(t, nrow, ent, seg, pos);
        if (nrow == 0) continue;  // the same for the whole warp
        float f[H];
        {
          // the tile's factors exp2(max_tile - max) / sum, from its piece's global statistics
          const float* st = reinterpret_cast<const float*>(ulist + ent * kRec + 8);
#pragma unroll
          for (int h = 0; h < H; ++h) {
            const float M = st[2 * h], il = st[2 * h + 1];
            const float mt = tsm[t * H + h];
            f[h] = (il > 0.0f && mt > -INFINITY) ? exp2f(mt - M) * il : 0.0f;
          }
        }
        const float* et = ebuf + (t - T0) * TR * H;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int r = hf * 32 + lane;
          float ev[H];
#pragma unroll
          for (int h = 0; h < H; ++h) ev[h] = 0.0f;
          if (r < nrow) lds_heads<H>(et + r * H, ev);
          float wgt[H];
          bool need = false;
          uint32_t kh = 0, kbits = 0;
          const bool valid = r < nrow;
#pragma unroll
          for (int h = 0; h < H; ++h) {
            const float p = ev[h] * f[h];
            const bool keep = valid && !(p < tau);
            wgt[h] = keep ? p : 0.0f;
            need |= keep;
            kh += keep ? 1u : 0u;
            kbits |= keep ? (1u << h) : 0u;
          }
          kh_lane += kh;
          kr_lane += need ? 1u : 0u;
          kv_lane += valid ? 1u : 0u;
          const unsigned bal = __ballot_sync(kFull, need);
          if (need) {
            const int o = n_w + __popc(bal & ((1u << lane) - 1u));
            if (o < wcap) {
              krow[warp * wcap + o] = (t * TR + r) | (ent << kCandRowBits);
              store_heads<H>(kw + (warp * wcap + o) * H, wgt);
              const int uu = ulist[ent * kRec];
              const int vr = pos + r;
              const int rbv = seg ? D * VB1 / 8 : D * VB0 / 8;
              const long long pr = PAGED ? unit_row<PAGED>(a, uu, vr) : (long long)uu * d.T_cap + vr;
              prefetch_l2(d.vc[seg] + pr * rbv);
              if ((seg ? VB1 : VB0) < 16) prefetch_l2(d.vsz[seg] + pr * ng * 2);
            }
          }
          n_w += __popc(bal);
          if (smask != nullptr || mass_out != nullptr) {
            // the optional outputs: skip mask and the group's mean attention
            const int uu = ulist[ent * kRec];
            const int b = uu / d.Hkv, g = uu % d.Hkv;
            if (r < nrow) {
              float ms = 0.0f;
#pragma unroll
              for (int h = 0; h < H; ++h) {
                ms += ev[h] * f[h];
                if (smask) smask[((long long)b * d.Hq + g * H + h) * d.T_cap + pos + r] = ((kbits >> h) & 1u) ? 0 : 1;
              }
              if (mass_out) mass_out[((long long)b * d.Hkv + g) * d.T_cap + pos + r] = ms * (1.0f / H);
            }
          }
        }
      }
      __syncthreads();  // the next round reuses the e-value buffer
    }
    if (n_w > wcap) s_ovf = 1;
    if (lane == 0) s_nw[warp] = min(n_w, wcap);
    (void)kbase;
  }
  __syncthreads();
  const bool sparse = sparse_try && !*static_cast<volatile int*>(&s_ovf);
  if (sparse_try && !sparse) {  // the list overflowed: the per-piece scan below needs the factors
    tile_factors();
    __syncthreads();
  }
  if (sparse) {
    if (tid == 0) {
      int acc_n = 0;
      for (int w2 = 0; w2 < CW; ++w2) { s_pref[w2] = acc_n; acc_n += s_nw[w2]; }
      s_pref[CW] = acc_n;
    }
    // counts: every valid (row, head) of the CTA minus the kept ones
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      kh_lane += __shfl_xor_sync(kFull, kh_lane, off);
      kr_lane += __shfl_xor_sync(kFull, kr_lane, off);
      kv_lane += __shfl_xor_sync(kFull, kv_lane, off);
    }
    if (lane == 0) { atomicAdd(&s_kept[0], (int)kh_lane); atomicAdd(&s_kept[1], (int)kr_lane); atomicAdd(&s_valid, (int)kv_lane); }
    if (tid < CW * 2) s_spiece[tid] = -1;
    // 2. the CTA's kept rows are split evenly over the warps; each warp
    //    brings its rows' V codes and (scale, zero) into its staging slots
    //    (slot = list position; rows past the slots are read from global
    //    memory), then accumulates.  A warp's share is cut where the unit
    //    piece changes; the first and last pieces of the share go to the
    //    warp's two partial-output slots, pieces in between (whole pieces,
    //    owned by this CTA) straight to the output.
    __syncthreads();
    const int n_all = s_pref[CW];
    const int wcap = lcap / CW;
    // physical list index of CTA list position gidx (warp lists in warp order)
    auto pidx = [&](int gidx) {
      int lo2 = 0, hi2 = CW - 1;
      while (lo2 < hi2) { const int mid = (lo2 + hi2 + 1) >> 1; if (s_pref[mid] <= gidx) lo2 = mid; else hi2 = mid - 1; }
      return lo2 * wcap + gidx - s_pref[lo2];
    };
    const int per = ((n_all + CW - 1) / CW + RPW - 1) / RPW * RPW;
    const int g_lo = min(n_all, warp * per), g_hi = min(n_all, g_lo + per);
    // one row per lane: its codes and (scale, zero) in 16-byte copies
    for (int i = g_lo + lane; i < min(g_hi, stage_slots); i += 32) {
      const int rowe = krow[pidx(i)];
      const int ent = rowe >> kCandRowBits, row = rowe & ((1 << kCandRowBits) - 1);
      const Unit x = load_unit(ulist + ent * kRec);
      const ChunkRows cr = chunk_rows(x, (k0 + row / kChunk) - x.cb);
      const int vr = cr.row0 + row % kChunk;
      const int rbv = cr.seg ? D * VB1 / 8 : D * VB0 / 8;
      const int szb = (cr.seg ? VB1 : VB0) == 16 ? 0 : (ng == 1 ? 16 : ng * 8);
      uint8_t* slot = stage0 + (size_t)i * kSlotBytes;
      const long long pr = PAGED ? unit_row<PAGED>(a, x.u, vr) : (long long)x.u * d.T_cap + vr;
      for (int c = 0; c < rbv; c += 16) cp_async16(slot + c, d.vc[cr.seg] + pr * rbv + c);
      if (szb > 0) {
        // ng == 1: the 16 bytes of the even/odd row pair (T_cap is even then)
        const long long pr0 = ng == 1 ? (pr & ~1ll) : pr;
        const uint8_t* zs = reinterpret_cast<const uint8_t*>(d.vsz[cr.seg] + pr0 * ng * 2);
        for (int c = 0; c < szb; c += 16) cp_async16(slot + kVRowMax + c, zs + c);
      }
    }
    cp_async_wait_all();
    __syncwarp();
    int seg_lo = g_lo;
    while (seg_lo < g_hi) {
      // the segment [seg_lo, seg_hi): the share's rows of one piece
      const int pc = krow[pidx(seg_lo)] >> kCandRowBits;
      int seg_hi;
      {
        int lo2 = seg_lo + 1, hi2 = g_hi;  // first index of a later piece
        while (lo2 < hi2) { const int mid = (lo2 + hi2) >> 1; if ((krow[pidx(mid)] >> kCandRowBits) == pc) lo2 = mid + 1; else hi2 = mid; }
        seg_hi = lo2;
      }
      const Unit x = load_unit(ulist + pc * kRec);
      float2 acc[H][8];
      float Z[H];
#pragma unroll
      for (int h = 0; h < H; ++h) {
        Z[h] = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[h][i] = make_float2(0.0f, 0.0f);
      }
      int sw = 0;
      {
        const int g0 = min(seg_lo + lane / LPR, n_all - 1);
        int lo2 = 0, hi2 = CW - 1;
        while (lo2 < hi2) { const int mid = (lo2 + hi2 + 1) >> 1; if (s_pref[mid] <= g0) lo2 = mid; else hi2 = mid - 1; }
        sw = lo2;
      }
      for (int i0 = seg_lo; i0 < seg_hi; i0 += RPW) {
        const int gidx = i0 + lane / LPR;
        if (gidx >= seg_hi) break;  // the lanes of a row agree
        while (gidx >= s_pref[sw + 1]) ++sw;
        float wgt[H];
        const int pi = sw * wcap + gidx - s_pref[sw];
        lds_heads<H>(kw + pi * H, wgt);
        const int row = krow[pi] & ((1 << kCandRowBits) - 1);
        const int v = (k0 - x.cb) * kChunk + row;
        const ChunkRows cr = chunk_rows(x, v / kChunk);
        const int vr = cr.row0 + v % kChunk;
        LaneWords<VB0> w0;
        LaneWords<(VB0 == VB1) ? 2 : VB1> w1;
        float2 sz;
        if (gidx < stage_slots) {
          const uint8_t* src = stage0 + (size_t)gidx * kSlotBytes;
          const float* szp = reinterpret_cast<const float*>(src + kVRowMax) + (ng == 1 ? (vr & 1) * 2 : gi * 2);
          sz = (cr.seg ? VB1 : VB0) == 16 ? make_float2(0.0f, 0.0f) : *reinterpret_cast<const float2*>(szp);
          if (cr.seg == 0 || VB0 == VB1) lds_lane_words<VB0>(src + j * 2 * VB0, w0);
          else if constexpr (VB0 != VB1) lds_lane_words<VB1>(src + j * 2 * VB1, w1);
        } else {
          const long long pr = PAGED ? unit_row<PAGED>(a, x.u, vr) : (long long)x.u * d.T_cap + vr;
          if (cr.seg == 0 || VB0 == VB1) ldg_v<VB0>(d.vc[cr.seg] + pr * (D * VB0 / 8), d.vsz[cr.seg] + pr * ng * 2, j, gi, w0, sz);
          else if constexpr (VB0 != VB1) ldg_v<VB1>(d.vc[1] + pr * (D * VB1 / 8), d.vsz[1] + pr * ng * 2, j, gi, w1, sz);
        }
        if (cr.seg == 0 || VB0 == VB1) accumulate_v<H, VB0>(w0, sz, wgt, acc, Z);
        else if constexpr (VB0 != VB1) accumulate_v<H, VB1>(w1, sz, wgt, acc, Z);
      }
      // add the warp's row slots with shuffles
#pragma unroll
      for (int h = 0; h < H; ++h)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float2 v2 = make_float2(acc[h][i].x + Z[h], acc[h][i].y + Z[h]);
#pragma unroll
          for (int off = LPR; off < 32; off <<= 1) {
            v2.x += __shfl_xor_sync(kFull, v2.x, off);
            v2.y += __shfl_xor_sync(kFull, v2.y, off);
          }
          acc[h][i] = v2;
        }
      const bool first = seg_lo == g_lo, last = seg_hi == g_hi;
      if (first || last) {
        // the share's last piece to the warp's slot in shared memory, a
        // different first piece to its slot in the workspace
        const int k = last ? 1 : 0;
        float* dst = last ? red2 + warp * H * D : a.wslot + ((long long)cta * CW + warp) * H * D;
        if (lane < LPR) {
#pragma unroll
          for (int h = 0; h < H; ++h)
#pragma unroll
            for (int i = 0; i < 8; i += 2)
              *reinterpret_cast<float4*>(dst + h * D + j * kDimsPerLane + 2 * i) =
                  make_float4(acc[h][i].x, acc[h][i].y, acc[h][i + 1].x, acc[h][i + 1].y);
        }
        if (lane == 0) s_spiece[warp * 2 + k] = pc;
      } else if (lane < LPR) {
        // a whole piece between two others: owned by this CTA, and only this warp holds its rows
        const int b = x.u / d.Hkv, g = x.u % d.Hkv;
#pragma unroll
        for (int h = 0; h < H; ++h)
#pragma unroll
          for (int i = 0; i < 8; i += 2)
            *reinterpret_cast<float4*>(d.out + ((long long)b * d.Hq + g * H + h) * D + j * kDimsPerLane + 2 * i) =
                make_float4(acc[h][i].x, acc[h][i].y, acc[h][i + 1].x, acc[h][i + 1].y);
        if (lane == 0) s_pdone[pc] = 1;
      }
      seg_lo = seg_hi;
    }
    __syncthreads();
    // 3. the output of every piece not yet written: the sum of the slots
    //    that hold it, in warp order (zero when no head kept any row); a
    //    piece's slots lie in one range of the warp-ordered slot list
    for (int e = 0; e < n_work; ++e) {
      if (s_pdone[e]) continue;
      const Unit x = load_unit(ulist + e * kRec);
      const int b = x.u / d.Hkv, g = x.u % d.Hkv;
      for (int o = tid; o < H * D; o += NTHR) {
        float s2 = 0.0f;
        for (int k2 = 0; k2 < CW * 2; ++k2)
          if (s_spiece[k2] == e)
            s2 += (k2 & 1) ? red2[(k2 >> 1) * H * D + o] : __ldcg(a.wslot + ((long long)cta * CW + (k2 >> 1)) * H * D + o);
        const int h = o / D, dd = o % D;
        if (x.owned) {
          d.out[((long long)b * d.Hq + g * H + h) * D + dd] = s2;
        } else {
          if (e == 0) a.ppart[(((long long)cta * 2 + 0) * H + h) * D + dd] = s2;
          if (e == nent - 1) a.ppart[(((long long)cta * 2 + 1) * H + h) * D + dd] = s2;
        }
      }
    }
    __syncthreads();
    // 4. shared units: publish the partial; the last CTA to arrive adds them
    if (tid == 0) {
      __threadfence();  // every thread's partial before the arrivals
      for (int c = 0; c < 2; ++c) {
        const int e = c == 0 ? 0 : nent - 1;
        if (c == 1 && nent == 1) break;
        const Unit x = load_unit(ulist + e * kRec);
        s_lastu[c] = -1;
        if (x.owned) continue;
        const int i_first = x.cb / cpc, i_last = (x.cb + x.nc - 1) / cpc;
        const int old = atomicAdd(a.arrive2 + x.u, 1);
        if (old == i_last - i_first) s_lastu[c] = e;
      }
    }
    __syncthreads();
    for (int c = 0; c < 2; ++c) {
      const int e = s_lastu[c];
      if (e < 0 || (c == 1 && nent == 1)) continue;
      __threadfence();
      const Unit x = load_unit(ulist + e * kRec);
      const int i_first = x.cb / cpc, i_last = (x.cb + x.nc - 1) / cpc;
      const int b = x.u / d.Hkv, g = x.u % d.Hkv;
      for (int o = tid; o < H * D; o += NTHR) {
        float s2 = 0.0f;
        for (int i = i_first; i <= i_last; ++i) {
          const int slot = (i == i_first) ? 1 : 0;
          s2 += __ldcg(a.ppart + (((long long)i * 2 + slot) * H) * D + o);
        }
        d.out[((long long)b * d.Hq + g * H + o / D) * D + o % D] = s2;
      }
      if (tid == 0) {
        a.arrive1[x.u] = 0;
        a.arrive2[x.u] = 0;
      }
    }
    __syncthreads();
    if (tid == 0) {
      const long long valid = s_valid;  // every valid row of the CTA passed the scan once
      cnt_heads = (unsigned long long)(valid * H - s_kept[0]);
      cnt_rows = (unsigned long long)(valid - s_kept[1]);
    }
  }
  int* lists = reinterpret_cast<int*>(ring);
  float* wts = reinterpret_cast<float*>(ring + kWarps * kListCap * 4);
  int dense_uses[2] = {0, 0};
  for (int e = 0; e < (sparse ? 0 : n_work); ++e) {
    int* rec = ulist + e * kRec;
    const Unit x = load_unit(rec);
    const int b = x.u / d.Hkv, g = x.u % d.Hkv;
    const int i_first = x.cb / cpc, i_last = (x.cb + x.nc - 1) / cpc;
    const int ga = max(x.cb, k0), gb = min(x.cb + x.nc, k1);
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
          uint64_t* bar = &dbar[warp * 2 + buf];
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
          if (!mbar_wait(&dbar[warp * 2 + buf], dense_uses[buf] & 1, limit_ns)) {
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
            // not unrolled: the body is large and the instruction cache small
#pragma unroll 1
            for (int s2 = 0; s2 < 32 / RPW; ++s2) {
              const int i = s2 * RPW + lane / LPR;
              if (i >= rows) continue;  // the lanes of a row agree
              float ev[H], wgt[H];
              lds_heads<H>(lgs + i * H, ev);
              float ms = 0.0f;
#pragma unroll
              for (int h = 0; h < H; ++h) { wgt[h] = ev[h] * f[h]; ms += wgt[h]; }
              if (j == 0) {
                if (smask) {
#pragma unroll
                  for (int h = 0; h < H; ++h) smask[((long long)b * d.Hq + g * H + h) * d.T_cap + v0 + i] = 0;
                }
                if (mass_out) mass_out[((long long)b * d.Hkv + g) * d.T_cap + v0 + i] = ms * (1.0f / H);
              }
              const float2 sz = *reinterpret_cast<const float2*>(szs + ((sz_skip + i) * ng + gi) * 2);
              if (cr.seg == 0) {
                LaneWords<VB0> lwd;
                lds_lane_words<VB0>(src + i * (D * VB0 / 8) + j * 2 * VB0, lwd);
                accumulate_v<H, VB0>(lwd, sz, wgt, acc, Z);
              } else {
                LaneWords<VB1> lwd;
                lds_lane_words<VB1>(src + i * (D * VB1 / 8) + j * 2 * VB1, lwd);
                accumulate_v<H, VB1>(lwd, sz, wgt, acc, Z);
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
          mbar_wait(&dbar[warp * 2 + buf], dense_uses[buf] & 1, limit_ns);
          ++dense_uses[buf];
        }
    } else {
      for (int vb = v_lo; vb < v_hi; vb += CW * 32 * kBatchBlocks) {
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
        // split evenly over the warps, in order
        if (lane == 0) s_nw[warp] = n_w;
        __syncthreads();
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
              accumulate_v<H, VB0>(w0[s2], szv[s2], wgt, acc, Z);
            } else {
              if (v / kChunk < x.nc0) accumulate_v<H, VB0>(w0[s2], szv[s2], wgt, acc, Z);
              else accumulate_v<H, VB1>(w1[s2], szv[s2], wgt, acc, Z);
            }
          }
        }
        __syncthreads();  // other warps read this batch's lists
      }
    }
    // fold the per-group constant, add the warp's row slots with shuffles
#pragma unroll
    for (int h = 0; h < H; ++h)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float2 v2 = make_float2(acc[h][i].x + Z[h], acc[h][i].y + Z[h]);
#pragma unroll
        for (int off = LPR; off < 32; off <<= 1) {
          v2.x += __shfl_xor_sync(kFull, v2.x, off);
          v2.y += __shfl_xor_sync(kFull, v2.y, off);
        }
        acc[h][i] = v2;
      }
    if (lane < LPR) {
#pragma unroll
      for (int h = 0; h < H; ++h)
#pragma unroll
        for (int i = 0; i < 8; i += 2)
          *reinterpret_cast<float4*>(red + (warp * H + h) * D + j * kDimsPerLane + 2 * i) =
              make_float4(acc[h][i].x, acc[h][i].y, acc[h][i + 1].x, acc[h][i + 1].y);
    }
    __syncthreads();
    for (int o = tid; o < H * D; o += NTHR) {
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
      __syncthreads();
      if (tid == 0) {
        __threadfence();  // every thread's partial before the arrival
        const int old = atomicAdd(a.arrive2 + x.u, 1);
        s_last = (old == i_last - i_first) ? 1 : 0;
      }
      __syncthreads();
      if (s_last) {
        __threadfence();
        for (int o = tid; o < H * D; o += NTHR) {
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
    __syncthreads();
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
  __syncthreads();
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
