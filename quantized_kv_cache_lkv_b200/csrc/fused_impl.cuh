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
//  phase 1  a producer warp streams the K rows of the CTA's chunks through a
//           ring of shared-memory stages with 1-D bulk copies (TMA, evict-
//           first in L2) completing on mbarriers.  Three groups of four
//           consumer warps take the tiles in turn and turn them into base-2
//           logits for the group's query heads, kept in shared memory, while
//           tracking each chunk's maximum.
//  stats    per chunk: sum of exp2(s - max) (logits become e = exp2(s - max));
//           per unit piece: the merged statistics.  A unit owned by one CTA
//           needs nothing else; a unit shared by neighbouring CTAs exchanges
//           piece statistics through the workspace (bounded wait on a
//           per-unit arrival counter).
//  phase 2  p = e * exp2(max_chunk - max) / sum.  A (b, h, t) with p < tau is
//           skipped; the V rows some head keeps are listed per warp in row
//           order, gathered from HBM and accumulated as p * vhat.  Shared
//           units publish partial outputs; the last CTA to arrive adds them.
//
// Dequantization is folded into the dot products: codes become exact
// integers (unpack16_int) and, with the group's (scale, zero),
//   sum_d q_d * (scale * c_d + zero) = scale * sum_d q_d c_d + zero * sum_d q_d.
#pragma once
#include <cfloat>

#include "lkv_kernels.cuh"

namespace lkv {
namespace fused {

constexpr int kGroupWarps = 4;                 // consumer warps sharing a tile
constexpr int kGroups = 3;                     // tiles are dealt to groups in turn
constexpr int kConsumerWarps = kGroupWarps * kGroups;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;      // + producer warp
constexpr int kChunk = 256;    // tokens per chunk (softmax statistics granularity)
constexpr int kTile = 64;      // tokens per bulk-copy tile
constexpr int kMaxStages = 15; // multiple of kGroups
constexpr int kListCap = 512;  // V-row list entries per warp per batch
constexpr int kBatchBlocks = kListCap / 32;
constexpr int kRec = 16;       // ints per unit-list record
constexpr int kGatherUnroll = 2;
constexpr int kCsCap = 64;     // chunk statistics kept in shared memory up to this many chunks
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kBarCons = 1;    // named barrier of the consumer warps
constexpr int kHeader = 4096;  // bytes of shared memory before the ring

// Shared header layout (bytes): barriers [0, 256), tile descriptors
// [256, 768), misc ints [768, 1024), chunk statistics [1024, 4096).
constexpr int kDescOff = 256;
constexpr int kMiscOff = 768;
constexpr int kCsOff = 1024;

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

// Order-preserving map of floats to ints (for atomicMax on floats).
__device__ __forceinline__ int f2ord(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float ord2f(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7FFFFFFF); }

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

template <int D, int KB>
struct Geo {
  static constexpr int LPR = D / kDimsPerLane;  // lanes per row
  static constexpr int RPW = 32 / LPR;          // rows per warp step
  static constexpr int RB = D * KB / 8;         // packed K row bytes
  static constexpr int kStageCodes = kTile * RB;
  static constexpr int kStageSz = (kTile + 2) * (D / 32) * 8;  // ng <= D/32, plus alignment rows
  static constexpr int kStageBytes = (kStageCodes + kStageSz + 127) / 128 * 128;
};

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

template <int NH, int OFF>
struct ReduceScatter {
  static __device__ __forceinline__ void run(float* v, int lane, int& hidx) {
    if constexpr (OFF >= 1) {
      if constexpr (NH > 1) {
        constexpr int half = NH / 2;
        const bool up = (lane & OFF) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
          const float send = up ? v[i] : v[half + i];
          const float keep = up ? v[half + i] : v[i];
          v[i] = keep + __shfl_xor_sync(kFull, send, OFF);
        }
        if (up) hidx += half;
        ReduceScatter<half, OFF / 2>::run(v, lane, hidx);
      } else {
        v[0] += __shfl_xor_sync(kFull, v[0], OFF);
        ReduceScatter<1, OFF / 2>::run(v, lane, hidx);
      }
    }
  }
};

template <int H, int LPR>
__device__ __forceinline__ int head_of_lane(int lane) {
  float dummy[H];
#pragma unroll
  for (int h = 0; h < H; ++h) dummy[h] = 0.0f;
  int hidx = 0;
  ReduceScatter<H, LPR / 2>::run(dummy, lane, hidx);
  return hidx;
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
__device__ __forceinline__ void store_heads(float* p, const float (&x)[H]) {
  if constexpr (H == 4) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  } else if constexpr (H == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
  } else {
    p[0] = x[0];
  }
}

// Exponent fields of the unpack's magic floats, kept in registers so that
// each code costs a single AND-OR (an immediate mask plus this register).
template <int BITS>
struct Magic {
  uint32_t m[32];
  __device__ __forceinline__ void load(const int* src) {
#pragma unroll
    for (int k = 0; k < 24 - BITS; ++k) m[k] = (uint32_t)src[k];
  }
};

template <int BITS, int I>
__device__ __forceinline__ float code_plus_magic_r(const LaneWords<BITS>& lw, const Magic<BITS>& mg) {
  constexpr int s = copy_shift<BITS>(I);
  constexpr int kk = I * BITS - s;
  constexpr uint32_t mask = ((1u << BITS) - 1u) << kk;
  return __uint_as_float((stream_bits<BITS>(lw, s) & mask) | mg.m[kk]);
}

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
  int kk, seg, row0, rows, entry, pad0, pad1, pad2;
};

// ------------------------------------------------------------------ kernel

template <int D, int H, int KB, int VB0, int VB1>
__global__ void __launch_bounds__(kThreads, 1) fused_decode_kernel(FusedArgs a) {
  using Gk = Geo<D, KB>;
  constexpr int LPR = Gk::LPR, RPW = Gk::RPW;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cta = blockIdx.x, grid = gridDim.x;
  const DecodeArgs& d = a.d;
  const int units = d.B * d.Hkv;
  const int ng = D / d.G;
  const int S = a.stages;
  const uint64_t limit_ns = (a.timeout_ns && *a.timeout_ns) ? *a.timeout_ns : 2000000000ull;
  const int j = lane % LPR;                 // lane's 16-channel slice of a row
  const int gi = (j * kDimsPerLane) / d.G;  // its quantization group

  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw);
  uint64_t* empty = full + kMaxStages;
  TileDesc* desc = reinterpret_cast<TileDesc*>(smem_raw + kDescOff);
  int* misc = reinterpret_cast<int*>(smem_raw + kMiscOff);   // 64 ints
  uint8_t* ring = smem_raw + kHeader;
  float* s_logits = reinterpret_cast<float*>(ring + a.ring_bytes);

  int& s_total = misc[0];
  int& s_e0 = misc[1];
  int& s_nent = misc[2];
  int& s_abort = misc[3];
  int& s_carry_c = misc[4];
  int& s_carry_n = misc[5];
  int& s_last = misc[6];
  float* s_glob = reinterpret_cast<float*>(misc + 8);   // (max, 1/sum) x 4 heads
  int* s_wsum = misc + 16;                             // 2 x 12 warp partials
  int* s_magic = misc + 40;                            // 24 magic exponent fields

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGroupWarps);
    }
    fence_mbar_init();
    s_total = 0; s_e0 = 0; s_nent = 0; s_abort = 0; s_carry_c = 0; s_carry_n = 0; s_last = 0;
  }
  if (tid < 24) s_magic[tid] = (150 - tid) << 23;
  __syncthreads();

  // ------------------------------------------------------------ unit list
  const bool consumer = warp < kConsumerWarps;
  if (consumer) {
    int part = 0;
    for (int u = tid; u < units; u += kConsumers) {
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
    if (tid == 0 && cta == 0) {
      for (int u = 0; u < (d.len_mode == 0 ? d.B : units); ++u) {
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
  int* ulist = a.ulist + (long long)cta * a.cpc_max * kRec;
  if (consumer) {
    for (int base = 0; base < units; base += kConsumers) {
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
      if (lane == 31) { s_wsum[warp] = sc; s_wsum[12 + warp] = sn; }
      named_barrier(kBarCons, kConsumers);
      int wc = 0, wn = 0, tc = 0, tn = 0;
      for (int w = 0; w < kConsumerWarps; ++w) {
        if (w < warp) { wc += s_wsum[w]; wn += s_wsum[12 + w]; }
        tc += s_wsum[w]; tn += s_wsum[12 + w];
      }
      const int cb = s_carry_c + wc + sc - nc;
      const int ne_idx = s_carry_n + wn + sn - ne;
      if (ne && cb <= k0 && k0 < cb + nc) s_e0 = ne_idx;
      named_barrier(kBarCons, kConsumers);
      if (ne && cb < k1 && cb + nc > k0) {
        const int idx = ne_idx - s_e0;
        int* rec = ulist + (long long)idx * kRec;
        rec[0] = u; rec[1] = cb; rec[2] = nc; rec[3] = n0; rec[4] = n1;
        rec[5] = (cb >= k0 && cb + nc <= k1) ? 1 : 0;
        rec[6] = nc0;
        atomicMax(&s_nent, idx + 1);
      }
      named_barrier(kBarCons, kConsumers);
      if (tid == 0) { s_carry_c += tc; s_carry_n += tn; }
      named_barrier(kBarCons, kConsumers);
    }
  }
  // chunk statistics: in shared memory unless the CTA has many chunks
  int* cmx;
  float *csm, *cfc;
  if (nck <= kCsCap) {
    cmx = reinterpret_cast<int*>(smem_raw + kCsOff);
    csm = reinterpret_cast<float*>(cmx + kCsCap * 4);
    cfc = csm + kCsCap * 4;
  } else {
    cmx = reinterpret_cast<int*>(a.gstats + (long long)cta * a.cpc_max * 12);
    csm = reinterpret_cast<float*>(cmx + a.cpc_max * 4);
    cfc = csm + a.cpc_max * 4;
  }
  for (int i = tid; i < nck * H; i += kThreads) cmx[i] = f2ord(-INFINITY);
  __syncthreads();  // list complete, maxima reset
  const int nent = s_nent;

  float* lg = ((long long)nck * kChunk * H <= a.smem_logit_floats)
                  ? s_logits
                  : a.glogits + (long long)cta * a.cpc_max * kChunk * H;

  // ------------------------------------------------------------ phase 1
  if (!consumer) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int t = 0;
      bool ok = true;
      auto acquire_stage = [&](int tt) -> bool {
        if (tt < S) return true;
        const int st = tt % S;
        if (mbar_wait(&empty[st], ((tt / S) - 1) & 1, limit_ns)) return true;
        atomicExch(d.status, kStatusTimeout);
        atomicExch(&s_abort, 1);
        return false;
      };
      for (int e = 0; e < nent && ok; ++e) {
        const Unit x = load_unit(ulist + (long long)e * kRec);
        const long long ubase = (long long)x.u * d.T_cap;
        const int ga = max(x.cb, k0), gb = min(x.cb + x.nc, k1);
        for (int g = ga; g < gb && ok; ++g) {
          const ChunkRows cr = chunk_rows(x, g - x.cb);
          for (int r = 0; r < cr.rows && ok; r += kTile) {
            const int rows = min(kTile, cr.rows - r);
            const int row = cr.row0 + r;
            if (!acquire_stage(t)) { ok = false; break; }
            const int stage = t % S;
            const int r0 = (ng == 1) ? (row & ~1) : row;
            const int r1 = (ng == 1) ? ((row + rows + 1) & ~1) : row + rows;
            const uint32_t cbytes = (uint32_t)rows * Gk::RB;
            const uint32_t sbytes = (uint32_t)(r1 - r0) * ng * 8;
            TileDesc td;
            td.kk = g - k0; td.seg = cr.seg; td.row0 = row; td.rows = rows; td.entry = e;
            desc[stage] = td;
            uint8_t* dst = ring + (size_t)stage * Gk::kStageBytes;
            mbar_arrive_expect_tx(&full[stage], cbytes + sbytes);
            bulk_g2s(dst, d.kc[cr.seg] + (ubase + row) * Gk::RB, cbytes, &full[stage], pol);
            bulk_g2s(dst + Gk::kStageCodes, d.ksz[cr.seg] + (ubase + r0) * ng * 2, sbytes, &full[stage], pol);
            ++t;
          }
        }
      }
      // one end marker per consumer group (a plain arrival completes the phase)
      for (int k = 0; k < kGroups && ok; ++k) {
        if (!acquire_stage(t)) { ok = false; break; }
        const int stage = t % S;
        desc[stage].rows = -1;
        mbar_arrive(&full[stage]);
        ++t;
      }
      // Never leave copies in flight: wait for the last stages issued.
      for (int k = max(0, t - S); k < t; ++k) mbar_wait(&full[k % S], (k / S) & 1, limit_ns);
    }
    return;  // the producer warp takes no further part
  }

  // consumers
  {
    const int grp = warp / kGroupWarps, wig = warp % kGroupWarps;
    const int hidx_lane = head_of_lane<H, LPR>(lane);
    const bool leader = (lane % (LPR / H)) == 0;
    Magic<KB> mg;
    mg.load(s_magic);
    float2 qf[H][8];
    float Q[H];
    int cur_e = -1;
    volatile int* abort_flag = &s_abort;
    for (int t = grp;; t += kGroups) {
      const int stage = t % S;
      if (*abort_flag) break;
      if (!mbar_wait(&full[stage], (t / S) & 1, limit_ns)) {
        atomicExch(d.status, kStatusTimeout);
        atomicExch(&s_abort, 1);
        break;
      }
      const TileDesc td = desc[stage];
      if (td.rows < 0) break;
      if (td.entry != cur_e) {
        cur_e = td.entry;
        const Unit x = load_unit(ulist + (long long)cur_e * kRec);
        const int b = x.u / d.Hkv, g = x.u % d.Hkv;
#pragma unroll
        for (int h = 0; h < H; ++h) {
          float xq[16];
          load16_bf16(d.q + ((long long)b * d.Hq + g * H + h) * D + j * kDimsPerLane, xq);
          float s = 0.0f;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            qf[h][i] = make_float2(xq[2 * i] * d.q_scale, xq[2 * i + 1] * d.q_scale);
            s += qf[h][i].x + qf[h][i].y;
          }
          Q[h] = s;
        }
      }
      const uint8_t* codes = ring + (size_t)stage * Gk::kStageBytes;
      const float* szs = reinterpret_cast<const float*>(codes + Gk::kStageCodes) +
                         ((ng == 1) ? (td.row0 & 1) : 0) * ng * 2;
      float* lgt = lg + (td.kk * kChunk + (td.row0 % kChunk)) * H;
      const int nrs = (td.rows + RPW - 1) / RPW;
      float tmax = -INFINITY;
      for (int rs = wig; rs < nrs; rs += kGroupWarps) {
        const int i = rs * RPW + lane / LPR;
        const bool valid = i < td.rows;
        float dot[H];
#pragma unroll
        for (int h = 0; h < H; ++h) dot[h] = 0.0f;
        if (valid) {
          LaneWords<KB> lw;
          lds_lane_words<KB>(codes + i * Gk::RB + j * (2 * KB), lw);
          const float2 sz = *reinterpret_cast<const float2*>(szs + (i * ng + gi) * 2);
          float2 c[8];
          unpack16_int_r<KB>(lw, mg, c);
#pragma unroll
          for (int h = 0; h < H; ++h) {
            float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int p = 0; p < 8; ++p) acc = __ffma2_rn(qf[h][p], c[p], acc);
            dot[h] = fmaf(sz.x, acc.x + acc.y, sz.y * Q[h]);
          }
        }
        int hidx = 0;
        ReduceScatter<H, LPR / 2>::run(dot, lane, hidx);
        if (valid && leader) {
          lgt[i * H + hidx] = dot[0];
          tmax = fmaxf(tmax, dot[0]);
        }
      }
      // tile maximum per head -> the chunk's running maximum
#pragma unroll
      for (int off = LPR; off < 32; off <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, off));
      if (lane < LPR && leader && tmax > -INFINITY) atomicMax(&cmx[td.kk * H + hidx_lane], f2ord(tmax));
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
    }
  }
  named_barrier(kBarCons, kConsumers);
  // After a timed-out wait a bulk copy may still land in the ring, which
  // phase 2 reuses: skip straight to the end (the status word says why).
  const bool aborted = *static_cast<volatile int*>(&s_abort) != 0;
  const int n_work = aborted ? 0 : nent;
  const int n_chunks_work = aborted ? 0 : nck;

  // ------------------------------------------------------------ chunk sums
  for (int kk = warp; kk < n_chunks_work; kk += kConsumerWarps) {
    const int g_chunk = k0 + kk;
    int lo = 0, hi = nent - 1;  // entry holding chunk g_chunk
    while (lo < hi) {
      const int mid = (lo + hi + 1) / 2;
      if (ulist[(long long)mid * kRec + 1] <= g_chunk) lo = mid; else hi = mid - 1;
    }
    const Unit x = load_unit(ulist + (long long)lo * kRec);
    const int rows = chunk_rows(x, g_chunk - x.cb).rows;
    float* base = lg + (long long)kk * kChunk * H;
    float m[H], l[H];
#pragma unroll
    for (int h = 0; h < H; ++h) { m[h] = ord2f(cmx[kk * H + h]); l[h] = 0.0f; }
    for (int i = lane; i < rows; i += 32) {
      float s[H];
      load_heads<H>(base + (long long)i * H, s);
#pragma unroll
      for (int h = 0; h < H; ++h) {
        s[h] = exp2f(s[h] - m[h]);
        l[h] += s[h];
      }
      store_heads<H>(base + (long long)i * H, s);
    }
#pragma unroll
    for (int h = 0; h < H; ++h)
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) l[h] += __shfl_xor_sync(kFull, l[h], off);
    if (lane < H) csm[kk * H + lane] = l[lane];
  }
  named_barrier(kBarCons, kConsumers);

  // ------------------------------------------------------------ piece statistics
  for (int e = warp; e < n_work; e += kConsumerWarps) {
    int* rec = ulist + (long long)e * kRec;
    const Unit x = load_unit(rec);
    const int ga = max(x.cb, k0), gb = min(x.cb + x.nc, k1);
#pragma unroll
    for (int h = 0; h < H; ++h) {
      float m = -INFINITY, l = 0.0f;
      for (int g2 = ga + lane; g2 < gb; g2 += 32) merge_ml(m, l, ord2f(cmx[(g2 - k0) * H + h]), csm[(g2 - k0) * H + h]);
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
  named_barrier(kBarCons, kConsumers);
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
  int* lists = reinterpret_cast<int*>(ring);                                    // [12][kListCap]
  float* red = reinterpret_cast<float*>(ring + kConsumerWarps * kListCap * 4);  // [12][H][D]
  Magic<VB0> mg0;
  mg0.load(s_magic);
  Magic<VB1> mg1;
  mg1.load(s_magic);
  unsigned long long cnt_heads = 0, cnt_rows = 0;
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
      named_barrier(kBarCons, kConsumers);
      const int ga = max(x.cb, k0), gb = min(x.cb + x.nc, k1);
      // per-chunk factors exp2(max_c - max) / sum
      for (int q = tid; q < (gb - ga) * H; q += kConsumers) {
        const int kk = ga - k0 + q / H, h = q % H;
        const float M = s_glob[2 * h], il = s_glob[2 * h + 1];
        cfc[kk * H + h] = (il > 0.0f) ? exp2f(ord2f(cmx[kk * H + h]) - M) * il : 0.0f;
      }
      named_barrier(kBarCons, kConsumers);

      const float* lgu = lg + (long long)(x.cb - k0) * kChunk * H;
      const float* cfu = cfc + (x.cb - k0) * H;
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
      for (int vb = v_lo; vb < v_hi; vb += kConsumers * kBatchBlocks) {
        // scan: 32-row blocks round robin over warps, row order kept per warp
        int* list = lists + warp * kListCap;
        int n_w = 0;
        for (int blk = warp; blk < kConsumerWarps * kBatchBlocks; blk += kConsumerWarps) {
          if (vb + blk * 32 >= v_hi) break;
          const int v = vb + blk * 32 + lane;
          const int c = v / kChunk;
          const ChunkRows cr = chunk_rows(x, c);
          bool need = false;
          if (v % kChunk < cr.rows) {
            float ev[H];
            load_heads<H>(lgu + (long long)v * H, ev);
            int nskip = 0;
#pragma unroll
            for (int h = 0; h < H; ++h) {
              const float p = ev[h] * cfu[c * H + h];
              const bool keep = !(p < d.tau);
              need |= keep;
              nskip += keep ? 0 : 1;
              if (d.skip_mask) d.skip_mask[((long long)b * d.Hq + g * H + h) * d.T_cap + v] = keep ? 0 : 1;
            }
            cnt_heads += nskip;
            cnt_rows += need ? 0 : 1;
          }
          const unsigned bal = __ballot_sync(kFull, need);
          if (need) list[n_w + __popc(bal & ((1u << lane) - 1u))] = v;
          n_w += __popc(bal);
        }
        __syncwarp();
        // gather and accumulate this warp's rows
        for (int i0 = 0; i0 < n_w; i0 += kGatherUnroll * RPW) {
          constexpr bool kOneWidth = (VB0 == VB1);
          LaneWords<VB0> w0[kGatherUnroll];
          LaneWords<kOneWidth ? 2 : VB1> w1[kOneWidth ? 1 : kGatherUnroll];
          float2 szv[kGatherUnroll];
          int vv[kGatherUnroll];
#pragma unroll
          for (int s = 0; s < kGatherUnroll; ++s) {
            const int idx = i0 + s * RPW + lane / LPR;
            vv[s] = idx < n_w ? list[idx] : -1;
            if (vv[s] >= 0) {
              const int v = vv[s];
              const ChunkRows cr = chunk_rows(x, v / kChunk);
              const long long row = ubase + cr.row0 + v % kChunk;
              if constexpr (kOneWidth) {
                ldg_v<VB0>(d.vc[cr.seg] + row * (D * VB0 / 8), d.vsz[cr.seg] + row * ng * 2, j, gi, w0[s], szv[s]);
              } else if (cr.seg == 0) {
                ldg_v<VB0>(d.vc[0] + row * (D * VB0 / 8), d.vsz[0] + row * ng * 2, j, gi, w0[s], szv[s]);
              } else {
                ldg_v<VB1>(d.vc[1] + row * (D * VB1 / 8), d.vsz[1] + row * ng * 2, j, gi, w1[s], szv[s]);
              }
            }
          }
#pragma unroll
          for (int s = 0; s < kGatherUnroll; ++s) {
            const int v = vv[s];
            if (v < 0) continue;
            const int c = v / kChunk;
            float ev[H], w[H];
            load_heads<H>(lgu + (long long)v * H, ev);
#pragma unroll
            for (int h = 0; h < H; ++h) {
              const float p = ev[h] * cfu[c * H + h];
              w[h] = (p < d.tau) ? 0.0f : p;
            }
            if constexpr (kOneWidth) {
              accumulate_v<H, VB0>(w0[s], mg0, szv[s], w, acc, Z);
            } else {
              if (c < x.nc0) accumulate_v<H, VB0>(w0[s], mg0, szv[s], w, acc, Z);
              else accumulate_v<H, VB1>(w1[s], mg1, szv[s], w, acc, Z);
            }
          }
        }
        __syncwarp();
      }
      // fold the per-group constant, reduce the row slots of the warp
#pragma unroll
      for (int h = 0; h < H; ++h)
#pragma unroll
        for (int i = 0; i < 8; ++i) { acc[h][i].x += Z[h]; acc[h][i].y += Z[h]; }
#pragma unroll
      for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
        for (int h = 0; h < H; ++h)
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            acc[h][i].x += __shfl_xor_sync(kFull, acc[h][i].x, off);
            acc[h][i].y += __shfl_xor_sync(kFull, acc[h][i].y, off);
          }
      if (lane < LPR) {
#pragma unroll
        for (int h = 0; h < H; ++h)
#pragma unroll
          for (int i = 0; i < 8; ++i)
            *reinterpret_cast<float2*>(red + (warp * H + h) * D + j * kDimsPerLane + 2 * i) = acc[h][i];
      }
      named_barrier(kBarCons, kConsumers);
      for (int o = tid; o < H * D; o += kConsumers) {
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) s += red[w * H * D + o];
        const int h = o / D, dd = o % D;
        if (x.owned) {
          d.out[((long long)b * d.Hq + g * H + h) * D + dd] = s;
        } else {
          if (e == 0) a.ppart[(((long long)cta * 2 + 0) * H + h) * D + dd] = s;
          if (e == nent - 1) a.ppart[(((long long)cta * 2 + 1) * H + h) * D + dd] = s;
        }
      }
      if (!x.owned) {
        named_barrier(kBarCons, kConsumers);
        if (tid == 0) {
          __threadfence();  // every thread's partial before the arrival
          const int old = atomicAdd(a.arrive2 + x.u, 1);
          s_last = (old == i_last - i_first) ? 1 : 0;
        }
        named_barrier(kBarCons, kConsumers);
        if (s_last) {
          __threadfence();
          for (int o = tid; o < H * D; o += kConsumers) {
            float s = 0.0f;
            for (int i = i_first; i <= i_last; ++i) {
              const int slot = (i == i_first) ? 1 : 0;
              s += __ldcg(a.ppart + (((long long)i * 2 + slot) * H) * D + o);
            }
            const int h = o / D, dd = o % D;
            d.out[((long long)b * d.Hq + g * H + h) * D + dd] = s;
          }
          if (tid == 0) {
            a.arrive1[x.u] = 0;
            a.arrive2[x.u] = 0;
          }
        }
      }
      named_barrier(kBarCons, kConsumers);
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
  named_barrier(kBarCons, kConsumers);
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
