// quantize.cu -- bf16 K/V rows to packed low-bit codes plus (scale, zero).
//
// Asymmetric min-max quantization per group of G head_dim channels
// ("Super KV Compression", §第一层：自适应非对称量化; "TurboQuant",
// §TurboQuant的核心创新: asymmetric and group-wise).  The kernel is bound by
// HBM traffic (2*D bytes in, D*bits/8 + 8*D/G bytes out per row and tensor),
// so it streams rows with 16-byte vector loads and keeps everything else in
// registers: one lane quantizes 32 channels (16 in the repack and append
// kernels), the lanes of a group share their min/max by warp shuffles, and
// each lane packs its codes and stores them itself.
#include <algorithm>

#include "lkv_kernels.cuh"

namespace lkv {

// Streaming 16-byte load that does not keep the line in L1 (each bf16 row is
// read exactly once).
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// The 16 bf16 channels [16j, 16j + 16) of one row of K and of V, in flight.
struct LaneRows {
  uint4 k0, k1, v0, v1;
};

__device__ __forceinline__ void fetch_lane_rows(const uint16_t* k, const uint16_t* v, LaneRows& r) {
  r.k0 = ld_stream(k); r.k1 = ld_stream(k + 8);
  r.v0 = ld_stream(v); r.v1 = ld_stream(v + 8);
}

// Quantize one lane's 16 channels of a row (raw bf16 words w0, w1) and store
// its codes and, for the group's first lane, the (scale, zero) pair.
template <int BITS>
__device__ __forceinline__ void quantize_lane(const uint4& w0, const uint4& w1, uint8_t* __restrict__ codes,
                                              float* __restrict__ sz, int j, int lpg, unsigned mask, float one) {
  if constexpr (BITS == 16) {  // passthrough width: the bf16 values themselves, no (scale, zero)
    *reinterpret_cast<uint4*>(codes + j * 32) = w0;
    *reinterpret_cast<uint4*>(codes + j * 32 + 16) = w1;
  } else {
    const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    LaneWords<BITS> lw;
    float scale, zero;
    quantize16<BITS>(w, lpg, mask, one, lw, scale, zero);
    store_lane_words<BITS>(codes + j * (2 * BITS), lw);
    if (j % lpg == 0) *reinterpret_cast<float2*>(sz + 2 * (j / lpg)) = make_float2(scale, zero);
  }
}

// ------------------------------------------------------------ 32 channels per lane
// The full-cache quantizer gives each lane 32 channels (two 16-channel
// slices): the per-lane work of a group -- min/max, the two divisions, the
// group shuffles -- is shared by twice as many values, and for G = 32 a lane
// holds a whole group.

constexpr int kLaneDims32 = 32;

struct LaneRows32 {
  uint4 k[4], v[4];
};

__device__ __forceinline__ void fetch_lane_rows32(const uint16_t* k, const uint16_t* v, LaneRows32& r) {
#pragma unroll
  for (int i = 0; i < 4; ++i) r.k[i] = ld_stream(k + 8 * i);
#pragma unroll
  for (int i = 0; i < 4; ++i) r.v[i] = ld_stream(v + 8 * i);
}

// Magic-rounded codes rb[i] = 0x4B400000 + code_i for 32 codes, packed LSB
// first into BITS words (see pack16_magic).
template <int BITS>
constexpr uint32_t magic_pack_const32(int wi) {
  uint32_t c = 0u;
  for (int i = 0; i < 32; ++i) {
    const int bit = i * BITS;
    if ((bit >> 5) == wi) c -= 0x4B400000u << (bit & 31);
  }
  return c;
}

template <int BITS>
__device__ __forceinline__ void pack32_magic(const uint32_t (&rb)[32], uint32_t (&out)[BITS]) {
  constexpr uint32_t mask = (1u << BITS) - 1u;
#pragma unroll
  for (int wi = 0; wi < BITS; ++wi) {
    uint32_t acc = magic_pack_const32<BITS>(wi);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int bit = i * BITS, w0 = bit >> 5, pos = bit & 31;
      if (w0 == wi) acc += rb[i] << pos;
      else if (w0 + 1 == wi && pos + BITS > 32) acc += (rb[i] & mask) >> (32 - pos);
    }
    out[wi] = acc;
  }
}

template <int BITS>
__device__ __forceinline__ void pack32(const uint32_t (&c)[32], uint32_t (&out)[BITS]) {
#pragma unroll
  for (int i = 0; i < BITS; ++i) out[i] = 0u;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int bit = i * BITS, wi = bit >> 5, pos = bit & 31;
    out[wi] |= c[i] << pos;
    if (pos + BITS > 32) out[wi + 1] |= c[i] >> (32 - pos);
  }
}

// quantize16 for 32 values (16 raw bf16 words); LPG = G / 32 lanes share a
// group.  The same fixed fp32 formula, the same two paths.
template <int BITS, int LPG>
__device__ __forceinline__ void quantize32(const uint32_t (&w)[16], unsigned mask, float one, uint32_t (&out)[BITS],
                                           float& scale, float& zero) {
  __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&w[0]), hi = lo;
#pragma unroll
  for (int i = 1; i < 16; ++i) {
    const __nv_bfloat162 p = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
    lo = __hmin2(lo, p);
    hi = __hmax2(hi, p);
  }
  float mn = fminf(__low2float(lo), __high2float(lo));
  float mx = fmaxf(__low2float(hi), __high2float(hi));
#pragma unroll
  for (int off = 1; off < LPG; off <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(mask, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(mask, mx, off));
  }
  constexpr uint32_t cmask = (1u << BITS) - 1u;
  const float qmax = static_cast<float>(cmask);
  const float d = __fsub_rn(mx, mn);
  float inv = 0.0f;
  scale = 0.0f;
  if (d != 0.0f) {
    scale = __fdiv_rn(d, qmax);
    inv = __fdiv_rn(qmax, d);
  }
  zero = __fadd_rn(mn, 0.0f);
  if (d <= 3.4028234663852886e38f && inv <= 3.4028234663852886e38f) {
    const __nv_bfloat162 mn_b = __floats2bfloat162_rn(mn, mn);
    const float2 nmn = make_float2(-mn, -mn), inv2 = make_float2(inv, inv), one2 = make_float2(one, one);
    const float2 rnd = make_float2(12582912.0f, 12582912.0f);
    uint32_t rb[32];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const __nv_bfloat162 p = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]), mn_b);
      const uint32_t u = *reinterpret_cast<const uint32_t*>(&p);
      const float2 x = make_float2(bf16_lo(u), bf16_hi(u));
      const float2 y = exact_mul2(exact_add2(x, nmn), inv2);
      const float2 r = exact_fma2(y, one2, rnd);  // y rounded half-even (see quantize16)
      rb[2 * i] = __float_as_uint(r.x);
      rb[2 * i + 1] = __float_as_uint(r.y);
    }
    pack32_magic<BITS>(rb, out);
  } else {
    const WideQuant wq = wide_quant_setup(mn, mx, d, qmax, inv, scale);
    uint32_t c[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float x = (i & 1) ? bf16_hi(w[i / 2]) : bf16_lo(w[i / 2]);
      c[i] = wide_quant_code(wq, x, mn, (int)cmask);
    }
    pack32<BITS>(c, out);
  }
}

// Store a lane's BITS words (4 * BITS bytes at a multiple of 4 * BITS).
template <int BITS>
__device__ __forceinline__ void store_words32(uint8_t* p, const uint32_t (&w)[BITS]) {
  if constexpr (BITS % 4 == 0) {
#pragma unroll
    for (int i = 0; i < BITS; i += 4) *reinterpret_cast<uint4*>(p + 4 * i) = make_uint4(w[i], w[i + 1], w[i + 2], w[i + 3]);
  } else {
#pragma unroll
    for (int i = 0; i < BITS; i += 2) *reinterpret_cast<uint2*>(p + 4 * i) = make_uint2(w[i], w[i + 1]);
  }
}

template <int BITS, int LPG>
__device__ __forceinline__ void quantize_lane32(const uint4 (&w4)[4], uint8_t* __restrict__ codes,
                                                float* __restrict__ sz, int j, unsigned mask, float one) {
  if constexpr (BITS == 16) {  // passthrough width: the bf16 values themselves, no (scale, zero)
#pragma unroll
    for (int i = 0; i < 4; ++i) *reinterpret_cast<uint4*>(codes + j * 64 + 16 * i) = w4[i];
  } else {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) { w[4 * i] = w4[i].x; w[4 * i + 1] = w4[i].y; w[4 * i + 2] = w4[i].z; w[4 * i + 3] = w4[i].w; }
    uint32_t out[BITS];
    float scale, zero;
    quantize32<BITS, LPG>(w, mask, one, out, scale, zero);
    store_words32<BITS>(codes + j * (4 * BITS), out);
    if (j % LPG == 0) *reinterpret_cast<float2*>(sz + 2 * (j / LPG)) = make_float2(scale, zero);
  }
}

// Row batches: batch (b, g, tb) covers tokens tb * RPW ... of KV head g of
// sequence b, one row per D/16 lanes.  Warp w of the grid takes batches w,
// w + W, w + 2W, ... in (b, g, tb) order, stepping its coordinates without
// divisions, and issues the next batch's loads before quantizing the current
// one, so two batches of K and V per warp are in flight.
template <int D, int KB, int VB, int LPG>
__global__ void __launch_bounds__(256, 2) quantize_kv_kernel(QuantizeArgs a) {
  constexpr int LPR = D / kLaneDims32;
  constexpr int RPW = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const int j = lane % LPR, sub = lane / LPR;
  const unsigned mask = row_lane_mask<LPR>(lane);
  const int ng = D / a.G;
  const uint32_t nbu = (uint32_t)(a.T_cap + RPW - 1) / RPW;  // batches per (b, g)
  const uint32_t W = gridDim.x * (blockDim.x / 32);
  const uint32_t w0 = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  // position (b, g, tb) of batch w0 and the step W in the same coordinates
  uint32_t tb = w0 % nbu, g = (w0 / nbu) % (uint32_t)a.Hkv, b = (w0 / nbu) / (uint32_t)a.Hkv;
  const uint32_t s_tb = W % nbu, s_g = (W / nbu) % (uint32_t)a.Hkv, s_b = (W / nbu) / (uint32_t)a.Hkv;
  auto step = [&](uint32_t& b_, uint32_t& g_, uint32_t& tb_) {
    tb_ += s_tb;
    uint32_t c = tb_ >= nbu ? 1u : 0u;
    tb_ -= c * nbu;
    g_ += s_g + c;
    c = g_ >= (uint32_t)a.Hkv ? 1u : 0u;
    g_ -= c * (uint32_t)a.Hkv;
    b_ += s_b + c;
  };
  auto fetch = [&](uint32_t b_, uint32_t g_, uint32_t tb_, LaneRows32& r, long long& row) -> bool {
    if (b_ >= (uint32_t)a.B) return false;
    const int t = (int)tb_ * RPW + sub;
    if (t >= clamp_len(__ldg(a.seq_lens + b_), a.T_cap)) return false;
    const long long src = ((long long)b_ * a.Hkv + g_) * a.T_cap + t;
    row = cache_row(a.block_table, a.pages_per_seq, a.num_pages, a.Hkv, a.T_cap, (int)b_, (int)g_, t);
    if (row < 0) return false;  // a page outside the pool: nothing is written
    fetch_lane_rows32(a.k + src * D + j * kLaneDims32, a.v + src * D + j * kLaneDims32, r);
    return true;
  };
  LaneRows32 cur, nxt;
  long long row = 0, row_n = 0;
  bool ok = fetch(b, g, tb, cur, row);
  while (b < (uint32_t)a.B) {
    uint32_t bn = b, gn = g, tbn = tb;
    step(bn, gn, tbn);
    const bool ok_n = fetch(bn, gn, tbn, nxt, row_n);
    // The lanes of one row share `ok`, so the group shuffles inside
    // quantize32 only ever pair lanes that are both active.
    if (ok) {
      quantize_lane32<KB, LPG>(cur.k, a.k_codes + row * (D * KB / 8), a.k_sz + row * ng * 2, j, mask, a.one);
      quantize_lane32<VB, LPG>(cur.v, a.v_codes + row * (D * VB / 8), a.v_sz + row * ng * 2, j, mask, a.one);
    }
    cur = nxt; row = row_n; ok = ok_n;
    b = bn; g = gn; tb = tbn;
  }
}

// Append: the new token of every (b, g) -- bf16 K and V rows [B][Hkv][D] --
// quantized into slot pos[b] of the packed cache, with the formula of
// quantize_kv_kernel (the step just before decode in a decode loop).  A
// position outside [0, T_cap) writes nothing.
template <int D, int KB, int VB>
__global__ void __launch_bounds__(256) append_kv_kernel(QuantizeArgs a) {
  constexpr int LPR = D / kDimsPerLane;
  constexpr int RPW = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const int j = lane % LPR, sub = lane / LPR;
  const unsigned mask = row_lane_mask<LPR>(lane);
  const int ng = D / a.G, lpg = a.G / kDimsPerLane;
  const long long unit = ((long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32) * RPW + sub;
  if (unit >= (long long)a.B * a.Hkv) return;  // the lanes of a row agree
  const int t = __ldg(a.seq_lens + unit / a.Hkv);
  if (t < 0 || t >= a.T_cap) return;
  const long long row = cache_row(a.block_table, a.pages_per_seq, a.num_pages, a.Hkv, a.T_cap,
                                  (int)(unit / a.Hkv), (int)(unit % a.Hkv), t);
  if (row < 0) return;  // a page outside the pool: nothing is written
  LaneRows r;
  fetch_lane_rows(a.k + unit * D + j * kDimsPerLane, a.v + unit * D + j * kDimsPerLane, r);
  quantize_lane<KB>(r.k0, r.k1, a.k_codes + row * (D * KB / 8), a.k_sz + row * ng * 2, j, lpg, mask, a.one);
  quantize_lane<VB>(r.v0, r.v1, a.v_codes + row * (D * VB / 8), a.v_sz + row * ng * 2, j, lpg, mask, a.one);
}

// Tier repack: row i of segment A (tier 2) or B (tier 1) of (b, g) is the
// token at pos[b][g][i], quantized from bf16 with K at 6 bits and V at 6 (A)
// or 4 (B) bits ("Super KV Compression", §第二层 items 1-2).  Block
// (bg * S + s, seg) walks only the n rows that segment seg of unit bg holds,
// S blocks per unit and segment, with the same one-ahead loads as above.
template <int D, int LPG>
__global__ void __launch_bounds__(256, 2) tier_repack_kernel(RepackArgs a, int S) {
  constexpr int LPR = D / kLaneDims32;
  constexpr int RPW = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const int j = lane % LPR, sub = lane / LPR;
  const unsigned mask = row_lane_mask<LPR>(lane);
  const int ng = D / a.G;
  const int seg = blockIdx.y;  // 0: segment A, 1: segment B
  const long long bg = blockIdx.x / S;
  const int s = blockIdx.x % S;
  const int n = clamp_len(a.counts[2 * bg + seg], a.T_cap);
  const int32_t* pos = (seg == 0 ? a.pos_a : a.pos_b) + bg * a.T_cap;
  const int nw = blockDim.x / 32;
  const int stride = S * nw * RPW;
  auto fetch = [&](int i, LaneRows32& r) -> bool {
    if (i >= n) return false;
    int t = __ldg(pos + i);
    t = t < 0 ? 0 : (t >= a.T_cap ? a.T_cap - 1 : t);
    const long long src = bg * a.T_cap + t;
    fetch_lane_rows32(a.k + src * D + j * kLaneDims32, a.v + src * D + j * kLaneDims32, r);
    return true;
  };
  int i = (s * nw + (int)threadIdx.x / 32) * RPW + sub;
  LaneRows32 cur, nxt;
  bool ok = fetch(i, cur);
  for (; i - sub < n; i += stride) {
    const bool ok_n = fetch(i + stride, nxt);
    if (ok) {
      const long long slot = bg * a.T_cap + i;
      if (seg == 0) {
        quantize_lane32<6, LPG>(cur.k, a.a_kc + slot * (D * 6 / 8), a.a_ksz + slot * ng * 2, j, mask, a.one);
        quantize_lane32<6, LPG>(cur.v, a.a_vc + slot * (D * 6 / 8), a.a_vsz + slot * ng * 2, j, mask, a.one);
      } else {
        quantize_lane32<6, LPG>(cur.k, a.b_kc + slot * (D * 6 / 8), a.b_ksz + slot * ng * 2, j, mask, a.one);
        quantize_lane32<4, LPG>(cur.v, a.b_vc + slot * (D * 4 / 8), a.b_vsz + slot * ng * 2, j, mask, a.one);
      }
    }
    cur = nxt; ok = ok_n;
  }
}

// The same repack over a grid of resident blocks, with the rows of every
// (segment, unit) pair laid end to end (segment A's units, then segment B's)
// and dealt out evenly, so that a unit's short segment A and long segment B
// cost the same per row.  Each block rebuilds the pairs' first rows in shared
// memory from the clamped counts.
constexpr int kRepackMaxPairs = 8192;

template <int D, int LPG>
__global__ void __launch_bounds__(256, 2) tier_repack_flat_kernel(RepackArgs a) {
  constexpr int LPR = D / kLaneDims32;
  constexpr int RPW = 32 / LPR;
  extern __shared__ int s_first[];  // [pairs + 1]: first row of pair p = seg * units + unit, then the total
  __shared__ int s_wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x / 32;
  const int j = lane % LPR, sub = lane / LPR;
  const unsigned mask = row_lane_mask<LPR>(lane);
  const int ng = D / a.G;
  const int units = a.B * a.Hkv, pairs = 2 * units;
  auto rows_of = [&](int p) { return clamp_len(a.counts[2 * (p % units) + p / units], a.T_cap); };
  // exclusive scan of the pairs' row counts: a run of pairs per thread
  const int per = (pairs + (int)blockDim.x - 1) / (int)blockDim.x;
  const int p0 = min(pairs, tid * per), p1 = min(pairs, p0 + per);
  int mine = 0;
  for (int p = p0; p < p1; ++p) mine += rows_of(p);
  int incl = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) s_wsum[warp] = incl;
  __syncthreads();
  int run = incl - mine;
  for (int w = 0; w < warp; ++w) run += s_wsum[w];
  for (int p = p0; p < p1; ++p) { s_first[p] = run; run += rows_of(p); }
  if (tid == (int)blockDim.x - 1) s_first[pairs] = run;  // the last thread's inclusive prefix: every row
  __syncthreads();
  const int total = s_first[pairs];
  // Row r: its pair (segment, unit) is the last whose first row is <= r
  // (empty pairs are passed over), its slot in the segment, and where its
  // position lives.  The position is loaded two rows ahead of use and the
  // bf16 rows one ahead, so the two dependent loads of a row never meet on
  // the critical path.
  struct Loc {
    bool ok;
    int seg;
    long long bg, slot;
    int t;  // position (loaded ahead)
  };
  auto locate = [&](int r) {
    Loc l{false, 0, 0, 0, 0};
    if (r >= total) return l;
    int lo = 0, hi = pairs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_first[mid] <= r) lo = mid; else hi = mid - 1;
    }
    l.ok = true;
    l.seg = lo / units;
    l.bg = lo % units;
    const int i = r - s_first[lo];
    l.slot = l.bg * a.T_cap + i;
    l.t = __ldg((l.seg == 0 ? a.pos_a : a.pos_b) + l.slot);
    return l;
  };
  auto fetch = [&](const Loc& l, LaneRows32& x) {
    if (!l.ok) return;
    const int t = l.t < 0 ? 0 : (l.t >= a.T_cap ? a.T_cap - 1 : l.t);
    const long long src = l.bg * a.T_cap + t;
    fetch_lane_rows32(a.k + src * D + j * kLaneDims32, a.v + src * D + j * kLaneDims32, x);
  };
  const int stride = (int)gridDim.x * nw * RPW;
  int r = ((int)blockIdx.x * nw + warp) * RPW + sub;
  LaneRows32 cur, nxt;
  Loc l0 = locate(r), l1 = locate(r + stride);
  fetch(l0, cur);
  for (; r - sub < total; r += stride) {  // r - sub is the same for the whole warp
    const Loc l2 = locate(r + 2 * stride);
    fetch(l1, nxt);
    if (l0.ok) {
      const long long slot = l0.slot;
      if (l0.seg == 0) {
        quantize_lane32<6, LPG>(cur.k, a.a_kc + slot * (D * 6 / 8), a.a_ksz + slot * ng * 2, j, mask, a.one);
        quantize_lane32<6, LPG>(cur.v, a.a_vc + slot * (D * 6 / 8), a.a_vsz + slot * ng * 2, j, mask, a.one);
      } else {
        quantize_lane32<6, LPG>(cur.k, a.b_kc + slot * (D * 6 / 8), a.b_ksz + slot * ng * 2, j, mask, a.one);
        quantize_lane32<4, LPG>(cur.v, a.b_vc + slot * (D * 4 / 8), a.b_vsz + slot * ng * 2, j, mask, a.one);
      }
    }
    cur = nxt; l0 = l1; l1 = l2;
  }
}

// Resident blocks of 256 threads per SM for a kernel (cached per kernel and
// device by the caller's static).
static int resident_blocks(const void* kern) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 256, 0) != cudaSuccess || n < 1) n = 1;
  return n;
}

template <int D, int KB, int VB, int LPG>
static cudaError_t launch_quantize_g(const QuantizeArgs& a, cudaStream_t s) {
  constexpr int RPW = 32 / (D / kLaneDims32);
  static int per_sm[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (per_sm[dev] == 0) per_sm[dev] = resident_blocks((const void*)quantize_kv_kernel<D, KB, VB, LPG>);
  const long long n_batches = (long long)a.B * a.Hkv * ((a.T_cap + RPW - 1) / RPW);
  if (n_batches >= (1ll << 31)) return cudaErrorInvalidValue;
  long long blocks = std::min<long long>((long long)num_sms() * per_sm[dev], (n_batches + 7) / 8);
  quantize_kv_kernel<D, KB, VB, LPG><<<(int)std::max<long long>(blocks, 1), 256, 0, s>>>(a);
  return cudaGetLastError();
}

template <int D, int KB, int VB>
static cudaError_t launch_quantize_t(const QuantizeArgs& a, cudaStream_t s) {
  // lanes per group: G / 32 (groups never exceed D)
  if (a.G == 32) return launch_quantize_g<D, KB, VB, 1>(a, s);
  if (a.G == 64) return launch_quantize_g<D, KB, VB, 2>(a, s);
  if constexpr (D >= 128) return launch_quantize_g<D, KB, VB, 4>(a, s);
  return cudaErrorInvalidValue;
}

template <int D, int KB, int VB>
static cudaError_t launch_append_t(const QuantizeArgs& a, cudaStream_t s) {
  constexpr int RPW = 32 / (D / kDimsPerLane);
  const long long units = (long long)a.B * a.Hkv;
  const long long blocks = (units + 8 * RPW - 1) / (8 * RPW);
  if (blocks >= (1ll << 31)) return cudaErrorInvalidValue;
  append_kv_kernel<D, KB, VB><<<(unsigned)blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

template <int D, int KB>
static cudaError_t launch_quantize_vb(const QuantizeArgs& a, int vb, bool append, cudaStream_t s) {
  switch (vb) {
    case 2: return append ? launch_append_t<D, KB, 2>(a, s) : launch_quantize_t<D, KB, 2>(a, s);
    case 4: return append ? launch_append_t<D, KB, 4>(a, s) : launch_quantize_t<D, KB, 4>(a, s);
    case 6: return append ? launch_append_t<D, KB, 6>(a, s) : launch_quantize_t<D, KB, 6>(a, s);
    case 8: return append ? launch_append_t<D, KB, 8>(a, s) : launch_quantize_t<D, KB, 8>(a, s);
    case 16: return append ? launch_append_t<D, KB, 16>(a, s) : launch_quantize_t<D, KB, 16>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
static cudaError_t launch_quantize_d(const QuantizeArgs& a, int kb, int vb, bool append, cudaStream_t s) {
  switch (kb) {
    case 2: return launch_quantize_vb<D, 2>(a, vb, append, s);
    case 4: return launch_quantize_vb<D, 4>(a, vb, append, s);
    case 6: return launch_quantize_vb<D, 6>(a, vb, append, s);
    case 8: return launch_quantize_vb<D, 8>(a, vb, append, s);
    case 16: return launch_quantize_vb<D, 16>(a, vb, append, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_quantize_kv(const QuantizeArgs& a, int kb, int vb, int D, cudaStream_t s) {
  const long long n_rows = (long long)a.B * a.Hkv * a.T_cap;
  if (n_rows == 0) return cudaSuccess;
  if (D == 64) return launch_quantize_d<64>(a, kb, vb, false, s);
  if (D == 128) return launch_quantize_d<128>(a, kb, vb, false, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_append_kv(const QuantizeArgs& a, int kb, int vb, int D, cudaStream_t s) {
  if ((long long)a.B * a.Hkv * a.T_cap == 0) return cudaSuccess;
  if (D == 64) return launch_quantize_d<64>(a, kb, vb, true, s);
  if (D == 128) return launch_quantize_d<128>(a, kb, vb, true, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_tier_repack(const RepackArgs& a, int D, cudaStream_t s) {
  const long long units = (long long)a.B * a.Hkv;
  if (units == 0 || a.T_cap == 0) return cudaSuccess;
  if (2 * units <= kRepackMaxPairs && 2 * units * a.T_cap < (1ll << 30)) {
    const dim3 grid((unsigned)(num_sms() * 2));
    const size_t smem = (size_t)(2 * units + 1) * sizeof(int);
    if (D == 64 && a.G == 32) tier_repack_flat_kernel<64, 1><<<grid, 256, smem, s>>>(a);
    else if (D == 64 && a.G == 64) tier_repack_flat_kernel<64, 2><<<grid, 256, smem, s>>>(a);
    else if (D == 128 && a.G == 32) tier_repack_flat_kernel<128, 1><<<grid, 256, smem, s>>>(a);
    else if (D == 128 && a.G == 64) tier_repack_flat_kernel<128, 2><<<grid, 256, smem, s>>>(a);
    else if (D == 128 && a.G == 128) tier_repack_flat_kernel<128, 4><<<grid, 256, smem, s>>>(a);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
  }
  // about eight blocks per SM over both segments, at least one per unit
  const long long want = (long long)num_sms() * 8;
  const int S = (int)std::max<long long>(1, std::min<long long>(64, want / (2 * units)));
  if (units * S >= (1ll << 31)) return cudaErrorInvalidValue;
  dim3 grid((unsigned)(units * S), 2);
  if (D == 64 && a.G == 32) tier_repack_kernel<64, 1><<<grid, 256, 0, s>>>(a, S);
  else if (D == 64 && a.G == 64) tier_repack_kernel<64, 2><<<grid, 256, 0, s>>>(a, S);
  else if (D == 128 && a.G == 32) tier_repack_kernel<128, 1><<<grid, 256, 0, s>>>(a, S);
  else if (D == 128 && a.G == 64) tier_repack_kernel<128, 2><<<grid, 256, 0, s>>>(a, S);
  else if (D == 128 && a.G == 128) tier_repack_kernel<128, 4><<<grid, 256, 0, s>>>(a, S);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace lkv
