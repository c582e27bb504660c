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
  const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
  LaneWords<BITS> lw;
  float scale, zero;
  quantize16<BITS>(w, lpg, mask, one, lw, scale, zero);
  store_lane_words<BITS>(codes + j * (2 * BITS), lw);
  if (j % lpg == 0) *reinterpret_cast<float2*>(sz + 2 * (j / lpg)) = make_float2(scale, zero);
}

// Row batches: batch (b, g, tb) covers tokens tb * RPW ... of KV head g of
// sequence b, one row per D/16 lanes.  Warp w of the grid takes batches w,
// w + W, w + 2W, ... in (b, g, tb) order, stepping its coordinates without
// divisions, and issues the next batch's loads before quantizing the current
// one, so two batches of K and V per warp are in flight.
template <int D, int KB, int VB>
__global__ void __launch_bounds__(256, 4) quantize_kv_kernel(QuantizeArgs a) {
  constexpr int LPR = D / kDimsPerLane;
  constexpr int RPW = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const int j = lane % LPR, sub = lane / LPR;
  const unsigned mask = row_lane_mask<LPR>(lane);
  const int ng = D / a.G, lpg = a.G / kDimsPerLane;
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
  auto fetch = [&](uint32_t b_, uint32_t g_, uint32_t tb_, LaneRows& r, long long& row) -> bool {
    if (b_ >= (uint32_t)a.B) return false;
    const int t = (int)tb_ * RPW + sub;
    if (t >= clamp_len(__ldg(a.seq_lens + b_), a.T_cap)) return false;
    row = ((long long)b_ * a.Hkv + g_) * a.T_cap + t;
    fetch_lane_rows(a.k + row * D + j * kDimsPerLane, a.v + row * D + j * kDimsPerLane, r);
    return true;
  };
  LaneRows cur, nxt;
  long long row = 0, row_n = 0;
  bool ok = fetch(b, g, tb, cur, row);
  while (b < (uint32_t)a.B) {
    uint32_t bn = b, gn = g, tbn = tb;
    step(bn, gn, tbn);
    const bool ok_n = fetch(bn, gn, tbn, nxt, row_n);
    // The lanes of one row share `ok`, so the group shuffles inside
    // quantize16 only ever pair lanes that are both active.
    if (ok) {
      quantize_lane<KB>(cur.k0, cur.k1, a.k_codes + row * (D * KB / 8), a.k_sz + row * ng * 2, j, lpg, mask, a.one);
      quantize_lane<VB>(cur.v0, cur.v1, a.v_codes + row * (D * VB / 8), a.v_sz + row * ng * 2, j, lpg, mask, a.one);
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
  const long long row = unit * a.T_cap + t;
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
template <int D>
__global__ void __launch_bounds__(256, 4) tier_repack_kernel(RepackArgs a, int S) {
  constexpr int LPR = D / kDimsPerLane;
  constexpr int RPW = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const int j = lane % LPR, sub = lane / LPR;
  const unsigned mask = row_lane_mask<LPR>(lane);
  const int ng = D / a.G, lpg = a.G / kDimsPerLane;
  const int seg = blockIdx.y;  // 0: segment A, 1: segment B
  const long long bg = blockIdx.x / S;
  const int s = blockIdx.x % S;
  const int n = clamp_len(a.counts[2 * bg + seg], a.T_cap);
  const int32_t* pos = (seg == 0 ? a.pos_a : a.pos_b) + bg * a.T_cap;
  const int nw = blockDim.x / 32;
  const int stride = S * nw * RPW;
  auto fetch = [&](int i, LaneRows& r) -> bool {
    if (i >= n) return false;
    int t = __ldg(pos + i);
    t = t < 0 ? 0 : (t >= a.T_cap ? a.T_cap - 1 : t);
    const long long src = bg * a.T_cap + t;
    fetch_lane_rows(a.k + src * D + j * kDimsPerLane, a.v + src * D + j * kDimsPerLane, r);
    return true;
  };
  int i = (s * nw + (int)threadIdx.x / 32) * RPW + sub;
  LaneRows cur, nxt;
  bool ok = fetch(i, cur);
  for (; i - sub < n; i += stride) {
    const bool ok_n = fetch(i + stride, nxt);
    if (ok) {
      const long long slot = bg * a.T_cap + i;
      if (seg == 0) {
        quantize_lane<6>(cur.k0, cur.k1, a.a_kc + slot * (D * 6 / 8), a.a_ksz + slot * ng * 2, j, lpg, mask, a.one);
        quantize_lane<6>(cur.v0, cur.v1, a.a_vc + slot * (D * 6 / 8), a.a_vsz + slot * ng * 2, j, lpg, mask, a.one);
      } else {
        quantize_lane<6>(cur.k0, cur.k1, a.b_kc + slot * (D * 6 / 8), a.b_ksz + slot * ng * 2, j, lpg, mask, a.one);
        quantize_lane<4>(cur.v0, cur.v1, a.b_vc + slot * (D * 4 / 8), a.b_vsz + slot * ng * 2, j, lpg, mask, a.one);
      }
    }
    cur = nxt; ok = ok_n;
  }
}

// Resident blocks of 256 threads per SM for a kernel (cached per kernel and
// device by the caller's static).
static int resident_blocks(const void* kern) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 256, 0) != cudaSuccess || n < 1) n = 1;
  return n;
}

template <int D, int KB, int VB>
static cudaError_t launch_quantize_t(const QuantizeArgs& a, cudaStream_t s) {
  constexpr int RPW = 32 / (D / kDimsPerLane);
  static int per_sm[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (per_sm[dev] == 0) per_sm[dev] = resident_blocks((const void*)quantize_kv_kernel<D, KB, VB>);
  const long long n_batches = (long long)a.B * a.Hkv * ((a.T_cap + RPW - 1) / RPW);
  if (n_batches >= (1ll << 31)) return cudaErrorInvalidValue;
  long long blocks = std::min<long long>((long long)num_sms() * per_sm[dev], (n_batches + 7) / 8);
  quantize_kv_kernel<D, KB, VB><<<(int)std::max<long long>(blocks, 1), 256, 0, s>>>(a);
  return cudaGetLastError();
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
  // about eight blocks per SM over both segments, at least one per unit
  const long long want = (long long)num_sms() * 8;
  const int S = (int)std::max<long long>(1, std::min<long long>(64, want / (2 * units)));
  if (units * S >= (1ll << 31)) return cudaErrorInvalidValue;
  dim3 grid((unsigned)(units * S), 2);
  if (D == 64) tier_repack_kernel<64><<<grid, 256, 0, s>>>(a, S);
  else if (D == 128) tier_repack_kernel<128><<<grid, 256, 0, s>>>(a, S);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace lkv
