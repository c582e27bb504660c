// lkv_device.cuh -- device-side building blocks shared by the liblkv kernels.
//
// Packed row format (the contract of include/lkv.h): code j of a token row
// occupies bits [j*BITS, (j+1)*BITS) of the row read as one little-endian
// bit string; each (scale, zero) pair covers G contiguous channels.
//
// Lane mapping used by every kernel: a token row of D channels is handled by
// D/16 consecutive lanes, lane j owning channels [16j, 16j+16).  Those 16
// codes take 2*BITS bytes, always a whole number of 32-bit words at a 4-byte
// aligned offset, and they lie inside one quantization group (G >= 32).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace lkv {

constexpr int kDimsPerLane = 16;

// Status values written to the workspace status word (mirror of lkv_status).
constexpr int kStatusInvalidArg = 1;
constexpr int kStatusTimeout = 5;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ int clamp_len(int32_t t, int T_cap) {
  return t < 0 ? 0 : (t > T_cap ? T_cap : t);
}

// Words of one lane's 16 codes.
template <int BITS>
struct LaneWords {
  static constexpr int N = BITS / 2;  // 16 * BITS / 32
  uint32_t w[N];
};

template <int BITS>
__device__ __forceinline__ void load_lane_words(const uint8_t* __restrict__ p, LaneWords<BITS>& lw) {
  // p is 4-byte aligned; 8- and 16-byte alignment hold for 4- and 8-bit rows.
  if constexpr (BITS == 8) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    lw.w[0] = v.x; lw.w[1] = v.y; lw.w[2] = v.z; lw.w[3] = v.w;
  } else if constexpr (BITS == 4) {
    uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    lw.w[0] = v.x; lw.w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < LaneWords<BITS>::N; ++i) lw.w[i] = __ldg(reinterpret_cast<const uint32_t*>(p) + i);
  }
}

// Code i (0..15) of the lane, as an integer.
template <int BITS>
__device__ __forceinline__ uint32_t lane_code(const LaneWords<BITS>& lw, int i) {
  constexpr uint32_t mask = (1u << BITS) - 1u;
  const int bit = i * BITS, wi = bit >> 5, pos = bit & 31;
  if (pos + BITS <= 32) return (lw.w[wi] >> pos) & mask;
  return __funnelshift_r(lw.w[wi], lw.w[wi + 1], pos) & mask;
}

// Code i as the float 1 + code / 2^BITS, built exactly by placing the code in
// the top mantissa bits of 1.0f.  The constant 1 is folded out by callers.
template <int BITS>
__device__ __forceinline__ float lane_code_f(const LaneWords<BITS>& lw, int i) {
  return __uint_as_float(0x3F800000u | (lane_code<BITS>(lw, i) << (23 - BITS)));
}

template <int BITS>
__device__ __forceinline__ void unpack16_f(const LaneWords<BITS>& lw, float2 (&f)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = make_float2(lane_code_f<BITS>(lw, 2 * i), lane_code_f<BITS>(lw, 2 * i + 1));
}

// Pack 16 codes into the lane's words.
template <int BITS>
__device__ __forceinline__ void pack16(const uint32_t (&c)[16], LaneWords<BITS>& lw) {
#pragma unroll
  for (int i = 0; i < LaneWords<BITS>::N; ++i) lw.w[i] = 0u;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int bit = i * BITS, wi = bit >> 5, pos = bit & 31;
    lw.w[wi] |= c[i] << pos;
    if (pos + BITS > 32) lw.w[wi + 1] |= c[i] >> (32 - pos);
  }
}

template <int BITS>
__device__ __forceinline__ void store_lane_words(uint8_t* p, const LaneWords<BITS>& lw) {
  if constexpr (BITS == 8) {
    *reinterpret_cast<uint4*>(p) = make_uint4(lw.w[0], lw.w[1], lw.w[2], lw.w[3]);
  } else if constexpr (BITS == 4) {
    *reinterpret_cast<uint2*>(p) = make_uint2(lw.w[0], lw.w[1]);
  } else {
#pragma unroll
    for (int i = 0; i < LaneWords<BITS>::N; ++i) reinterpret_cast<uint32_t*>(p)[i] = lw.w[i];
  }
}

// Quantize the 16 values a lane holds, sharing min/max with the other lanes
// of its group (LPG = G / 16 consecutive lanes).  The formula is the fixed
// fp32 one of lkv_quantize_kv, every operation rounded separately.
// `mask` names the lanes of the calling row (all of them take this call).
template <int BITS>
__device__ __forceinline__ void quantize16(const float (&x)[16], int lpg, unsigned mask, uint32_t (&c)[16],
                                           float& scale, float& zero) {
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int i = 1; i < 16; ++i) { mn = fminf(mn, x[i]); mx = fmaxf(mx, x[i]); }
  for (int off = 1; off < lpg; off <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(mask, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(mask, mx, off));
  }
  const float qmax = static_cast<float>((1u << BITS) - 1u);
  const float d = __fsub_rn(mx, mn);
  float inv = 0.0f;
  scale = 0.0f;
  if (d != 0.0f) {
    scale = __fdiv_rn(d, qmax);
    inv = __fdiv_rn(qmax, d);
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float y = __fmul_rn(__fsub_rn(x[i], mn), inv);
    int ci = __float2int_rn(y);
    ci = ci < 0 ? 0 : ci;
    ci = ci > (int)((1u << BITS) - 1u) ? (int)((1u << BITS) - 1u) : ci;
    c[i] = static_cast<uint32_t>(ci);
  }
  zero = __fadd_rn(mn, 0.0f);
}

// Load 16 bf16 values (32 bytes, 32-byte aligned) as floats.
__device__ __forceinline__ void load16_bf16(const uint16_t* __restrict__ p, float (&x)[16]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
  uint4 a = __ldg(q), b = __ldg(q + 1);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) { x[2 * i] = bf16_lo(w[i]); x[2 * i + 1] = bf16_hi(w[i]); }
}

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// Lanes of the row that lane `lane` belongs to, LPR consecutive lanes per row.
template <int LPR>
__device__ __forceinline__ unsigned row_lane_mask(int lane) {
  constexpr unsigned m = LPR == 32 ? 0xFFFFFFFFu : ((1u << LPR) - 1u);
  return m << ((lane / LPR) * LPR);
}

}  // namespace lkv
