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

// Paged caches: a page holds kPageTokens consecutive tokens of one KV head;
// the pool is [num_pages][Hkv][kPageTokens][row], and block_table[b][i] is the
// page of tokens [i * kPageTokens, (i + 1) * kPageTokens) of sequence b.
constexpr int kPageTokens = 256;

// Physical row of token t of KV head g of sequence b: the contiguous cache
// row (b * Hkv + g) * T_cap + t, or its slot in the page that the block
// table names.  A page id outside [0, num_pages) gives -1.
__device__ __forceinline__ long long cache_row(const int32_t* block_table, int pages_per_seq, int num_pages,
                                               int Hkv, int T_cap, int b, int g, int t) {
  if (block_table == nullptr) return ((long long)b * Hkv + g) * T_cap + t;
  const int page = __ldg(block_table + (long long)b * pages_per_seq + t / kPageTokens);
  if (page < 0 || page >= num_pages) return -1;
  return ((long long)page * Hkv + g) * kPageTokens + (t % kPageTokens);
}

// Words of one lane's 16 codes.
template <int BITS>
struct LaneWords {
  static constexpr int N = BITS / 2;  // 16 * BITS / 32
  uint32_t w[N];
};

template <int BITS>
__device__ __forceinline__ void load_lane_words(const uint8_t* __restrict__ p, LaneWords<BITS>& lw) {
  // p is 4-byte aligned; 8- and 16-byte alignment hold for 4-, 8- and 16-bit rows.
  if constexpr (BITS == 16) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p)), u = __ldg(reinterpret_cast<const uint4*>(p) + 1);
    lw.w[0] = v.x; lw.w[1] = v.y; lw.w[2] = v.z; lw.w[3] = v.w;
    lw.w[4] = u.x; lw.w[5] = u.y; lw.w[6] = u.z; lw.w[7] = u.w;
  } else if constexpr (BITS == 8) {
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
  if constexpr (BITS == 16) {
    *reinterpret_cast<uint4*>(p) = make_uint4(lw.w[0], lw.w[1], lw.w[2], lw.w[3]);
    *reinterpret_cast<uint4*>(p + 16) = make_uint4(lw.w[4], lw.w[5], lw.w[6], lw.w[7]);
  } else if constexpr (BITS == 8) {
    *reinterpret_cast<uint4*>(p) = make_uint4(lw.w[0], lw.w[1], lw.w[2], lw.w[3]);
  } else if constexpr (BITS == 4) {
    *reinterpret_cast<uint2*>(p) = make_uint2(lw.w[0], lw.w[1]);
  } else {
#pragma unroll
    for (int i = 0; i < LaneWords<BITS>::N; ++i) reinterpret_cast<uint32_t*>(p)[i] = lw.w[i];
  }
}

// Packed fp32 add and multiply, each rounded to nearest even, written as PTX
// so that the compiler front end cannot reassociate them.  A multiply whose
// result feeds an add directly may still be contracted by the code generator;
// callers that need the product rounded separately put another operation
// between the two.
__device__ __forceinline__ uint64_t pack_f2(float2 a) {
  return ((uint64_t)__float_as_uint(a.y) << 32) | __float_as_uint(a.x);
}
__device__ __forceinline__ float2 unpack_f2(uint64_t r) {
  return make_float2(__uint_as_float((uint32_t)r), __uint_as_float((uint32_t)(r >> 32)));
}
__device__ __forceinline__ float2 exact_add2(float2 a, float2 b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pack_f2(a)), "l"(pack_f2(b)));
  return unpack_f2(r);
}
__device__ __forceinline__ float2 exact_mul2(float2 a, float2 b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pack_f2(a)), "l"(pack_f2(b)));
  return unpack_f2(r);
}

__device__ __forceinline__ float2 exact_fma2(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(pack_f2(a)), "l"(pack_f2(b)), "l"(pack_f2(c)));
  return unpack_f2(r);
}

// Magic-rounded codes: rb[i] = 0x4B400000 + code_i (the bits of 1.5 * 2^23 +
// code).  Packs them LSB first without masking: adding rb << pos for every
// code of a word and one constant that cancels the 0x4B400000 << pos terms
// (mod 2^32) leaves exactly the OR of code << pos.
template <int BITS>
constexpr uint32_t magic_pack_const(int wi) {
  uint32_t c = 0u;
  for (int i = 0; i < 16; ++i) {
    const int bit = i * BITS;
    if ((bit >> 5) == wi) c -= 0x4B400000u << (bit & 31);
  }
  return c;
}

template <int BITS>
__device__ __forceinline__ void pack16_magic(const uint32_t (&rb)[16], LaneWords<BITS>& lw) {
  constexpr uint32_t mask = (1u << BITS) - 1u;
#pragma unroll
  for (int wi = 0; wi < LaneWords<BITS>::N; ++wi) {
    uint32_t acc = magic_pack_const<BITS>(wi);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int bit = i * BITS, w0 = bit >> 5, pos = bit & 31;
      if (w0 == wi) acc += rb[i] << pos;
      else if (w0 + 1 == wi && pos + BITS > 32) acc += (rb[i] & mask) >> (32 - pos);
    }
    lw.w[wi] = acc;
  }
}

// The scalar path of the group quantizer for the two ranges of finite
// values whose formula leaves fp32 (each step rounded on its own):
//   tiny d, qmax / d overflowing: inv = qmax / (d * 2^64),
//     code = rint(((x - mn) * 2^64) * inv), scale = d / qmax unchanged;
//   huge d, mx - mn overflowing: dh = mx/2 - mn/2, inv = qmax / dh,
//     code = rint((x/2 - mn/2) * inv), scale = (dh / qmax) * 2.
// Every other group (and a NaN d) keeps code = rint((x - mn) * inv).
// Codes are clamped to [0, qmax]; a NaN code is 0.
struct WideQuant {
  int mode;   // 0: plain, 1: tiny d, 2: huge d
  float mnh;  // mn / 2 (mode 2)
  float inv;
};

__device__ __forceinline__ WideQuant wide_quant_setup(float mn, float mx, float d, float qmax, float inv,
                                                      float& scale) {
  WideQuant q{0, 0.0f, inv};
  if (d > 3.4028234663852886e38f) {
    const float dh = __fsub_rn(__fmul_rn(mx, 0.5f), __fmul_rn(mn, 0.5f));
    q.mode = 2;
    q.mnh = __fmul_rn(mn, 0.5f);
    scale = __fmul_rn(__fdiv_rn(dh, qmax), 2.0f);
    q.inv = __fdiv_rn(qmax, dh);
  } else if (inv > 3.4028234663852886e38f) {
    q.mode = 1;
    q.inv = __fdiv_rn(qmax, __fmul_rn(d, 18446744073709551616.0f));
  }
  return q;
}

__device__ __forceinline__ uint32_t wide_quant_code(const WideQuant& q, float x, float mn, int cmask) {
  float y;
  if (q.mode == 2) y = __fmul_rn(__fsub_rn(__fmul_rn(x, 0.5f), q.mnh), q.inv);
  else if (q.mode == 1) y = __fmul_rn(__fmul_rn(__fsub_rn(x, mn), 18446744073709551616.0f), q.inv);
  else y = __fmul_rn(__fsub_rn(x, mn), q.inv);
  int ci = __float2int_rn(y);  // NaN gives 0
  ci = ci < 0 ? 0 : ci;
  return static_cast<uint32_t>(ci > cmask ? cmask : ci);
}

// Quantize the 16 bf16 values a lane holds (raw words w, value 2i in the low
// half of w[i]), sharing min/max with the other lanes of its group (LPG =
// G / 16 consecutive lanes), and pack the codes into lw.  The formula is the
// fixed fp32 one of lkv_quantize_kv, every operation rounded separately:
//   d = mx - mn;  scale = d / qmax;  inv = qmax / d  (both 0 when d == 0);
//   code = clamp(rint((x - mn) * inv), 0, qmax);  zero = mn + 0.
// While d and inv are finite, x - mn <= d, so (x - mn) * inv < qmax + 1/2 and
// the clamp never bites: the code is rounded half-even by adding 1.5 * 2^23
// (two values per packed fp32 operation) and read from the low mantissa bits.
// `one` must be 1.0f, passed in at run time (see the rounding step).
// Otherwise (inv overflowing for a tiny d, or d overflowing) every value takes
// the scalar path of wide_quant_code.  `mask` names the lanes of the calling row.
template <int BITS>
__device__ __forceinline__ void quantize16(const uint32_t (&w)[8], int lpg, unsigned mask, float one,
                                           LaneWords<BITS>& lw, float& scale, float& zero) {
  // min and max are exact in bf16, two values per instruction
  __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&w[0]), hi = lo;
#pragma unroll
  for (int i = 1; i < 8; ++i) {
    const __nv_bfloat162 p = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
    lo = __hmin2(lo, p);
    hi = __hmax2(hi, p);
  }
  float mn = fminf(__low2float(lo), __high2float(lo));
  float mx = fmaxf(__low2float(hi), __high2float(hi));
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) {
    if (off < lpg) {
      mn = fminf(mn, __shfl_xor_sync(mask, mn, off));
      mx = fmaxf(mx, __shfl_xor_sync(mask, mx, off));
    }
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
    // a NaN input becomes mn (code 0), every other value is unchanged
    const __nv_bfloat162 mn_b = __floats2bfloat162_rn(mn, mn);
    const float2 nmn = make_float2(-mn, -mn), inv2 = make_float2(inv, inv), one2 = make_float2(one, one);
    const float2 rnd = make_float2(12582912.0f, 12582912.0f);
    uint32_t rb[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __nv_bfloat162 p = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]), mn_b);
      const uint32_t u = *reinterpret_cast<const uint32_t*>(&p);
      const float2 x = make_float2(bf16_lo(u), bf16_hi(u));
      const float2 y = exact_mul2(exact_add2(x, nmn), inv2);
      // y * one + 1.5 * 2^23 with one == 1.0 held in a register: the product
      // y * 1 is exact, so this is y + 1.5 * 2^23 rounded once, i.e. y rounded
      // half-even into the low mantissa bits.  (A plain add fed directly by
      // the multiply above would be contracted into one fused multiply-add,
      // skipping the rounding of y.)
      const float2 r = exact_fma2(y, one2, rnd);
      rb[2 * i] = __float_as_uint(r.x);
      rb[2 * i + 1] = __float_as_uint(r.y);
    }
    pack16_magic<BITS>(rb, lw);
  } else {
    const WideQuant wq = wide_quant_setup(mn, mx, d, qmax, inv, scale);
    uint32_t c[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float x = (i & 1) ? bf16_hi(w[i / 2]) : bf16_lo(w[i / 2]);
      c[i] = wide_quant_code(wq, x, mn, (int)cmask);
    }
    pack16<BITS>(c, lw);
  }
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

namespace lkv {

// ------------------------------------------------------------------ exact integer unpack
//
// A code c sitting at bits [kk, kk+BITS) of a 32-bit word x with kk + BITS <= 23
// becomes the float 2^(23-kk) + c with one AND-OR: the mantissa holds c * 2^kk
// and the exponent field is 150 - kk.  Subtracting 2^(23-kk) (two codes per
// packed fp32 add) leaves c exactly.  Codes further up the word are first
// brought down with one (funnel) shift shared by the codes that follow it.

// Stream offset of the shifted copy that code i is read from (greedy plan).
template <int BITS>
constexpr int copy_shift(int i) {
  int s = 0;
  for (int j = 0; j <= i; ++j) {
    const int p = j * BITS;
    if (!(p >= s && p - s + BITS <= 23)) s = p;
  }
  return s;
}

template <int BITS>
__device__ __forceinline__ uint32_t stream_bits(const LaneWords<BITS>& lw, int s) {
  const int wi = s >> 5, k = s & 31;
  if (k == 0) return lw.w[wi];
  const uint32_t hi = (wi + 1 < LaneWords<BITS>::N) ? lw.w[wi + 1] : 0u;
  return __funnelshift_r(lw.w[wi], hi, k);
}

template <int BITS, int I>
__device__ __forceinline__ float code_plus_magic(const LaneWords<BITS>& lw) {
  constexpr int s = copy_shift<BITS>(I);
  constexpr int kk = I * BITS - s;
  constexpr uint32_t mask = ((1u << BITS) - 1u) << kk;
  constexpr uint32_t magic = (uint32_t)(150 - kk) << 23;
  return __uint_as_float((stream_bits<BITS>(lw, s) & mask) | magic);
}

template <int BITS, int I>
__device__ __forceinline__ float magic_value() {
  constexpr int kk = I * BITS - copy_shift<BITS>(I);
  return __uint_as_float((uint32_t)(150 - kk) << 23);
}

template <int BITS, int P>
__device__ __forceinline__ float2 code_pair(const LaneWords<BITS>& lw) {
  const float2 m = make_float2(code_plus_magic<BITS, 2 * P>(lw), code_plus_magic<BITS, 2 * P + 1>(lw));
  return __fadd2_rn(m, make_float2(-magic_value<BITS, 2 * P>(), -magic_value<BITS, 2 * P + 1>()));
}

// The lane's 16 codes as exact floats, in channel pairs.
template <int BITS>
__device__ __forceinline__ void unpack16_int(const LaneWords<BITS>& lw, float2 (&c)[8]) {
  c[0] = code_pair<BITS, 0>(lw);
  c[1] = code_pair<BITS, 1>(lw);
  c[2] = code_pair<BITS, 2>(lw);
  c[3] = code_pair<BITS, 3>(lw);
  c[4] = code_pair<BITS, 4>(lw);
  c[5] = code_pair<BITS, 5>(lw);
  c[6] = code_pair<BITS, 6>(lw);
  c[7] = code_pair<BITS, 7>(lw);
}

// Lane words from shared memory (4-byte aligned; wider when the width allows).
template <int BITS>
__device__ __forceinline__ void lds_lane_words(const uint8_t* p, LaneWords<BITS>& lw) {
  if constexpr (BITS == 16) {
    const uint4 v = *reinterpret_cast<const uint4*>(p), u = *reinterpret_cast<const uint4*>(p + 16);
    lw.w[0] = v.x; lw.w[1] = v.y; lw.w[2] = v.z; lw.w[3] = v.w;
    lw.w[4] = u.x; lw.w[5] = u.y; lw.w[6] = u.z; lw.w[7] = u.w;
  } else if constexpr (BITS == 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    lw.w[0] = v.x; lw.w[1] = v.y; lw.w[2] = v.z; lw.w[3] = v.w;
  } else if constexpr (BITS == 4) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    lw.w[0] = v.x; lw.w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < LaneWords<BITS>::N; ++i) lw.w[i] = reinterpret_cast<const uint32_t*>(p)[i];
  }
}

// ------------------------------------------------------------------ mbarrier / bulk copy

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for a phase of an mbarrier, giving up after `limit_ns`.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

// 1-D bulk copy global -> shared, completing `bytes` on the mbarrier.  Both
// addresses and the size are multiples of 16 bytes.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
      ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// 16-byte asynchronous copy global -> shared through the load path (no
// tensor-memory-access unit), for many small scattered rows; both addresses
// are 16-byte aligned.  cp_async_wait_all waits for this thread's copies.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Start bringing the 128-byte line of p into L2 (no register result).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Orders this thread's earlier shared-memory accesses before later
// async-proxy (bulk copy) writes to shared memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Orders this thread's view of earlier global-memory writes (generic proxy)
// before its later bulk copies (async proxy) that read the same memory.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

}  // namespace lkv
