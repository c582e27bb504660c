// mma_k.cuh -- the K pass of the decode on tensor cores: packed K codes
// become exact fp16 integers in registers and meet q in mma.sync.m16n8k16.
//
// Why this is exact enough: a code c (at most 8 bits) is an integer, exact
// in fp16; q is a bf16 value, whose 8-bit significand fits fp16's 11 bits
// once the head's q is scaled by a power of two 2^E so that its largest
// magnitude lies in [2^14, 2^15).  Each product c * q * 2^E is then exact
// in the fp32 accumulator of the MMA and only the sums round, as they do in
// an fp32 FMA chain.  The affine part of the dequantization is folded once
// per group afterwards:
//   sum_d q_d (scale_g c_d + zero_g) = scale_g * sum_d q_d c_d + zero_g * sum_d q_d.
//
// Codes to fp16 without conversion instructions: a code sitting at bits
// [o, o + bits) of one 16-bit half, with o + bits <= 10, is OR-ed into the
// fp16 pattern 0x6400 (1024, unit spacing), giving 1024 + c * 2^o; one
// packed subtraction of 1024 leaves c * 2^o exactly, and the factor 2^-o is
// moved into q.  A "plan" lists, for each 16-code block of a lane's slice of
// a row, which 32-bit window of the packed bit stream and which masks give
// each register its two codes (found by search: 1.06 / 1.13 / 1.31
// instructions per code for 2 / 4 / 6 bits).  8-bit codes are whole bytes
// and are placed under the 0x64 exponent bytes by one byte permute.
//
// Fragment layout of mma.m16n8k16 (A row-major 16x16, B 16x8, C 16x8):
// lane = 4 * gid + tig; A registers {a0, a1, a2, a3} = rows {gid, gid + 8,
// gid, gid + 8}, k pairs {2tig, 2tig + 8}; B registers {b0, b1} = k pairs
// {2tig, 2tig + 8} of column gid; C = rows {gid, gid + 8} x columns
// {2tig, 2tig + 1}.  The k order inside a step is free as long as A and B
// agree, so lane tig owns a contiguous slice of D/4 channels of each row
// and register J of that slice feeds k-step J/2.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

namespace lkv {
namespace fused {

struct PlanEntry {
  int p;       // first bit of the window inside the 16-code block
  int lo, lo_off;  // code index (0..15) and its bit offset in the low half
  int hi, hi_off;  // the same for the high half
};

template <int KB>
struct Plan;
template <>
struct Plan<2> {
  static constexpr PlanEntry e[8] = {{0, 0, 0, 8, 0},  {0, 1, 2, 9, 2},   {0, 2, 4, 10, 4},  {0, 3, 6, 11, 6},
                                     {0, 4, 8, 12, 8}, {10, 5, 0, 13, 0}, {10, 6, 2, 14, 2}, {10, 7, 4, 15, 4}};
};
template <>
struct Plan<4> {
  static constexpr PlanEntry e[8] = {{0, 0, 0, 4, 0},   {0, 1, 4, 5, 4},   {8, 2, 0, 6, 0},   {8, 3, 4, 7, 4},
                                     {32, 8, 0, 12, 0}, {32, 9, 4, 13, 4}, {40, 10, 0, 14, 0}, {40, 11, 4, 15, 4}};
};
template <>
struct Plan<6> {
  static constexpr PlanEntry e[8] = {{0, 0, 0, 3, 2},   {5, 1, 1, 4, 3},   {11, 2, 1, 5, 3},  {32, 6, 4, 8, 0},
                                     {42, 7, 0, 10, 2}, {54, 9, 0, 12, 2}, {64, 11, 2, 14, 4}, {74, 13, 4, 15, 0}};
};
// 8-bit codes: register j of a block holds bytes (0, 2) or (1, 3) of word j / 2.
template <>
struct Plan<8> {
  static constexpr PlanEntry e[8] = {{0, 0, 0, 2, 0},   {0, 1, 0, 3, 0},   {32, 4, 0, 6, 0},  {32, 5, 0, 7, 0},
                                     {64, 8, 0, 10, 0}, {64, 9, 0, 11, 0}, {96, 12, 0, 14, 0}, {96, 13, 0, 15, 0}};
};

// Compile-time checks of a plan: every code of the block appears once, and
// each sits inside its window at the stated offset with room below bit 10.
template <int KB>
constexpr bool plan_ok() {
  int seen[16] = {0};
  for (int j = 0; j < 8; ++j) {
    const PlanEntry x = Plan<KB>::e[j];
    if (x.lo < 0 || x.lo > 15 || x.hi < 0 || x.hi > 15) return false;
    seen[x.lo]++;
    seen[x.hi]++;
    if (x.lo_off + KB > 10 || x.hi_off + KB > 10) return false;
    if (KB * x.lo - x.p != x.lo_off) return false;
    if (KB * x.hi - x.p != 16 + x.hi_off) return false;
  }
  for (int i = 0; i < 16; ++i)
    if (seen[i] != 1) return false;
  return true;
}
static_assert(plan_ok<2>() && plan_ok<4>() && plan_ok<6>(), "bad code extraction plan");

template <int KB>
constexpr bool plan8_ok() {
  int seen[16] = {0};
  for (int j = 0; j < 8; ++j) {
    const PlanEntry x = Plan<8>::e[j];
    if (x.p != 32 * (j / 2) || x.lo != 4 * (j / 2) + (j & 1) || x.hi != x.lo + 2) return false;
    seen[x.lo]++;
    seen[x.hi]++;
  }
  for (int i = 0; i < 16; ++i)
    if (seen[i] != 1) return false;
  return true;
}
static_assert(plan8_ok<8>(), "bad 8-bit plan");

constexpr uint32_t kF16Magic2 = 0x64006400u;  // (1024, 1024) in fp16

__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Register J (0 .. D/8 - 1) of a lane slice held in words w (the slice's
// D*KB/128 words): two codes as exact fp16 values c * 2^off.
template <int KB, int J, int SW>
__device__ __forceinline__ uint32_t a_reg_codes(const uint32_t (&w)[SW]) {
  constexpr PlanEntry pe = Plan<KB>::e[J % 8];
  constexpr int p = pe.p + (J / 8) * 16 * KB;  // first bit of the window in the slice
  constexpr int wi = p / 32, sh = p % 32;
  uint32_t r;
  if constexpr (KB == 8) {
    r = __byte_perm(w[wi], 0x64646464u, (J & 1) ? 0x4341 : 0x4240);
  } else {
    // highest bit of the window that holds code bits
    constexpr int top = sh + 16 + pe.hi_off + KB - 1;
    uint32_t win;
    if constexpr (sh == 0) {
      win = w[wi];
    } else if constexpr (top < 32) {
      win = w[wi] >> sh;
    } else {
      win = __funnelshift_r(w[wi], w[wi + 1], sh);
    }
    constexpr uint32_t m = (1u << KB) - 1u;
    constexpr uint32_t mask = (m << pe.lo_off) | (m << (16 + pe.hi_off));
    r = (win & mask) | kF16Magic2;
  }
  return hsub2_u32(r, kF16Magic2);
}

// At the 16-bit passthrough width the slice holds bf16 values: register J
// is word J, channels (2J, 2J + 1), used as it is by the bf16 MMA.
template <int KB, int J, int SW>
__device__ __forceinline__ uint32_t a_reg(const uint32_t (&w)[SW]) {
  if constexpr (KB == 16) {
    return w[J];
  } else {
    return a_reg_codes<KB, J, SW>(w);
  }
}

// Slice channels (0 .. D/4 - 1) and power-of-two offsets of register J.
template <int KB, int J>
struct RegChannels {
  static constexpr PlanEntry pe = Plan<KB>::e[J % 8];
  static constexpr int lo = (J / 8) * 16 + pe.lo;
  static constexpr int hi = (J / 8) * 16 + pe.hi;
  static constexpr int lo_off = pe.lo_off;
  static constexpr int hi_off = pe.hi_off;
};
template <int J>
struct RegChannels<16, J> {
  static constexpr int lo = 2 * J, hi = 2 * J + 1, lo_off = 0, hi_off = 0;
};

__device__ __forceinline__ void hmma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same with bf16 operands (the 16-bit passthrough width: bf16 K rows
// against the bf16 q; every product is exact in the fp32 accumulator).
__device__ __forceinline__ void hmma16816_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// fp16 pair (x, y), each scaled by its exact power of two (offsets 0: the
// two 16-bit patterns side by side, whatever their type).
template <int OFF_LO, int OFF_HI>
__device__ __forceinline__ uint32_t q_pair(__half x, __half y) {
  __half2 v = __halves2half2(x, y);
  if constexpr (OFF_LO != 0 || OFF_HI != 0) {
    const __half2 f = __floats2half2_rn(1.0f / (float)(1 << OFF_LO), 1.0f / (float)(1 << OFF_HI));
    v = __hmul2(v, f);
  }
  return *reinterpret_cast<uint32_t*>(&v);
}

// B fragments of one n-tile for lane (gid, tig): column n = 8 * nt + gid is
// (head n / ng, group n % ng); it is nonzero only on the channels of the
// lane's slice when they belong to that group.  qh points at the scaled
// fp16 q of the column's head (D values; for 16-bit K the raw bf16 q);
// bf[J] for J = 0 .. D/8 - 1.
template <int KB, int D, int J>
__device__ __forceinline__ void bfrag_one(const __half* qh, int base, bool on, uint32_t* bf) {
  using R = RegChannels<KB, J>;
  bf[J] = on ? q_pair<R::lo_off, R::hi_off>(qh[base + R::lo], qh[base + R::hi]) : 0u;
  if constexpr (J + 1 < D / 8) bfrag_one<KB, D, J + 1>(qh, base, on, bf);
}

}  // namespace fused
}  // namespace lkv
