// decode.cu -- single-token GQA decode attention over the packed KV cache,
// split along the sequence, with the sparse-V skip.
//
// "Super KV Compression" §第一层 gives the K/V widths, §第三层 the skip (a V
// row whose softmax probability is below tau is never dequantized) and
// §第二层 the tiered cache this same code reads as two segments.  The split
// into chunks with per-chunk (max, sum) statistics merged afterwards is the
// standard exact online-softmax decomposition ("TurboQuant" §与其他优化技术的
// 对比 names FlashAttention as the complementary technique).
//
// Three launches, stream ordered:
//   k_phase   per (chunk, b, kv head): dequant-K . q for the group's query
//             heads -> base-2 logits in the workspace + chunk (max, sum).
//   v_phase   per (chunk, b, kv head): global (max, sum) from all chunks,
//             p = exp2(s - max) / sum, skip p < tau; a V row is loaded only
//             when some head keeps it; accumulate p * vhat -> chunk partial.
//   combine   per (b, query head): out = sum of chunk partials.
//
// Dequantization is folded into the dot products.  A code c is turned into
// the float f = 1 + c / 2^bits exactly by bit placement, so with u = 2^bits *
// scale the reconstruction is khat = u * f + (zero - u), and
//   sum_d q_d khat_d = u * (sum_d q_d f_d - Q) + zero * Q,   Q = sum_d q_d
// over the 16 channels of a lane (they share one group).  The inner loop is
// then one packed fp32 multiply-add (two channels) per code and head.
#include <cfloat>

#include "lkv_kernels.cuh"

namespace lkv {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr unsigned kFull = 0xFFFFFFFFu;

struct SegLens {
  int n0, n1;
};

__device__ __forceinline__ SegLens seg_lens(const DecodeArgs& a, int b, int bg, bool flag_bad) {
  SegLens s;
  if (a.len_mode == 0) {
    const int raw = a.lens[b];
    if (flag_bad && (raw < 0 || raw > a.T_cap)) atomicExch(a.status, kStatusInvalidArg);
    s.n0 = clamp_len(raw, a.T_cap);
    s.n1 = 0;
  } else {
    const int r0 = a.lens[2 * bg], r1 = a.lens[2 * bg + 1];
    if (flag_bad && (r0 < 0 || r1 < 0 || (long long)r0 + r1 > a.T_cap)) atomicExch(a.status, kStatusInvalidArg);
    s.n0 = clamp_len(r0, a.T_cap);
    s.n1 = clamp_len(r1, a.T_cap - s.n0);
  }
  return s;
}

// Reduce-scatter of NH per-lane values over the lanes that differ in bits
// OFF, OFF/2, ..., 1: after the first log2(NH) steps each lane keeps one
// head (index accumulated in hidx), the remaining steps all-reduce it.
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

__device__ __forceinline__ void merge_ml(float& m, float& l, float m2, float l2) {
  const float M = fmaxf(m, m2);
  if (M == -INFINITY) return;  // both empty
  l = l * exp2f(m - M) + l2 * exp2f(m2 - M);
  m = M;
}

// ---------------------------------------------------------------- K phase

template <int D, int H, int KB>
__global__ void __launch_bounds__(kThreads) k_phase_kernel(DecodeArgs a) {
  constexpr int LPR = D / kDimsPerLane;
  constexpr int RPW = 32 / LPR;
  static_assert(H <= LPR, "heads per lane group");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int j = lane % LPR;
  const int bg = blockIdx.y, b = bg / a.Hkv, g = bg % a.Hkv, z = blockIdx.z;
  const int c = blockIdx.x;
  const int ng = D / a.G;
  const int gi = (j * kDimsPerLane) / a.G;

  if (blockIdx.x == 0 && bg == 0 && z == 0 && threadIdx.x == 0 && a.skip_counts) {
    a.skip_counts[0] = 0ull;
    a.skip_counts[1] = 0ull;
  }
  const SegLens sl = seg_lens(a, b, bg, c == 0 && z == 0 && threadIdx.x == 0);
  const int n = sl.n0 + sl.n1;
  const int v0 = c * a.chunk, v1 = min(v0 + a.chunk, n);
  float* st = a.stats + (((long long)bg * a.n_chunks + c) * a.r + z * H) * 2;
  if (v0 >= n) {
    if (threadIdx.x < H) { st[2 * threadIdx.x] = -INFINITY; st[2 * threadIdx.x + 1] = 0.0f; }
    return;
  }

  // The lane's 16 query channels for each head of this slice, pre-scaled so
  // that logits come out in base 2, and their sum Q.
  float2 qf[H][8];
  float Q[H];
#pragma unroll
  for (int h = 0; h < H; ++h) {
    const int hq = g * a.r + z * H + h;
    float x[16];
    load16_bf16(a.q + ((long long)b * a.Hq + hq) * D + j * kDimsPerLane, x);
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      qf[h][i] = make_float2(x[2 * i] * a.q_scale, x[2 * i + 1] * a.q_scale);
      s += qf[h][i].x + qf[h][i].y;
    }
    Q[h] = s;
  }

  float run_m = -INFINITY, run_l = 0.0f;
  int hidx = 0;
  const bool leader = (lane % (LPR / H)) == 0;
  for (int vb = v0 + warp * RPW; vb < v1; vb += kWarps * RPW) {
    const int v = vb + lane / LPR;
    const bool valid = v < v1;
    float dot[H];
#pragma unroll
    for (int h = 0; h < H; ++h) dot[h] = 0.0f;
    if (valid) {
      const int seg = v >= sl.n0;
      const long long row = (long long)bg * a.T_cap + (seg ? v - sl.n0 : v);
      LaneWords<KB> lw;
      load_lane_words<KB>(a.kc[seg] + row * (D * KB / 8) + j * (2 * KB), lw);
      if constexpr (KB == 16) {
        // passthrough width: the bf16 K values themselves
#pragma unroll
        for (int h = 0; h < H; ++h) {
          float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            acc = __ffma2_rn(qf[h][i], make_float2(__uint_as_float(lw.w[i] << 16), __uint_as_float(lw.w[i] & 0xFFFF0000u)),
                             acc);
          dot[h] = acc.x + acc.y;
        }
      } else {
        const float2 sz = __ldg(reinterpret_cast<const float2*>(a.ksz[seg] + (row * ng + gi) * 2));
        float2 f[8];
        unpack16_f<KB>(lw, f);
        const float u = sz.x * (float)(1 << KB);
#pragma unroll
        for (int h = 0; h < H; ++h) {
          float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc = __ffma2_rn(qf[h][i], f[i], acc);
          dot[h] = fmaf(u, (acc.x + acc.y) - Q[h], sz.y * Q[h]);
        }
      }
    }
    hidx = 0;
    ReduceScatter<H, LPR / 2>::run(dot, lane, hidx);
    if (valid && leader) {
      const float s = dot[0];
      a.logits[((long long)bg * a.T_cap + v) * a.r + z * H + hidx] = s;
      if (s > run_m) {
        run_l = run_l * exp2f(run_m - s) + 1.0f;
        run_m = s;
      } else {
        run_l += exp2f(s - run_m);
      }
    }
  }
  // hidx of a lane depends only on its lane bits: recompute for lanes whose
  // loop ran zero times.
  {
    float dummy[H];
#pragma unroll
    for (int h = 0; h < H; ++h) dummy[h] = 0.0f;
    hidx = 0;
    ReduceScatter<H, LPR / 2>::run(dummy, lane, hidx);
  }
  __shared__ float sm_m[kThreads], sm_l[kThreads];
  __shared__ int sm_h[kThreads];
  sm_m[threadIdx.x] = leader ? run_m : -INFINITY;
  sm_l[threadIdx.x] = leader ? run_l : 0.0f;
  sm_h[threadIdx.x] = hidx;
  __syncthreads();
  if (threadIdx.x < H) {
    float m = -INFINITY, l = 0.0f;
    for (int i = 0; i < kThreads; ++i)
      if (sm_h[i] == (int)threadIdx.x) merge_ml(m, l, sm_m[i], sm_l[i]);
    st[2 * threadIdx.x] = m;
    st[2 * threadIdx.x + 1] = l;
  }
}

// ---------------------------------------------------------------- V phase

template <int D, int H, int VB>
__device__ __forceinline__ void v_row_accumulate(const uint8_t* __restrict__ codes, const float* __restrict__ sz_row,
                                                 int j, int gi, const float (&p)[H], const bool (&keep)[H],
                                                 float2 (&acc)[H][8], float (&Z)[H]) {
  LaneWords<VB> lw;
  load_lane_words<VB>(codes + j * (2 * VB), lw);
  if constexpr (VB == 16) {
    // passthrough width: the bf16 V values themselves
#pragma unroll
    for (int h = 0; h < H; ++h) {
      const float w = keep[h] ? p[h] : 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        acc[h][i] = __ffma2_rn(f2(w), make_float2(__uint_as_float(lw.w[i] << 16), __uint_as_float(lw.w[i] & 0xFFFF0000u)),
                               acc[h][i]);
    }
  } else {
    const float2 sz = __ldg(reinterpret_cast<const float2*>(sz_row + gi * 2));
    float2 f[8];
    unpack16_f<VB>(lw, f);
    const float u = sz.x * (float)(1 << VB);
    const float zu = sz.y - u;
#pragma unroll
    for (int h = 0; h < H; ++h) {
      const float w = keep[h] ? p[h] : 0.0f;
      const float wu = w * u;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[h][i] = __ffma2_rn(f2(wu), f[i], acc[h][i]);
      Z[h] = fmaf(w, zu, Z[h]);
    }
  }
}

template <int D, int H, int VB0, int VB1>
__global__ void __launch_bounds__(kThreads) v_phase_kernel(DecodeArgs a) {
  constexpr int LPR = D / kDimsPerLane;
  constexpr int RPW = 32 / LPR;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int j = lane % LPR;
  const int bg = blockIdx.y, b = bg / a.Hkv, g = bg % a.Hkv, z = blockIdx.z;
  const int c = blockIdx.x;
  const int ng = D / a.G;
  const int gi = (j * kDimsPerLane) / a.G;
  const SegLens sl = seg_lens(a, b, bg, false);
  const int n = sl.n0 + sl.n1;
  const int v0 = c * a.chunk, v1 = min(v0 + a.chunk, n);
  if (v0 >= n) return;
  const int n_used = (n + a.chunk - 1) / a.chunk;

  // Global (max, 1/sum) for every head of the group (all r heads: the
  // skipped-row count needs them), one warp per head.
  __shared__ float sm_m[64], sm_il[64];
  for (int h = warp; h < a.r; h += kWarps) {
    float m = -INFINITY, l = 0.0f;
    for (int cc = lane; cc < n_used; cc += 32) {
      const float* st = a.stats + (((long long)bg * a.n_chunks + cc) * a.r + h) * 2;
      merge_ml(m, l, st[0], st[1]);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const float m2 = __shfl_xor_sync(kFull, m, off), l2 = __shfl_xor_sync(kFull, l, off);
      merge_ml(m, l, m2, l2);
    }
    if (lane == 0) { sm_m[h] = m; sm_il[h] = l > 0.0f ? 1.0f / l : 0.0f; }
  }
  __syncthreads();

  float2 acc[H][8];
  float Z[H];
#pragma unroll
  for (int h = 0; h < H; ++h) {
    Z[h] = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[h][i] = make_float2(0.0f, 0.0f);
  }
  unsigned long long cnt_heads = 0, cnt_rows = 0;
  const bool counting = a.skip_counts != nullptr;
  for (int vb = v0 + warp * RPW; vb < v1; vb += kWarps * RPW) {
    const int v = vb + lane / LPR;
    if (v >= v1) continue;  // the lanes of a row agree; no shuffles below
    const long long lrow = (long long)bg * a.T_cap + v;
    float p[H];
    bool keep[H];
    bool need = false;
#pragma unroll
    for (int h = 0; h < H; ++h) {
      const int hh = z * H + h;
      const float s = a.logits[lrow * a.r + hh];
      p[h] = exp2f(s - sm_m[hh]) * sm_il[hh];
      keep[h] = !(p[h] < a.tau);
      need |= keep[h];
    }
    if (j == 0) {
      if (a.mass && z == 0) {  // the group's mean attention to the row, over all r heads
        float ms = 0.0f;
        for (int hh = 0; hh < a.r; ++hh) ms += exp2f(a.logits[lrow * a.r + hh] - sm_m[hh]) * sm_il[hh];
        a.mass[lrow] = ms * (1.0f / a.r);
      }
      if (a.skip_mask) {
#pragma unroll
        for (int h = 0; h < H; ++h)
          a.skip_mask[((long long)b * a.Hq + g * a.r + z * H + h) * a.T_cap + v] = keep[h] ? 0 : 1;
      }
      if (counting) {
#pragma unroll
        for (int h = 0; h < H; ++h) cnt_heads += keep[h] ? 0 : 1;
        if (z == 0) {
          bool all_skip = true;
          for (int hh = 0; hh < a.r; ++hh) {
            const float s = a.logits[lrow * a.r + hh];
            all_skip &= (exp2f(s - sm_m[hh]) * sm_il[hh]) < a.tau;
          }
          cnt_rows += all_skip ? 1 : 0;
        }
      }
    }
    if (!need) continue;
    const int seg = v >= sl.n0;
    const long long row = (long long)bg * a.T_cap + (seg ? v - sl.n0 : v);
    if (seg == 0)
      v_row_accumulate<D, H, VB0>(a.vc[0] + row * (D * VB0 / 8), a.vsz[0] + row * ng * 2, j, gi, p, keep, acc, Z);
    else
      v_row_accumulate<D, H, VB1>(a.vc[1] + row * (D * VB1 / 8), a.vsz[1] + row * ng * 2, j, gi, p, keep, acc, Z);
  }
  // Fold the per-group constant, then reduce the RPW row slots of the warp.
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
  __shared__ float red[kWarps][H][D];
  if (lane < LPR) {
#pragma unroll
    for (int h = 0; h < H; ++h)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        red[warp][h][j * kDimsPerLane + 2 * i] = acc[h][i].x;
        red[warp][h][j * kDimsPerLane + 2 * i + 1] = acc[h][i].y;
      }
  }
  __syncthreads();
  float* part = a.partial + (((long long)bg * a.n_chunks + c) * a.r + z * H) * D;
  for (int e = threadIdx.x; e < H * D; e += kThreads) {
    const int h = e / D, d = e % D;
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += red[w][h][d];
    part[(long long)h * D + d] = s;
  }
  if (counting) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      cnt_heads += __shfl_xor_sync(kFull, cnt_heads, off);
      cnt_rows += __shfl_xor_sync(kFull, cnt_rows, off);
    }
    if (lane == 0 && (cnt_heads | cnt_rows)) {
      atomicAdd(a.skip_counts, cnt_heads);
      atomicAdd(a.skip_counts + 1, cnt_rows);
    }
  }
}

// ---------------------------------------------------------------- combine

__global__ void combine_kernel(DecodeArgs a, int D) {
  const int bh = blockIdx.x, b = bh / a.Hq, h = bh % a.Hq, g = h / a.r, bg = b * a.Hkv + g;
  const SegLens sl = seg_lens(a, b, bg, false);
  const int n = sl.n0 + sl.n1;
  const int n_used = (n + a.chunk - 1) / a.chunk;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float s = 0.0f;
    for (int c = 0; c < n_used; ++c)
      s += a.partial[(((long long)bg * a.n_chunks + c) * a.r + (h - g * a.r)) * D + d];
    a.out[((long long)b * a.Hq + h) * D + d] = s;
  }
}

template <int D, int H, int KB>
cudaError_t launch_k(const DecodeArgs& a, dim3 grid, cudaStream_t s) {
  k_phase_kernel<D, H, KB><<<grid, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

template <int D, int H>
cudaError_t launch_k_bits(const DecodeArgs& a, int kb, dim3 grid, cudaStream_t s) {
  switch (kb) {
    case 2: return launch_k<D, H, 2>(a, grid, s);
    case 4: return launch_k<D, H, 4>(a, grid, s);
    case 6: return launch_k<D, H, 6>(a, grid, s);
    case 8: return launch_k<D, H, 8>(a, grid, s);
    case 16: return launch_k<D, H, 16>(a, grid, s);
  }
  return cudaErrorInvalidValue;
}

template <int D, int H>
cudaError_t launch_v_bits(const DecodeArgs& a, int vb0, int vb1, dim3 grid, cudaStream_t s) {
  if (vb0 == vb1) {
    switch (vb0) {
      case 2: v_phase_kernel<D, H, 2, 2><<<grid, kThreads, 0, s>>>(a); return cudaGetLastError();
      case 4: v_phase_kernel<D, H, 4, 4><<<grid, kThreads, 0, s>>>(a); return cudaGetLastError();
      case 6: v_phase_kernel<D, H, 6, 6><<<grid, kThreads, 0, s>>>(a); return cudaGetLastError();
      case 8: v_phase_kernel<D, H, 8, 8><<<grid, kThreads, 0, s>>>(a); return cudaGetLastError();
      case 16: v_phase_kernel<D, H, 16, 16><<<grid, kThreads, 0, s>>>(a); return cudaGetLastError();
    }
  } else if (vb0 == 6 && vb1 == 4) {
    v_phase_kernel<D, H, 6, 4><<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
  }
  return cudaErrorInvalidValue;
}

template <int D>
cudaError_t launch_decode_d(const DecodeArgs& a, int H, int kb, int vb0, int vb1, dim3 grid, cudaStream_t s) {
  cudaError_t e;
  switch (H) {
    case 1: e = launch_k_bits<D, 1>(a, kb, grid, s); if (e) return e; return launch_v_bits<D, 1>(a, vb0, vb1, grid, s);
    case 2: e = launch_k_bits<D, 2>(a, kb, grid, s); if (e) return e; return launch_v_bits<D, 2>(a, vb0, vb1, grid, s);
    case 4: e = launch_k_bits<D, 4>(a, kb, grid, s); if (e) return e; return launch_v_bits<D, 4>(a, vb0, vb1, grid, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, int D, int kb, int vb0, int vb1, cudaStream_t s) {
  if ((long long)a.B * a.Hkv == 0) return cudaSuccess;
  const int H = a.r < 4 ? a.r : 4;
  dim3 grid(a.n_chunks, a.B * a.Hkv, a.r / H);
  cudaError_t e;
  if (D == 64) e = launch_decode_d<64>(a, H, kb, vb0, vb1, grid, s);
  else if (D == 128) e = launch_decode_d<128>(a, H, kb, vb0, vb1, grid, s);
  else return cudaErrorInvalidValue;
  if (e != cudaSuccess) return e;
  combine_kernel<<<a.B * a.Hq, D, 0, s>>>(a, D);
  return cudaGetLastError();
}

}  // namespace lkv
