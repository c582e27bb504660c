/*
 * lkv.h -- C ABI of liblkv: low-bit quantized KV cache and single-token
 * decode attention over the packed cache, for NVIDIA B200 (sm_100a).
 *
 * The method comes from two web pages:
 *   [SKV] "Super KV Compression: 突破LLM推理内存瓶颈的三层压缩架构解析"
 *         §第一层：自适应非对称量化      -- K at 6 bits, V at 4 bits, asymmetric
 *         §第二层：注意力感知的Token淘汰机制 -- V at 6 / 4 bits or evicted by attention
 *         §第三层：稀疏V跳过加速          -- do not dequantize low-attention V
 *   [TQ]  "TurboQuant：将LLM KV缓存压缩5-7倍的突破性技术"
 *         §TurboQuant的核心创新           -- asymmetric, group-wise quantization
 *
 * Conventions for every entry point
 * ---------------------------------
 * - All tensor arguments are DEVICE pointers to caller-owned memory; the
 *   library allocates nothing and keeps no state between calls.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  Every call only enqueues work on it and returns at once; no
 *   call synchronizes, except lkv_workspace_status().
 * - Arguments are validated on the host before anything is launched; a
 *   failed check returns a nonzero lkv_status and enqueues nothing.
 *   Launch failures return LKV_ERR_CUDA.
 * - Sequence lengths live on the device, so the host cannot see them:
 *   kernels clamp each length into [0, T_cap]; the decode entry points also
 *   record an out-of-range length in the workspace status word.
 * - bf16 inputs must be finite.  NaN or infinity gives unspecified values
 *   but never an out-of-bounds access.
 * - Index arithmetic is 64-bit: any tensor that fits in device memory works.
 *
 * Shapes and layouts (row-major, innermost last)
 *   B batch, Hq query heads, Hkv KV heads (Hq % Hkv == 0), r = Hq / Hkv;
 *   query head h reads KV head h / r.  D head_dim (64 or 128).  G group:
 *   G contiguous head_dim channels of one token share one (scale, zero);
 *   G in {32, 64, 128}, G divides D, ng = D / G.  T_cap cache capacity
 *   in tokens; T_b = seq_lens[b] valid tokens of sequence b.  bits in
 *   {2, 4, 6, 8, 16}.  16 is the passthrough width of outlier layers
 *   ([SKV] §第一层 "异常层处理": kept in 16-bit floating point): the row
 *   holds the bf16 values unchanged (the codes below with bits = 16 are the
 *   bf16 bit patterns), and that tensor has no (scale, zero) -- its sz
 *   pointer is ignored and may be NULL.  A per-layer width policy is a
 *   table on the caller's side: each layer's cache has its own lkv_qspec.
 *
 *   K, V (bf16)  [B][Hkv][T_cap][D]
 *   codes (u8)   [B][Hkv][T_cap][D*bits/8]   one packed row per token:
 *                code j of the row occupies bits [j*bits, (j+1)*bits) of the
 *                row read as one little-endian bit string.
 *   sz (f32)     [B][Hkv][T_cap][ng][2]      (scale, zero) per group.
 *   q (bf16)     [B][Hq][D];  out (f32) [B][Hq][D].
 *
 * Every device pointer must be 16-byte aligned, and T_cap * ng must be even
 * (the per-token (scale, zero) rows are then 16-byte aligned in bulk).
 */
#ifndef LKV_H
#define LKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define LKV_API __attribute__((visibility("default")))
#else
#define LKV_API
#endif

/* Status codes returned by every entry point and kept in the workspace. */
enum lkv_status {
    LKV_OK = 0,
    LKV_ERR_INVALID_ARG = 1, /* null pointer, bad shape, misalignment, bad seq_len */
    LKV_ERR_UNSUPPORTED = 2, /* a shape or bit width this build does not handle */
    LKV_ERR_WORKSPACE = 3,   /* workspace smaller than the *_workspace_bytes query */
    LKV_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
    LKV_ERR_TIMEOUT = 5      /* a bounded cross-block wait gave up (device side) */
};

/* Quantizer settings: bit widths of K and V codes and the group size. */
typedef struct {
    int32_t k_bits; /* 2, 4, 6, 8, or 16 (passthrough bf16, no scale/zero) */
    int32_t v_bits; /* 2, 4, 6, 8, or 16 (passthrough bf16, no scale/zero) */
    int32_t group;  /* 32, 64 or 128; divides D */
} lkv_qspec;

/* One packed cache segment: codes and (scale, zero) for K and V. */
typedef struct {
    void *k_codes;
    float *k_sz;
    void *v_codes;
    float *v_sz;
} lkv_segment;

/* Human-readable name of a status code (static string, never NULL). */
LKV_API const char *lkv_status_string(int status);

/* ABI version of this header (major * 100 + minor). */
LKV_API int lkv_version(void);

/* Bytes of one packed token row: D * bits / 8.  0 for unsupported input. */
LKV_API size_t lkv_row_bytes(int bits, int D);

/* Bytes of one token's (scale, zero) row: 8 * D / group.  0 if unsupported. */
LKV_API size_t lkv_sz_row_bytes(int D, int group);

/*
 * lkv_quantize_kv -- [SKV] §第一层 (K and V at their own widths, asymmetric),
 * [TQ] §核心创新 (group-wise).  For every valid token t < T_b of every
 * (b, kv head) and every group of G channels x_0..x_{G-1}, in fp32 with each
 * operation rounded on its own (no fused multiply-add):
 *   mn = min x_i, mx = max x_i, d = mx - mn, qmax = 2^bits - 1
 *   scale = d / qmax, inv = qmax / d      (both 0 when d == 0)
 *   code_i = clamp(round_half_even((x_i - mn) * inv), 0, qmax)
 *   stored (scale, zero) = (scale, mn + 0.0f)
 * and reconstruction is code * scale + zero.  K uses spec.k_bits, V uses
 * spec.v_bits.  Rows t >= T_b are not written.
 *
 *   k, v       in   bf16 [B][Hkv][T_cap][D]
 *   seq_lens   in   int32 [B] (device)
 *   k_codes    out  u8  [B][Hkv][T_cap][D*k_bits/8]
 *   k_sz       out  f32 [B][Hkv][T_cap][D/group][2]
 *   v_codes    out  u8  [B][Hkv][T_cap][D*v_bits/8]
 *   v_sz       out  f32 [B][Hkv][T_cap][D/group][2]
 */
LKV_API int lkv_quantize_kv(lkv_qspec spec, int B, int Hkv, int T_cap, int D,
                    const int32_t *seq_lens, const void *k, const void *v,
                    void *k_codes, float *k_sz, void *v_codes, float *v_sz,
                    void *stream);

/*
 * lkv_append_kv -- quantize the newest token of every (b, g) into the packed
 * cache in place: the step before decode in a decode loop ([LKV]
 * §实现细节与工程考量: quantization must keep pace with generation).  Row
 * pos[b] of every KV head of sequence b receives the codes and (scale, zero)
 * that lkv_quantize_kv would write for that token; no other row changes.
 *
 *   pos          in   int32 [B], device: the slot to write (normally the
 *                     length before this token); a value outside [0, T_cap)
 *                     writes nothing for that sequence
 *   k_new, v_new in   bf16 [B][Hkv][D]
 *   k_codes...   in/out  the packed cache of lkv_quantize_kv
 */
LKV_API int lkv_append_kv(lkv_qspec spec, int B, int Hkv, int T_cap, int D, const int32_t *pos,
                  const void *k_new, const void *v_new, void *k_codes, float *k_sz, void *v_codes,
                  float *v_sz, void *stream);

/*
 * Paged caches ([TQ] §与其他优化技术的对比: the quantized cache is meant to
 * work with paged KV management).  A page holds LKV_PAGE_TOKENS consecutive
 * tokens of one KV head; the four pools are
 *   codes  [num_pages][Hkv][LKV_PAGE_TOKENS][D * bits / 8]
 *   sz     [num_pages][Hkv][LKV_PAGE_TOKENS][D / group][2]
 * and block_table (int32 [B][pages_per_seq], device) names the page of
 * tokens [i * LKV_PAGE_TOKENS, (i + 1) * LKV_PAGE_TOKENS) of sequence b.
 * The logical capacity is T_cap = pages_per_seq * LKV_PAGE_TOKENS.  Codes,
 * (scale, zero) and all results are those of the contiguous calls on the
 * same tokens.  A page id outside [0, num_pages) makes quantize and append
 * skip that token; the decode reads page 0 instead and sets
 * LKV_ERR_INVALID_ARG in its workspace status word.
 * Returns LKV_ERR_INVALID_ARG for pages_per_seq or num_pages < 1 or a
 * missing block table.
 */
#define LKV_PAGE_TOKENS 256

/* lkv_quantize_kv into a paged cache; k, v are bf16 [B][Hkv][T_cap][D]. */
LKV_API int lkv_quantize_kv_paged(lkv_qspec spec, int B, int Hkv, int pages_per_seq, int num_pages,
                         int D, const int32_t *seq_lens, const void *k, const void *v,
                         const int32_t *block_table, void *k_pool, float *k_sz_pool, void *v_pool,
                         float *v_sz_pool, void *stream);

/* lkv_append_kv into a paged cache (pos[b] is the logical token index). */
LKV_API int lkv_append_kv_paged(lkv_qspec spec, int B, int Hkv, int pages_per_seq, int num_pages,
                         int D, const int32_t *pos, const void *k_new, const void *v_new,
                         const int32_t *block_table, void *k_pool, float *k_sz_pool, void *v_pool,
                         float *v_sz_pool, void *stream);

/*
 * lkv_decode_attention over a paged cache.  Groups of 1, 2 or 4 query heads
 * and widths below 16 bits (LKV_ERR_UNSUPPORTED otherwise).  The workspace is that of
 * lkv_decode_attention with T_cap = pages_per_seq * LKV_PAGE_TOKENS; the
 * skip mask is [B][Hq][T_cap] over logical positions.
 */
LKV_API int lkv_decode_attention_paged(lkv_qspec spec, int B, int Hq, int Hkv, int pages_per_seq,
                         int num_pages, int D, const int32_t *seq_lens, const void *q,
                         const int32_t *block_table, const void *k_pool, const float *k_sz_pool,
                         const void *v_pool, const float *v_sz_pool, float softmax_scale,
                         float tau, float *out, uint8_t *skip_mask, int64_t *skip_counts,
                         void *workspace, size_t ws_bytes, void *stream);

/*
 * Workspace bytes that lkv_decode_attention needs for these sizes on the
 * current device (the size depends on its SM count).  The workspace is
 * caller-owned device memory (256-byte aligned).  It must be zero-filled
 * before its first use (lkv_workspace_reset); every successful call leaves
 * it ready for the next one.  Calls that overlap on the GPU must not share a
 * workspace.  Layout of its first 256 bytes:
 *   bytes [0, 4)   device status word (an lkv_status); a call sets it on a
 *                  device-side error and it stays set until a reset;
 *   bytes [8, 16)  optional limit, in nanoseconds, of every bounded wait of
 *                  the single-launch decode (0 = 2 s).  A wait that runs out
 *                  sets LKV_ERR_TIMEOUT, abandons the rest of the call and
 *                  leaves finite but meaningless outputs; reset the
 *                  workspace before reusing it.
 */
LKV_API size_t lkv_decode_workspace_bytes(lkv_qspec spec, int B, int Hq, int Hkv, int T_cap, int D);

/*
 * lkv_decode_attention -- one decode step of grouped-query attention read
 * straight from the packed cache, with the sparse-V skip of [SKV] §第三层.
 * For every (b, h) with g = h / r and T = T_b:
 *   khat_t, vhat_t = dequantized rows t < T of KV head g
 *   s_t  = softmax_scale * sum_d q[b,h,d] * khat_t[d]
 *   p_t  = exp(s_t - max_u s_u) / sum_u exp(s_u - max_u s_u)
 *   skip_t = p_t < tau        (the V row is never dequantized for this head)
 *   out[b,h,:] = sum_{t : !skip_t} p_t * vhat_t     (no renormalisation)
 * A V row is read from memory only if some head of its group keeps it.
 * T == 0 gives out = 0.  Arithmetic is fp32; the sequence is split into
 * chunks whose partial softmax statistics and outputs are merged exactly.
 *
 *   q            in   bf16 [B][Hq][D]
 *   k_codes...   in   the packed cache written by lkv_quantize_kv
 *   out          out  f32 [B][Hq][D]
 *   skip_mask    out  u8  [B][Hq][T_cap], nullable; 1 = skipped; only t < T_b written
 *   skip_counts  out  int64 [2], nullable; {skipped (b, h, t), V rows skipped
 *                     by every head of their group}
 *   workspace    in/out  lkv_decode_workspace_bytes() bytes, see above
 */
LKV_API int lkv_decode_attention(lkv_qspec spec, int B, int Hq, int Hkv, int T_cap, int D,
                         const int32_t *seq_lens, const void *q, const void *k_codes,
                         const float *k_sz, const void *v_codes, const float *v_sz,
                         float softmax_scale, float tau, float *out, uint8_t *skip_mask,
                         int64_t *skip_counts, void *workspace, size_t ws_bytes,
                         void *stream);

/*
 * lkv_decode_attention_mass -- lkv_decode_attention that also emits, for
 * every token, the attention its KV group paid to it in this step: the
 * input of the next step's lkv_tier_classify ([SKV] §第二层: the attention
 * weights are the signal that ranks tokens into tiers).
 *
 *   mass  out  f32 [B][Hkv][T_cap], not NULL (4-byte aligned):
 *              mass[b][g][t] = (1/r) * sum over the r query heads h of group
 *              g of p[b][h][t], the softmax probability before the sparse-V
 *              skip, for t < T_b; slots t >= T_b are not written.  Over t it
 *              sums to 1 for every (b, g) with T_b > 0.
 * Every other argument and the return value are those of
 * lkv_decode_attention.  Arithmetic is fp32.
 */
LKV_API int lkv_decode_attention_mass(lkv_qspec spec, int B, int Hq, int Hkv, int T_cap, int D,
                         const int32_t *seq_lens, const void *q, const void *k_codes,
                         const float *k_sz, const void *v_codes, const float *v_sz,
                         float softmax_scale, float tau, float *out, uint8_t *skip_mask,
                         int64_t *skip_counts, float *mass, void *workspace, size_t ws_bytes,
                         void *stream);

/*
 * Size of the fixed device scratch that lkv_decode_attention_static uses:
 * 32 MiB on each device.  Whether a shape fits depends on the device, since
 * the decode's scratch layout scales with the SM count: the test is
 * lkv_decode_workspace_bytes(...) <= LKV_STATIC_WORKSPACE_BYTES, called with
 * the target device current.  On a 148-SM B200, B = 16, Hkv = 8,
 * T_cap = 8192, D = 128 with groups of 4 query heads needs about 23 MiB.
 */
#define LKV_STATIC_WORKSPACE_BYTES (32u << 20)

/*
 * lkv_decode_attention_static -- lkv_decode_attention without a caller
 * workspace and without allocating: its scratch is a fixed array of
 * LKV_STATIC_WORKSPACE_BYTES bytes of device memory inside the library, one
 * per device.  The paper has no counterpart; it exists for callers that
 * cannot hand out device memory (a plain-C host with no device allocator,
 * or a process whose memory another allocator has reserved in full).
 * Arguments, outputs and numerics are those of lkv_decode_attention.
 *
 *   status  out  nullable device int32: the call's device-side status (an
 *                lkv_status: LKV_OK, LKV_ERR_INVALID_ARG for a length outside
 *                [0, T_cap], LKV_ERR_TIMEOUT), written on `stream` after the
 *                decode.  Bounded waits use the default 2 s limit.
 *
 * Returns LKV_ERR_WORKSPACE, before enqueueing anything, when the decode
 * needs more than LKV_STATIC_WORKSPACE_BYTES (lkv_decode_workspace_bytes
 * gives the need).  Nothing is allocated or freed.  Each call first clears,
 * on `stream`, the part of the scratch that must start at zero, so an
 * earlier failed call leaves nothing behind.  Every call looks up the
 * scratch's address in the current context (so a device reset or another
 * context is safe); the first one on a device may load the library's device
 * code, so make it before any stream capture.  All calls on one device share
 * the one scratch: calls that overlap on the GPU (other streams, other host
 * threads) race and give wrong results, so order them (one stream, or
 * events).
 */
LKV_API int lkv_decode_attention_static(lkv_qspec spec, int B, int Hq, int Hkv, int T_cap, int D,
                         const int32_t *seq_lens, const void *q, const void *k_codes,
                         const float *k_sz, const void *v_codes, const float *v_sz,
                         float softmax_scale, float tau, float *out, uint8_t *skip_mask,
                         int64_t *skip_counts, int32_t *status, void *stream);

/* Zero-fill a workspace (enqueued on stream). */
LKV_API int lkv_workspace_reset(void *workspace, size_t ws_bytes, void *stream);

/*
 * Copy the workspace status word to *status (an lkv_status), synchronizing
 * `stream` first.  The only synchronizing call of the library.
 */
LKV_API int lkv_workspace_status(const void *workspace, void *stream, int32_t *status);

/*
 * lkv_tier_classify -- [SKV] §第二层 (attention-aware tiers).  From the
 * previous step's attention mass a of each token:
 *   tier 2 (keep, V at 6 bits) if a > tau_high
 *   tier 1 (keep, V at 4 bits) if tau_low <= a <= tau_high
 *   tier 0 (evict K and V)     otherwise (including NaN), and for t >= T_b
 * Then, per (b, kv head), the positions of tier-2 and of tier-1 tokens are
 * listed in ascending order (a stable compaction).
 *
 *   mass    in   f32 [B][Hkv][T_cap]
 *   tier    out  i8  [B][Hkv][T_cap]   all T_cap entries written
 *   counts  out  i32 [B][Hkv][2]       {n2, n1}
 *   pos_a   out  i32 [B][Hkv][T_cap]   first n2 entries: tier-2 positions
 *   pos_b   out  i32 [B][Hkv][T_cap]   first n1 entries: tier-1 positions
 */
LKV_API int lkv_tier_classify(int B, int Hkv, int T_cap, const int32_t *seq_lens, const float *mass,
                      float tau_low, float tau_high, int8_t *tier, int32_t *counts,
                      int32_t *pos_a, int32_t *pos_b, void *stream);

/*
 * lkv_tier_repack -- [SKV] §第二层 items 1 and 2: every kept token is
 * quantized again from its bf16 K and V with the lkv_quantize_kv formula --
 * K at 6 bits in both segments, V at 6 bits in segment A (tier 2) and at 4
 * bits in segment B (tier 1).  Row i of segment A / B of (b, kv head) holds
 * position pos_a / pos_b [b][g][i]; rows i >= the count are not written.
 *
 *   k, v      in   bf16 [B][Hkv][T_cap][D]
 *   counts, pos_a, pos_b   in  as written by lkv_tier_classify
 *   seg_a     out  k_codes u8 [B][Hkv][T_cap][D*6/8], k_sz, v_codes [..][D*6/8], v_sz
 *   seg_b     out  k_codes u8 [B][Hkv][T_cap][D*6/8], k_sz, v_codes [..][D*4/8], v_sz
 */
LKV_API int lkv_tier_repack(int B, int Hkv, int T_cap, int D, int group, const void *k, const void *v,
                    const int32_t *counts, const int32_t *pos_a, const int32_t *pos_b,
                    lkv_segment seg_a, lkv_segment seg_b, void *stream);

/* Workspace bytes for lkv_tiered_attention / lkv_tiered_decode (same rules). */
LKV_API size_t lkv_tiered_workspace_bytes(int B, int Hq, int Hkv, int T_cap, int D, int group);

/*
 * lkv_tiered_attention -- decode attention over the kept tokens only
 * ([SKV] §第二层: evicted tokens are gone): one softmax over segment A
 * (K6, V6) followed by segment B (K6, V4), with the sparse-V skip at tau as
 * in lkv_decode_attention.  n2 + n1 == 0 gives out = 0.
 *
 *   counts   in  i32 [B][Hkv][2]  {rows of segment A, rows of segment B}
 *   q        in  bf16 [B][Hq][D];  out  f32 [B][Hq][D]
 *   skip_counts  nullable int64 [2] as in lkv_decode_attention
 */
LKV_API int lkv_tiered_attention(int B, int Hq, int Hkv, int T_cap, int D, int group,
                         const int32_t *counts, const void *q, lkv_segment seg_a,
                         lkv_segment seg_b, float softmax_scale, float tau, float *out,
                         int64_t *skip_counts, void *workspace, size_t ws_bytes, void *stream);

/*
 * lkv_tiered_decode -- the whole attention-tiered step of [SKV] §第二层 in one
 * call: lkv_tier_classify, then lkv_tier_repack, then lkv_tiered_attention,
 * enqueued in that order on `stream`.  Arguments as in those three calls.
 */
LKV_API int lkv_tiered_decode(int B, int Hq, int Hkv, int T_cap, int D, int group,
                      const int32_t *seq_lens, const float *mass, float tau_low,
                      float tau_high, const void *k, const void *v, const void *q,
                      int8_t *tier, int32_t *counts, int32_t *pos_a, int32_t *pos_b,
                      lkv_segment seg_a, lkv_segment seg_b, float softmax_scale, float tau,
                      float *out, int64_t *skip_counts, void *workspace, size_t ws_bytes,
                      void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LKV_H */
