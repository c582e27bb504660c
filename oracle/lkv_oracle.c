/*
 * lkv_oracle.c -- plain, slow CPU oracle for the quantized-KV decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code, header or constant table with
 * the CUDA library: the packed format is re-derived here from its definition.
 *
 * Sources (web pages, cited by title and section):
 *   [SKV]  "Super KV Compression: 突破LLM推理内存瓶颈的三层压缩架构解析"
 *          §第一层：自适应非对称量化 (K at 6 bits, V at 4 bits, asymmetric),
 *          §第二层：注意力感知的Token淘汰机制 (three attention tiers),
 *          §第三层：稀疏V跳过加速 (skip dequantization of low-attention V).
 *   [TQ]   "TurboQuant：将LLM KV缓存压缩5-7倍的突破性技术"
 *          §TurboQuant的核心创新 (asymmetric + group-wise quantization).
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes): a group is G contiguous head_dim channels of one token; the
 * zero-point is the group minimum stored as an fp32 offset; codes use one
 * division per group and round half to even; bits are packed LSB-first per
 * token row; skipped probability mass is dropped, not renormalised; a
 * sequence with no tokens attends to nothing and yields zeros.
 *
 * Precision: the quantizer is an encoding and runs in fp32 with every
 * operation rounded separately (compile with -ffp-contract=off, never
 * -ffast-math).  Attention is an exact definition and runs in fp64.
 *
 * Parity status: every function below is pinned by tests that do not route
 * through this file alone (closed forms, brute force, a float64 library
 * softmax, values the pages print).
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1

/* bf16 is the upper half of an IEEE binary32, so widening is exact. */
static float bf16_to_float(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* 16 is the passthrough width of [SKV] §第一层 "异常层处理" (outlier layers
 * kept in 16-bit floating point): the row holds the bf16 values unchanged,
 * with no (scale, zero). */
static int bits_supported(int bits)
{
    return bits == 2 || bits == 4 || bits == 6 || bits == 8 || bits == 16;
}

/* Bytes of one packed token row: D codes of `bits` bits each. */
long long lkv_oracle_row_bytes(int bits, int D)
{
    return (long long)D * bits / 8;
}

/*
 * Asymmetric min-max quantization of one group ([SKV] §第一层, [TQ]
 * §核心创新 "非对称量化和分组量化"):
 *   1. mn, mx = smallest and largest value of the group;
 *   2. d = mx - mn, qmax = 2^bits - 1;
 *   3. scale = d / qmax and inv = qmax / d (0 and 0 when d == 0);
 *   4. code_i = clamp(round_half_even((x_i - mn) * inv), 0, qmax);
 *   5. the record is (scale, zero) with zero = mn (+0.0 makes a minus zero
 *      into plus zero, so the stored bits do not depend on which of two
 *      equal zeros was found first).
 * Two ranges of finite values leave fp32 in steps 3-4 and take the same
 * formula on exactly rescaled values (each step rounded on its own):
 *   - d so small that qmax / d overflows: the differences and d are
 *     scaled by 2^64 first, inv = qmax / (d * 2^64) and
 *     code_i = round((x_i - mn) * 2^64 * inv); scale = d / qmax as above;
 *   - d itself overflowing (mx - mn above the largest float): the group is
 *     quantized at half size, d_h = mx/2 - mn/2, inv = qmax / d_h,
 *     code_i = round((x_i/2 - mn/2) * inv), and scale = (d_h / qmax) * 2.
 * Both keep |x - xhat| <= scale / 2 (up to the fp32 rounding of the
 * formula) and the group minimum's exact reconstruction for every finite
 * group.
 */
void lkv_oracle_quantize_group(const float *x, int n, int bits,
                               uint32_t *codes, float *scale_out, float *zero_out)
{
    float mn = x[0], mx = x[0];
    for (int i = 1; i < n; ++i) {
        if (x[i] < mn) mn = x[i];
        if (x[i] > mx) mx = x[i];
    }
    const float qmax = (float)((1u << bits) - 1u);
    const float d = mx - mn;
    float scale = 0.0f, inv = 0.0f;
    int regime = 0;              /* 0: as written; 1: tiny range; 2: huge range */
    const float two64 = 18446744073709551616.0f;
    float mnh = 0.0f;
    if (d != 0.0f) {
        scale = d / qmax;
        inv = qmax / d;
        if (d > FLT_MAX) {               /* mx - mn overflowed */
            const float dh = mx * 0.5f - mn * 0.5f;
            mnh = mn * 0.5f;
            scale = (dh / qmax) * 2.0f;
            inv = qmax / dh;
            regime = 2;
        } else if (inv > FLT_MAX) {      /* qmax / d overflowed */
            inv = qmax / (d * two64);
            regime = 1;
        }
    }
    for (int i = 0; i < n; ++i) {
        float y;
        if (regime == 1) {
            float diff = x[i] - mn;
            float big = diff * two64;
            y = big * inv;
        } else if (regime == 2) {
            float half = x[i] * 0.5f;
            float diff = half - mnh;
            y = diff * inv;
        } else {
            float diff = x[i] - mn;
            y = diff * inv;
        }
        float r = nearbyintf(y); /* default rounding mode: half to even */
        if (!(r >= 0.0f)) r = 0.0f; /* also NaN (inputs outside the contract) */
        if (r > qmax) r = qmax;
        codes[i] = (uint32_t)r;
    }
    *scale_out = scale;
    *zero_out = mn + 0.0f;
}

/* Reconstruction of one code: code * scale + zero, rounded once to fp32
 * (a product that does not fit fp32 on its own -- the group maximum of a
 * range wider than the largest float -- still gives a finite value). */
float lkv_oracle_dequant(uint32_t code, float scale, float zero)
{
    return fmaf((float)code, scale, zero);
}

/*
 * Bit packing of one token row: code j occupies bits [j*bits, (j+1)*bits) of
 * the row read as one little-endian bit string (bit k of byte i is string
 * bit 8*i + k).  The pages only ask that the cache layout be reorganised for
 * the quantized format (LeanKV, §实现细节与工程考量); this order is our choice.
 */
void lkv_oracle_pack_row(const uint32_t *codes, int D, int bits, uint8_t *row)
{
    const long long nbytes = lkv_oracle_row_bytes(bits, D);
    memset(row, 0, (size_t)nbytes);
    for (int j = 0; j < D; ++j) {
        for (int k = 0; k < bits; ++k) {
            long long s = (long long)j * bits + k;
            uint32_t bit = (codes[j] >> k) & 1u;
            row[s / 8] |= (uint8_t)(bit << (s % 8));
        }
    }
}

void lkv_oracle_unpack_row(const uint8_t *row, int D, int bits, uint32_t *codes)
{
    for (int j = 0; j < D; ++j) {
        uint32_t c = 0;
        for (int k = 0; k < bits; ++k) {
            long long s = (long long)j * bits + k;
            uint32_t bit = (row[s / 8] >> (s % 8)) & 1u;
            c |= bit << k;
        }
        codes[j] = c;
    }
}

/* Quantize and pack one token row of D bf16 values in groups of G.  At the
 * passthrough width the "code" of a value is its own bf16 bit pattern and
 * sz_row is not touched. */
static void quantize_row(const uint16_t *src, int D, int G, int bits,
                         uint8_t *codes_row, float *sz_row)
{
    float xs[256];
    uint32_t cs[256];
    if (bits == 16) {
        for (int d = 0; d < D; ++d) cs[d] = src[d];
        lkv_oracle_pack_row(cs, D, bits, codes_row);
        return;
    }
    for (int d = 0; d < D; ++d) xs[d] = bf16_to_float(src[d]);
    for (int g = 0; g < D / G; ++g) {
        lkv_oracle_quantize_group(xs + g * G, G, bits, cs + g * G,
                                  &sz_row[2 * g], &sz_row[2 * g + 1]);
    }
    lkv_oracle_pack_row(cs, D, bits, codes_row);
}

/* Dequantize one packed token row into D floats. */
static void dequant_row(const uint8_t *codes_row, const float *sz_row, int D, int G,
                        int bits, float *out)
{
    uint32_t cs[256];
    lkv_oracle_unpack_row(codes_row, D, bits, cs);
    if (bits == 16) {  /* passthrough: the bf16 value itself */
        for (int d = 0; d < D; ++d) out[d] = bf16_to_float((uint16_t)cs[d]);
        return;
    }
    for (int d = 0; d < D; ++d) {
        int g = d / G;
        out[d] = lkv_oracle_dequant(cs[d], sz_row[2 * g], sz_row[2 * g + 1]);
    }
}

static int shape_ok(int bits, int G, int D)
{
    return bits_supported(bits) && G > 0 && D > 0 && D <= 256 && D % G == 0 &&
           (D * bits) % 8 == 0;
}

/* Dequantize n consecutive packed rows (codes [n][row_bytes], sz [n][D/G][2]). */
int lkv_oracle_dequant_rows(const uint8_t *codes, const float *sz, long long n, int D, int G,
                            int bits, float *out)
{
    if (!shape_ok(bits, G, D) || n < 0) return ORACLE_BAD_ARG;
    const long long rb = lkv_oracle_row_bytes(bits, D);
    const int ng = D / G;
    for (long long i = 0; i < n; ++i)
        dequant_row(codes + i * rb, sz + i * ng * 2, D, G, bits, out + i * D);
    return ORACLE_OK;
}

/*
 * Quantize the valid rows (t < seq_lens[b]) of K and V, laid out
 * [B][Hkv][T_cap][D] in bf16, into packed codes [B][Hkv][T_cap][row_bytes]
 * and (scale, zero) pairs [B][Hkv][T_cap][D/G][2].  Rows t >= seq_lens[b]
 * are left as they are.
 */
int lkv_oracle_quantize_kv(int kb, int vb, int G, int B, int Hkv, int T_cap, int D,
                           const int32_t *seq_lens, const uint16_t *k, const uint16_t *v,
                           uint8_t *k_codes, float *k_sz, uint8_t *v_codes, float *v_sz)
{
    if (!shape_ok(kb, G, D) || !shape_ok(vb, G, D) || B < 0 || Hkv <= 0 || T_cap < 0)
        return ORACLE_BAD_ARG;
    const long long kr = lkv_oracle_row_bytes(kb, D), vr = lkv_oracle_row_bytes(vb, D);
    const int ng = D / G;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long u = 0; u < (long long)B * Hkv; ++u) {
        const int b = (int)(u / Hkv);
        const int T = seq_lens[b];
        for (int t = 0; t < T && t < T_cap; ++t) {
            long long row = u * T_cap + t;
            quantize_row(k + row * D, D, G, kb, k_codes + row * kr, k_sz + row * ng * 2);
            quantize_row(v + row * D, D, G, vb, v_codes + row * vr, v_sz + row * ng * 2);
        }
    }
    return ORACLE_OK;
}

/*
 * Softmax attention of one query head over n dequantized rows, in fp64,
 * with the sparse-V skip of [SKV] §第三层: a row whose probability is below
 * tau contributes nothing (its V is never dequantized) and the kept mass is
 * not renormalised.  k_rows/v_rows point at row i via a row stride; rows can
 * come from two segments, so the caller passes per-row pointers.
 *
 *   s_t = softmax_scale * sum_d q_d * khat_{t,d}
 *   p_t = exp(s_t - max s) / sum_u exp(s_u - max s)
 *   out = sum_{t : p_t >= tau} p_t * vhat_t
 *
 * skip[t] receives 1 for a skipped row and 0 otherwise; p_out (nullable)
 * receives p_t.  With n == 0 the output is all zeros.
 */
static void attend_one_head(const float *qf, int D, int n, const float *const *khat,
                            const float *const *vhat, float softmax_scale, float tau,
                            double *s_buf, float *out, uint8_t *skip, double *p_out)
{
    double acc[256];
    for (int d = 0; d < D; ++d) acc[d] = 0.0;
    if (n > 0) {
        double m = -INFINITY;
        for (int t = 0; t < n; ++t) {
            double dot = 0.0;
            for (int d = 0; d < D; ++d) dot += (double)qf[d] * (double)khat[t][d];
            s_buf[t] = (double)softmax_scale * dot;
            if (s_buf[t] > m) m = s_buf[t];
        }
        double l = 0.0;
        for (int t = 0; t < n; ++t) l += exp(s_buf[t] - m);
        for (int t = 0; t < n; ++t) {
            double p = exp(s_buf[t] - m) / l;
            int skipped = p < (double)tau;
            if (skip) skip[t] = (uint8_t)skipped;
            if (p_out) p_out[t] = p;
            if (!skipped)
                for (int d = 0; d < D; ++d) acc[d] += p * (double)vhat[t][d];
        }
    }
    for (int d = 0; d < D; ++d) out[d] = (float)acc[d];
}

/*
 * Grouped-query decode attention over the packed cache.  Query head h reads
 * KV head h / (Hq / Hkv).  q is bf16 [B][Hq][D]; out is f32 [B][Hq][D];
 * skip_mask (nullable) is u8 [B][Hq][T_cap] and only entries t < T_b are
 * written; skip_counts (nullable) receives {skipped (b, h, t) triples,
 * V rows skipped by every head of their group}; p_out (nullable) is f64
 * [B][Hq][T_cap] and receives the probabilities p_t for t < T_b.
 */
int lkv_oracle_decode_attention(int kb, int vb, int G, int B, int Hq, int Hkv, int T_cap,
                                int D, const int32_t *seq_lens, const uint16_t *q,
                                const uint8_t *k_codes, const float *k_sz,
                                const uint8_t *v_codes, const float *v_sz,
                                float softmax_scale, float tau, float *out,
                                uint8_t *skip_mask, int64_t *skip_counts, double *p_out)
{
    if (!shape_ok(kb, G, D) || !shape_ok(vb, G, D) || Hkv <= 0 || Hq % Hkv != 0 || B < 0)
        return ORACLE_BAD_ARG;
    const int r = Hq / Hkv, ng = D / G;
    const long long kr = lkv_oracle_row_bytes(kb, D), vr = lkv_oracle_row_bytes(vb, D);
    long long skipped_heads = 0, skipped_rows = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : skipped_heads, skipped_rows)
    for (long long u = 0; u < (long long)B * Hkv; ++u) {
        const int b = (int)(u / Hkv), g = (int)(u % Hkv);
        int T = seq_lens[b];
        if (T > T_cap) T = T_cap;
        if (T < 0) T = 0;
        float *kh = malloc(sizeof(float) * (size_t)(T > 0 ? T : 1) * D);
        float *vh = malloc(sizeof(float) * (size_t)(T > 0 ? T : 1) * D);
        const float **kp = malloc(sizeof(float *) * (size_t)(T > 0 ? T : 1));
        const float **vp = malloc(sizeof(float *) * (size_t)(T > 0 ? T : 1));
        double *s = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        uint8_t *sk = malloc((size_t)(T > 0 ? T : 1) * r);
        for (int t = 0; t < T; ++t) {
            long long row = u * T_cap + t;
            dequant_row(k_codes + row * kr, k_sz + row * ng * 2, D, G, kb, kh + (long long)t * D);
            dequant_row(v_codes + row * vr, v_sz + row * ng * 2, D, G, vb, vh + (long long)t * D);
            kp[t] = kh + (long long)t * D;
            vp[t] = vh + (long long)t * D;
        }
        for (int j = 0; j < r; ++j) {
            const int h = g * r + j;
            float qf[256];
            for (int d = 0; d < D; ++d) qf[d] = bf16_to_float(q[((long long)b * Hq + h) * D + d]);
            attend_one_head(qf, D, T, kp, vp, softmax_scale, tau, s,
                            out + ((long long)b * Hq + h) * D, sk + (long long)j * (T > 0 ? T : 1),
                            p_out ? p_out + ((long long)b * Hq + h) * T_cap : NULL);
            if (skip_mask)
                for (int t = 0; t < T; ++t)
                    skip_mask[((long long)b * Hq + h) * T_cap + t] = sk[(long long)j * (T > 0 ? T : 1) + t];
        }
        for (int t = 0; t < T; ++t) {
            int all = 1;
            for (int j = 0; j < r; ++j) {
                int sj = sk[(long long)j * (T > 0 ? T : 1) + t];
                skipped_heads += sj;
                all &= sj;
            }
            skipped_rows += all;
        }
        free(kh); free(vh); free(kp); free(vp); free(s); free(sk);
    }
    if (skip_counts) {
        skip_counts[0] = skipped_heads;
        skip_counts[1] = skipped_rows;
    }
    return ORACLE_OK;
}

/*
 * Attention-aware tiers ([SKV] §第二层): with a the previous step's
 * attention mass of a token,
 *   tier 2 (keep, V at 6 bits)  if a > tau_high,
 *   tier 1 (keep, V at 4 bits)  if tau_low <= a <= tau_high,
 *   tier 0 (evict K and V)      otherwise (a < tau_low, or a is NaN).
 * Positions t >= T_b get tier 0.  counts[b][g] = {n2, n1}; pos2 / pos1 list
 * the positions of each kept tier in ascending order (first n entries).
 */
int lkv_oracle_tier_classify(int B, int Hkv, int T_cap, const int32_t *seq_lens,
                             const float *mass, float tau_low, float tau_high, int8_t *tier,
                             int32_t *counts, int32_t *pos2, int32_t *pos1)
{
    if (B < 0 || Hkv <= 0 || T_cap < 0) return ORACLE_BAD_ARG;
    for (long long u = 0; u < (long long)B * Hkv; ++u) {
        const int b = (int)(u / Hkv);
        const int T = seq_lens[b];
        int n2 = 0, n1 = 0;
        for (int t = 0; t < T_cap; ++t) {
            const long long i = u * T_cap + t;
            int8_t c = 0;
            if (t < T) {
                const float a = mass[i];
                if (a > tau_high) c = 2;
                else if (a >= tau_low && a <= tau_high) c = 1;
                else c = 0;
            }
            tier[i] = c;
            if (c == 2) pos2[u * T_cap + n2++] = t;
            if (c == 1) pos1[u * T_cap + n1++] = t;
        }
        counts[2 * u] = n2;
        counts[2 * u + 1] = n1;
    }
    return ORACLE_OK;
}

/*
 * Tier repack ([SKV] §第二层 items 1-2): every kept token is quantized again
 * from its bf16 K and V with the group quantizer above -- K at 6 bits in both
 * segments, V at 6 bits in segment A (tier 2) and at 4 bits in segment B
 * (tier 1).  Segment row i of (b, g) holds position pos[b][g][i].
 */
int lkv_oracle_tier_repack(int B, int Hkv, int T_cap, int D, int G, const uint16_t *k,
                           const uint16_t *v, const int32_t *counts, const int32_t *pos2,
                           const int32_t *pos1, uint8_t *a_kc, float *a_ksz, uint8_t *a_vc,
                           float *a_vsz, uint8_t *b_kc, float *b_ksz, uint8_t *b_vc,
                           float *b_vsz)
{
    if (!shape_ok(6, G, D) || !shape_ok(4, G, D) || B < 0 || Hkv <= 0) return ORACLE_BAD_ARG;
    const int ng = D / G;
    const long long r6 = lkv_oracle_row_bytes(6, D), r4 = lkv_oracle_row_bytes(4, D);
    for (long long u = 0; u < (long long)B * Hkv; ++u) {
        for (int i = 0; i < counts[2 * u]; ++i) {
            const long long src = u * T_cap + pos2[u * T_cap + i], dst = u * T_cap + i;
            quantize_row(k + src * D, D, G, 6, a_kc + dst * r6, a_ksz + dst * ng * 2);
            quantize_row(v + src * D, D, G, 6, a_vc + dst * r6, a_vsz + dst * ng * 2);
        }
        for (int i = 0; i < counts[2 * u + 1]; ++i) {
            const long long src = u * T_cap + pos1[u * T_cap + i], dst = u * T_cap + i;
            quantize_row(k + src * D, D, G, 6, b_kc + dst * r6, b_ksz + dst * ng * 2);
            quantize_row(v + src * D, D, G, 4, b_vc + dst * r4, b_vsz + dst * ng * 2);
        }
    }
    return ORACLE_OK;
}

/*
 * Decode attention over the kept tokens only: one softmax over segment A
 * (K6, V6) together with segment B (K6, V4); evicted tokens are absent.
 * The sparse-V skip at tau applies as in plain decode.
 */
int lkv_oracle_tiered_attention(int B, int Hq, int Hkv, int T_cap, int D, int G,
                                const int32_t *counts, const uint16_t *q,
                                const uint8_t *a_kc, const float *a_ksz, const uint8_t *a_vc,
                                const float *a_vsz, const uint8_t *b_kc, const float *b_ksz,
                                const uint8_t *b_vc, const float *b_vsz, float softmax_scale,
                                float tau, float *out, int64_t *skip_counts, double *p_out)
{
    if (!shape_ok(6, G, D) || !shape_ok(4, G, D) || Hkv <= 0 || Hq % Hkv != 0 || B < 0)
        return ORACLE_BAD_ARG;
    const int r = Hq / Hkv, ng = D / G;
    const long long r6 = lkv_oracle_row_bytes(6, D), r4 = lkv_oracle_row_bytes(4, D);
    long long skipped_heads = 0, skipped_rows = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : skipped_heads, skipped_rows)
    for (long long u = 0; u < (long long)B * Hkv; ++u) {
        const int b = (int)(u / Hkv), g = (int)(u % Hkv);
        const int na = counts[2 * u], nb = counts[2 * u + 1], n = na + nb;
        const size_t cap = (size_t)(n > 0 ? n : 1);
        float *kh = malloc(sizeof(float) * cap * D);
        float *vh = malloc(sizeof(float) * cap * D);
        const float **kp = malloc(sizeof(float *) * cap);
        const float **vp = malloc(sizeof(float *) * cap);
        double *s = malloc(sizeof(double) * cap);
        uint8_t *sk = malloc(cap * r);
        for (int i = 0; i < n; ++i) {
            const int in_a = i < na;
            const long long row = u * T_cap + (in_a ? i : i - na);
            dequant_row((in_a ? a_kc : b_kc) + row * r6, (in_a ? a_ksz : b_ksz) + row * ng * 2,
                        D, G, 6, kh + (long long)i * D);
            if (in_a)
                dequant_row(a_vc + row * r6, a_vsz + row * ng * 2, D, G, 6, vh + (long long)i * D);
            else
                dequant_row(b_vc + row * r4, b_vsz + row * ng * 2, D, G, 4, vh + (long long)i * D);
            kp[i] = kh + (long long)i * D;
            vp[i] = vh + (long long)i * D;
        }
        for (int j = 0; j < r; ++j) {
            const int h = g * r + j;
            float qf[256];
            for (int d = 0; d < D; ++d) qf[d] = bf16_to_float(q[((long long)b * Hq + h) * D + d]);
            attend_one_head(qf, D, n, kp, vp, softmax_scale, tau, s,
                            out + ((long long)b * Hq + h) * D, sk + (size_t)j * cap,
                            p_out ? p_out + ((long long)b * Hq + h) * T_cap : NULL);
        }
        for (int i = 0; i < n; ++i) {
            int all = 1;
            for (int j = 0; j < r; ++j) {
                int sj = sk[(size_t)j * cap + i];
                skipped_heads += sj;
                all &= sj;
            }
            skipped_rows += all;
        }
        free(kh); free(vh); free(kp); free(vp); free(s); free(sk);
    }
    if (skip_counts) {
        skip_counts[0] = skipped_heads;
        skip_counts[1] = skipped_rows;
    }
    return ORACLE_OK;
}

/*
 * Softmax attention over the unquantized bf16 cache, in fp64: the quantity
 * the quantized decode approximates ([SKV] §第一层 judges K6V4 by the
 * change it makes to the model's output; [TQ] §TurboQuant的核心创新).
 * Query head h reads KV head h / (Hq / Hkv); k, v are bf16 [B][Hkv][T_cap][D];
 * out is f32 [B][Hq][D].  No skip: every row contributes.
 */
int lkv_oracle_attention_bf16(int B, int Hq, int Hkv, int T_cap, int D,
                              const int32_t *seq_lens, const uint16_t *q, const uint16_t *k,
                              const uint16_t *v, float softmax_scale, float *out)
{
    if (Hkv <= 0 || Hq % Hkv != 0 || B < 0 || D <= 0 || D > 256) return ORACLE_BAD_ARG;
    const int r = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long u = 0; u < (long long)B * Hkv; ++u) {
        const int b = (int)(u / Hkv), g = (int)(u % Hkv);
        int T = seq_lens[b];
        if (T > T_cap) T = T_cap;
        if (T < 0) T = 0;
        float *kh = malloc(sizeof(float) * (size_t)(T > 0 ? T : 1) * D);
        float *vh = malloc(sizeof(float) * (size_t)(T > 0 ? T : 1) * D);
        const float **kp = malloc(sizeof(float *) * (size_t)(T > 0 ? T : 1));
        const float **vp = malloc(sizeof(float *) * (size_t)(T > 0 ? T : 1));
        double *s = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        for (int t = 0; t < T; ++t) {
            const long long row = (u * T_cap + t) * D;
            for (int d = 0; d < D; ++d) {
                kh[(long long)t * D + d] = bf16_to_float(k[row + d]);
                vh[(long long)t * D + d] = bf16_to_float(v[row + d]);
            }
            kp[t] = kh + (long long)t * D;
            vp[t] = vh + (long long)t * D;
        }
        for (int j = 0; j < r; ++j) {
            const int h = g * r + j;
            float qf[256];
            for (int d = 0; d < D; ++d) qf[d] = bf16_to_float(q[((long long)b * Hq + h) * D + d]);
            attend_one_head(qf, D, T, kp, vp, softmax_scale, 0.0f, s,
                            out + ((long long)b * Hq + h) * D, NULL, NULL);
        }
        free(kh); free(vh); free(kp); free(vp); free(s);
    }
    return ORACLE_OK;
}

/* Thread count of the parallel loops above (the CPU baseline times the
 * oracle both on every core and on one). */
void lkv_oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int lkv_oracle_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
