// lkv_kernels.cuh -- kernel argument blocks and launchers (internal to liblkv).
#pragma once
#include "lkv_device.cuh"

namespace lkv {

struct QuantizeArgs {
  int B, Hkv, T_cap, G;
  float one;  // 1.0f, read at run time by the rounding step of the quantizer
  const int32_t* block_table;  // nullable: contiguous [B][Hkv][T_cap] cache
  int pages_per_seq, num_pages;
  const int32_t* seq_lens;
  const uint16_t* k;
  const uint16_t* v;
  uint8_t* k_codes;
  float* k_sz;
  uint8_t* v_codes;
  float* v_sz;
};

struct RepackArgs {
  int B, Hkv, T_cap, G;
  float one;  // 1.0f, as in QuantizeArgs
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* counts;
  const int32_t* pos_a;
  const int32_t* pos_b;
  uint8_t *a_kc, *a_vc, *b_kc, *b_vc;
  float *a_ksz, *a_vsz, *b_ksz, *b_vsz;
};

struct ClassifyArgs {
  int B, Hkv, T_cap;
  const int32_t* seq_lens;
  const float* mass;
  float tau_low, tau_high;
  int8_t* tier;
  int32_t* counts;
  int32_t* pos_a;
  int32_t* pos_b;
};

// A decode problem: per (b, kv head) up to two packed segments that together
// form one sequence (segment 0 rows first).  Plain decode has one segment of
// seq_lens[b] rows; the tiered cache has segment A (V6) then segment B (V4)
// with counts[b][g][0..1] rows.
struct DecodeArgs {
  int B, Hq, Hkv, T_cap, G;
  int r;                 // Hq / Hkv
  const int32_t* lens;   // seq_lens [B] (len_mode 0) or counts [B][Hkv][2] (len_mode 1)
  int len_mode;
  const uint16_t* q;
  const uint8_t* kc[2];
  const float* ksz[2];
  const uint8_t* vc[2];
  const float* vsz[2];
  float q_scale;         // softmax_scale * log2(e): logits are kept in base 2
  float tau;
  float* out;
  uint8_t* skip_mask;    // nullable, [B][Hq][T_cap] (plain decode only)
  float* mass;           // nullable, [B][Hkv][T_cap]: mean over the group's heads of p (plain decode only)
  unsigned long long* skip_counts;  // nullable, [2]
  // workspace
  int* status;
  int chunk;             // rows per chunk
  int n_chunks;          // chunks per (b, g) = ceil(2 * T_cap / chunk) for two segments
  float* logits;         // [B][Hkv][n_chunks * chunk][r]
  float* stats;          // [B][Hkv][n_chunks][r][2]  (max, sum of exp2)
  float* partial;        // [B][Hkv][n_chunks][r][D]
};

// Single-launch decode (fused_impl.cuh): DecodeArgs plus its workspace.
struct FusedArgs {
  DecodeArgs d;
  int cpc_max;                   // upper bound of chunks per CTA
  int stages;                    // ring stages in use
  int ring_bytes;                // shared-memory ring size
  int cand_cap;                  // sparse mode: kept rows one CTA can list (0: sparse mode off)
  long long smem_logit_floats;   // logits that fit in shared memory per CTA
  const unsigned long long* timeout_ns;  // workspace word: wait limit override (0 = default)
  int* arrive1;                  // [units] piece statistics published
  int* arrive2;                  // [units] partial outputs published
  float* pstats;                 // [grid][2][H][2]
  float* ppart;                  // [grid][2][H][D]
  float* wslot;                  // [grid][kWarps][H][D] sparse mode: a warp's first piece when its share holds more than one
  float* cstats;                 // [chunks][H][2]
  int* ulist;                    // [grid][cpc_max][16]
  float* glogits;                // [grid][cpc_max * chunk][H] (when shared memory is short)
  float* gstats;                 // [grid][cpc_max * 8][12] tile statistics (when there are many tiles)
  float* qbuf;                   // [units][H][D] fp16 q scaled by a power of two (units past the shared slots)
  float* qgsum;                  // [units][H][8] fold constants: q_scale * group sums of q [4], q_scale * 2^-E
  unsigned long long* wcounts;   // [2] skip-count accumulators
  int* done;                     // CTAs finished
  // paged cache (plain decode only): block table [B][pages_per_seq], T_cap = pages_per_seq * kPageTokens
  const int32_t* block_table;
  int pages_per_seq, num_pages;
};

// Dispatch on (D, H, V widths) for one K width; smem = dynamic shared bytes.
cudaError_t launch_fused_k2(const FusedArgs& a, int D, int H, int vb0, int vb1, size_t smem, int grid, cudaStream_t s);
cudaError_t launch_fused_k4(const FusedArgs& a, int D, int H, int vb0, int vb1, size_t smem, int grid, cudaStream_t s);
cudaError_t launch_fused_k6(const FusedArgs& a, int D, int H, int vb0, int vb1, size_t smem, int grid, cudaStream_t s);
cudaError_t launch_fused_k8(const FusedArgs& a, int D, int H, int vb0, int vb1, size_t smem, int grid, cudaStream_t s);
cudaError_t launch_fused_k16(const FusedArgs& a, int D, int H, int vb0, int vb1, size_t smem, int grid, cudaStream_t s);
// The same over a paged cache (plain decode: one V width).
cudaError_t launch_fused_paged_k2(const FusedArgs& a, int D, int H, int vb, size_t smem, int grid, cudaStream_t s);
cudaError_t launch_fused_paged_k4(const FusedArgs& a, int D, int H, int vb, size_t smem, int grid, cudaStream_t s);
cudaError_t launch_fused_paged_k6(const FusedArgs& a, int D, int H, int vb, size_t smem, int grid, cudaStream_t s);
cudaError_t launch_fused_paged_k8(const FusedArgs& a, int D, int H, int vb, size_t smem, int grid, cudaStream_t s);

int num_sms();

cudaError_t launch_quantize_kv(const QuantizeArgs& a, int kb, int vb, int D, cudaStream_t s);
// seq_lens holds the slot to write per sequence; k, v hold [B][Hkv][D].
cudaError_t launch_append_kv(const QuantizeArgs& a, int kb, int vb, int D, cudaStream_t s);
cudaError_t launch_tier_repack(const RepackArgs& a, int D, cudaStream_t s);
cudaError_t launch_tier_classify(const ClassifyArgs& a, cudaStream_t s);
// vb0 / vb1: V bit widths of segment 0 / 1 (equal for plain decode).
cudaError_t launch_decode(const DecodeArgs& a, int D, int kb, int vb0, int vb1, cudaStream_t s);

}  // namespace lkv
