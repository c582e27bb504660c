// api.cu -- the extern "C" entry points of liblkv (declared in include/lkv.h):
// host-side validation, workspace carving and kernel launches.  Nothing here
// allocates device memory or synchronizes (except lkv_workspace_status).
#include <cmath>
#include <cstdint>
#include <cstring>

#include "../../include/lkv.h"
#include <algorithm>

#include "fused_impl.cuh"
#include "lkv_kernels.cuh"

namespace lkv {

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

namespace {

constexpr int kChunk = 256;       // decode rows per chunk
constexpr size_t kAlign = 256;
constexpr size_t kHeaderBytes = 256;  // status, wait limit, done counter, skip-count accumulators

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// 16 is the passthrough width: the row holds the bf16 values, with no (scale, zero)
bool bits_ok(int b) { return b == 2 || b == 4 || b == 6 || b == 8 || b == 16; }
bool dim_ok(int D) { return D == 64 || D == 128; }
bool group_ok(int G, int D) { return (G == 32 || G == 64 || G == 128) && G <= D && D % G == 0; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// A pointer that must be valid when its tensor is non-empty.
bool ptr_ok(const void* p, bool nonempty) { return !nonempty || (p != nullptr && aligned16(p)); }

int from_cuda(cudaError_t e) { return e == cudaSuccess ? LKV_OK : LKV_ERR_CUDA; }

struct WsLayout {
  size_t status, logits, stats, partial, total;
  int n_chunks;
};

WsLayout ws_layout(int B, int Hq, int Hkv, int T_cap, int D) {
  WsLayout w{};
  const int r = Hq / Hkv;
  w.n_chunks = T_cap > 0 ? (T_cap + kChunk - 1) / kChunk : 1;
  const size_t units = (size_t)B * (size_t)Hkv;
  w.status = 0;
  w.logits = kHeaderBytes;
  w.stats = w.logits + align_up(units * (size_t)T_cap * r * sizeof(float));
  w.partial = w.stats + align_up(units * (size_t)w.n_chunks * r * 2 * sizeof(float));
  w.total = w.partial + align_up(units * (size_t)w.n_chunks * r * D * sizeof(float));
  return w;
}

// The single-launch decode handles GQA groups of 1, 2 or 4 query heads.
bool fused_ok(int r) { return r == 1 || r == 2 || r == 4; }

struct FusedLayout {
  int grid, H, cpc_max, ring_bytes, stages, cand_cap;
  size_t smem_bytes;
  size_t arrive1, arrive2, pstats, ppart, wslot, ulist, glogits, gstats, qbuf, qgsum, total;
  bool need_gstats;
};

constexpr int kMaxSmem = 227 * 1024;  // dynamic shared memory of one CTA on sm_100

FusedLayout fused_layout(int B, int Hq, int Hkv, int T_cap, int D, int KB) {
  FusedLayout L{};
  L.grid = num_sms();
  L.H = Hq / Hkv;
  const long long units = (long long)B * Hkv;
  // A little fewer units than SMs: one CTA per unit instead of all SMs.  With
  // equal lengths every unit is then owned by one CTA, which saves the
  // exchange of statistics and partial outputs between CTAs (worth more
  // than the idle SMs cost the bandwidth-bound first phase).
  if (units >= (3 * L.grid) / 4 && units < L.grid) L.grid = (int)units;
  // each segment rounds up to whole chunks: at most one more chunk per unit
  const long long per_unit = T_cap > 0 ? (T_cap + kChunk - 1) / kChunk + 1 : 1;
  const long long chunks_max = units * per_unit > 0 ? units * per_unit : 1;
  L.cpc_max = (int)((chunks_max + L.grid - 1) / L.grid);
  // phase 1: as many ring stages as shared memory holds (at most kMaxStages);
  // phase 2 reuses the ring: the sparse-mode list of kept rows (2048 per
  // CTA), one partial output per warp and V staging slots, the fallback
  // scan's lists, or the dense-mode buffers, each followed by the warps'
  // partial outputs
  const int sb = fused::stage_bytes_host(D, KB);
  const int red = fused::kWarps * L.H * D * 4;
  const int slot = D * 8 / 8 + 8 * std::max(2, D / 32);  // widest V row plus (scale, zero)
  int lcap = 2048;  // kept rows one CTA can list (more fall back to a per-piece scan)
  if ((long long)L.cpc_max * kChunk >= (1ll << fused::kCandRowBits) || L.cpc_max >= 2048) lcap = 0;
  const int sparse = (lcap * (1 + L.H) * 4 + 127) / 128 * 128 + red + 128 * slot;
  const int scan_fb = fused::kWarps * fused::kListCap * 4 * (1 + L.H) + red;
  const int dense = fused::kDenseStaging + red;
  const int phase2 = std::max(sparse, std::max(scan_fb, dense));
  L.stages = std::min(fused::kMaxStages, (kMaxSmem - fused::kHeader) / sb);
  L.ring_bytes = (std::max(L.stages * sb, phase2) + 127) / 128 * 128;
  L.cand_cap = lcap;
  L.smem_bytes = fused::kHeader + L.ring_bytes;
  const int tpc = fused::kTilesPerChunk;
  L.need_gstats = (long long)L.cpc_max * tpc > fused::kTsCap;
  size_t off = kHeaderBytes;
  L.arrive1 = off; off = align_up(off + units * 4);
  L.arrive2 = off; off = align_up(off + units * 4);
  L.pstats = off; off = align_up(off + (size_t)L.grid * 2 * L.H * 2 * 4);
  L.ppart = off; off = align_up(off + (size_t)L.grid * 2 * L.H * D * 4);
  L.wslot = off; off = align_up(off + (size_t)L.grid * fused::kWarps * L.H * D * 4);
  L.ulist = off; off = align_up(off + (size_t)L.grid * L.cpc_max * fused::kRec * 4);
  L.glogits = off; off = align_up(off + (size_t)L.grid * L.cpc_max * kChunk * L.H * 4);
  L.gstats = off;
  if (L.need_gstats) off = align_up(off + (size_t)L.grid * L.cpc_max * 8 * 12 * 4);
  L.qbuf = off; off = align_up(off + (size_t)units * L.H * D * 2);
  L.qgsum = off; off = align_up(off + (size_t)units * L.H * 8 * 4);
  L.total = off;
  return L;
}

size_t attention_ws_bytes(int B, int Hq, int Hkv, int T_cap, int D, int KB) {
  if (fused_ok(Hq / Hkv)) return fused_layout(B, Hq, Hkv, T_cap, D, KB).total;
  return ws_layout(B, Hq, Hkv, T_cap, D).total;
}

// Launch the decode of `a` on the single-launch kernel when the group fits,
// else on the three-launch path.
int run_attention(DecodeArgs& a, int D, int kb, int vb0, int vb1, void* ws, size_t ws_bytes, cudaStream_t s,
                  const int32_t* block_table = nullptr, int pages_per_seq = 0, int num_pages = 0) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return LKV_ERR_INVALID_ARG;
  char* base = static_cast<char*>(ws);
  a.status = reinterpret_cast<int*>(base);
  if (!fused_ok(a.r)) {
    const WsLayout w = ws_layout(a.B, a.Hq, a.Hkv, a.T_cap, D);
    if (ws_bytes < w.total) return LKV_ERR_WORKSPACE;
    a.logits = reinterpret_cast<float*>(base + w.logits);
    a.stats = reinterpret_cast<float*>(base + w.stats);
    a.partial = reinterpret_cast<float*>(base + w.partial);
    a.chunk = kChunk;
    a.n_chunks = w.n_chunks;
    return from_cuda(launch_decode(a, D, kb, vb0, vb1, s));
  }
  const FusedLayout L = fused_layout(a.B, a.Hq, a.Hkv, a.T_cap, D, kb);
  if (ws_bytes < L.total) return LKV_ERR_WORKSPACE;
  FusedArgs f{};
  f.d = a;
  f.cpc_max = L.cpc_max;
  f.stages = L.stages;
  f.ring_bytes = L.ring_bytes;
  f.cand_cap = L.cand_cap;
  f.smem_logit_floats = 0;
  f.timeout_ns = reinterpret_cast<const unsigned long long*>(base + 8);
  f.done = reinterpret_cast<int*>(base + 16);
  f.wcounts = reinterpret_cast<unsigned long long*>(base + 32);
  f.arrive1 = reinterpret_cast<int*>(base + L.arrive1);
  f.arrive2 = reinterpret_cast<int*>(base + L.arrive2);
  f.pstats = reinterpret_cast<float*>(base + L.pstats);
  f.ppart = reinterpret_cast<float*>(base + L.ppart);
  f.wslot = reinterpret_cast<float*>(base + L.wslot);
  f.cstats = nullptr;
  f.ulist = reinterpret_cast<int*>(base + L.ulist);
  f.glogits = reinterpret_cast<float*>(base + L.glogits);
  f.gstats = L.need_gstats ? reinterpret_cast<float*>(base + L.gstats) : nullptr;
  f.qbuf = reinterpret_cast<float*>(base + L.qbuf);
  f.qgsum = reinterpret_cast<float*>(base + L.qgsum);
  f.block_table = block_table;
  f.pages_per_seq = pages_per_seq;
  f.num_pages = num_pages;
  cudaError_t e;
  if (block_table != nullptr) {
    if (vb0 != vb1 || kb == 16 || vb0 == 16) return LKV_ERR_UNSUPPORTED;
    switch (kb) {
      case 2: e = launch_fused_paged_k2(f, D, L.H, vb0, L.smem_bytes, L.grid, s); break;
      case 4: e = launch_fused_paged_k4(f, D, L.H, vb0, L.smem_bytes, L.grid, s); break;
      case 6: e = launch_fused_paged_k6(f, D, L.H, vb0, L.smem_bytes, L.grid, s); break;
      case 8: e = launch_fused_paged_k8(f, D, L.H, vb0, L.smem_bytes, L.grid, s); break;
      default: return LKV_ERR_UNSUPPORTED;
    }
    return from_cuda(e);
  }
  switch (kb) {
    case 2: e = launch_fused_k2(f, D, L.H, vb0, vb1, L.smem_bytes, L.grid, s); break;
    case 4: e = launch_fused_k4(f, D, L.H, vb0, vb1, L.smem_bytes, L.grid, s); break;
    case 6: e = launch_fused_k6(f, D, L.H, vb0, vb1, L.smem_bytes, L.grid, s); break;
    case 8: e = launch_fused_k8(f, D, L.H, vb0, vb1, L.smem_bytes, L.grid, s); break;
    case 16: e = launch_fused_k16(f, D, L.H, vb0, vb1, L.smem_bytes, L.grid, s); break;
    default: return LKV_ERR_UNSUPPORTED;
  }
  return from_cuda(e);
}

// Shapes shared by every attention call.
int check_attention_shape(int B, int Hq, int Hkv, int T_cap, int D, int G) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || T_cap < 0) return LKV_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return LKV_ERR_INVALID_ARG;
  if (!dim_ok(D) || !group_ok(G, D)) return LKV_ERR_UNSUPPORTED;
  const int r = Hq / Hkv;
  if (r > 64 || !(r == 1 || r == 2 || r % 4 == 0)) return LKV_ERR_UNSUPPORTED;
  if (((long long)T_cap * (D / G)) % 2 != 0) return LKV_ERR_UNSUPPORTED;
  return LKV_OK;
}

int check_cache_shape(int B, int Hkv, int T_cap, int D, int G) {
  if (B < 0 || Hkv <= 0 || T_cap < 0) return LKV_ERR_INVALID_ARG;
  if (!dim_ok(D) || !group_ok(G, D)) return LKV_ERR_UNSUPPORTED;
  if (((long long)T_cap * (D / G)) % 2 != 0) return LKV_ERR_UNSUPPORTED;
  return LKV_OK;
}

bool segment_ok(const lkv_segment& s, bool nonempty) {
  return ptr_ok(s.k_codes, nonempty) && ptr_ok(s.k_sz, nonempty) && ptr_ok(s.v_codes, nonempty) &&
         ptr_ok(s.v_sz, nonempty);
}

}  // namespace
}  // namespace lkv

using namespace lkv;

// ---------------------------------------------------------------- fixed scratch
// Scratch of lkv_decode_attention_static: a fixed array of device memory that
// belongs to this library's module, so that callers which cannot allocate
// device memory still get a decode.  Examples: a host embedding the library
// from plain C with no device allocator of its own, or a serving process
// whose memory is all reserved up front by another allocator, where a new
// cudaMalloc would fail and a cudaFree would synchronize the whole device.
// Its size is fixed at LKV_STATIC_WORKSPACE_BYTES; larger decodes are
// rejected.  Host code never uses the array's name as a device address: the
// address comes from cudaGetSymbolAddress, looked up on every call.
static __device__ __align__(256) unsigned char g_static_ws[LKV_STATIC_WORKSPACE_BYTES];

namespace {

// Device address of g_static_ws in the current context, looked up on every
// call (cheap once the module is loaded): after a device reset, or in
// another context, the array can sit at another address.
int static_scratch(void** ptr) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || p == nullptr) return LKV_ERR_CUDA;
  *ptr = p;
  return LKV_OK;
}

// Bytes at the start of the scratch that a decode expects to find zero: the
// status word, the wait limit and the cross-CTA counters.  Everything past
// them is written before it is read.
size_t static_zero_prefix(int B, int Hq, int Hkv, int T_cap, int D, int KB) {
  if (fused_ok(Hq / Hkv)) return fused_layout(B, Hq, Hkv, T_cap, D, KB).pstats;
  return kHeaderBytes;
}

}  // namespace

namespace {

// A paged cache: block_table [B][pps] of page ids in [0, pages); nullptr
// table = the contiguous [B][Hkv][T_cap] layout.
struct Paging {
  const int32_t* table = nullptr;
  int pps = 0, pages = 0;
  int T_cap() const { return pps * kPageTokens; }
};

int check_paging(const Paging& pg, int B) {
  if (pg.pps <= 0 || pg.pages <= 0) return LKV_ERR_INVALID_ARG;
  if ((long long)pg.pps * kPageTokens > (1ll << 30)) return LKV_ERR_UNSUPPORTED;
  if (B > 0 && (pg.table == nullptr || (reinterpret_cast<uintptr_t>(pg.table) & 3u) != 0)) return LKV_ERR_INVALID_ARG;
  return LKV_OK;
}

int quantize_impl(lkv_qspec spec, int B, int Hkv, int T_cap, int D, const int32_t* seq_lens, const void* k,
                  const void* v, const Paging& pg, void* k_codes, float* k_sz, void* v_codes, float* v_sz,
                  void* stream) {
  if (!bits_ok(spec.k_bits) || !bits_ok(spec.v_bits)) return LKV_ERR_UNSUPPORTED;
  int rc = check_cache_shape(B, Hkv, T_cap, D, spec.group);
  if (rc) return rc;
  const bool ne = (long long)B * Hkv * T_cap > 0;
  if (!ptr_ok(seq_lens, B > 0) || !ptr_ok(k, ne) || !ptr_ok(v, ne) || !ptr_ok(k_codes, ne) || !ptr_ok(k_sz, ne && spec.k_bits < 16) ||
      !ptr_ok(v_codes, ne) || !ptr_ok(v_sz, ne && spec.v_bits < 16))
    return LKV_ERR_INVALID_ARG;
  if (!ne) return LKV_OK;
  QuantizeArgs a{};
  a.B = B; a.Hkv = Hkv; a.T_cap = T_cap; a.G = spec.group; a.one = 1.0f;
  a.block_table = pg.table; a.pages_per_seq = pg.pps; a.num_pages = pg.pages;
  a.seq_lens = seq_lens;
  a.k = static_cast<const uint16_t*>(k);
  a.v = static_cast<const uint16_t*>(v);
  a.k_codes = static_cast<uint8_t*>(k_codes);
  a.k_sz = k_sz;
  a.v_codes = static_cast<uint8_t*>(v_codes);
  a.v_sz = v_sz;
  return from_cuda(launch_quantize_kv(a, spec.k_bits, spec.v_bits, D, static_cast<cudaStream_t>(stream)));
}

int append_impl(lkv_qspec spec, int B, int Hkv, int T_cap, int D, const int32_t* pos, const void* k_new,
                const void* v_new, const Paging& pg, void* k_codes, float* k_sz, void* v_codes, float* v_sz,
                void* stream) {
  if (!bits_ok(spec.k_bits) || !bits_ok(spec.v_bits)) return LKV_ERR_UNSUPPORTED;
  int rc = check_cache_shape(B, Hkv, T_cap, D, spec.group);
  if (rc) return rc;
  const bool ne = (long long)B * Hkv * T_cap > 0;
  if (!ptr_ok(pos, ne) || !ptr_ok(k_new, ne) || !ptr_ok(v_new, ne) || !ptr_ok(k_codes, ne) || !ptr_ok(k_sz, ne && spec.k_bits < 16) ||
      !ptr_ok(v_codes, ne) || !ptr_ok(v_sz, ne && spec.v_bits < 16))
    return LKV_ERR_INVALID_ARG;
  if (!ne) return LKV_OK;
  QuantizeArgs a{};
  a.B = B; a.Hkv = Hkv; a.T_cap = T_cap; a.G = spec.group; a.one = 1.0f;
  a.block_table = pg.table; a.pages_per_seq = pg.pps; a.num_pages = pg.pages;
  a.seq_lens = pos;
  a.k = static_cast<const uint16_t*>(k_new);
  a.v = static_cast<const uint16_t*>(v_new);
  a.k_codes = static_cast<uint8_t*>(k_codes);
  a.k_sz = k_sz;
  a.v_codes = static_cast<uint8_t*>(v_codes);
  a.v_sz = v_sz;
  return from_cuda(launch_append_kv(a, spec.k_bits, spec.v_bits, D, static_cast<cudaStream_t>(stream)));
}

}  // namespace

namespace {
int decode_impl(lkv_qspec spec, int B, int Hq, int Hkv, int T_cap, int D, const int32_t* seq_lens, const void* q,
                const void* k_codes, const float* k_sz, const void* v_codes, const float* v_sz, float softmax_scale,
                float tau, float* out, uint8_t* skip_mask, int64_t* skip_counts, float* mass, void* workspace,
                size_t ws_bytes, void* stream, const Paging& pg);
}  // namespace

extern "C" {

const char* lkv_status_string(int status) {
  switch (status) {
    case LKV_OK: return "LKV_OK";
    case LKV_ERR_INVALID_ARG: return "LKV_ERR_INVALID_ARG";
    case LKV_ERR_UNSUPPORTED: return "LKV_ERR_UNSUPPORTED";
    case LKV_ERR_WORKSPACE: return "LKV_ERR_WORKSPACE";
    case LKV_ERR_CUDA: return "LKV_ERR_CUDA";
    case LKV_ERR_TIMEOUT: return "LKV_ERR_TIMEOUT";
  }
  return "LKV_ERR_UNKNOWN";
}

int lkv_version(void) { return 100; }

size_t lkv_row_bytes(int bits, int D) {
  if (!bits_ok(bits) || D <= 0 || (D * bits) % 8 != 0) return 0;
  return (size_t)D * bits / 8;
}

size_t lkv_sz_row_bytes(int D, int group) {
  if (!group_ok(group, D)) return 0;
  return (size_t)8 * (D / group);
}

int lkv_quantize_kv(lkv_qspec spec, int B, int Hkv, int T_cap, int D, const int32_t* seq_lens, const void* k,
                    const void* v, void* k_codes, float* k_sz, void* v_codes, float* v_sz, void* stream) {
  return quantize_impl(spec, B, Hkv, T_cap, D, seq_lens, k, v, Paging{}, k_codes, k_sz, v_codes, v_sz, stream);
}

int lkv_quantize_kv_paged(lkv_qspec spec, int B, int Hkv, int pages_per_seq, int num_pages, int D,
                          const int32_t* seq_lens, const void* k, const void* v, const int32_t* block_table,
                          void* k_pool, float* k_sz_pool, void* v_pool, float* v_sz_pool, void* stream) {
  Paging pg{block_table, pages_per_seq, num_pages};
  int rc = check_paging(pg, B);
  if (rc) return rc;
  return quantize_impl(spec, B, Hkv, pg.T_cap(), D, seq_lens, k, v, pg, k_pool, k_sz_pool, v_pool, v_sz_pool,
                       stream);
}

int lkv_append_kv(lkv_qspec spec, int B, int Hkv, int T_cap, int D, const int32_t* pos, const void* k_new,
                  const void* v_new, void* k_codes, float* k_sz, void* v_codes, float* v_sz, void* stream) {
  return append_impl(spec, B, Hkv, T_cap, D, pos, k_new, v_new, Paging{}, k_codes, k_sz, v_codes, v_sz, stream);
}

int lkv_append_kv_paged(lkv_qspec spec, int B, int Hkv, int pages_per_seq, int num_pages, int D, const int32_t* pos,
                        const void* k_new, const void* v_new, const int32_t* block_table, void* k_pool,
                        float* k_sz_pool, void* v_pool, float* v_sz_pool, void* stream) {
  Paging pg{block_table, pages_per_seq, num_pages};
  int rc = check_paging(pg, B);
  if (rc) return rc;
  return append_impl(spec, B, Hkv, pg.T_cap(), D, pos, k_new, v_new, pg, k_pool, k_sz_pool, v_pool, v_sz_pool,
                     stream);
}

size_t lkv_decode_workspace_bytes(lkv_qspec spec, int B, int Hq, int Hkv, int T_cap, int D) {
  if (!bits_ok(spec.k_bits) || !bits_ok(spec.v_bits)) return 0;
  if (check_attention_shape(B, Hq, Hkv, T_cap, D, spec.group)) return 0;
  return attention_ws_bytes(B, Hq, Hkv, T_cap, D, spec.k_bits);
}

int lkv_decode_attention(lkv_qspec spec, int B, int Hq, int Hkv, int T_cap, int D, const int32_t* seq_lens,
                         const void* q, const void* k_codes, const float* k_sz, const void* v_codes,
                         const float* v_sz, float softmax_scale, float tau, float* out, uint8_t* skip_mask,
                         int64_t* skip_counts, void* workspace, size_t ws_bytes, void* stream) {
  return decode_impl(spec, B, Hq, Hkv, T_cap, D, seq_lens, q, k_codes, k_sz, v_codes, v_sz, softmax_scale, tau,
                     out, skip_mask, skip_counts, nullptr, workspace, ws_bytes, stream, Paging{});
}

int lkv_decode_attention_paged(lkv_qspec spec, int B, int Hq, int Hkv, int pages_per_seq, int num_pages, int D,
                               const int32_t* seq_lens, const void* q, const int32_t* block_table,
                               const void* k_pool, const float* k_sz_pool, const void* v_pool,
                               const float* v_sz_pool, float softmax_scale, float tau, float* out,
                               uint8_t* skip_mask, int64_t* skip_counts, void* workspace, size_t ws_bytes,
                               void* stream) {
  Paging pg{block_table, pages_per_seq, num_pages};
  int rc = check_paging(pg, B);
  if (rc) return rc;
  if (Hkv > 0 && !fused_ok(Hq / Hkv)) return LKV_ERR_UNSUPPORTED;  // paged: groups of 1, 2 or 4 query heads
  return decode_impl(spec, B, Hq, Hkv, pg.T_cap(), D, seq_lens, q, k_pool, k_sz_pool, v_pool, v_sz_pool,
                     softmax_scale, tau, out, skip_mask, skip_counts, nullptr, workspace, ws_bytes, stream, pg);
}

int lkv_decode_attention_mass(lkv_qspec spec, int B, int Hq, int Hkv, int T_cap, int D, const int32_t* seq_lens,
                              const void* q, const void* k_codes, const float* k_sz, const void* v_codes,
                              const float* v_sz, float softmax_scale, float tau, float* out, uint8_t* skip_mask,
                              int64_t* skip_counts, float* mass, void* workspace, size_t ws_bytes, void* stream) {
  if (mass == nullptr && (long long)B * Hkv * T_cap > 0) return LKV_ERR_INVALID_ARG;
  return decode_impl(spec, B, Hq, Hkv, T_cap, D, seq_lens, q, k_codes, k_sz, v_codes, v_sz, softmax_scale, tau,
                     out, skip_mask, skip_counts, mass, workspace, ws_bytes, stream, Paging{});
}

}  // extern "C"

namespace {

int decode_impl(lkv_qspec spec, int B, int Hq, int Hkv, int T_cap, int D, const int32_t* seq_lens, const void* q,
                const void* k_codes, const float* k_sz, const void* v_codes, const float* v_sz, float softmax_scale,
                float tau, float* out, uint8_t* skip_mask, int64_t* skip_counts, float* mass, void* workspace,
                size_t ws_bytes, void* stream, const Paging& pg) {
  if (!bits_ok(spec.k_bits) || !bits_ok(spec.v_bits)) return LKV_ERR_UNSUPPORTED;
  int rc = check_attention_shape(B, Hq, Hkv, T_cap, D, spec.group);
  if (rc) return rc;
  if (!std::isfinite(softmax_scale) || std::isnan(tau)) return LKV_ERR_INVALID_ARG;
  const bool ne = (long long)B * Hkv * T_cap > 0;
  if (!ptr_ok(seq_lens, B > 0) || !ptr_ok(q, B > 0) || !ptr_ok(out, B > 0) || !ptr_ok(k_codes, ne) ||
      !ptr_ok(k_sz, ne && spec.k_bits < 16) || !ptr_ok(v_codes, ne) || !ptr_ok(v_sz, ne && spec.v_bits < 16))
    return LKV_ERR_INVALID_ARG;
  if (skip_counts && !aligned16(skip_counts)) return LKV_ERR_INVALID_ARG;
  if (mass && (reinterpret_cast<uintptr_t>(mass) & 3u) != 0) return LKV_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return LKV_ERR_INVALID_ARG;
  if (ws_bytes < attention_ws_bytes(B, Hq, Hkv, T_cap, D, spec.k_bits)) return LKV_ERR_WORKSPACE;
  DecodeArgs a{};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (B == 0) {
    if (skip_counts) return from_cuda(cudaMemsetAsync(skip_counts, 0, 2 * sizeof(int64_t), s));
    return LKV_OK;
  }
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.T_cap = T_cap; a.G = spec.group; a.r = Hq / Hkv;
  a.lens = seq_lens; a.len_mode = 0;
  a.q = static_cast<const uint16_t*>(q);
  a.kc[0] = a.kc[1] = static_cast<const uint8_t*>(k_codes);
  a.ksz[0] = a.ksz[1] = k_sz;
  a.vc[0] = a.vc[1] = static_cast<const uint8_t*>(v_codes);
  a.vsz[0] = a.vsz[1] = v_sz;
  a.q_scale = softmax_scale * 1.4426950408889634f;
  a.tau = tau;
  a.out = out;
  a.skip_mask = skip_mask;
  a.mass = mass;
  a.skip_counts = reinterpret_cast<unsigned long long*>(skip_counts);
  return run_attention(a, D, spec.k_bits, spec.v_bits, spec.v_bits, workspace, ws_bytes, s, pg.table,
                       pg.pps, pg.pages);
}

}  // namespace

extern "C" {

int lkv_decode_attention_static(lkv_qspec spec, int B, int Hq, int Hkv, int T_cap, int D, const int32_t* seq_lens,
                                const void* q, const void* k_codes, const float* k_sz, const void* v_codes,
                                const float* v_sz, float softmax_scale, float tau, float* out,
                                uint8_t* skip_mask, int64_t* skip_counts, int32_t* status, void* stream) {
  if (!bits_ok(spec.k_bits) || !bits_ok(spec.v_bits)) return LKV_ERR_UNSUPPORTED;
  int rc = check_attention_shape(B, Hq, Hkv, T_cap, D, spec.group);
  if (rc) return rc;
  if (!std::isfinite(softmax_scale) || std::isnan(tau)) return LKV_ERR_INVALID_ARG;
  const bool ne = (long long)B * Hkv * T_cap > 0;
  if (!ptr_ok(seq_lens, B > 0) || !ptr_ok(q, B > 0) || !ptr_ok(out, B > 0) || !ptr_ok(k_codes, ne) ||
      !ptr_ok(k_sz, ne && spec.k_bits < 16) || !ptr_ok(v_codes, ne) || !ptr_ok(v_sz, ne && spec.v_bits < 16))
    return LKV_ERR_INVALID_ARG;
  if (skip_counts && !aligned16(skip_counts)) return LKV_ERR_INVALID_ARG;
  if (status && (reinterpret_cast<uintptr_t>(status) & 3u) != 0) return LKV_ERR_INVALID_ARG;
  const size_t need = attention_ws_bytes(B, Hq, Hkv, T_cap, D, spec.k_bits);
  if (need > (size_t)LKV_STATIC_WORKSPACE_BYTES) return LKV_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (B == 0) {
    if (skip_counts) rc = from_cuda(cudaMemsetAsync(skip_counts, 0, 2 * sizeof(int64_t), s));
    if (rc == LKV_OK && status) rc = from_cuda(cudaMemsetAsync(status, 0, sizeof(int32_t), s));
    return rc;
  }
  void* ws = nullptr;
  rc = static_scratch(&ws);
  if (rc) return rc;
  // Clear what must start at zero, so that a failed earlier call (a timeout,
  // a bad length) leaves nothing behind for this one.
  rc = from_cuda(cudaMemsetAsync(ws, 0, static_zero_prefix(B, Hq, Hkv, T_cap, D, spec.k_bits), s));
  if (rc) return rc;
  DecodeArgs a{};
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.T_cap = T_cap; a.G = spec.group; a.r = Hq / Hkv;
  a.lens = seq_lens; a.len_mode = 0;
  a.q = static_cast<const uint16_t*>(q);
  a.kc[0] = a.kc[1] = static_cast<const uint8_t*>(k_codes);
  a.ksz[0] = a.ksz[1] = k_sz;
  a.vc[0] = a.vc[1] = static_cast<const uint8_t*>(v_codes);
  a.vsz[0] = a.vsz[1] = v_sz;
  a.q_scale = softmax_scale * 1.4426950408889634f;
  a.tau = tau;
  a.out = out;
  a.skip_mask = skip_mask;
  a.skip_counts = reinterpret_cast<unsigned long long*>(skip_counts);
  rc = run_attention(a, D, spec.k_bits, spec.v_bits, spec.v_bits, ws, LKV_STATIC_WORKSPACE_BYTES, s);
  if (rc == LKV_OK && status)
    rc = from_cuda(cudaMemcpyAsync(status, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, s));
  return rc;
}

int lkv_workspace_reset(void* workspace, size_t ws_bytes, void* stream) {
  if (workspace == nullptr && ws_bytes > 0) return LKV_ERR_INVALID_ARG;
  if (ws_bytes == 0) return LKV_OK;
  return from_cuda(cudaMemsetAsync(workspace, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

int lkv_workspace_status(const void* workspace, void* stream, int32_t* status) {
  if (workspace == nullptr || status == nullptr) return LKV_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return LKV_ERR_CUDA;
  *status = v;
  return LKV_OK;
}

int lkv_tier_classify(int B, int Hkv, int T_cap, const int32_t* seq_lens, const float* mass, float tau_low,
                      float tau_high, int8_t* tier, int32_t* counts, int32_t* pos_a, int32_t* pos_b, void* stream) {
  if (B < 0 || Hkv <= 0 || T_cap < 0) return LKV_ERR_INVALID_ARG;
  const bool ne = (long long)B * Hkv * T_cap > 0;
  if (!ptr_ok(seq_lens, B > 0) || !ptr_ok(counts, B > 0) || !ptr_ok(mass, ne) || !ptr_ok(tier, ne) ||
      !ptr_ok(pos_a, ne) || !ptr_ok(pos_b, ne))
    return LKV_ERR_INVALID_ARG;
  if (B == 0) return LKV_OK;
  ClassifyArgs a{};
  a.B = B; a.Hkv = Hkv; a.T_cap = T_cap;
  a.seq_lens = seq_lens; a.mass = mass; a.tau_low = tau_low; a.tau_high = tau_high;
  a.tier = tier; a.counts = counts; a.pos_a = pos_a; a.pos_b = pos_b;
  return from_cuda(launch_tier_classify(a, static_cast<cudaStream_t>(stream)));
}

int lkv_tier_repack(int B, int Hkv, int T_cap, int D, int group, const void* k, const void* v, const int32_t* counts,
                    const int32_t* pos_a, const int32_t* pos_b, lkv_segment seg_a, lkv_segment seg_b, void* stream) {
  int rc = check_cache_shape(B, Hkv, T_cap, D, group);
  if (rc) return rc;
  const bool ne = (long long)B * Hkv * T_cap > 0;
  if (!ptr_ok(counts, B > 0) || !ptr_ok(k, ne) || !ptr_ok(v, ne) || !ptr_ok(pos_a, ne) || !ptr_ok(pos_b, ne) ||
      !segment_ok(seg_a, ne) || !segment_ok(seg_b, ne))
    return LKV_ERR_INVALID_ARG;
  if (!ne) return LKV_OK;
  RepackArgs a{};
  a.B = B; a.Hkv = Hkv; a.T_cap = T_cap; a.G = group; a.one = 1.0f;
  a.k = static_cast<const uint16_t*>(k);
  a.v = static_cast<const uint16_t*>(v);
  a.counts = counts; a.pos_a = pos_a; a.pos_b = pos_b;
  a.a_kc = static_cast<uint8_t*>(seg_a.k_codes); a.a_ksz = seg_a.k_sz;
  a.a_vc = static_cast<uint8_t*>(seg_a.v_codes); a.a_vsz = seg_a.v_sz;
  a.b_kc = static_cast<uint8_t*>(seg_b.k_codes); a.b_ksz = seg_b.k_sz;
  a.b_vc = static_cast<uint8_t*>(seg_b.v_codes); a.b_vsz = seg_b.v_sz;
  return from_cuda(launch_tier_repack(a, D, static_cast<cudaStream_t>(stream)));
}

size_t lkv_tiered_workspace_bytes(int B, int Hq, int Hkv, int T_cap, int D, int group) {
  if (check_attention_shape(B, Hq, Hkv, T_cap, D, group)) return 0;
  return attention_ws_bytes(B, Hq, Hkv, T_cap, D, 6);
}

int lkv_tiered_attention(int B, int Hq, int Hkv, int T_cap, int D, int group, const int32_t* counts, const void* q,
                         lkv_segment seg_a, lkv_segment seg_b, float softmax_scale, float tau, float* out,
                         int64_t* skip_counts, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_attention_shape(B, Hq, Hkv, T_cap, D, group);
  if (rc) return rc;
  if (!std::isfinite(softmax_scale) || std::isnan(tau)) return LKV_ERR_INVALID_ARG;
  const bool ne = (long long)B * Hkv * T_cap > 0;
  if (!ptr_ok(counts, B > 0) || !ptr_ok(q, B > 0) || !ptr_ok(out, B > 0) || !segment_ok(seg_a, ne) ||
      !segment_ok(seg_b, ne))
    return LKV_ERR_INVALID_ARG;
  if (skip_counts && !aligned16(skip_counts)) return LKV_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return LKV_ERR_INVALID_ARG;
  if (ws_bytes < attention_ws_bytes(B, Hq, Hkv, T_cap, D, 6)) return LKV_ERR_WORKSPACE;
  DecodeArgs a{};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (B == 0) {
    if (skip_counts) return from_cuda(cudaMemsetAsync(skip_counts, 0, 2 * sizeof(int64_t), s));
    return LKV_OK;
  }
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.T_cap = T_cap; a.G = group; a.r = Hq / Hkv;
  a.lens = counts; a.len_mode = 1;
  a.q = static_cast<const uint16_t*>(q);
  a.kc[0] = static_cast<const uint8_t*>(seg_a.k_codes); a.kc[1] = static_cast<const uint8_t*>(seg_b.k_codes);
  a.ksz[0] = seg_a.k_sz; a.ksz[1] = seg_b.k_sz;
  a.vc[0] = static_cast<const uint8_t*>(seg_a.v_codes); a.vc[1] = static_cast<const uint8_t*>(seg_b.v_codes);
  a.vsz[0] = seg_a.v_sz; a.vsz[1] = seg_b.v_sz;
  a.q_scale = softmax_scale * 1.4426950408889634f;
  a.tau = tau;
  a.out = out;
  a.skip_mask = nullptr;
  a.skip_counts = reinterpret_cast<unsigned long long*>(skip_counts);
  return run_attention(a, D, 6, 6, 4, workspace, ws_bytes, s);
}

int lkv_tiered_decode(int B, int Hq, int Hkv, int T_cap, int D, int group, const int32_t* seq_lens, const float* mass,
                      float tau_low, float tau_high, const void* k, const void* v, const void* q, int8_t* tier,
                      int32_t* counts, int32_t* pos_a, int32_t* pos_b, lkv_segment seg_a, lkv_segment seg_b,
                      float softmax_scale, float tau, float* out, int64_t* skip_counts, void* workspace,
                      size_t ws_bytes, void* stream) {
  // Validate all three stages before enqueueing any of them.
  int rc = check_attention_shape(B, Hq, Hkv, T_cap, D, group);
  if (rc) return rc;
  if (!std::isfinite(softmax_scale) || std::isnan(tau)) return LKV_ERR_INVALID_ARG;
  const bool ne = (long long)B * Hkv * T_cap > 0;
  if (!ptr_ok(seq_lens, B > 0) || !ptr_ok(counts, B > 0) || !ptr_ok(q, B > 0) || !ptr_ok(out, B > 0) ||
      !ptr_ok(mass, ne) || !ptr_ok(tier, ne) || !ptr_ok(pos_a, ne) || !ptr_ok(pos_b, ne) || !ptr_ok(k, ne) ||
      !ptr_ok(v, ne) || !segment_ok(seg_a, ne) || !segment_ok(seg_b, ne))
    return LKV_ERR_INVALID_ARG;
  if (skip_counts && !aligned16(skip_counts)) return LKV_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) % 256) != 0) return LKV_ERR_INVALID_ARG;
  if (ws_bytes < lkv_tiered_workspace_bytes(B, Hq, Hkv, T_cap, D, group)) return LKV_ERR_WORKSPACE;
  rc = lkv_tier_classify(B, Hkv, T_cap, seq_lens, mass, tau_low, tau_high, tier, counts, pos_a, pos_b, stream);
  if (rc) return rc;
  rc = lkv_tier_repack(B, Hkv, T_cap, D, group, k, v, counts, pos_a, pos_b, seg_a, seg_b, stream);
  if (rc) return rc;
  return lkv_tiered_attention(B, Hq, Hkv, T_cap, D, group, counts, q, seg_a, seg_b, softmax_scale, tau, out,
                              skip_counts, workspace, ws_bytes, stream);
}

}  // extern "C"
