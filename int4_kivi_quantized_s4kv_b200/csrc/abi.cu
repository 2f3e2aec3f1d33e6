// Host side of the s4kv C ABI: argument validation, workspace sizing and
// kernel launches.  Every host-visible argument is checked before anything
// is launched; the library allocates no memory and keeps no state: launch
// shapes are worked out and kernel attributes set at every call.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "kernels.cuh"
#include "prefill.cuh"

using namespace s4kv;

namespace {


struct DeviceShape {
  int num_sms = 0;
  int num_ctas[3] = {0, 0, 0};     // decode grid for 4-bit / 8-bit / 2-bit pages
  int num_workers[3] = {0, 0, 0};  // worker warps of that grid
  int max_workers = 0;          // sizes the (shared) decode workspace
};

int fmt_index(int bits) { return bits == 8 ? 1 : bits == 2 ? 2 : 0; }
int fmt_bits(int index) { return index == 1 ? 8 : index == 2 ? 2 : 4; }
int cache_bits(const s4kv_cache_t *c) { return c->bits == 8 || c->bits == 2 ? c->bits : 4; }
size_t block_bytes(int bits) {
  return bits == 8 ? S4KV_BLOCK_BYTES_INT8 : bits == 2 ? S4KV_BLOCK_BYTES_INT2 : S4KV_BLOCK_BYTES;
}
size_t record_bytes(const s4kv_cache_t *c) { return static_cast<size_t>(c->num_kv_heads) * block_bytes(cache_bits(c)); }

// Decode launch shape of the current device, worked out at every call (the
// library keeps no state): one persistent CTA per SM.
int device_shape(DeviceShape *out) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    cudaGetLastError();
    return S4KV_ERR_CUDA;
  }
  DeviceShape d;
  d.num_sms = sms;
  for (int f = 0; f < 3; ++f) {
    d.num_ctas[f] = sms;
    d.num_workers[f] = sms * decode_warps_per_cta(fmt_bits(f));
    d.max_workers = d.num_workers[f] > d.max_workers ? d.num_workers[f] : d.max_workers;
  }
  *out = d;
  return S4KV_OK;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_cache(const s4kv_cache_t *c) {
  if (c == nullptr) return S4KV_ERR_INVALID_ARG;
  if (c->head_dim != S4KV_HEAD_DIM || c->page_tokens != S4KV_PAGE_TOKENS) return S4KV_ERR_UNSUPPORTED;
  if (c->pool == nullptr || c->res_k == nullptr || c->res_v == nullptr) return S4KV_ERR_INVALID_ARG;
  if (c->num_pages <= 0 || c->num_kv_heads <= 0 || c->max_seqs <= 0) return S4KV_ERR_INVALID_ARG;
  if (!aligned(c->pool, 128) || !aligned(c->res_k, 16) || !aligned(c->res_v, 16)) return S4KV_ERR_INVALID_ARG;
  if (c->err_flag != nullptr && !aligned(c->err_flag, 4)) return S4KV_ERR_INVALID_ARG;
  if (c->bits != 0 && c->bits != 2 && c->bits != 4 && c->bits != 8) return S4KV_ERR_UNSUPPORTED;
  return S4KV_OK;
}

// Workspace carve-up: [m,l: 2*workers*8 float2] [partial O:
// 2*workers*8*128 float] [tickets: batch*kv_heads u32].  The two partial
// regions depend only on the device's worker count, so they sit first and a
// workspace sized for a large batch serves any smaller one: a call touches
// a prefix of the ticket region, which it leaves at zero, and never reads
// partial results as tickets.
struct WsLayout {
  size_t tickets, ml, part, total;
};

WsLayout ws_layout(int batch, int num_kv_heads, int num_workers) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  WsLayout w;
  w.ml = 0;
  w.part = up(static_cast<size_t>(2) * num_workers * 8 * 2 * sizeof(float));
  w.tickets = w.part + up(static_cast<size_t>(2) * num_workers * 8 * S4KV_HEAD_DIM * sizeof(float));
  w.total = w.tickets + static_cast<size_t>(batch) * num_kv_heads * sizeof(uint32_t);
  return w;
}

int launch_records(const uint8_t *src, uint8_t *dst, const int32_t *src_idx, const int32_t *dst_idx,
                   long long rec_bytes, int n, int src_limit, int dst_limit, uint32_t *err, uint32_t err_bit,
                   void *stream) {
  MoveParams p;
  p.src_base = src;
  p.dst_base = dst;
  p.src_idx = src_idx;
  p.dst_idx = dst_idx;
  p.err = err;
  p.rec_bytes = rec_bytes;
  p.n = n;
  p.src_limit = src_limit;
  p.dst_limit = dst_limit;
  p.err_bit = err_bit;
  launch_move(p, static_cast<cudaStream_t>(stream));
  if (cudaGetLastError() != cudaSuccess) return S4KV_ERR_CUDA;
  return S4KV_OK;
}

}  // namespace

extern "C" {

int s4kv_version(void) { return S4KV_VERSION; }

const char *s4kv_status_string(int status) {
  switch (status) {
    case S4KV_OK: return "ok";
    case S4KV_ERR_INVALID_ARG: return "invalid argument";
    case S4KV_ERR_UNSUPPORTED: return "unsupported model shape (head_dim 128, 16-token pages, GQA group <= 8 only)";
    case S4KV_ERR_CUDA: return "CUDA runtime error";
    case S4KV_ERR_DEVICE_CHECK: return "device-side check failed (err_flag set)";
    case S4KV_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int s4kv_check_model(int head_dim, int page_tokens, int num_q_heads, int num_kv_heads) {
  if (head_dim <= 0 || page_tokens <= 0 || num_q_heads <= 0 || num_kv_heads <= 0) return S4KV_ERR_INVALID_ARG;
  if (head_dim != S4KV_HEAD_DIM || page_tokens != S4KV_PAGE_TOKENS) return S4KV_ERR_UNSUPPORTED;
  if (num_q_heads % num_kv_heads != 0) return S4KV_ERR_UNSUPPORTED;
  const int g = num_q_heads / num_kv_heads;
  if (g < 1 || g > S4KV_MAX_GQA_GROUP) return S4KV_ERR_UNSUPPORTED;
  return S4KV_OK;
}

int s4kv_cache_layout(int num_pages, int num_kv_heads, int max_seqs, size_t *pool_bytes,
                      size_t *residual_bytes) {
  if (num_pages <= 0 || num_kv_heads <= 0 || max_seqs <= 0) return S4KV_ERR_INVALID_ARG;
  if (pool_bytes) *pool_bytes = static_cast<size_t>(num_pages) * num_kv_heads * S4KV_BLOCK_BYTES;
  if (residual_bytes)
    *residual_bytes = static_cast<size_t>(max_seqs) * num_kv_heads * S4KV_PAGE_TOKENS * S4KV_HEAD_DIM * 2;
  return S4KV_OK;
}

int s4kv_cache_layout_bits(int num_pages, int num_kv_heads, int max_seqs, int bits, size_t *pool_bytes,
                           size_t *residual_bytes) {
  if (bits != 2 && bits != 4 && bits != 8) return S4KV_ERR_UNSUPPORTED;
  const int rc = s4kv_cache_layout(num_pages, num_kv_heads, max_seqs, pool_bytes, residual_bytes);
  if (rc == S4KV_OK && pool_bytes) *pool_bytes = static_cast<size_t>(num_pages) * num_kv_heads * block_bytes(bits);
  return rc;
}

int s4kv_append(const s4kv_cache_t *cache, const void *k, const void *v, int n_tokens,
                const int64_t *slot_mapping, const int32_t *cu_new, const int32_t *seq_lens,
                const int32_t *block_tables, int batch, int max_pages_per_seq, int max_new_per_seq,
                void *stream) {
  int rc = check_cache(cache);
  if (rc != S4KV_OK) return rc;
  if (n_tokens < 0 || batch < 0 || batch > cache->max_seqs || max_pages_per_seq <= 0) return S4KV_ERR_INVALID_ARG;
  if (n_tokens == 0 || batch == 0) return S4KV_OK;
  if (max_new_per_seq <= 0 || max_new_per_seq > n_tokens) return S4KV_ERR_INVALID_ARG;
  if (!k || !v || !slot_mapping || !cu_new || !seq_lens || !block_tables) return S4KV_ERR_INVALID_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(slot_mapping, 8) || !aligned(cu_new, 4) ||
      !aligned(seq_lens, 4) || !aligned(block_tables, 4))
    return S4KV_ERR_INVALID_ARG;
  const long long slots = (S4KV_PAGE_TOKENS - 1 + static_cast<long long>(max_new_per_seq) + S4KV_PAGE_TOKENS - 1) / S4KV_PAGE_TOKENS;
  if (slots > 0x7FFFFFFF || batch > 65535 || cache->num_kv_heads > 65535) return S4KV_ERR_INVALID_ARG;
  AppendParams p;
  p.pool = static_cast<uint8_t *>(cache->pool);
  p.res_k = static_cast<__half *>(cache->res_k);
  p.res_v = static_cast<__half *>(cache->res_v);
  p.err = cache->err_flag;
  p.k = static_cast<const __half *>(k);
  p.v = static_cast<const __half *>(v);
  p.slot_mapping = slot_mapping;
  p.cu_new = cu_new;
  p.seq_lens = seq_lens;
  p.block_tables = block_tables;
  p.num_pages = cache->num_pages;
  p.num_kv_heads = cache->num_kv_heads;
  p.max_pages = max_pages_per_seq;
  p.max_new = max_new_per_seq;
  p.n_tokens = n_tokens;
  p.bits = cache_bits(cache);
  launch_append(p, batch, max_new_per_seq, static_cast<cudaStream_t>(stream));
  if (cudaGetLastError() != cudaSuccess) return S4KV_ERR_CUDA;
  return S4KV_OK;
}

int s4kv_decode_workspace_size(int batch, int num_kv_heads, size_t *bytes) {
  if (batch < 0 || num_kv_heads <= 0 || bytes == nullptr) return S4KV_ERR_INVALID_ARG;
  DeviceShape d;
  const int rc = device_shape(&d);
  if (rc != S4KV_OK) return rc;
  *bytes = ws_layout(batch, num_kv_heads, d.max_workers).total;
  return S4KV_OK;
}

int s4kv_decode_attention(const s4kv_cache_t *cache, const void *q, int num_q_heads,
                          const int32_t *seq_lens, const int32_t *block_tables, int batch,
                          int max_pages_per_seq, float sm_scale, void *out, void *workspace,
                          size_t workspace_bytes, void *stream) {
  return s4kv::decode_call(cache, nullptr, nullptr, q, num_q_heads, seq_lens, block_tables, batch,
                           max_pages_per_seq, sm_scale, out, workspace, workspace_bytes, stream, false);
}

int s4kv_append_decode(const s4kv_cache_t *cache, const void *k_new, const void *v_new, const void *q,
                       int num_q_heads, const int32_t *seq_lens, const int32_t *block_tables, int batch,
                       int max_pages_per_seq, float sm_scale, void *out, void *workspace, size_t workspace_bytes,
                       void *stream) {
  if (batch > 0 && (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16))) return S4KV_ERR_INVALID_ARG;
  return s4kv::decode_call(cache, k_new, v_new, q, num_q_heads, seq_lens, block_tables, batch,
                           max_pages_per_seq, sm_scale, out, workspace, workspace_bytes, stream, false);
}

}  // extern "C"

namespace s4kv {

int decode_call(const s4kv_cache_t *cache, const void *k_new, const void *v_new, const void *q, int num_q_heads,
                const int32_t *seq_lens, const int32_t *block_tables, int batch, int max_pages_per_seq,
                float sm_scale, void *out, void *workspace, size_t workspace_bytes, void *stream,
                bool clear_tickets) {
  int rc = check_cache(cache);
  if (rc != S4KV_OK) return rc;
  rc = s4kv_check_model(cache->head_dim, cache->page_tokens, num_q_heads, cache->num_kv_heads);
  if (rc != S4KV_OK) return rc;
  if (batch < 0 || batch > cache->max_seqs || max_pages_per_seq <= 0) return S4KV_ERR_INVALID_ARG;
  // the step's append grid has one CTA per (sequence, kv head)
  if (k_new && static_cast<long long>(batch) * cache->num_kv_heads > 0x7FFFFFFF) return S4KV_ERR_INVALID_ARG;
  if (!(std::isfinite(sm_scale)) || sm_scale <= 0.0f) return S4KV_ERR_INVALID_ARG;
  if (batch == 0) return S4KV_OK;
  if (!q || !seq_lens || !block_tables || !out) return S4KV_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 8) || !aligned(seq_lens, 4) || !aligned(block_tables, 4))
    return S4KV_ERR_INVALID_ARG;
  DeviceShape d;
  rc = device_shape(&d);
  if (rc != S4KV_OK) return rc;
  const WsLayout w = ws_layout(batch, cache->num_kv_heads, d.max_workers);
  const int fi = fmt_index(cache_bits(cache));
  if (workspace == nullptr || workspace_bytes < w.total || !aligned(workspace, 16)) return S4KV_ERR_WORKSPACE;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  // every argument has been checked: only now may the tickets be cleared
  if (clear_tickets && cudaMemsetAsync(ws + w.tickets, 0, w.total - w.tickets, static_cast<cudaStream_t>(stream)) !=
                           cudaSuccess) {
    cudaGetLastError();
    return S4KV_ERR_CUDA;
  }
  DecodeParams p;
  p.pool = static_cast<const uint8_t *>(cache->pool);
  p.res_k = static_cast<const __half *>(cache->res_k);
  p.res_v = static_cast<const __half *>(cache->res_v);
  p.q = static_cast<const __half *>(q);
  p.out = static_cast<__half *>(out);
  p.seq_lens = seq_lens;
  p.block_tables = block_tables;
  p.tickets = reinterpret_cast<uint32_t *>(ws + w.tickets);
  p.part_ml = reinterpret_cast<float2 *>(ws + w.ml);
  p.part = reinterpret_cast<float *>(ws + w.part);
  p.err = cache->err_flag;
  p.batch = batch;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = cache->num_kv_heads;
  p.group = num_q_heads / cache->num_kv_heads;
  p.max_pages = max_pages_per_seq;
  p.num_pages = cache->num_pages;
  p.scale_log2 = static_cast<float>(static_cast<double>(sm_scale) * 1.4426950408889634);
  p.num_workers = d.num_workers[fi];
  FusedAppend f;
  f.k_new = static_cast<const __half *>(k_new);
  f.v_new = static_cast<const __half *>(v_new);
  if (launch_decode(p, f, cache_bits(cache), d.num_ctas[fi], static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return S4KV_ERR_CUDA;
  }
  return S4KV_OK;
}

}  // namespace s4kv

extern "C" {

int s4kv_prefill_workspace_size(int num_kv_heads, int batch, int max_pages_per_seq, size_t *bytes) {
  if (!bytes || num_kv_heads <= 0 || batch < 0 || max_pages_per_seq <= 0) return S4KV_ERR_INVALID_ARG;
  const unsigned long long tiles = static_cast<unsigned long long>(prefill_tiles_per_seq(max_pages_per_seq));
  const unsigned long long n = tiles * static_cast<unsigned long long>(batch) * num_kv_heads;
  if (n > (1ull << 40) / prefill_tile_bytes()) return S4KV_ERR_INVALID_ARG;
  *bytes = static_cast<size_t>(n * prefill_tile_bytes());
  return S4KV_OK;
}

int s4kv_prefill_attention(const s4kv_cache_t *cache, const void *q, int num_q_heads, int n_tokens,
                           const int32_t *cu_new, const int32_t *seq_lens, const int32_t *block_tables,
                           int batch, int max_pages_per_seq, int max_new_per_seq, float sm_scale, void *out,
                           void *workspace, size_t workspace_bytes, void *stream) {
  int rc = check_cache(cache);
  if (rc != S4KV_OK) return rc;
  rc = s4kv_check_model(cache->head_dim, cache->page_tokens, num_q_heads, cache->num_kv_heads);
  if (rc != S4KV_OK) return rc;
  if (n_tokens < 0 || batch < 0 || batch > cache->max_seqs || max_pages_per_seq <= 0) return S4KV_ERR_INVALID_ARG;
  if (!(std::isfinite(sm_scale)) || sm_scale <= 0.0f) return S4KV_ERR_INVALID_ARG;
  if (n_tokens == 0 || batch == 0) return S4KV_OK;
  if (max_new_per_seq <= 0 || max_new_per_seq > n_tokens) return S4KV_ERR_INVALID_ARG;
  if (!q || !cu_new || !seq_lens || !block_tables || !out) return S4KV_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(cu_new, 4) || !aligned(seq_lens, 4) ||
      !aligned(block_tables, 4))
    return S4KV_ERR_INVALID_ARG;
  size_t need = 0;
  rc = s4kv_prefill_workspace_size(cache->num_kv_heads, batch, max_pages_per_seq, &need);
  if (rc != S4KV_OK) return rc;
  if (!workspace || !aligned(workspace, 16) || workspace_bytes < need) return S4KV_ERR_WORKSPACE;
  const int group = num_q_heads / cache->num_kv_heads;
  const long long tiles = (static_cast<long long>(max_new_per_seq) + (128 / group) - 1) / (128 / group);
  if (tiles > 0x7FFFFFFF || batch > 65535 || cache->num_kv_heads > 65535) return S4KV_ERR_INVALID_ARG;
  PrefillParams p;
  p.pool = static_cast<const uint8_t *>(cache->pool);
  p.res_k = static_cast<const __half *>(cache->res_k);
  p.res_v = static_cast<const __half *>(cache->res_v);
  p.q = static_cast<const __half *>(q);
  p.out = static_cast<__half *>(out);
  p.cu_new = cu_new;
  p.seq_lens = seq_lens;
  p.block_tables = block_tables;
  p.err = cache->err_flag;
  p.n_tokens = n_tokens;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = cache->num_kv_heads;
  p.group = group;
  p.max_pages = max_pages_per_seq;
  p.num_pages = cache->num_pages;
  p.scale_log2 = static_cast<float>(static_cast<double>(sm_scale) * 1.4426950408889634);
  p.ws = static_cast<uint8_t *>(workspace);
  p.tiles_per_seq = prefill_tiles_per_seq(max_pages_per_seq);
  p.bits = cache_bits(cache);
  if (launch_prefill(p, batch, max_new_per_seq, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return S4KV_ERR_CUDA;
  }
  return S4KV_OK;
}

int s4kv_dequant_page(const s4kv_cache_t *cache, int physical_page, void *out_k, void *out_v,
                      int out_fp32, void *stream) {
  int rc = check_cache(cache);
  if (rc != S4KV_OK) return rc;
  if (physical_page < 0 || physical_page >= cache->num_pages) return S4KV_ERR_INVALID_ARG;
  if (!out_k || !out_v || !aligned(out_k, 16) || !aligned(out_v, 16)) return S4KV_ERR_INVALID_ARG;
  DequantParams p;
  p.pool = static_cast<const uint8_t *>(cache->pool);
  p.out_k = out_k;
  p.out_v = out_v;
  p.pages = nullptr;
  p.err = cache->err_flag;
  p.physical_page = physical_page;
  p.n_pages = 1;
  p.num_pages = cache->num_pages;
  p.num_kv_heads = cache->num_kv_heads;
  p.out_fp32 = out_fp32 ? 1 : 0;
  p.bits = cache_bits(cache);
  launch_dequant(p, static_cast<cudaStream_t>(stream));
  if (cudaGetLastError() != cudaSuccess) return S4KV_ERR_CUDA;
  return S4KV_OK;
}

int s4kv_dequant_pages(const s4kv_cache_t *cache, const int32_t *pages, int n, void *out_k, void *out_v,
                       int out_fp32, void *stream) {
  int rc = check_cache(cache);
  if (rc != S4KV_OK) return rc;
  if (n < 0 || n > 65535) return S4KV_ERR_INVALID_ARG;
  if (n == 0) return S4KV_OK;
  if (!pages || !out_k || !out_v || !aligned(pages, 4) || !aligned(out_k, 16) || !aligned(out_v, 16))
    return S4KV_ERR_INVALID_ARG;
  DequantParams p;
  p.pool = static_cast<const uint8_t *>(cache->pool);
  p.out_k = out_k;
  p.out_v = out_v;
  p.pages = pages;
  p.err = cache->err_flag;
  p.physical_page = 0;
  p.n_pages = n;
  p.num_pages = cache->num_pages;
  p.num_kv_heads = cache->num_kv_heads;
  p.out_fp32 = out_fp32 ? 1 : 0;
  p.bits = cache_bits(cache);
  launch_dequant(p, static_cast<cudaStream_t>(stream));
  if (cudaGetLastError() != cudaSuccess) return S4KV_ERR_CUDA;
  return S4KV_OK;
}

int s4kv_page_record_bytes(const s4kv_cache_t *cache, size_t *bytes) {
  const int rc = check_cache(cache);
  if (rc != S4KV_OK) return rc;
  if (bytes == nullptr) return S4KV_ERR_INVALID_ARG;
  *bytes = record_bytes(cache);
  return S4KV_OK;
}

int s4kv_gather_pages(const s4kv_cache_t *cache, const int32_t *pages, int n, void *dst, void *stream) {
  int rc = check_cache(cache);
  if (rc != S4KV_OK) return rc;
  if (n < 0) return S4KV_ERR_INVALID_ARG;
  if (n == 0) return S4KV_OK;
  if (!pages || !dst || !aligned(pages, 4) || !aligned(dst, 16)) return S4KV_ERR_INVALID_ARG;
  return launch_records(static_cast<const uint8_t *>(cache->pool), static_cast<uint8_t *>(dst), pages, nullptr,
                        static_cast<long long>(record_bytes(cache)), n, cache->num_pages, n,
                        cache->err_flag, S4KV_EFLAG_PAGE_RANGE, stream);
}

int s4kv_scatter_pages(const s4kv_cache_t *cache, const int32_t *pages, int n, const void *src, void *stream) {
  int rc = check_cache(cache);
  if (rc != S4KV_OK) return rc;
  if (n < 0) return S4KV_ERR_INVALID_ARG;
  if (n == 0) return S4KV_OK;
  if (!pages || !src || !aligned(pages, 4) || !aligned(src, 16)) return S4KV_ERR_INVALID_ARG;
  return launch_records(static_cast<const uint8_t *>(src), static_cast<uint8_t *>(cache->pool), nullptr, pages,
                        static_cast<long long>(record_bytes(cache)), n, n, cache->num_pages,
                        cache->err_flag, S4KV_EFLAG_PAGE_RANGE, stream);
}

int s4kv_copy_pages(const s4kv_cache_t *cache, const int32_t *src_pages, const int32_t *dst_pages, int n,
                    void *stream) {
  int rc = check_cache(cache);
  if (rc != S4KV_OK) return rc;
  if (n < 0) return S4KV_ERR_INVALID_ARG;
  if (n == 0) return S4KV_OK;
  if (!src_pages || !dst_pages || !aligned(src_pages, 4) || !aligned(dst_pages, 4)) return S4KV_ERR_INVALID_ARG;
  return launch_records(static_cast<const uint8_t *>(cache->pool), static_cast<uint8_t *>(cache->pool), src_pages,
                        dst_pages, static_cast<long long>(record_bytes(cache)), n,
                        cache->num_pages, cache->num_pages, cache->err_flag, S4KV_EFLAG_PAGE_RANGE, stream);
}

int s4kv_fork_residual(const s4kv_cache_t *cache, const int32_t *src_rows, const int32_t *dst_rows, int n,
                       void *stream) {
  int rc = check_cache(cache);
  if (rc != S4KV_OK) return rc;
  if (n < 0) return S4KV_ERR_INVALID_ARG;
  if (n == 0) return S4KV_OK;
  if (!src_rows || !dst_rows || !aligned(src_rows, 4) || !aligned(dst_rows, 4)) return S4KV_ERR_INVALID_ARG;
  const long long rec = static_cast<long long>(cache->num_kv_heads) * S4KV_PAGE_TOKENS * S4KV_HEAD_DIM * 2;
  rc = launch_records(static_cast<const uint8_t *>(cache->res_k), static_cast<uint8_t *>(cache->res_k), src_rows,
                      dst_rows, rec, n, cache->max_seqs, cache->max_seqs, cache->err_flag, S4KV_EFLAG_SLOT, stream);
  if (rc != S4KV_OK) return rc;
  return launch_records(static_cast<const uint8_t *>(cache->res_v), static_cast<uint8_t *>(cache->res_v), src_rows,
                        dst_rows, rec, n, cache->max_seqs, cache->max_seqs, cache->err_flag, S4KV_EFLAG_SLOT, stream);
}

int s4kv_swap_out(const s4kv_cache_t *cache, const int32_t *pages, int n, void *staging, void *host_dst,
                  void *stream) {
  int rc = s4kv_gather_pages(cache, pages, n, staging, stream);
  if (rc != S4KV_OK || n == 0) return rc;
  if (host_dst == nullptr) return S4KV_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(n) * record_bytes(cache);
  if (cudaMemcpyAsync(host_dst, staging, bytes, cudaMemcpyDeviceToHost, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess) {
    cudaGetLastError();
    return S4KV_ERR_CUDA;
  }
  return S4KV_OK;
}

int s4kv_swap_in(const s4kv_cache_t *cache, const int32_t *pages, int n, void *staging, const void *host_src,
                 void *stream) {
  int rc = check_cache(cache);
  if (rc != S4KV_OK) return rc;
  if (n < 0) return S4KV_ERR_INVALID_ARG;
  if (n == 0) return S4KV_OK;
  if (host_src == nullptr || staging == nullptr || !aligned(staging, 16)) return S4KV_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(n) * record_bytes(cache);
  if (cudaMemcpyAsync(staging, host_src, bytes, cudaMemcpyHostToDevice, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess) {
    cudaGetLastError();
    return S4KV_ERR_CUDA;
  }
  return s4kv_scatter_pages(cache, pages, n, staging, stream);
}

int s4kv_get_error(const s4kv_cache_t *cache, uint32_t *flags, int clear, void *stream) {
  if (cache == nullptr || flags == nullptr) return S4KV_ERR_INVALID_ARG;
  *flags = 0;
  if (cache->err_flag == nullptr) return S4KV_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t host = 0;
  if (cudaMemcpyAsync(&host, cache->err_flag, sizeof(uint32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return S4KV_ERR_CUDA;
  }
  if (clear && host != 0) {
    if (cudaMemsetAsync(cache->err_flag, 0, sizeof(uint32_t), s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
      cudaGetLastError();
      return S4KV_ERR_CUDA;
    }
  }
  *flags = host;
  return host ? S4KV_ERR_DEVICE_CHECK : S4KV_OK;
}

}  // extern "C"
