// s4kv_decode_attention_noalloc: decode attention whose scratch memory is a
// fixed array inside this library instead of a caller-allocated workspace.
//
// Some callers cannot call cudaMalloc: a plugin running inside a host engine
// that owns the device's whole memory pool and forbids allocations outside
// it, or a latency-critical path that cannot afford cudaMalloc's implicit
// device-wide synchronisation.  For them this entry point takes the same
// inputs and outputs as s4kv_decode_attention but no workspace.
//
// The scratch is one file-scope device array of S4KV_NOALLOC_SCRATCH_BYTES.
// Every GPU that loads the library holds it until the process exits, and
// all calls on a device share it, so calls whose kernels overlap on the GPU
// (different streams without ordering between them) race on it.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "kernels.cuh"

namespace {

constexpr int kMaxDevices = 64;

// The scratch array.  In host code this name is only a host-side stand-in:
// its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[S4KV_NOALLOC_SCRATCH_BYTES];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device, looked up once
// per device with that device current.
int scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return S4KV_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void *ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return S4KV_ERR_CUDA;
    }
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return S4KV_OK;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" int s4kv_decode_attention_noalloc(const s4kv_cache_t *cache, const void *q, int num_q_heads,
                                             const int32_t *seq_lens, const int32_t *block_tables,
                                             int batch, int max_pages_per_seq, float sm_scale,
                                             void *out, void *stream) {
  // the same host checks s4kv_decode_attention makes, done here first so a
  // rejected call launches nothing (not even the scratch clear below)
  if (cache == nullptr) return S4KV_ERR_INVALID_ARG;
  int rc = s4kv_check_model(cache->head_dim, cache->page_tokens, num_q_heads, cache->num_kv_heads);
  if (rc != S4KV_OK) return rc;
  if (cache->pool == nullptr || cache->res_k == nullptr || cache->res_v == nullptr ||
      cache->num_pages <= 0 || cache->max_seqs <= 0 || !aligned(cache->pool, 128) ||
      !aligned(cache->res_k, 16) || !aligned(cache->res_v, 16))
    return S4KV_ERR_INVALID_ARG;
  if (batch < 0 || batch > cache->max_seqs || max_pages_per_seq <= 0) return S4KV_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale) || sm_scale <= 0.0f) return S4KV_ERR_INVALID_ARG;
  if (batch == 0) return S4KV_OK;
  if (!q || !seq_lens || !block_tables || !out || !aligned(q, 16) || !aligned(out, 8) ||
      !aligned(seq_lens, 4) || !aligned(block_tables, 4))
    return S4KV_ERR_INVALID_ARG;

  // the decode workspace this batch needs must fit in the fixed scratch
  size_t need = 0;
  rc = s4kv_decode_workspace_size(batch, cache->num_kv_heads, &need);
  if (rc != S4KV_OK) return rc;
  if (need > static_cast<size_t>(S4KV_NOALLOC_SCRATCH_BYTES)) return S4KV_ERR_WORKSPACE;

  void *scratch = nullptr;
  rc = scratch_address(&scratch);
  if (rc != S4KV_OK) return rc;

  // The decode workspace begins with one ticket word per (sequence, kv head)
  // that must be zero when a call starts; the scratch keeps whatever the
  // last call left, so clear them on the caller's stream.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t ticket_bytes = static_cast<size_t>(batch) * cache->num_kv_heads * sizeof(uint32_t);
  if (cudaMemsetAsync(scratch, 0, ticket_bytes, s) != cudaSuccess) {
    cudaGetLastError();
    return S4KV_ERR_CUDA;
  }
  return s4kv_decode_attention(cache, q, num_q_heads, seq_lens, block_tables, batch, max_pages_per_seq,
                               sm_scale, out, scratch, static_cast<size_t>(S4KV_NOALLOC_SCRATCH_BYTES),
                               stream);
}
