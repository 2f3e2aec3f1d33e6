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

}  // namespace

extern "C" int s4kv_decode_attention_noalloc(const s4kv_cache_t *cache, const void *q, int num_q_heads,
                                             const int32_t *seq_lens, const int32_t *block_tables,
                                             int batch, int max_pages_per_seq, float sm_scale,
                                             void *out, void *stream) {
  if (cache == nullptr) return S4KV_ERR_INVALID_ARG;
  // the decode workspace this batch needs must fit in the fixed scratch
  // (a pure size query: nothing is launched)
  size_t need = 0;
  int rc = s4kv_decode_workspace_size(batch, cache->num_kv_heads, &need);
  if (rc != S4KV_OK) return rc;
  if (need > static_cast<size_t>(S4KV_NOALLOC_SCRATCH_BYTES)) return S4KV_ERR_WORKSPACE;

  void *scratch = nullptr;
  rc = scratch_address(&scratch);
  if (rc != S4KV_OK) return rc;

  // The decode workspace holds one ticket word per (sequence, kv head) that
  // must be zero when a call starts; the scratch keeps whatever the last call
  // left.  decode_call checks every argument first and only then clears the
  // tickets on the caller's stream and launches, so a rejected call touches
  // neither the scratch nor the GPU.
  return s4kv::decode_call(cache, nullptr, nullptr, q, num_q_heads, seq_lens, block_tables, batch,
                           max_pages_per_seq, sm_scale, out, scratch,
                           static_cast<size_t>(S4KV_NOALLOC_SCRATCH_BYTES), stream, true);
}
