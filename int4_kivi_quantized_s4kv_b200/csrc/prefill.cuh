// Launch parameters and launchers of the prefill (chunked-append) attention
// kernels (internal).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace s4kv {

struct PrefillParams {
  const uint8_t *pool;
  const __half *res_k;
  const __half *res_v;
  const __half *q;        // [n_tokens][num_q_heads][128]
  __half *out;            // [n_tokens][num_q_heads][128]
  const int32_t *cu_new;  // [batch + 1]
  const int32_t *seq_lens;
  const int32_t *block_tables;
  uint32_t *err;
  int n_tokens;
  int num_q_heads;
  int num_kv_heads;
  int group;
  int max_pages;
  int num_pages;
  float scale_log2;       // sm_scale * log2(e)
  uint8_t *ws;            // operand tiles [batch][num_kv_heads][tiles_per_seq][tile bytes]
  int tiles_per_seq;      // key tiles of max_pages pages
  int bits;               // code width, 2, 4 or 8
};

cudaError_t launch_prefill(const PrefillParams &p, int batch, int max_new, cudaStream_t stream);
size_t prefill_smem_bytes();
size_t prefill_tile_bytes();
int prefill_tiles_per_seq(int max_pages);

}  // namespace s4kv
