// Launch parameters and launchers of the s4kv kernels (internal).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace s4kv {

struct AppendParams {
  uint8_t *pool;
  __half *res_k;
  __half *res_v;
  uint32_t *err;
  const __half *k;
  const __half *v;
  const int64_t *slot_mapping;
  const int32_t *cu_new;
  const int32_t *seq_lens;
  const int32_t *block_tables;
  int num_pages;
  int num_kv_heads;
  int max_pages;
  int max_new;
  int n_tokens;
  int bits;  // code width, 4 or 8
};

struct DequantParams {
  const uint8_t *pool;
  void *out_k;
  void *out_v;
  const int32_t *pages;  // device page list, or nullptr: the one physical_page
  uint32_t *err;
  int physical_page;
  int n_pages;
  int num_pages;
  int num_kv_heads;
  int out_fp32;
  int bits;  // code width, 4 or 8
};

// Copy of whole records: item i copies rec_bytes from
// src_base + (src_idx ? src_idx[i] : i) * rec_bytes to
// dst_base + (dst_idx ? dst_idx[i] : i) * rec_bytes.  An index outside
// [0, src_limit) / [0, dst_limit) sets err_bit and the item is skipped.
struct MoveParams {
  const uint8_t *src_base;
  uint8_t *dst_base;
  const int32_t *src_idx;
  const int32_t *dst_idx;
  uint32_t *err;
  long long rec_bytes;  // a multiple of 16
  int n;
  int src_limit;
  int dst_limit;
  uint32_t err_bit;
};

struct DecodeParams {
  const uint8_t *pool;
  const __half *res_k;
  const __half *res_v;
  const __half *q;
  __half *out;
  const int32_t *seq_lens;
  const int32_t *block_tables;
  float *part;        // [2 * num_workers][8][128] partial O (unnormalised)
  float2 *part_ml;    // [2 * num_workers][8] (running max m, sum l)
  uint32_t *tickets;  // [batch * num_kv_heads], zero between calls
  uint32_t *err;
  int batch;
  int num_q_heads;
  int num_kv_heads;
  int group;
  int max_pages;
  int num_pages;
  float scale_log2;   // sm_scale * log2(e)
  int num_workers;
};

// The append of a decode step (s4kv_append_decode): each sequence's new
// token (fp16 [batch][kv_heads][128]) is written into the cache by an append
// grid that the decode grid depends on.  Both nullptr for a plain decode.
struct FusedAppend {
  const __half *k_new;
  const __half *v_new;
};

void launch_append(const AppendParams &p, int batch, int max_new, cudaStream_t stream);
void launch_dequant(const DequantParams &p, cudaStream_t stream);
void launch_move(const MoveParams &p, cudaStream_t stream);
cudaError_t launch_decode(const DecodeParams &p, const FusedAppend &f, int bits, int num_ctas, cudaStream_t stream);
int decode_warps_per_cta(int bits);
size_t decode_smem_bytes(int bits);

// Host entry of every decode call (plain, fused append, no-alloc): checks all
// arguments, then -- only when they pass and clear_tickets is set -- zeroes
// the workspace's ticket words on `stream`, then launches.  Returns an
// S4KV_* status; an invalid call touches nothing.
int decode_call(const s4kv_cache_t *cache, const void *k_new, const void *v_new, const void *q, int num_q_heads,
                const int32_t *seq_lens, const int32_t *block_tables, int batch, int max_pages_per_seq,
                float sm_scale, void *out, void *workspace, size_t workspace_bytes, void *stream,
                bool clear_tickets);

}  // namespace s4kv
