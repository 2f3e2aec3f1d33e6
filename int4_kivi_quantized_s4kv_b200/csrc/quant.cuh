// Page quantization by one 128-thread CTA, shared by s4kv_append and the
// fused append of s4kv_append_decode so that both write the same bytes.
//
// KIVI split ("S4 KV -- int4 KV-Cache-Kompression fuer vLLM", "Funktionsweise"
// step 1): keys asymmetric int4 per channel (one group = one channel over the
// page's 16 tokens), values int4 per token (groups of 32 channels).
#pragma once

#include "common.cuh"

namespace s4kv {

// Quantize one page of one kv head.  ks / vs: the page's fp16 keys and values
// [16][128] in shared memory (complete before the call); kc / vc: [16][128]
// byte scratch in shared memory; blk: the 2816-byte block in global memory.
// Called by all 128 threads of the CTA (tid = threadIdx.x, whole warps);
// contains CTA barriers.
__device__ __forceinline__ void quantize_page_cta(const __half (*ks)[kHeadDim], const __half (*vs)[kHeadDim],
                                                  uint8_t (*kc)[kHeadDim], uint8_t (*vc)[kHeadDim], uint8_t *blk,
                                                  int tid) {
  // keys: thread c quantizes channel c over the 16 tokens
  {
    const int c = tid;
    float mn = __half2float(ks[0][c]), mx = mn;
#pragma unroll
    for (int t = 1; t < kPage; ++t) {
      const float x = __half2float(ks[t][c]);
      if (total_less(x, mn)) mn = x;
      if (total_less(mx, x)) mx = x;
    }
    const float s = group_scale(mn, mx);
    const float inv = __frcp_rn(s);
#pragma unroll
    for (int t = 0; t < kPage; ++t)
      kc[t][c] = static_cast<uint8_t>(group_code_fast(__half2float(ks[t][c]), mn, s, inv));
    reinterpret_cast<__half *>(blk + kKScaleOff)[c] = __float2half_rn(s);
    // zero points in the MMA k order: tile (c%32)/4, slot 2(c/32) + (c%2) + 8((c%4)/2)
    const int zslot = 16 * ((c & 31) >> 2) + 2 * (c >> 5) + (c & 1) + 8 * ((c & 3) >> 1);
    reinterpret_cast<__half *>(blk + kKZeroOff)[zslot] = __float2half_rn(mn);
  }
  // values: one (token, 32-channel group) per thread pair; each thread takes
  // 16 channels and the pair combines its minima and maxima
  {
    const int t = tid >> 3, g = (tid >> 1) & 3, c0 = g * kVGroup + (tid & 1) * (kVGroup / 2);
    float mn = __half2float(vs[t][c0]), mx = mn;
#pragma unroll
    for (int j = 1; j < kVGroup / 2; ++j) {
      const float x = __half2float(vs[t][c0 + j]);
      if (total_less(x, mn)) mn = x;
      if (total_less(mx, x)) mx = x;
    }
    const float omn = __shfl_xor_sync(0xFFFFFFFFu, mn, 1), omx = __shfl_xor_sync(0xFFFFFFFFu, mx, 1);
    if (total_less(omn, mn)) mn = omn;
    if (total_less(mx, omx)) mx = omx;
    const float s = group_scale(mn, mx);
    const float inv = __frcp_rn(s);
#pragma unroll
    for (int j = 0; j < kVGroup / 2; ++j)
      vc[t][c0 + j] = static_cast<uint8_t>(group_code_fast(__half2float(vs[t][c0 + j]), mn, s, inv));
    if ((tid & 1) == 0) {
      reinterpret_cast<__half *>(blk + kVScaleOff)[g * kPage + t] = __float2half_rn(s);
      reinterpret_cast<__half *>(blk + kVZeroOff)[g * kPage + t] = __float2half_rn(mn);
    }
  }
  __syncthreads();
  // pack: word w = 128*hh + 4*lane + q; nibble j is register j&3, half j>>2
  // of that lane's m16n8k16 operand fragment (tile = 4*hh + q)
  for (int w = tid; w < 256; w += 128) {
    const int hh = w >> 7, lane = (w >> 2) & 31, q = w & 3;
    const int n = lane >> 2, i = lane & 3, tile = 4 * hh + q;
    uint32_t kw = 0, vw = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      // keys: row = token, k axis = channel 32i + 4*tile + {0,1 | 2,3}
      const int kt = 8 * (j & 1) + n;
      const int kch = 32 * i + 4 * tile + 2 * ((j >> 1) & 1) + (j >> 2);
      kw |= static_cast<uint32_t>(kc[kt][kch]) << (4 * j);
      // values: row = channel of M-tile `tile`, k axis = token
      const int vt = 2 * i + (j >> 2) + 8 * ((j >> 1) & 1);
      const int vch = 32 * (tile >> 1) + 4 * n + 2 * (tile & 1) + (j & 1);
      vw |= static_cast<uint32_t>(vc[vt][vch]) << (4 * j);
    }
    reinterpret_cast<uint32_t *>(blk + kKCodeOff)[w] = kw;
    reinterpret_cast<uint32_t *>(blk + kVCodeOff)[w] = vw;
  }
}

}  // namespace s4kv
