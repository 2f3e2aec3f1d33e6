// Page quantization by one 128-thread CTA, shared by s4kv_append and the
// step append grid of s4kv_append_decode so that both write the same bytes.
//
// KIVI split ("S4 KV -- int4 KV-Cache-Kompression fuer vLLM", "Funktionsweise"
// step 1): keys asymmetric int4 per channel (one group = one channel over the
// page's 16 tokens), values int4 per token (groups of 32 channels); the INT8
// variant ("KV-Cache-Optimierung -- PagedAttention, quantisierter KV,
// Speculative Cache", "Warum es zaehlt": INT8/INT4 KV) uses 255 levels and
// the 2-bit one (KIVI's own width) 3.
#pragma once

#include "common.cuh"

namespace s4kv {

// Quantize one page of one kv head.  ks / vs: the page's fp16 keys and values
// [16][128] in shared memory (complete before the call); kc / vc: [16][128]
// byte scratch in shared memory; blk: the 2816-byte block in global memory.
// Called by every thread of the CTA (tid = threadIdx.x, at least 128
// threads, whole warps): threads 0..127 do the work, and all of them meet at
// the CTA barrier inside.
template <int kBits>
__device__ __forceinline__ void quantize_page_cta(const __half (*ks)[kHeadDim], const __half (*vs)[kHeadDim],
                                                  uint8_t (*kc)[kHeadDim], uint8_t (*vc)[kHeadDim], uint8_t *blk,
                                                  int tid) {
  using F = Fmt<kBits>;
  // keys: thread c quantizes channel c over the 16 tokens
  if (tid < 128) {
    const int c = tid;
    float mn = __half2float(ks[0][c]), mx = mn;
#pragma unroll
    for (int t = 1; t < kPage; ++t) {
      const float x = __half2float(ks[t][c]);
      if (total_less(x, mn)) mn = x;
      if (total_less(mx, x)) mx = x;
    }
    const float s = group_scale(mn, mx, F::kLevels);
    const float inv = __frcp_rn(s);
#pragma unroll
    for (int t = 0; t < kPage; ++t)
      kc[t][c] = static_cast<uint8_t>(group_code_fast(__half2float(ks[t][c]), mn, s, inv, F::kLevels));
    reinterpret_cast<__half *>(blk + F::kKScale)[c] = __float2half_rn(s);
    // zero points in the MMA k order: tile (c%32)/4, slot 2(c/32) + (c%2) + 8((c%4)/2)
    const int zslot = 16 * ((c & 31) >> 2) + 2 * (c >> 5) + (c & 1) + 8 * ((c & 3) >> 1);
    reinterpret_cast<__half *>(blk + F::kKZero)[zslot] = __float2half_rn(mn);
  }
  // values: one (token, 32-channel group) per thread pair; each thread takes
  // 16 channels and the pair combines its minima and maxima
  if (tid < 128) {
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
    const float s = group_scale(mn, mx, F::kLevels);
    const float inv = __frcp_rn(s);
#pragma unroll
    for (int j = 0; j < kVGroup / 2; ++j)
      vc[t][c0 + j] = static_cast<uint8_t>(group_code_fast(__half2float(vs[t][c0 + j]), mn, s, inv, F::kLevels));
    if ((tid & 1) == 0) {
      reinterpret_cast<__half *>(blk + F::kVScale)[value_scale_slot(t, g)] = __float2half_rn(s);
      reinterpret_cast<__half *>(blk + F::kVZero)[g * kPage + t] = __float2half_rn(mn);
    }
  }
  __syncthreads();
  if (tid >= 128) return;
  // (token, channel) at register r, half e of the operand fragment of tile
  // `tile`, lane = 4n + i
  auto key_tc = [](int tile, int n, int i, int r, int e, int &t, int &c) {
    t = 8 * (r & 1) + n;                               // row = token
    c = 32 * i + 4 * tile + 2 * (r >> 1) + e;          // k axis = channel
  };
  auto val_tc = [](int tile, int n, int i, int r, int e, int &t, int &c) {
    t = 2 * i + e + 8 * (r >> 1);                             // k axis = token
    c = 32 * (tile >> 1) + 4 * n + 2 * (tile & 1) + (r & 1);  // row = channel
  };
  if (kBits == 4) {
    // word w = 128*hh + 4*lane + q is lane's fragment of tile 4*hh + q;
    // register r, half e at nibble nibble_of(r, e)
    for (int w = tid; w < 256; w += 128) {
      const int hh = w >> 7, lane = (w >> 2) & 31, q = w & 3;
      const int n = lane >> 2, i = lane & 3, tile = 4 * hh + q;
      uint32_t kw = 0, vw = 0;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          int t, c;
          key_tc(tile, n, i, r, e, t, c);
          kw |= static_cast<uint32_t>(kc[t][c]) << (4 * nibble_of(r, e));
          val_tc(tile, n, i, r, e, t, c);
          vw |= static_cast<uint32_t>(vc[t][c]) << (4 * nibble_of(r, e));
        }
      }
      reinterpret_cast<uint32_t *>(blk + F::kKCode)[w] = kw;
      reinterpret_cast<uint32_t *>(blk + F::kVCode)[w] = vw;
    }
  } else if (kBits == 2) {
    // word 4 lane + m holds tiles 2m, 2m + 1 of the lane: register r, half e
    // of tile 2m + p at bit 16 e + 2 (4 p + r)
    for (int w = tid; w < 128; w += 128) {
      const int lane = w >> 2, m = w & 3;
      const int n = lane >> 2, i = lane & 3;
      uint32_t kw = 0, vw = 0;
#pragma unroll
      for (int p = 0; p < 2; ++p) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int bit = 16 * e + 2 * (4 * p + r);
            int t, c;
            key_tc(2 * m + p, n, i, r, e, t, c);
            kw |= static_cast<uint32_t>(kc[t][c]) << bit;
            val_tc(2 * m + p, n, i, r, e, t, c);
            vw |= static_cast<uint32_t>(vc[t][c]) << bit;
          }
        }
      }
      reinterpret_cast<uint32_t *>(blk + F::kKCode)[w] = kw;
      reinterpret_cast<uint32_t *>(blk + F::kVCode)[w] = vw;
    }
  } else {
    // byte (32 m + lane) * 16 + 8 (tile % 2) + 2 r + e holds register r, half
    // e of tile 2m + tile % 2
    for (int w = tid; w < 512; w += 128) {
      const int chunk = w >> 2, within = w & 3;
      const int m = chunk >> 5, lane = chunk & 31;
      const int tile = 2 * m + (within >> 1), r0 = 2 * (within & 1);
      const int n = lane >> 2, i = lane & 3;
      uint32_t kw = 0, vw = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int r = r0 + (b >> 1), e = b & 1;
        int t, c;
        key_tc(tile, n, i, r, e, t, c);
        kw |= static_cast<uint32_t>(kc[t][c]) << (8 * b);
        val_tc(tile, n, i, r, e, t, c);
        vw |= static_cast<uint32_t>(vc[t][c]) << (8 * b);
      }
      reinterpret_cast<uint32_t *>(blk + F::kKCode)[w] = kw;
      reinterpret_cast<uint32_t *>(blk + F::kVCode)[w] = vw;
    }
  }
}

}  // namespace s4kv
