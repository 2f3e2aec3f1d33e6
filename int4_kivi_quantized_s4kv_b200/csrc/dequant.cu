// s4kv_dequant_page / s4kv_dequant_pages device side: physical pages, all kv
// heads, back to natural [token][channel] order (page i of a list goes to
// output slot i).  x = code * scale + zero in fp32 (the
// product of a 4- or 8-bit code and an fp16 scale is exact, so this is a
// single rounding); the fp16 output is that fp32 value rounded to nearest
// even.
#include "kernels.cuh"

namespace s4kv {

// The code at 4-bit position (word, nibble): that nibble, or with 8-bit
// codes the byte holding the same fragment place (tile 4*(word/128) +
// word%4, lane (word/4)%32, register nibble%4, half nibble/4).
__device__ __forceinline__ uint32_t code_at(const uint8_t *region, int word, int nibble, int bits) {
  if (bits == 8) {
    const int tile = 4 * (word >> 7) + (word & 3), lane = (word >> 2) & 31;
    return region[((tile >> 1) * 32 + lane) * 16 + (tile & 1) * 8 + 2 * (nibble & 3) + (nibble >> 2)];
  }
  if (bits == 2) {
    const int tile = 4 * (word >> 7) + (word & 3), lane = (word >> 2) & 31;
    const uint32_t w = reinterpret_cast<const uint32_t *>(region)[4 * lane + (tile >> 1)];
    return (w >> (16 * (nibble >> 2) + 2 * (4 * (tile & 1) + (nibble & 3)))) & 3u;
  }
  const uint32_t w = reinterpret_cast<const uint32_t *>(region)[word];
  return (w >> (4 * nibble)) & 0xFu;
}

__global__ void __launch_bounds__(128) dequant_kernel(const DequantParams p) {
  const int h = blockIdx.x;
  const int c = threadIdx.x;  // channel
  const int slot = blockIdx.y;
  int page = p.physical_page;
  if (p.pages != nullptr) {
    page = __ldg(p.pages + slot);
    if (static_cast<unsigned>(page) >= static_cast<unsigned>(p.num_pages)) {
      if (c == 0) flag_error(p.err, S4KV_EFLAG_PAGE_RANGE);
      return;
    }
  }
  // regions of the block: codes, then the same 768 bytes of fp16 metadata
  const int code_bytes = kPage * kHeadDim * p.bits / 8;
  const int kcode_off = 0, vcode_off = code_bytes;
  const int kscale_off = 2 * code_bytes, kzero_off = kscale_off + 2 * kHeadDim;
  const int vscale_off = kzero_off + 2 * kHeadDim, vzero_off = vscale_off + 2 * kPage * (kHeadDim / kVGroup);
  const uint8_t *blk = p.pool + (static_cast<long>(page) * p.num_kv_heads + h) * block_bytes_for(p.bits);
  const float ks = __half2float(reinterpret_cast<const __half *>(blk + kscale_off)[c]);
  const int zslot = 16 * ((c & 31) >> 2) + 2 * (c >> 5) + (c & 1) + 8 * ((c & 3) >> 1);
  const float kz = __half2float(reinterpret_cast<const __half *>(blk + kzero_off)[zslot]);
  const int g = c / kVGroup;
  // key fragment coordinates of channel c: lane quarter i, tile kt, pair e
  const int ki = c >> 5, kt = (c & 31) >> 2, ke = c & 3;
  // value fragment coordinates of channel c: M-tile m, row group n
  const int vn = (c & 31) >> 2, ve = c & 3, vm = 2 * g + (ve >> 1);
  for (int t = 0; t < kPage; ++t) {
    const int kword = 128 * (kt >> 2) + 4 * (4 * (t & 7) + ki) + (kt & 3);
    const int knib = (t >> 3) + 2 * (ke >> 1) + 4 * (ke & 1);
    const int vi = (t & 7) >> 1;
    const int vword = 128 * (vm >> 2) + 4 * (4 * vn + vi) + (vm & 3);
    const int vnib = (ve & 1) + 2 * (t >> 3) + 4 * (t & 1);
    const float kcode = static_cast<float>(code_at(blk + kcode_off, kword, knib, p.bits));
    const float vcode = static_cast<float>(code_at(blk + vcode_off, vword, vnib, p.bits));
    const float vs = __half2float(reinterpret_cast<const __half *>(blk + vscale_off)[g * kPage + t]);
    const float vz = __half2float(reinterpret_cast<const __half *>(blk + vzero_off)[g * kPage + t]);
    const float kx = __fadd_rn(__fmul_rn(kcode, ks), kz);
    const float vx = __fadd_rn(__fmul_rn(vcode, vs), vz);
    const long o = ((static_cast<long>(slot) * p.num_kv_heads + h) * kPage + t) * kHeadDim + c;
    if (p.out_fp32) {
      static_cast<float *>(p.out_k)[o] = kx;
      static_cast<float *>(p.out_v)[o] = vx;
    } else {
      static_cast<__half *>(p.out_k)[o] = __float2half_rn(kx);
      static_cast<__half *>(p.out_v)[o] = __float2half_rn(vx);
    }
  }
}

void launch_dequant(const DequantParams &p, cudaStream_t stream) {
  dequant_kernel<<<dim3(p.num_kv_heads, p.n_pages), 128, 0, stream>>>(p);
}

}  // namespace s4kv
