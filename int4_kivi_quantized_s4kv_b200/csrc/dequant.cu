// s4kv_dequant_page / s4kv_dequant_pages device side: physical pages, all kv
// heads, back to natural [token][channel] order (page i of a list goes to
// output slot i).  x = code * scale + zero in fp32 (the
// product of a code of at most 8 bits and an fp16 scale is exact, so this is
// a single rounding); the fp16 output is that fp32 value rounded to nearest
// even.
#include "code_map.cuh"
#include "kernels.cuh"

namespace s4kv {

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
  const float kz = __half2float(reinterpret_cast<const __half *>(blk + kzero_off)[key_zero_slot(c)]);
  const int g = c / kVGroup;
  for (int t = 0; t < kPage; ++t) {
    int kword, knib, vword, vnib;
    key_position(t, c, kword, knib);
    value_position(t, c, vword, vnib);
    const float kcode = static_cast<float>(code_at(blk + kcode_off, kword, knib, p.bits));
    const float vcode = static_cast<float>(code_at(blk + vcode_off, vword, vnib, p.bits));
    const float vs = __half2float(reinterpret_cast<const __half *>(blk + vscale_off)[value_scale_slot(t, g)]);
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
