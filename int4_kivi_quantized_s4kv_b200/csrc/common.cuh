// Internal device helpers of the s4kv CUDA library (sm_100a only).
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "s4kv.h"

namespace s4kv {

constexpr int kHeadDim = S4KV_HEAD_DIM;
constexpr int kPage = S4KV_PAGE_TOKENS;
constexpr int kVGroup = S4KV_VALUE_GROUP;
constexpr int kBlockBytes = S4KV_BLOCK_BYTES;
constexpr int kKCodeOff = 0;
constexpr int kVCodeOff = 1024;
constexpr int kKScaleOff = 2048;
constexpr int kKZeroOff = 2304;
constexpr int kVScaleOff = 2560;
constexpr int kVZeroOff = 2688;

// Block layout of one (page, kv head) with kBits-bit codes (2, 4 or 8): K codes,
// V codes, K scale fp16 [128], K zero fp16 [128] (MMA k order), V scale fp16
// [64] (lane-major, value_scale_slot), V zero fp16 [4][16].  Fmt<4> is the
// 2816-byte int4 block above.
// 8-bit codes keep the int4 assignment of (token, channel) to MMA operand
// fragments with bytes for nibbles: a lane's 8 codes of one tile are 8
// consecutive bytes (register r at bytes 2r, 2r + 1) and the 16 bytes of
// tiles 2m, 2m + 1 of lane l sit at (32 m + l) * 16.  2-bit codes keep it
// with bit pairs: the 16 codes of tiles 2m, 2m + 1 of lane l are word
// 4 l + m, half 0 of every register in the low 16 bits and half 1 in the
// high 16 bits, register r of tile 2m + p at bits 2 (4 p + r) of its half.
template <int kBits>
struct Fmt {
  static constexpr int kCodeBytes = kPage * kHeadDim * kBits / 8;
  static constexpr int kKCode = 0;
  static constexpr int kVCode = kCodeBytes;
  static constexpr int kKScale = 2 * kCodeBytes;
  static constexpr int kKZero = kKScale + 2 * kHeadDim;
  static constexpr int kVScale = kKZero + 2 * kHeadDim;
  static constexpr int kVZero = kVScale + 2 * kPage * (kHeadDim / kVGroup);
  static constexpr int kBlock = kVZero + 2 * kPage * (kHeadDim / kVGroup);
  static constexpr int kLevels = (1 << kBits) - 1;
};
static_assert(Fmt<4>::kBlock == kBlockBytes && Fmt<4>::kVZero == kVZeroOff, "int4 block layout");
static_assert(Fmt<8>::kBlock == S4KV_BLOCK_BYTES_INT8, "int8 block layout");
static_assert(Fmt<2>::kBlock == S4KV_BLOCK_BYTES_INT2, "int2 block layout");

__host__ __device__ constexpr int block_bytes_for(int bits) {
  return bits == 8 ? Fmt<8>::kBlock : bits == 2 ? Fmt<2>::kBlock : Fmt<4>::kBlock;
}

__device__ __forceinline__ void flag_error(uint32_t *err, uint32_t bits) {
  if (err != nullptr) atomicOr(err, bits);
}

// ------------------------------------------------------------ quantizer --

// a < b in IEEE total order for non-NaN values (-0 below +0).
__device__ __forceinline__ bool total_less(float a, float b) {
  return a < b || (a == b && signbit(a) && !signbit(b));
}

// One quantization group in fp32: s = (max - min) / 15 and
// code = s == 0 ? 0 : clamp(rint((x - min) / s), 0, 15), every operation
// IEEE-rounded (no contraction, no fast math).
__device__ __forceinline__ float group_scale(float mn, float mx, int levels = 15) {
  return __fdiv_rn(__fsub_rn(mx, mn), static_cast<float>(levels));
}
__device__ __forceinline__ uint32_t group_code(float x, float mn, float s) {
  if (s == 0.0f) return 0u;
  float r = rintf(__fdiv_rn(__fsub_rn(x, mn), s));
  r = fminf(fmaxf(r, 0.0f), 15.0f);
  return static_cast<uint32_t>(r);
}

// The same code with the division replaced by a product with inv_s =
// RN(1 / s) wherever that cannot change it: with x_ = x - min and x_ / s <=
// 256, the product is within 2^-15 of x_ / s and RN(x_ / s) within 2^-16, so
// the two round to the same integer unless the product lies within 2^-10 of
// a half-integer; only then is the division done.
__device__ __forceinline__ uint32_t group_code_fast(float x, float mn, float s, float inv_s, int levels = 15) {
  if (s == 0.0f) return 0u;
  const float d = __fsub_rn(x, mn);
  const float q = __fmul_rn(d, inv_s);
  float r = rintf(q);
  if (fabsf(fabsf(__fsub_rn(q, r)) - 0.5f) < 0x1p-10f) r = rintf(__fdiv_rn(d, s));
  r = fminf(fmaxf(r, 0.0f), static_cast<float>(levels));
  return static_cast<uint32_t>(r);
}

// ---------------------------------------------------------------- bit ops --

// (a & b) | c in one LOP3.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) {
  return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) {
  return *reinterpret_cast<__half2 *>(&u);
}

// Place of a code in a lane's m16n8k16 operand fragment (register r, half e)
// <-> nibble of the lane's packed 32-bit word: the low nibbles of the word's
// bytes 0-1 are register 0 and those of bytes 2-3 register 2, the high
// nibbles of bytes 0-1 register 1 and of bytes 2-3 register 3, the lower
// byte of each pair in the lower half.
__host__ __device__ constexpr int nibble_of(int r, int e) { return (r & 1) + 2 * e + 4 * (r >> 1); }
__host__ __device__ constexpr int reg_of_nibble(int j) { return (j & 1) + 2 * (j >> 2); }
__host__ __device__ constexpr int half_of_nibble(int j) { return (j >> 1) & 1; }

// Position (in halves) of the value scale of (token t, group g): lane quad
// i = (t%8)/2 reads the token pairs 2i + 8e, 2i + 8e + 1 (e = t/8) of all four
// groups as 32 consecutive bytes.
__host__ __device__ constexpr int value_scale_slot(int t, int g) {
  return 16 * ((t & 7) >> 1) + 8 * (t >> 3) + 2 * g + (t & 1);
}

// fp8 e4m3 pair -> f16x2, the lower byte into the lower half.  A 4-bit code c
// in the low nibble of an e4m3 byte (sign and upper exponent bits zero) is
// c * 2^-9 exactly: codes 0..7 are the subnormals m * 2^-9 and codes 8..15
// the first normal binade 2^-6 (1 + m/8), whose step is the same 2^-9.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t x) {
  uint32_t d;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(x));
  return d;
}

// Eight 4-bit codes of a packed word -> the four f16x2 registers of one
// lane's m16n8k16 operand fragment, each value code * 2^-9 (exact): the low
// and the high nibble of every byte masked into bytes of their own (one
// shift, two LOP3), then one conversion per byte pair.
__device__ __forceinline__ void unpack_codes_s9(uint32_t w, uint32_t &a0, uint32_t &a1, uint32_t &a2,
                                                uint32_t &a3) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
  uint16_t l0, l1, h0, h1;
  asm("mov.b32 {%0,%1}, %2;" : "=h"(l0), "=h"(l1) : "r"(lo));
  asm("mov.b32 {%0,%1}, %2;" : "=h"(h0), "=h"(h1) : "r"(hi));
  a0 = e4m3x2_to_f16x2(l0);
  a1 = e4m3x2_to_f16x2(h0);
  a2 = e4m3x2_to_f16x2(l1);
  a3 = e4m3x2_to_f16x2(h1);
}

// The same registers holding the codes themselves (the exact factor 512
// applied in fp16).
__device__ __forceinline__ void unpack_codes(uint32_t w, uint32_t &a0, uint32_t &a1, uint32_t &a2, uint32_t &a3) {
  unpack_codes_s9(w, a0, a1, a2, a3);
  const __half2 k512 = u32_as_h2(0x60006000u);
  a0 = h2_as_u32(__hmul2(u32_as_h2(a0), k512));
  a1 = h2_as_u32(__hmul2(u32_as_h2(a1), k512));
  a2 = h2_as_u32(__hmul2(u32_as_h2(a2), k512));
  a3 = h2_as_u32(__hmul2(u32_as_h2(a3), k512));
}

// One lane's 8-bit tile fragment (two words, registers 0-1 in w0 and 2-3 in
// w1, the low half of a register in its lower byte) -> the four f16x2
// registers: each byte pair is laid into the mantissa of 1024 (0x64 high
// bytes, one byte permute) and the 1024 removed exactly in fp16.
__device__ __forceinline__ void unpack_codes8(uint32_t w0, uint32_t w1, uint32_t &a0, uint32_t &a1,
                                              uint32_t &a2, uint32_t &a3) {
  const __half2 k1024 = u32_as_h2(0x64006400u);
  uint32_t p0, p1, p2, p3;
  asm("prmt.b32 %0, %1, %2, 0x7170;" : "=r"(p0) : "r"(w0), "r"(0x64646464u));
  asm("prmt.b32 %0, %1, %2, 0x7372;" : "=r"(p1) : "r"(w0), "r"(0x64646464u));
  asm("prmt.b32 %0, %1, %2, 0x7170;" : "=r"(p2) : "r"(w1), "r"(0x64646464u));
  asm("prmt.b32 %0, %1, %2, 0x7372;" : "=r"(p3) : "r"(w1), "r"(0x64646464u));
  a0 = h2_as_u32(__hsub2(u32_as_h2(p0), k1024));
  a1 = h2_as_u32(__hsub2(u32_as_h2(p1), k1024));
  a2 = h2_as_u32(__hsub2(u32_as_h2(p2), k1024));
  a3 = h2_as_u32(__hsub2(u32_as_h2(p3), k1024));
}

// One register of a lane's 2-bit tile fragment: codes at bit 2k of both
// halves of `w` (k = 4 * tile parity + register).  Below bit 10 a code c is
// laid into the mantissa of 1024 as 1024 + c * 4^k (exact: at most 1792) and
// scaled back exactly by one fp16 multiply-add; codes above are first moved
// down by 10 bits.
template <int k>
__device__ __forceinline__ uint32_t unpack_code2(uint32_t w, uint32_t w10) {
  constexpr int kk = k <= 4 ? k : k - 5;
  const uint32_t src = k <= 4 ? w : w10;
  const uint32_t x = and_or(src, 0x00030003u << (2 * kk), 0x64006400u);
  if (kk == 0) return h2_as_u32(__hsub2(u32_as_h2(x), u32_as_h2(0x64006400u)));
  // fp16 pairs of 4^-kk (1/4, 1/16, 1/64, 1/256) and -1024 * 4^-kk
  constexpr uint32_t kScale = kk == 1 ? 0x34003400u : kk == 2 ? 0x2C002C00u : kk == 3 ? 0x24002400u : 0x1C001C00u;
  constexpr uint32_t kBias = kk == 1 ? 0xDC00DC00u : kk == 2 ? 0xD400D400u : kk == 3 ? 0xCC00CC00u : 0xC400C400u;
  return h2_as_u32(__hfma2(u32_as_h2(x), u32_as_h2(kScale), u32_as_h2(kBias)));
}

template <int kParity>
__device__ __forceinline__ void unpack_codes2(uint32_t w, uint32_t &a0, uint32_t &a1, uint32_t &a2, uint32_t &a3) {
  const uint32_t w10 = w >> 10;
  a0 = unpack_code2<4 * kParity + 0>(w, w10);
  a1 = unpack_code2<4 * kParity + 1>(w, w10);
  a2 = unpack_code2<4 * kParity + 2>(w, w10);
  a3 = unpack_code2<4 * kParity + 3>(w, w10);
}

// ------------------------------------------------------------- warp MMA --

// Register-only instructions are emitted as plain (non-volatile) asm so the
// compiler may schedule them freely around each other; S4KV_ASM_VOLATILE=1
// pins them in program order instead.
#ifndef S4KV_ASM_VOLATILE
#define S4KV_ASM_VOLATILE 0
#endif
#if S4KV_ASM_VOLATILE
#define S4KV_ASM asm volatile
#else
#define S4KV_ASM asm
#endif

// D += A * B, m16n8k16, A row-major f16, B col-major f16, fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                         uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  S4KV_ASM(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose of an 8x8 b16 matrix held as one b16x2 register per lane.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  S4KV_ASM("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// --------------------------------------------------------- shared memory --

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared loads at [base + OFF] with OFF folded into the instruction.
template <int OFF>
__device__ __forceinline__ uint4 lds128(uint32_t base) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4+%5];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(base), "n"(OFF));
  return v;
}

template <int OFF>
__device__ __forceinline__ uint32_t lds32(uint32_t base) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(base), "n"(OFF));
  return v;
}

// Four 8x8 b16 matrices from shared memory at [addr + OFF], one row address
// per lane (lanes 8m..8m+7 give matrix m's rows), straight into an MMA
// operand fragment.
template <int OFF>
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                            uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4+%5];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr), "n"(OFF));
}

// ------------------------------------------------- packed fp32 pairs --

// Two IEEE fp32 operations in one instruction (sm_100 f32x2 forms); each
// lane of the pair rounds exactly like the scalar operation.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  S4KV_ASM("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
           "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
           : "=f"(d.x), "=f"(d.y)
           : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  S4KV_ASM("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
           "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
           : "=f"(d.x), "=f"(d.y)
           : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  float2 d;
  S4KV_ASM("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
           "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
           : "=f"(d.x), "=f"(d.y)
           : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  S4KV_ASM("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
           "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
           : "=f"(d.x), "=f"(d.y)
           : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// ------------------------------------------------ mbarrier + bulk copies --

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy accesses (a bulk copy reusing a stage).
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// One 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// No multicast.  dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                              uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Test (and, for up to S4KV_WAIT_HINT_NS nanoseconds, wait) for completion
// of the barrier phase with the given parity.  A suspended warp leaves its
// issue slots to the other warps instead of spinning.
#ifndef S4KV_WAIT_HINT_NS
#define S4KV_WAIT_HINT_NS 0
#endif
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
#if S4KV_WAIT_HINT_NS > 0
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity), "n"(S4KV_WAIT_HINT_NS)
      : "memory");
#else
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
#endif
  return done != 0;
}

// Bounded wait for the phase with the given parity: gives up after roughly
// `limit_cycles` SM clock cycles and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  long long limit_cycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > limit_cycles) return false;
  }
}

}  // namespace s4kv
