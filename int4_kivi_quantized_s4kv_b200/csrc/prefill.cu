// s4kv_prefill_attention device side: causal attention of a chunk of new
// query tokens over the paged cache (4-bit codes, or the 8- and 2-bit
// variants) after the chunk was appended (the prefill / chunked-append side
// of the cache that decode attention reads).
//
// What it computes: sequence b owns query rows cu_new[b] .. cu_new[b+1]-1;
// with n new tokens and L tokens after the append, row j sits at position
// L - n + j and, for each query head (GQA: kv head = head / G, "KV-Cache-
// Optimierung -- PagedAttention, quantisierter KV, Speculative Cache",
// "Begriffe auf dieser Seite"), attends to tokens 0 .. L - n + j of the
// cache: full pages dequantized (code * scale + zero, "S4 KV -- int4
// KV-Cache-Kompression fuer vLLM", "Funktionsweise" step 1), the partial last
// page from the fp16 residual.
//
// How (B200): this is a dense contraction, so it runs on the fifth-generation
// tensor cores, in two launches.
//  1. prefill_operands_kernel dequantizes every key tile (128 keys, 8 pages)
//     of every (sequence, kv head) ONCE into a workspace tile of 80 KB that
//     holds the MMA operands exactly as shared memory wants them (128-byte
//     swizzled, K-major): K_hi, K_lo and V^T.  A key is code * scale + zero
//     in fp32 (exact product, one rounding, the value the oracle's
//     dequantization gives) split into an fp16 hi part and the e5m2 rounding
//     of the remainder (at most 2^-12 of the key, so its 2^-3 relative error
//     leaves the key carried to about 2^-14 relative; keys of outlier
//     channels are large, and a single fp16 rounding of them moves the logits
//     visibly).  A value is the fused fp16 multiply-add
//     code * scale + zero (the correctly rounded fp16), stored transposed.
//     Every query tile of the sequence then reads these bytes (mostly from
//     L2) instead of dequantizing the same pages again.  One CTA writes half
//     a tile; int4 pages are read in their MMA-fragment order, 8- and 2-bit
//     pages code by code through the code map.  Only this launch depends on
//     the code width.
//  2. prefill_kernel: one CTA takes one (query tile, sequence, kv head); the
//     tile's 128 MMA rows are (token, head of the group) pairs, so a tile
//     holds floor(128 / G) tokens.  Warps with separate roles hand buffers
//     over through mbarriers:
//      * two producer warps bring each key tile's K_hi, K_lo (48 KB) and V^T
//        (32 KB) into one of two K and one of two V buffers with 1-D bulk
//        copies (TMA engine, no multicast); a K buffer is refilled as soon as
//        the S MMAs that read it complete, a V buffer once the PV MMAs have,
//        each by its own warp so that neither copy queues behind the other's
//        buffer;
//      * one warp issues S(k) = Q K_hi^T + Q8 K_lo^T (M = 128, N = 128 keys,
//        one accumulation: the 128 channels of Q, read from tensor memory,
//        against K_hi with fp16 MMAs, then those of Q8, an e5m2 copy of Q in
//        shared memory, against K_lo with e5m2 MMAs at twice the rate) into
//        one of two tensor-memory S buffers, another issues O += P(k) V(k) (N = 128,
//        K = 128) with P read from tensor memory, so that S(k+1) never
//        queues behind a PV that waits for its softmax; with two S buffers
//        S(k+1) never waits for the softmax to have read S(k);
//      * 4 softmax warps (one tensor-memory lane, i.e. one row, per thread)
//        read S back, apply the causal mask and an online softmax
//        in the exp2 domain whose reference moves only when a row maximum
//        passes it by more than 8 (weights stay <= 256, fine for fp16),
//        rescale that row of O in tensor memory when it moves, and write P
//        (fp16 pairs) into tensor memory; three exponentials in eight are
//        computed on the FMA pipe (exp2_poly2), the rest on the MUFU pipe.
//     The Q tile sits in tensor memory too, so every MMA reads only its B
//     operand (K or V) from shared memory.
// Every wait is bounded; a timeout sets a CTA-wide abort flag and an error
// bit, and every role then leaves its loop.
#include <cfloat>

#include "code_map.cuh"
#include "kernels.cuh"
#include "prefill.cuh"
#include "tc05.cuh"

namespace s4kv {

namespace {

constexpr int kSoftmaxWarps = 4;   // warps 0..3: one row per thread
constexpr int kMmaWarp = 4;        // S MMAs
constexpr int kKProducerWarp = 5;  // K tiles
constexpr int kVProducerWarp = 6;  // V tiles
constexpr int kPvWarp = 7;         // PV MMAs
constexpr int kThreadsP = 32 * 8;
constexpr int kKeyTile = 128;                    // keys per tile
constexpr int kPagesPerTile = kKeyTile / kPage;  // 8
constexpr int kOpPages = kPagesPerTile / 2;       // operand kernel: half a key tile per CTA
constexpr int kOpThreads = 64 * kOpPages;        // 64 threads per page
constexpr int kStages = 2;                       // K and V buffers each
constexpr uint32_t kKHiBytes = kKeyTile * 128 * 2;     // K_hi [128][128] fp16
constexpr uint32_t kKLoBytes = kKeyTile * 128;         // K_lo [128][128] e5m2
constexpr uint32_t kKBytes = kKHiBytes + kKLoBytes;    // one K buffer
constexpr uint32_t kVBytes = 128 * kKeyTile * 2;       // V^T [128][128] fp16
constexpr uint32_t kTileBytes = kKBytes + kVBytes;     // workspace tile
constexpr uint32_t kHalfTileBytes = kTileBytes / 2;
constexpr uint32_t kQ8Bytes = 128 * 128;               // Q [128][128] e5m2
constexpr float kSlack = 8.0f;                   // log2 slack of the softmax reference
#ifndef S4KV_PREFILL_POLY_OF8
#define S4KV_PREFILL_POLY_OF8 3
#endif
constexpr int kPolyOf8 = S4KV_PREFILL_POLY_OF8;  // eighths of the exponentials on the FMA pipe
constexpr long long kWaitLimit = 2000000000LL;   // about one second
// S: M = 128, N = 128 keys (Q against K_hi, fp16 K = 16 per MMA, then Q8
// against K_lo, e5m2 K = 32 per MMA, accumulated); PV: M = 128, N = 128
constexpr uint32_t kIdescS = tc05::idesc_f16_f32(128, kKeyTile);
constexpr uint32_t kIdescO = tc05::idesc_f16_f32(128, 128);
constexpr uint32_t kIdescS8 = tc05::idesc_e5m2_f32(128, kKeyTile);  // Q8 . K_lo^T
// tensor memory (512 columns): two S buffers at 0 and 128, O at 256, P (fp16
// pairs, the PV A operand) at 384, Q (fp16 pairs, the S A operand) at 448.
// With both A operands in tensor memory, each MMA reads only its B operand
// from shared memory.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384, kColQ = 448;

// attention kernel smem (1024-aligned operands): two K and two V buffers,
// barriers
constexpr uint32_t kOffK = 0;                                    // [2]
constexpr uint32_t kOffV = kOffK + kStages * kKBytes;            // [2]
constexpr uint32_t kOffQ8 = kOffV + kStages * kVBytes;
constexpr uint32_t kOffBar = kOffQ8 + kQ8Bytes;
// barriers (8 bytes each): k_full[2], k_empty[2], v_full[2], v_empty[2],
// s_full[2], s_empty[2], p_full, p_empty; then the tensor-memory address and
// the abort flag
constexpr uint32_t kNumBars = 14;
constexpr uint32_t kOffSlot = kOffBar + 8 * kNumBars;
constexpr uint32_t kOffAbort = kOffSlot + 4;
constexpr uint32_t kSmemBytes = kOffAbort + 4 + 1024;  // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "prefill shared memory");
static_assert(kKHiBytes % 1024 == 0 && kKBytes % 1024 == 0 && kVBytes % 1024 == 0 && kOffQ8 % 1024 == 0 &&
                  kOffBar % 1024 == 0,
              "1024-byte operand alignment");

// operand kernel smem: the output half tile, then the staged page blocks
template <int kBits>
constexpr uint32_t op_smem_bytes() {
  return kHalfTileBytes + kOpPages * Fmt<kBits>::kBlock + 1024;
}

// Bounded wait for a barrier phase; gives up after about a second or as soon
// as another role has raised the CTA's abort flag.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, const volatile int *abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort || clock64() - t0 > kWaitLimit) return false;
  }
}

// Bounded wait used while draining copies before the CTA exits (time only).
__device__ __forceinline__ void wait_landed(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity) && clock64() - t0 <= kWaitLimit) {
  }
}

// 2^x for a pair, on the FMA/ALU pipes instead of the MUFU pipe.  Cody and
// Waite's range reduction: x = j + f with j = rint(x) (adding 1.5 * 2^23
// rounds x to an integer held in the sum's low mantissa bits) and
// f in [-1/2, 1/2]; 2^f from a cubic; 2^j applied by adding j to the
// exponent field (the sum's bits shifted left by 23 are j << 23, since the
// constant's own bits vanish under the shift).  The cubic was fitted for this
// kernel by iteratively reweighted least squares towards the smallest maximum
// relative error over [-1/2, 1/2]: 7.5e-5 in fp32 Horner evaluation, well
// below the 2^-11 of the fp16 rounding P goes through.  x is clamped at -125,
// so that 2^j * p(f) stays a normal number (weights below 2^-125 are 0 to
// fp16 and nothing to the fp32 row sum).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const float2 xc = make_float2(fmaxf(x.x, -125.0f), fmaxf(x.y, -125.0f));
  const float2 t = add2(xc, make_float2(kRound, kRound));
  const float2 f = sub2(xc, sub2(t, make_float2(kRound, kRound)));
  float2 q = fma2(f, make_float2(0.0551716685f, 0.0551716685f), make_float2(0.2426111400f, 0.2426111400f));
  q = fma2(q, f, make_float2(0.6932609677f, 0.6932609677f));
  q = fma2(q, f, make_float2(0.9999280572f, 0.9999280572f));
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void sts64(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t a) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
}
__device__ __forceinline__ void sts16(uint32_t addr, uint16_t a) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(a) : "memory");
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 lds128_at(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds32_at(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds64_at(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// max of three floats in one instruction (sm_100); a NaN operand is ignored
// as by fmaxf
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
  return h2_as_u32(__hfma2(u32_as_h2(a), u32_as_h2(b), u32_as_h2(c)));
}

// Two fp32 values rounded to e5m2 (round to nearest even, saturating), the
// first in the low byte.
__device__ __forceinline__ uint16_t e5m2x2(float first, float second) {
  uint16_t d;
  asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(d) : "f"(second), "f"(first));
  return d;
}
// Two fp16 values (a pair in one word, the lower element in the low half)
// rounded to e5m2, the lower element in the low byte.
__device__ __forceinline__ uint16_t e5m2x2_of_f16x2(uint32_t x) {
  uint16_t d;
  asm("cvt.rn.satfinite.e5m2x2.f16x2 %0, %1;" : "=h"(d) : "r"(x));
  return d;
}

// Two keys (fp16 codes in `codes`) dequantized in fp32 (code * scale + zero:
// the product is exact, so one rounding) and split into an fp16 hi part and
// the e5m2 rounding of the remainder (lo, the lower key in the low byte).
__device__ __forceinline__ void split_key(uint32_t codes, float2 sc, float2 z, uint32_t &hi, uint16_t &lo) {
  const float2 c = __half22float2(u32_as_h2(codes));
  const float2 k = fma2(c, sc, z);
  const __half2 h = __floats2half2_rn(k.x, k.y);
  const float2 r = sub2(k, __half22float2(h));
  hi = h2_as_u32(h);
  lo = e5m2x2(r.x, r.y);
}

// Byte offset of element (r, k) of a [rows][128] 8-bit K-major operand in the
// 128-byte-swizzled layout (one 128-byte row per r).
__device__ __forceinline__ uint32_t sw128_offset_b8(int r, int k) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((((k >> 4) ^ (r & 7))) << 4) + (k & 15));
}

// The rows of sequence b that the chunk holds, checked against the cache.
// Returns false (and flags bad lengths once, from the attention kernel's
// first CTA of the sequence) when there is nothing to do.
struct SeqRows {
  int c_lo, n, L;
};
__device__ __forceinline__ bool seq_rows(const PrefillParams &p, int b, bool flag, SeqRows &r) {
  r.c_lo = __ldg(p.cu_new + b);
  const int c_hi = __ldg(p.cu_new + b + 1);
  r.n = c_hi - r.c_lo;
  if (r.n <= 0) return false;
  r.L = __ldg(p.seq_lens + b);
  if (r.c_lo < 0 || c_hi > p.n_tokens || r.L < r.n || r.L > p.max_pages * kPage) {
    if (flag) flag_error(p.err, S4KV_EFLAG_SEQ_LEN);
    return false;
  }
  return true;
}

}  // namespace

// ---------------------------------------------------------------------------
// Launch 1: one CTA per (half key tile, sequence, kv head) writes that half
// of the tile's operands to the workspace: K_hi and V^T [128][128] fp16,
// K_lo [128][128] e5m2, each 128-byte swizzled K-major.  Half hh holds keys
// 64 hh .. 64 hh + 63: rows 64 hh .. of both column blocks of K_hi (8 KB
// each, the same bytes a 64-row operand has), rows 64 hh .. of K_lo (8 KB)
// and column block hh of V^T (16 KB).  Keys at or past L (the rest of the partial last page, pages
// after it) are written as zeros, so masked keys hold finite values.
template <int kBits>
__global__ void __launch_bounds__(kOpThreads) prefill_operands_kernel(const PrefillParams p) {
  using F = Fmt<kBits>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  // half tile in smem: K_hi [64][128] (two 8 KB column blocks), K_lo
  // [64][128] e5m2 (8 KB), then V^T [128][64]
  const uint32_t sK = base, sKlo = base + kKHiBytes / 2, sV = base + kKBytes / 2;
  const uint32_t stage = base + kHalfTileBytes;
  const int ht = blockIdx.x, b = blockIdx.y, h = blockIdx.z, H = p.num_kv_heads;
  const int kt = ht >> 1, hh = ht & 1;
  const int t = threadIdx.x;
  SeqRows sr;
  if (!seq_rows(p, b, false, sr)) return;
  const int L = sr.L;
  // a tile the attention reads is written whole: a half past L is zeros
  if (kt * kKeyTile >= L) return;
  const int nfull = L / kPage;
  const int np = (L + kPage - 1) / kPage;
  const int pg0 = ht * kOpPages;  // first page of this half tile

  // ---- the half tile's full pages into shared memory, 16-byte loads
  const int q = max(0, min(kOpPages, nfull - pg0));
  const int32_t *bt = p.block_tables + static_cast<long>(b) * p.max_pages + pg0;
  constexpr int kChunks = F::kBlock / 16;
  for (int i = t; i < q * kChunks; i += kOpThreads) {
    const int k = i / kChunks, c = i - k * kChunks;
    int phys = __ldg(bt + k);
    if (static_cast<unsigned>(phys) >= static_cast<unsigned>(p.num_pages)) {
      if (c == 0) flag_error(p.err, S4KV_EFLAG_PAGE_RANGE);
      phys = 0;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(
        p.pool + (static_cast<long long>(phys) * H + h) * F::kBlock);
    sts128(stage + k * F::kBlock + 16 * c, __ldg(src + c));
  }
  __syncthreads();

  // ---- dequantize: 64 threads per page
  const int dpage = t >> 6, widx = t & 63;
  const int dq = widx & 3, dlane0 = widx >> 2;
  const int pg = pg0 + dpage;
  if (pg < nfull && kBits != 4) {
    // 8- and 2-bit codes: element by element through the code map; two
    // channels per thread, the page's 16 tokens
    const uint8_t *blk = smem_raw + (stage + dpage * F::kBlock - raw);
    const __half *kscale = reinterpret_cast<const __half *>(blk + F::kKScale);
    const __half *kzero = reinterpret_cast<const __half *>(blk + F::kKZero);
    const __half *vscale = reinterpret_cast<const __half *>(blk + F::kVScale);
    const __half *vzero = reinterpret_cast<const __half *>(blk + F::kVZero);
    const int c0 = 2 * widx;
    const float ks0 = __half2float(kscale[c0]), ks1 = __half2float(kscale[c0 + 1]);
    const float kz0 = __half2float(kzero[key_zero_slot(c0)]), kz1 = __half2float(kzero[key_zero_slot(c0 + 1)]);
    const int g = c0 / kVGroup;
    for (int t = 0; t < kPage; ++t) {
      int w0, n0, w1, n1;
      key_position(t, c0, w0, n0);
      key_position(t, c0 + 1, w1, n1);
      uint32_t hi;
      uint16_t lo;
      const uint32_t codes = h2_as_u32(__floats2half2_rn(static_cast<float>(code_at(blk + F::kKCode, w0, n0, kBits)),
                                                         static_cast<float>(code_at(blk + F::kKCode, w1, n1, kBits))));
      split_key(codes, make_float2(ks0, ks1), make_float2(kz0, kz1), hi, lo);
      const int key = dpage * 16 + t;  // within the half tile
      sts32(sK + tc05::sw128_offset(key, c0, kKeyTile / 2), hi);
      sts16(sKlo + sw128_offset_b8(key, c0), lo);
      const __half vs = vscale[value_scale_slot(t, g)], vz = vzero[g * kPage + t];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        int vw, vn;
        value_position(t, c0 + j, vw, vn);
        const __half code = __float2half_rn(static_cast<float>(code_at(blk + F::kVCode, vw, vn, kBits)));
        sts16(sV + tc05::sw128_offset(c0 + j, key, 128), __half_as_ushort(__hfma(code, vs, vz)));
      }
    }
  } else if (pg < nfull) {
    const uint32_t blk = stage + dpage * F::kBlock;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int w = widx + 64 * e;
      const int ln = dlane0 + 16 * (e & 1), tt = 4 * (e >> 1) + dq;
      const int dn = ln >> 2, di = ln & 3;
      // keys: tokens dn, dn + 8 of the page; channels c0 .. c0 + 3
      {
        uint32_t a0, a1, a2, a3;
        unpack_codes(lds32_at(blk + kKCodeOff + 4 * w), a0, a1, a2, a3);
        const int c0 = 32 * di + 4 * tt;
        const uint2 sc = lds64_at(blk + kKScaleOff + 2 * c0);
        const uint32_t zslot = 16 * tt + 2 * di;
        const uint32_t z01 = lds32_at(blk + kKZeroOff + 2 * zslot);
        const uint32_t z23 = lds32_at(blk + kKZeroOff + 2 * (zslot + 8));
        const float2 s01 = __half22float2(u32_as_h2(sc.x)), s23 = __half22float2(u32_as_h2(sc.y));
        const float2 zf01 = __half22float2(u32_as_h2(z01)), zf23 = __half22float2(u32_as_h2(z23));
        uint32_t hi0, hi1, hi2, hi3;
        uint16_t lo0, lo1, lo2, lo3;
        split_key(a0, s01, zf01, hi0, lo0);
        split_key(a1, s01, zf01, hi1, lo1);
        split_key(a2, s23, zf23, hi2, lo2);
        split_key(a3, s23, zf23, hi3, lo3);
        const uint32_t ko = tc05::sw128_offset(dpage * 16 + dn, c0, kKeyTile / 2);
        sts64(sK + ko, hi0, hi2);
        sts64(sK + ko + 1024, hi1, hi3);
        // tokens dn and dn + 8 are 8 rows (1024 bytes) apart in both layouts
        const uint32_t ko8 = sw128_offset_b8(dpage * 16 + dn, c0);
        sts32(sKlo + ko8, static_cast<uint32_t>(lo0) | (static_cast<uint32_t>(lo2) << 16));
        sts32(sKlo + ko8 + 1024, static_cast<uint32_t>(lo1) | (static_cast<uint32_t>(lo3) << 16));
      }
      // values: channels cb, cb + 1; tokens 2 di, 2 di + 1 (+ 8)
      {
        uint32_t a0, a1, a2, a3;
        unpack_codes(lds32_at(blk + kVCodeOff + 4 * w), a0, a1, a2, a3);
        const int g = tt >> 1;
        const uint32_t sv_lo = lds32_at(blk + kVScaleOff + 2 * value_scale_slot(2 * di, g));
        const uint32_t sv_hi = lds32_at(blk + kVScaleOff + 2 * value_scale_slot(2 * di + 8, g));
        const uint32_t zv_lo = lds32_at(blk + kVZeroOff + 2 * (16 * g + 2 * di));
        const uint32_t zv_hi = lds32_at(blk + kVZeroOff + 2 * (16 * g + 2 * di + 8));
        const int cb = 32 * (tt >> 1) + 4 * dn + 2 * (tt & 1);
        const int key = dpage * 16 + 2 * di;
        sts32(sV + tc05::sw128_offset(cb, key, 128), hfma2_u32(a0, sv_lo, zv_lo));
        sts32(sV + tc05::sw128_offset(cb + 1, key, 128), hfma2_u32(a1, sv_lo, zv_lo));
        sts32(sV + tc05::sw128_offset(cb, key + 8, 128), hfma2_u32(a2, sv_hi, zv_hi));
        sts32(sV + tc05::sw128_offset(cb + 1, key + 8, 128), hfma2_u32(a3, sv_hi, zv_hi));
      }
    }
  } else {
    // the partial last page (fp16 residual rows < L % 16) or no page: copy
    // the valid rows, zero the rest
    const int rres = (pg == nfull && pg < np) ? L - nfull * kPage : 0;
    const long res_base = (static_cast<long>(b) * H + h) * kPage * kHeadDim;
    const __half *rk = p.res_k + res_base;
    const __half *rv = p.res_v + res_base;
    for (int e = widx; e < kPage * kHeadDim / 2; e += 64) {
      const int tk = e >> 6, c = 2 * (e & 63);
      uint32_t kb = 0;
      if (tk < rres) kb = *reinterpret_cast<const uint32_t *>(rk + tk * kHeadDim + c);
      // residual keys are fp16 already: K_lo is zero
      sts32(sK + tc05::sw128_offset(dpage * 16 + tk, c, kKeyTile / 2), kb);
      sts16(sKlo + sw128_offset_b8(dpage * 16 + tk, c), 0);
    }
    for (int e = widx; e < kPage * kHeadDim; e += 64) {
      const int tk = e >> 7, c = e & 127;
      uint16_t vb = 0;
      if (tk < rres) vb = __half_as_ushort(rv[tk * kHeadDim + c]);
      sts16(sV + tc05::sw128_offset(c, dpage * 16 + tk, 128), vb);
    }
  }
  __syncthreads();

  // ---- the half tile to its places in the workspace tile, coalesced 16-byte
  // stores: smem 8 KB pieces 0, 1 (K_hi column blocks) go to
  // 16 KB * piece + 8 KB * hh, the 8 KB of K_lo to K_hi bytes + 8 KB * hh,
  // the 16 KB of V^T to K bytes + 16 KB * hh
  uint8_t *tile = p.ws + ((static_cast<long long>(b) * H + h) * p.tiles_per_seq + kt) * kTileBytes;
  for (int i = t; i < static_cast<int>(kHalfTileBytes / 16); i += kOpThreads) {
    const uint32_t off = 16u * i;
    const uint32_t dst = off < kKHiBytes / 2 ? (off >> 13) * 16384u + 8192u * hh + (off & 8191u)
                         : off < kKBytes / 2 ? kKHiBytes + 8192u * hh + (off - kKHiBytes / 2)
                                             : kKBytes + 16384u * hh + (off - kKBytes / 2);
    *reinterpret_cast<uint4 *>(tile + dst) = lds128_at(base + off);
  }
}

// ---------------------------------------------------------------------------
// Launch 2: the attention itself, reading the operand tiles of launch 1.
__global__ void __launch_bounds__(kThreadsP, 1) prefill_kernel(const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t bars = base + kOffBar;
  const uint32_t tslot = base + kOffSlot;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem_raw + (base + kOffAbort - raw));
  auto kbuf = [&](int s) { return base + kOffK + s * kKBytes; };
  auto vbuf = [&](int s) { return base + kOffV + s * kVBytes; };
  auto k_full = [&](int s) { return bars + 8u * (0 + s); };
  auto k_empty = [&](int s) { return bars + 8u * (2 + s); };
  auto v_full = [&](int s) { return bars + 8u * (4 + s); };
  auto v_empty = [&](int s) { return bars + 8u * (6 + s); };
  auto s_full = [&](int s) { return bars + 8u * (8 + s); };
  auto s_empty = [&](int s) { return bars + 8u * (10 + s); };
  const uint32_t p_full = bars + 8u * 12, p_empty = bars + 8u * 13;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.group, H = p.num_kv_heads;
  const int Tq = 128 / G;                                   // tokens per query tile
  const int b = blockIdx.y, h = blockIdx.z;
  const int tile = static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x);  // long tiles first

  // ---- this CTA's rows (uniform across the CTA; exits before any allocation)
  SeqRows sr;
  if (!seq_rows(p, b, tile == 0 && h == 0 && tid == 0, sr)) return;
  const int c_lo = sr.c_lo, n = sr.n, L = sr.L;
  // more rows than max_new_per_seq sized the grid for: the rows past the
  // last tile are not computed, which the caller learns from the flag
  if (tile == 0 && h == 0 && tid == 0 && n > static_cast<int>(gridDim.x) * Tq) flag_error(p.err, S4KV_EFLAG_SEQ_LEN);
  const int t0 = tile * Tq;
  if (t0 >= n) return;
  const int tq = min(Tq, n - t0);
  const int rows = tq * G;
  const int pos_first = L - n + t0;
  const int n_keys = pos_first + tq;                         // keys 0 .. pos_last
  const int n_ktiles = (n_keys + kKeyTile - 1) / kKeyTile;

  // ---- setup: tensor memory, barriers, Q
  if (warp == 0) {
    tc05::tmem_alloc(tslot, kTmemCols);
    tc05::tmem_relinquish();
    tc05::fence_before_sync();
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full(s), 1);
      mbar_init(s_empty(s), 32 * kSoftmaxWarps);
    }
    mbar_init(p_full, 32 * kSoftmaxWarps);
    mbar_init(p_empty, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = lds32_at(tslot);
  auto tS = [&](int s) { return tmem + kColS + 128u * s; };
  const uint32_t tO = tmem + kColO, tP = tmem + kColP, tQ = tmem + kColQ;
  // Q tile into tensor memory: row r = (token r / G, head r % G), one row
  // per softmax thread (its lane), channels 2c and 2c + 1 in column c; rows
  // >= rows are zero
  if (warp < kSoftmaxWarps) {
    const int r = tid, tl = r / G, g = r - (r / G) * G;
    const uint4 *src = reinterpret_cast<const uint4 *>(
        p.q + (static_cast<long>(c_lo + t0 + tl) * p.num_q_heads + h * G + g) * kHeadDim);
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 x = r < rows ? __ldg(src + 8 * hc + c) : make_uint4(0, 0, 0, 0);
        v[4 * c] = x.x;
        v[4 * c + 1] = x.y;
        v[4 * c + 2] = x.z;
        v[4 * c + 3] = x.w;
      }
      tc05::tmem_st32(tQ + (static_cast<uint32_t>(32 * warp) << 16) + 32 * hc, v);
      // the same channels in e5m2 into the Q8 tile (shared memory, the A
      // operand of Q8 . K_lo^T): 16-byte chunks 4 hc .. 4 hc + 3 of row r
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          w[i] = static_cast<uint32_t>(e5m2x2_of_f16x2(v[8 * cc + 2 * i])) |
                 (static_cast<uint32_t>(e5m2x2_of_f16x2(v[8 * cc + 2 * i + 1])) << 16);
        sts128(base + kOffQ8 + sw128_offset_b8(r, 16 * (4 * hc + cc)), make_uint4(w[0], w[1], w[2], w[3]));
      }
    }
    tc05::tmem_wait_st();
    tc05::fence_before_sync();
    fence_proxy_async();  // the Q8 tile is read by the MMAs (async proxy)
  }
  __syncthreads();
  tc05::fence_after_sync();
  bool failed = false;
  auto fail = [&]() {
    failed = true;
    *abort_flag = 1;
  };

  if (warp == kKProducerWarp || warp == kVProducerWarp) {
    // --------------------------------------------------------- producers
    // one warp per operand, so that neither waits behind the other's buffer:
    // K(kt) into K buffer kt % 2 once S(kt - 2) has read it, V(kt) into V
    // buffer kt % 2 once O += P(kt - 2) V(kt - 2) has
    if (lane == 0) {
      const bool is_k = warp == kKProducerWarp;
      const uint32_t bytes = is_k ? kKBytes : kVBytes;
      const uint8_t *tiles = p.ws + (static_cast<long long>(b) * H + h) * p.tiles_per_seq * kTileBytes + (is_k ? 0 : kKBytes);
      auto full = [&](int s) { return is_k ? k_full(s) : v_full(s); };
      int issued = 0;
      for (int kt = 0; kt < n_ktiles; ++kt) {
        const int s = kt % kStages, u = kt / kStages;
        if (kt >= kStages && !wait_bounded(is_k ? k_empty(s) : v_empty(s), (u - 1) & 1, abort_flag)) {
          fail();
          break;
        }
        mbar_arrive_expect_tx(full(s), bytes);
        bulk_copy_g2s(is_k ? kbuf(s) : vbuf(s), tiles + static_cast<long long>(kt) * kTileBytes, bytes, full(s));
        issued = kt + 1;
      }
      // before the CTA exits, the copies in flight must have landed (bounded
      // by time only, also after an abort): at most the last kStages
      for (int kt = max(0, issued - kStages); kt < issued; ++kt) wait_landed(full(kt % kStages), (kt / kStages) & 1);
    }
  } else if (warp == kMmaWarp || warp == kPvWarp) {
    // -------------------------------------------------------- MMA issuers
    // Two warps issue: S(kt) goes out as soon as K(kt) has landed and the
    // softmax has read S(kt - 2) from its buffer, without waiting behind
    // O += P V of an earlier tile, whose issue waits for that tile's softmax.
    // Each warp runs its loop on all lanes (descriptors and decisions stay
    // warp-uniform); one elected lane issues each MMA and commit, and a
    // commit tracks the MMAs of its own thread only.
    auto wait_w = [&](uint32_t bar, uint32_t parity) {
      return __all_sync(0xFFFFFFFFu, wait_bounded(bar, parity, abort_flag));
    };
    if (warp == kPvWarp) {
      const uint64_t dv0 = tc05::smem_desc_sw128(vbuf(0)), dv1 = tc05::smem_desc_sw128(vbuf(1));
      for (int k = 0; k < n_ktiles; ++k) {
        // O += P(k) V(k), P read from tensor memory, once V(k) has landed and
        // the softmax has written P(k)
        const int vs = k % kStages;
        const bool vf = mbar_try_wait(v_full(vs), (k / kStages) & 1);
        const bool pf = mbar_try_wait(p_full, k & 1);
        if (!__all_sync(0xFFFFFFFFu, vf && pf) &&
            (!wait_w(v_full(vs), (k / kStages) & 1) || !wait_w(p_full, k & 1))) {
          fail();
          break;
        }
        tc05::fence_after_sync();
        const uint64_t dv = vs ? dv1 : dv0;
#pragma unroll
        for (int j = 0; j < kKeyTile / 16; ++j)
          tc05::mma_f16_ts(tO, tP + 8 * j, dv + (((j >> 2) * (kVBytes / 2) + (j & 3) * 32) >> 4), kIdescO,
                       (k > 0 || j > 0) ? 1u : 0u);
        tc05::mma_commit(p_empty);
        tc05::mma_commit(v_empty(vs));
      }
    } else {
      const uint64_t dk0 = tc05::smem_desc_sw128(kbuf(0)), dk1 = tc05::smem_desc_sw128(kbuf(1));
      const uint64_t dq8 = tc05::smem_desc_sw128(base + kOffQ8);
      for (int kt = 0; kt < n_ktiles; ++kt) {
        const int ks = kt % kStages;
        // S(kt) = Q K_hi^T + Q K_lo^T into S buffer kt % 2 once K(kt) has
        // landed and the softmax has read S(kt - 2) from that buffer
        const int sb = kt & 1;
        // both barriers tested back to back (their latencies overlap); the
        // bounded waits only when one of them is not complete yet
        const bool kf = mbar_try_wait(k_full(ks), (kt / kStages) & 1);
        const bool se = kt < 2 || mbar_try_wait(s_empty(sb), ((kt >> 1) - 1) & 1);
        if (!__all_sync(0xFFFFFFFFu, kf && se) &&
            (!wait_w(k_full(ks), (kt / kStages) & 1) || (kt >= 2 && !wait_w(s_empty(sb), ((kt >> 1) - 1) & 1)))) {
          fail();
          break;
        }
        tc05::fence_after_sync();
        const uint64_t dk = ks ? dk1 : dk0;
        // Q channels 16 j .. + 15 (tensor-memory columns 8 j ..) against the
        // same channels of K_hi (fp16, K = 16 per MMA) ...
#pragma unroll
        for (int j = 0; j < 8; ++j)
          tc05::mma_f16_ts(tS(sb), tQ + 8 * j, dk + ((((j >> 2) * (kKHiBytes / 2)) + (j & 3) * 32) >> 4), kIdescS,
                       j > 0 ? 1u : 0u);
        // ... then Q8 channels 32 j .. + 31 against K_lo (e5m2, K = 32)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tc05::mma_e5m2_ss(tS(sb), dq8 + ((32 * j) >> 4), dk + ((kKHiBytes + 32 * j) >> 4), kIdescS8, 1u);
        tc05::mma_commit(s_full(sb));
        tc05::mma_commit(k_empty(ks));
      }
    }
  } else {
    // ---------------------------------------------------- softmax (rows)
    const int row = tid;  // tensor-memory lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
    const bool row_ok = row < rows;
    const int pos_row = pos_first + (row_ok ? row / G : 0);
    float ref = -INFINITY;
    float2 lsum = make_float2(0.f, 0.f);
    const float sl2 = p.scale_log2;
    // the warp takes every decision together (its lanes run warp-wide
    // tensor-memory loads and votes)
    auto wait_warp = [&](uint32_t bar, uint32_t parity) {
      return __all_sync(0xFFFFFFFFu, wait_bounded(bar, parity, abort_flag));
    };
    // barrier tests whose answer is needed only later are made while a
    // tensor-memory load or store is in flight (an S(kt + 1) test after P(kt)
    // goes out, a P-buffer test after S(kt) is requested), so that a
    // complete barrier costs no wait of its own
    bool s_ready = false;
    for (int kt = 0; kt < n_ktiles; ++kt) {
      const int sb = kt & 1;
      if (!__all_sync(0xFFFFFFFFu, s_ready) && !wait_warp(s_full(sb), (kt >> 1) & 1)) {
        fail();
        break;
      }
      tc05::fence_after_sync();
      uint32_t sv[kKeyTile];
#pragma unroll
      for (int c = 0; c < kKeyTile / 32; ++c) {
        uint32_t (&w)[32] = *reinterpret_cast<uint32_t (*)[32]>(&sv[32 * c]);
        tc05::tmem_ld32(tS(sb) + lane_base + 32 * c, w);
      }
      const bool p_ready = kt == 0 || mbar_try_wait(p_empty, (kt - 1) & 1);
      tc05::tmem_wait_ld();
      tc05::fence_before_sync();
      mbar_arrive(s_empty(sb));
      // a key tile wholly before the tile's first query position needs no
      // mask (rows past the last row hold q = 0: finite logits, never written)
      const int key0 = kt * kKeyTile;
      const bool full = key0 + kKeyTile - 1 <= pos_first;
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (!full) {
#pragma unroll
        for (int j = 0; j < kKeyTile; ++j) sv[j] = (row_ok && key0 + j <= pos_row) ? sv[j] : __float_as_uint(-INFINITY);
      }
#pragma unroll
      for (int j = 0; j < kKeyTile; j += 2)
        m4[(j >> 1) & 3] = fmax3(m4[(j >> 1) & 3], __uint_as_float(sv[j]), __uint_as_float(sv[j + 1]));
      const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
      // the reference moves only when the row maximum passes it by > 8
      const bool move = mx > ref + kSlack;
      const float new_ref = move ? mx : ref;
      const float alpha = move ? fast_exp2(ref - new_ref) : 1.0f;  // 0 when ref was -inf
      // weights exp2(s * scale - ref); masked logits are -inf and give 0 (a
      // row without a valid key keeps a -inf reference, replaced by 0 so that
      // no inf - inf appears).  The row sum adds the fp32 weights; their fp16
      // roundings, which the MMA multiplies with, differ from them by
      // independent errors below 2^-11 relative that average out in the sum.
      const float nref = new_ref == -INFINITY ? 0.f : -new_ref;
      const float2 sc = make_float2(sl2, sl2), nr = make_float2(nref, nref);
      uint32_t hp[kKeyTile / 2];
      float2 ts0 = make_float2(0.f, 0.f), ts1 = make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < kKeyTile; j += 2) {
        const float2 x = fma2(make_float2(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])), sc, nr);
        // the exponentials are split between the MUFU pipe and the FMA pipe
        // (both are otherwise the softmax's bound): pairs m % 8 < kPolyOf8
        // of the tile's 64 take the polynomial
        const float2 e = ((j >> 1) % 8 < kPolyOf8) ? exp2_poly2(x) : make_float2(fast_exp2(x.x), fast_exp2(x.y));
        if (j & 2) ts1 = add2(ts1, e);
        else ts0 = add2(ts0, e);
        hp[j >> 1] = h2_as_u32(__floats2half2_rn(e.x, e.y));
      }
      lsum = add2(mul2(lsum, make_float2(alpha, alpha)), add2(ts0, ts1));
      // O and P are idle once O += P(kt-1) V has completed
      if (kt >= 1) {
        if (!__all_sync(0xFFFFFFFFu, p_ready) && !wait_warp(p_empty, (kt - 1) & 1)) {
          fail();
          break;
        }
        tc05::fence_after_sync();
        // a moved reference rescales O
        if (__any_sync(0xFFFFFFFFu, move)) {
          const float2 a2 = make_float2(alpha, alpha);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tc05::tmem_ld32(tO + lane_base + 32 * c, o);
            tc05::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float2 r = mul2(make_float2(__uint_as_float(o[j]), __uint_as_float(o[j + 1])), a2);
              o[j] = __float_as_uint(r.x);
              o[j + 1] = __float_as_uint(r.y);
            }
            tc05::tmem_st32(tO + lane_base + 32 * c, o);
          }
        }
      }
      ref = new_ref;
      // P into tensor memory (fp16 pairs, the A operand of O += P V)
      {
        uint32_t (&h0)[32] = *reinterpret_cast<uint32_t (*)[32]>(&hp[0]);
        uint32_t (&h1)[32] = *reinterpret_cast<uint32_t (*)[32]>(&hp[32]);
        tc05::tmem_st32(tP + lane_base, h0);
        tc05::tmem_st32(tP + lane_base + 32, h1);
      }
      s_ready = kt + 1 < n_ktiles && mbar_try_wait(s_full(sb ^ 1), ((kt + 1) >> 1) & 1);
      tc05::tmem_wait_st();
      tc05::fence_before_sync();
      mbar_arrive(p_full);
    }
    // ---- out = O / l once the last O += P V has completed
    if (!failed && !wait_warp(p_empty, (n_ktiles - 1) & 1)) fail();
    if (!failed) {
      tc05::fence_after_sync();
      const float l = lsum.x + lsum.y;
      const float inv = row_ok && l > 0.f ? 1.0f / l : 0.f;
      const int tl = row / G, g = row - (row / G) * G;
      __half *dst = p.out + (static_cast<long>(c_lo + t0 + tl) * p.num_q_heads + h * G + g) * kHeadDim;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tc05::tmem_ld32(tO + lane_base + 32 * c, o);
        tc05::tmem_wait_ld();
        if (row_ok) {
          uint32_t hv[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2)
            hv[j >> 1] = h2_as_u32(__floats2half2_rn(__uint_as_float(o[j]) * inv, __uint_as_float(o[j + 1]) * inv));
          uint4 *o4 = reinterpret_cast<uint4 *>(dst + 32 * c);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            o4[q4] = make_uint4(hv[4 * q4], hv[4 * q4 + 1], hv[4 * q4 + 2], hv[4 * q4 + 3]);
        }
      }
    }
  }

  if (failed) flag_error(p.err, S4KV_EFLAG_TIMEOUT);
  tc05::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc05::fence_after_sync();
    tc05::tmem_dealloc(tmem, kTmemCols);
  }
}

size_t prefill_smem_bytes() { return kSmemBytes; }
size_t prefill_tile_bytes() { return kTileBytes; }
int prefill_tiles_per_seq(int max_pages) {
  return static_cast<int>((static_cast<long long>(max_pages) + kPagesPerTile - 1) / kPagesPerTile);
}

// Both launches of a call; their shared-memory allowances are set at every
// call (the library keeps no record of what it configured).
template <int kBits>
cudaError_t launch_operands(const PrefillParams &p, dim3 grid, cudaStream_t stream) {
  const cudaError_t e = cudaFuncSetAttribute(prefill_operands_kernel<kBits>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(op_smem_bytes<kBits>()));
  if (e != cudaSuccess) return e;
  prefill_operands_kernel<kBits><<<grid, kOpThreads, op_smem_bytes<kBits>(), stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_prefill(const PrefillParams &p, int batch, int max_new, cudaStream_t stream) {
  const dim3 og(2 * p.tiles_per_seq, batch, p.num_kv_heads);
  cudaError_t e = p.bits == 8 ? launch_operands<8>(p, og, stream)
                  : p.bits == 2 ? launch_operands<2>(p, og, stream) : launch_operands<4>(p, og, stream);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const int Tq = 128 / p.group;
  const int tiles = (max_new + Tq - 1) / Tq;
  const dim3 grid(tiles, batch, p.num_kv_heads);
  prefill_kernel<<<grid, kThreadsP, kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace s4kv
