// s4kv_prefill_attention device side: causal attention of a chunk of new
// query tokens over the int4 paged cache after the chunk was appended (the
// prefill / chunked-append side of the cache that decode attention reads).
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
// tensor cores.  One CTA takes one (query tile, sequence, kv head); the tile's
// 128 MMA rows are (token, head of the group) pairs, so a tile holds
// floor(128 / G) tokens.  Keys are walked in tiles of 128 (8 pages):
//  * the 8 page blocks of the next key tile are fetched by 1-D bulk copies
//    (TMA engine, no multicast) into a second staging buffer while the
//    current one is used;
//  * all 128 threads dequantize the current tile into the 128-byte-swizzled
//    fp16 operands.  A key is code * scale + zero in fp32 (exact product, one
//    rounding, the value the oracle's dequantization gives) split into an
//    fp16 hi part and the fp16 rounding of the remainder, so K_hi + K_lo
//    carries it to about 22 bits: keys of outlier channels are large, and a
//    single fp16 rounding of them moves the logits visibly.  A value is the
//    fused fp16 multiply-add code * scale + zero (the correctly rounded fp16),
//    stored transposed (V^T [channel][key]);
//  * one thread issues S = Q K_hi^T + Q K_lo^T (16 tcgen05.mma, M = N = 128,
//    K = 16 each) into tensor memory; the four warps read S back one row per thread, apply
//    the causal mask and an online softmax in the exp2 domain whose reference
//    moves only when a row maximum passes it by more than 8 (weights stay
//    <= 256, fine for fp16), and write P (fp16) to shared memory;
//  * one thread issues O += P V (8 tcgen05.mma) into a second tensor-memory
//    accumulator; when a row's reference moves, that row of O is rescaled in
//    tensor memory first.
// Every wait is bounded; a timeout or a bad page id sets a bit in err_flag.
#include <cfloat>

#include "kernels.cuh"
#include "tc05.cuh"

namespace s4kv {

namespace {

constexpr int kThreadsP = 512;
constexpr int kKeyTile = 128;                    // keys per tile (MMA N of S)
constexpr int kPagesPerTile = kKeyTile / kPage;  // 8
constexpr uint32_t kOpBytes = 128 * 128 * 2;     // one fp16 [128][128] operand
constexpr uint32_t kStageBytes = kPagesPerTile * kBlockBytes;
constexpr float kSlack = 8.0f;                   // log2 slack of the softmax reference
constexpr long long kWaitLimit = 2000000000LL;   // about one second
constexpr uint32_t kIdesc = tc05::idesc_f16_f32(128, 128);

// smem: Q, K hi, K lo, V^T, P operands (1024-aligned), two staging buffers,
// barriers
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOpBytes;
constexpr uint32_t kOffKlo = 2 * kOpBytes;
constexpr uint32_t kOffV = 3 * kOpBytes;
constexpr uint32_t kOffP = 4 * kOpBytes;
constexpr uint32_t kOffStage = 5 * kOpBytes;
constexpr uint32_t kOffBar = kOffStage + 2 * kStageBytes;  // 4 mbarriers + tmem slot
constexpr uint32_t kOffRed = kOffBar + 64;                 // [4][128] fp32 row partials
constexpr uint32_t kSmemBytes = kOffRed + 4 * 128 * 4 + 1024;  // + alignment slack

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > kWaitLimit) return false;
  }
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

__device__ __forceinline__ uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
  return h2_as_u32(__hfma2(u32_as_h2(a), u32_as_h2(b), u32_as_h2(c)));
}

// Two keys (fp16 codes in `codes`) dequantized in fp32 (code * scale + zero:
// the product is exact, so one rounding) and split into fp16 hi and lo parts.
__device__ __forceinline__ void split_key(uint32_t codes, float2 sc, float2 z, uint32_t &hi, uint32_t &lo) {
  const float2 c = __half22float2(u32_as_h2(codes));
  const float2 k = fma2(c, sc, z);
  const __half2 h = __floats2half2_rn(k.x, k.y);
  const float2 r = sub2(k, __half22float2(h));
  hi = h2_as_u32(h);
  lo = h2_as_u32(__floats2half2_rn(r.x, r.y));
}

}  // namespace

__global__ void __launch_bounds__(kThreadsP, 1) prefill_kernel(const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t sQ = base + kOffQ, sK = base + kOffK, sKlo = base + kOffKlo, sV = base + kOffV, sP = base + kOffP;
  const uint32_t stage0 = base + kOffStage;
  const uint32_t bar_stage0 = base + kOffBar, bar_s = base + kOffBar + 16, bar_o = base + kOffBar + 24;
  const uint32_t tslot = base + kOffBar + 32;

  const int tid = threadIdx.x, warp = tid >> 5;
  const int G = p.group, H = p.num_kv_heads;
  const int Tq = 128 / G;                                   // tokens per query tile
  const int b = blockIdx.y, h = blockIdx.z;
  const int tile = static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x);  // long tiles first

  // ---- this CTA's rows (uniform across the CTA; exits before any allocation)
  const int c_lo = __ldg(p.cu_new + b), c_hi = __ldg(p.cu_new + b + 1);
  const int n = c_hi - c_lo;
  const int t0 = tile * Tq;
  if (n <= 0 || t0 >= n) return;
  int L = __ldg(p.seq_lens + b);
  if (c_lo < 0 || c_hi > p.n_tokens || L < n || L > p.max_pages * kPage) {
    if (tid == 0 && t0 == 0 && h == 0) flag_error(p.err, S4KV_EFLAG_SEQ_LEN);
    return;
  }
  const int tq = min(Tq, n - t0);
  const int rows = tq * G;
  const int pos_first = L - n + t0;
  const int n_keys = pos_first + tq;                         // keys 0 .. pos_last
  const int n_ktiles = (n_keys + kKeyTile - 1) / kKeyTile;
  const int nfull = L / kPage;
  const int np = (L + kPage - 1) / kPage;
  const int32_t *bt = p.block_tables + static_cast<long>(b) * p.max_pages;
  const uint8_t *head_pool = p.pool + static_cast<long>(h) * kBlockBytes;
  const long long page_stride = static_cast<long long>(H) * kBlockBytes;

  // ---- setup: tensor memory (S at columns 0..127, O at 128..255), barriers
  if (warp == 0) {
    tc05::tmem_alloc(tslot, 256);
    tc05::tmem_relinquish();
    tc05::fence_before_sync();
  }
  if (tid == 0) {
    mbar_init(bar_stage0, 1);
    mbar_init(bar_stage0 + 8, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_barrier_init();
  }

  // producer: the quantized pages of key tile kt into staging buffer kt & 1
  int fetched = 0;  // tiles fetched so far (thread 0)
  auto fetch = [&](int kt) {
    ++fetched;
    const int s = kt & 1;
    const uint32_t bar = bar_stage0 + 8u * s, dst = stage0 + s * kStageBytes;
    const int pg0 = kt * kPagesPerTile;
    const int q = max(0, min(kPagesPerTile, nfull - pg0));
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(q) * kBlockBytes);
    for (int k = 0; k < q; ++k) {
      int phys = __ldg(bt + pg0 + k);
      if (static_cast<unsigned>(phys) >= static_cast<unsigned>(p.num_pages)) {
        flag_error(p.err, S4KV_EFLAG_PAGE_RANGE);
        phys = 0;
      }
      bulk_copy_g2s(dst + k * kBlockBytes, head_pool + phys * page_stride, kBlockBytes, bar);
    }
  };
  __syncthreads();
  if (tid == 0) fetch(0);

  // ---- Q tile: row r = (token r / G, head r % G); rows >= rows are zero.
  // Four threads per row, four 16-byte chunks each.
  {
    const int r = tid >> 2, cq = tid & 3;
    const int tl = r / G, g = r - tl * G;
    const uint4 *src = reinterpret_cast<const uint4 *>(
        p.q + (static_cast<long>(c_lo + t0 + tl) * p.num_q_heads + h * G + g) * kHeadDim);
#pragma unroll
    for (int c = 4 * cq; c < 4 * cq + 4; ++c) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < rows) v = __ldg(src + c);
      sts128(sQ + tc05::sw128_offset(r, 8 * c, 128), v);
    }
  }

  tc05::fence_after_sync();
  const uint32_t tmem = lds32_at(tslot);
  const uint32_t tS = tmem, tO = tmem + 128;

  // ---- dequant mapping: 64 threads per page of the key tile; thread word
  // w = widx + 64 e (e = 0..3) of a code region, i.e. MMA lane (w % 128) / 4
  // and tile 4 (w / 128) + w % 4
  const int dpage = tid >> 6, widx = tid & 63;
  const int dq = widx & 3, dlane0 = widx >> 2;
  // swizzled store offsets of this thread's words (they do not change from
  // tile to tile): keys row 16 dpage + dn (and + 8 rows = + 1024 bytes),
  // channels 32 di + 4 t; values rows cb, cb + 1, keys 16 dpage + 2 di (+ 8)
  uint32_t kofs[4], vofs[4][4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int lane = dlane0 + 16 * (e & 1), t = 4 * (e >> 1) + dq;
    const int dn = lane >> 2, di = lane & 3;
    kofs[e] = tc05::sw128_offset(dpage * 16 + dn, 32 * di + 4 * t, 128);
    const int cb = 32 * (t >> 1) + 4 * dn + 2 * (t & 1);
    const int key = dpage * 16 + 2 * di;
    vofs[e][0] = tc05::sw128_offset(cb, key, 128);
    vofs[e][1] = tc05::sw128_offset(cb + 1, key, 128);
    vofs[e][2] = tc05::sw128_offset(cb, key + 8, 128);
    vofs[e][3] = tc05::sw128_offset(cb + 1, key + 8, 128);
  }

  // ---- softmax mapping: warp w reads tensor-memory lanes 32 (w % 4) ..
  // (row r = 32 (w % 4) + lane) and key columns 32 (w / 4) .. + 31
  const int qd = warp & 3, cq = warp >> 2;
  const int row = 32 * qd + (tid & 31);
  const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
  const bool row_ok = row < rows;
  const int pos_row = pos_first + (row_ok ? row / G : 0);
  float ref = -INFINITY;
  float2 lsum = make_float2(0.f, 0.f);  // this thread's columns only
  const float sl2 = p.scale_log2;
  float *red = reinterpret_cast<float *>(smem_raw + (base + kOffRed - raw));  // [4][128]

  bool failed = false;
  int kt = 0;
  for (; kt < n_ktiles; ++kt) {
    const int s = kt & 1;
    if (tid == 0 && kt + 1 < n_ktiles) fetch(kt + 1);
    if (!wait_bounded(bar_stage0 + 8u * s, (kt >> 1) & 1)) failed = true;
    if (__syncthreads_or(failed)) {
      failed = true;
      break;
    }
    const uint32_t stg = stage0 + s * kStageBytes;
    const int pg = kt * kPagesPerTile + dpage;
    const uint32_t blk = stg + dpage * kBlockBytes;
    const int rres = (pg == nfull && pg < np) ? L - nfull * kPage : 0;  // residual rows of a partial page
    const long res_base = (static_cast<long>(b) * H + h) * kPage * kHeadDim;

    // ---- keys of tile kt -> sK (hi) and sKlo; S(kt-1) finished before the
    // softmax of kt-1, so both are free
    if (pg < nfull) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int w = widx + 64 * e;
        const int lane = dlane0 + 16 * (e & 1), t = 4 * (e >> 1) + dq;
        const int di = lane & 3;
        uint32_t a0, a1, a2, a3;
        unpack_codes(lds32_at(blk + kKCodeOff + 4 * w), a0, a1, a2, a3);
        const int c0 = 32 * di + 4 * t;
        const uint2 sc = lds64_at(blk + kKScaleOff + 2 * c0);
        const uint32_t zslot = 16 * t + 2 * di;
        const uint32_t z01 = lds32_at(blk + kKZeroOff + 2 * zslot);
        const uint32_t z23 = lds32_at(blk + kKZeroOff + 2 * (zslot + 8));
        const float2 s01 = __half22float2(u32_as_h2(sc.x)), s23 = __half22float2(u32_as_h2(sc.y));
        const float2 zf01 = __half22float2(u32_as_h2(z01)), zf23 = __half22float2(u32_as_h2(z23));
        uint32_t hi0, lo0, hi1, lo1, hi2, lo2, hi3, lo3;
        split_key(a0, s01, zf01, hi0, lo0);
        split_key(a1, s01, zf01, hi1, lo1);
        split_key(a2, s23, zf23, hi2, lo2);
        split_key(a3, s23, zf23, hi3, lo3);
        const uint32_t o0 = kofs[e], o1 = kofs[e] + 1024;
        sts64(sK + o0, hi0, hi2);
        sts64(sK + o1, hi1, hi3);
        sts64(sKlo + o0, lo0, lo2);
        sts64(sKlo + o1, lo1, lo3);
      }
    } else {
      // the partial last page (fp16 residual rows < L % 16) or no page: copy
      // the valid rows, zero the rest, so masked keys hold finite values
      const __half *rk = p.res_k + res_base;
#pragma unroll 4
      for (int e = widx; e < kPage * kHeadDim / 2; e += 64) {
        const int tk = e >> 6, c = 2 * (e & 63);
        uint32_t kb = 0;
        if (tk < rres) kb = *reinterpret_cast<const uint32_t *>(rk + tk * kHeadDim + c);
        const uint32_t ko = tc05::sw128_offset(dpage * 16 + tk, c, 128);
        sts32(sK + ko, kb);
        sts32(sKlo + ko, 0u);
      }
    }
    fence_proxy_async();
    tc05::fence_before_sync();
    __syncthreads();

    // ---- S = Q K_hi^T + Q K_lo^T (overlaps the value dequantization below)
    if (tid == 0) {
      tc05::fence_after_sync();
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t off = (k >> 2) * (kOpBytes / 2) + (k & 3) * 32;
        tc05::mma_f16_ss(tS, tc05::smem_desc_sw128(sQ + off), tc05::smem_desc_sw128(sK + off), kIdesc,
                         k > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t off = (k >> 2) * (kOpBytes / 2) + (k & 3) * 32;
        tc05::mma_f16_ss(tS, tc05::smem_desc_sw128(sQ + off), tc05::smem_desc_sw128(sKlo + off), kIdesc, 1u);
      }
      tc05::mma_commit(bar_s);
    }

    // ---- values of tile kt -> sV (transposed), once O += P V of kt-1 is done
    if (kt > 0 && !wait_bounded(bar_o, (kt - 1) & 1)) failed = true;
    if (pg < nfull) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int w = widx + 64 * e;
        const int lane = dlane0 + 16 * (e & 1), t = 4 * (e >> 1) + dq;
        const int di = lane & 3;
        uint32_t a0, a1, a2, a3;
        unpack_codes(lds32_at(blk + kVCodeOff + 4 * w), a0, a1, a2, a3);
        const int g = t >> 1;
        const uint32_t sv_lo = lds32_at(blk + kVScaleOff + 2 * (16 * g + 2 * di));
        const uint32_t sv_hi = lds32_at(blk + kVScaleOff + 2 * (16 * g + 2 * di + 8));
        const uint32_t zv_lo = lds32_at(blk + kVZeroOff + 2 * (16 * g + 2 * di));
        const uint32_t zv_hi = lds32_at(blk + kVZeroOff + 2 * (16 * g + 2 * di + 8));
        sts32(sV + vofs[e][0], hfma2_u32(a0, sv_lo, zv_lo));
        sts32(sV + vofs[e][1], hfma2_u32(a1, sv_lo, zv_lo));
        sts32(sV + vofs[e][2], hfma2_u32(a2, sv_hi, zv_hi));
        sts32(sV + vofs[e][3], hfma2_u32(a3, sv_hi, zv_hi));
      }
    } else {
      const __half *rv = p.res_v + res_base;
#pragma unroll 4
      for (int e = widx; e < kPage * kHeadDim; e += 64) {
        const int tk = e >> 7, c = e & 127;
        uint16_t vb = 0;
        if (tk < rres) vb = __half_as_ushort(rv[tk * kHeadDim + c]);
        sts16(sV + tc05::sw128_offset(c, dpage * 16 + tk, 128), vb);
      }
    }
    fence_proxy_async();
    if (!wait_bounded(bar_s, kt & 1)) failed = true;
    if (__syncthreads_or(failed)) {
      failed = true;
      break;
    }
    tc05::fence_after_sync();

    // ---- online softmax: row `row`, key columns 32 cq .. 32 cq + 31.  A key
    // tile wholly before the tile's first query position needs no mask
    // (rows past the tile's last row hold q = 0, so finite logits, and are
    // never written out).
    {
      const int key0 = kt * kKeyTile + 32 * cq;
      const bool full = kt * kKeyTile + kKeyTile - 1 <= pos_first;
      uint32_t v[32];
      tc05::tmem_ld32(tS + lane_base + 32 * cq, v);
      tc05::tmem_wait_ld();
      float mx = -INFINITY;
      if (full) {
#pragma unroll
        for (int j = 0; j < 32; ++j) mx = fmaxf(mx, __uint_as_float(v[j]));
        mx *= sl2;
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const bool ok = row_ok && key0 + j <= pos_row;
          const float x = ok ? __uint_as_float(v[j]) : -INFINITY;
          v[j] = __float_as_uint(x);
          mx = fmaxf(mx, x);
        }
        mx *= sl2;
      }
      red[cq * 128 + row] = mx;
      __syncthreads();
      mx = fmaxf(fmaxf(red[row], red[128 + row]), fmaxf(red[256 + row], red[384 + row]));
      // the reference moves only when the row maximum passes it by > 8
      const bool move = mx > ref + kSlack;
      const float new_ref = move ? mx : ref;
      const float alpha = move ? fast_exp2(ref - new_ref) : 1.0f;  // 0 when ref was -inf
      if (__any_sync(0xFFFFFFFFu, move) && kt > 0) {
        // this warp's rows, columns 32 cq .. of O (warp-wide tensor-memory access)
        uint32_t o[32];
        tc05::tmem_ld32(tO + lane_base + 32 * cq, o);
        tc05::tmem_wait_ld();
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 r = mul2(make_float2(__uint_as_float(o[j]), __uint_as_float(o[j + 1])), a2);
          o[j] = __float_as_uint(r.x);
          o[j + 1] = __float_as_uint(r.y);
        }
        tc05::tmem_st32(tO + lane_base + 32 * cq, o);
        tc05::tmem_wait_st();
      }
      lsum = mul2(lsum, make_float2(alpha, alpha));
      ref = new_ref;
      // weights exp2(s * scale - ref); masked logits are -inf and give 0
      // (ref is finite for every row with a valid key; a row without one has
      // only masked logits, and its -inf reference is replaced by 0 so that
      // no inf - inf appears)
      const float nref = ref == -INFINITY ? 0.f : -ref;
      const float2 sc = make_float2(sl2, sl2), nr = make_float2(nref, nref);
      uint32_t hp[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float2 x = fma2(make_float2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])), sc, nr);
        const __half2 ph = __floats2half2_rn(fast_exp2(x.x), fast_exp2(x.y));
        // the row sum takes the fp16 weights the MMA multiplies with, so a
        // dominant key's value comes through exactly
        lsum = add2(lsum, __half22float2(ph));
        hp[j >> 1] = h2_as_u32(ph);
      }
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        sts128(sP + tc05::sw128_offset(row, 32 * cq + 8 * q4, 128),
               make_uint4(hp[4 * q4], hp[4 * q4 + 1], hp[4 * q4 + 2], hp[4 * q4 + 3]));
    }
    fence_proxy_async();
    tc05::fence_before_sync();
    __syncthreads();

    // ---- O += P V (overlaps the next tile's key dequantization)
    if (tid == 0) {
      tc05::fence_after_sync();
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t off = (k >> 2) * (kOpBytes / 2) + (k & 3) * 32;
        tc05::mma_f16_ss(tO, tc05::smem_desc_sw128(sP + off), tc05::smem_desc_sw128(sV + off), kIdesc,
                         (kt > 0 || k > 0) ? 1u : 0u);
      }
      tc05::mma_commit(bar_o);
    }
  }
  if (!failed && !wait_bounded(bar_o, (n_ktiles - 1) & 1)) failed = true;
  failed = __syncthreads_or(failed);
  tc05::fence_after_sync();

  if (!failed) {
    // ---- out = O / l: l is the sum of the four column quarters' partial sums
    red[cq * 128 + row] = lsum.x + lsum.y;
    __syncthreads();
    const float l = (red[row] + red[128 + row]) + (red[256 + row] + red[384 + row]);
    const float inv = row_ok && l > 0.f ? 1.0f / l : 0.f;
    uint32_t v[32];
    tc05::tmem_ld32(tO + lane_base + 32 * cq, v);
    tc05::tmem_wait_ld();
    if (row_ok) {
      const int tl = row / G, g = row - tl * G;
      __half *dst = p.out + (static_cast<long>(c_lo + t0 + tl) * p.num_q_heads + h * G + g) * kHeadDim + 32 * cq;
      uint32_t hv[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2)
        hv[j >> 1] = h2_as_u32(__floats2half2_rn(__uint_as_float(v[j]) * inv, __uint_as_float(v[j + 1]) * inv));
      uint4 *o4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) o4[q4] = make_uint4(hv[4 * q4], hv[4 * q4 + 1], hv[4 * q4 + 2], hv[4 * q4 + 3]);
    }
  } else if (tid == 0) {
    flag_error(p.err, S4KV_EFLAG_TIMEOUT);
    // wait (bounded) for the bulk copies still in flight before the CTA exits
    for (int f = kt; f < fetched; ++f) wait_bounded(bar_stage0 + 8u * (f & 1), (f >> 1) & 1);
  }

  tc05::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc05::tmem_dealloc(tmem, 256);
}

size_t prefill_smem_bytes() { return kSmemBytes; }

cudaError_t prepare_prefill_kernel() {
  return cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemBytes));
}

void launch_prefill(const PrefillParams &p, int batch, int max_new, cudaStream_t stream) {
  const int Tq = 128 / p.group;
  const int tiles = (max_new + Tq - 1) / Tq;
  const dim3 grid(tiles, batch, p.num_kv_heads);
  prefill_kernel<<<grid, kThreadsP, kSmemBytes, stream>>>(p);
}

}  // namespace s4kv
