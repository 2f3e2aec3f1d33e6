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
// floor(128 / G) tokens.  Keys are walked in tiles of 64 (4 pages) by warps
// with separate roles, handing buffers over through mbarriers so that the
// dequantization, the tensor core and the softmax run at the same time:
//  * a producer warp brings each key tile's page blocks into one of two
//    staging buffers with 1-D bulk copies (TMA engine, no multicast);
//  * 8 dequantization warps turn a staged tile into the 128-byte-swizzled
//    fp16 operands of one of two operand buffers.  A key is code * scale +
//    zero in fp32 (exact product, one rounding, the value the oracle's
//    dequantization gives) split into an fp16 hi part and the fp16 rounding
//    of the remainder, so K_hi + K_lo carries it to about 22 bits (keys of
//    outlier channels are large, and a single fp16 rounding of them moves the
//    logits visibly).  A value is the fused fp16 multiply-add code * scale +
//    zero (the correctly rounded fp16), stored transposed (V^T);
//  * one thread issues S(k) = Q K_hi^T + Q K_lo^T (M = 128, N = 64) into one
//    of two tensor-memory buffers, then O += P(k-1) V(k-1) (N = 128, K = 64),
//    so the tensor core computes the next logits during the softmax;
//  * 4 softmax warps (one tensor-memory lane, i.e. one row, per thread) read
//    S back, apply the causal mask and an online softmax in the exp2 domain
//    whose reference moves only when a row maximum passes it by more than 8
//    (weights stay <= 256, fine for fp16), rescale that row of O in tensor
//    memory when it moves, and write P (fp16) to shared memory.
// Every wait is bounded; a timeout sets a CTA-wide abort flag and an error
// bit, and every role then leaves its loop.
#include <cfloat>

#include "kernels.cuh"
#include "tc05.cuh"

namespace s4kv {

namespace {

constexpr int kSoftmaxWarps = 4;   // warps 0..3: one row per thread
constexpr int kDequantWarps = 8;   // warps 4..11
constexpr int kMmaWarp = 12;
constexpr int kProducerWarp = 13;
constexpr int kThreadsP = 32 * 14;
constexpr int kDqThreads = 32 * kDequantWarps;
constexpr int kKeyTile = 64;                     // keys per tile (MMA N of S)
constexpr int kPagesPerTile = kKeyTile / kPage;  // 4
constexpr uint32_t kQBytes = 128 * 128 * 2;      // Q [128][128] fp16
constexpr uint32_t kKBytes = 64 * 128 * 2;       // K [64][128] fp16
constexpr uint32_t kVBytes = 128 * 64 * 2;       // V^T [128][64] fp16
constexpr uint32_t kPBytes = 128 * 64 * 2;       // P [128][64] fp16
constexpr uint32_t kStageBytes = kPagesPerTile * kBlockBytes;
constexpr float kSlack = 8.0f;                   // log2 slack of the softmax reference
constexpr long long kWaitLimit = 2000000000LL;   // about one second
constexpr uint32_t kIdescS = tc05::idesc_f16_f32(128, 64);
constexpr uint32_t kIdescO = tc05::idesc_f16_f32(128, 128);

// smem: operands (1024-aligned), two staging buffers, barriers
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKhi = kOffQ + kQBytes;         // [2]
constexpr uint32_t kOffKlo = kOffKhi + 2 * kKBytes;   // [2]
constexpr uint32_t kOffV = kOffKlo + 2 * kKBytes;     // [2]
constexpr uint32_t kOffP = kOffV + 2 * kVBytes;
constexpr uint32_t kOffStage = kOffP + kPBytes;       // [2]
constexpr uint32_t kOffBar = kOffStage + 2 * kStageBytes;
// barriers (8 bytes each): stage_full[2], stage_empty[2], kv_full[2],
// kv_empty[2], s_full[2], s_empty[2], p_full, p_empty; then the tensor-memory
// address and the abort flag
constexpr uint32_t kNumBars = 14;
constexpr uint32_t kOffSlot = kOffBar + 8 * kNumBars;
constexpr uint32_t kOffAbort = kOffSlot + 4;
constexpr uint32_t kSmemBytes = kOffAbort + 4 + 1024;  // + alignment slack

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
  const uint32_t sQ = base + kOffQ, sP = base + kOffP;
  const uint32_t stage0 = base + kOffStage;
  const uint32_t bars = base + kOffBar;
  const uint32_t tslot = base + kOffSlot;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem_raw + (base + kOffAbort - raw));
  auto khi = [&](int s) { return base + kOffKhi + s * kKBytes; };
  auto klo = [&](int s) { return base + kOffKlo + s * kKBytes; };
  auto vop = [&](int s) { return base + kOffV + s * kVBytes; };
  auto stage_full = [&](int s) { return bars + 8u * (0 + s); };
  auto stage_empty = [&](int s) { return bars + 8u * (2 + s); };
  auto kv_full = [&](int s) { return bars + 8u * (4 + s); };
  auto kv_empty = [&](int s) { return bars + 8u * (6 + s); };
  auto s_full = [&](int s) { return bars + 8u * (8 + s); };
  auto s_empty = [&](int s) { return bars + 8u * (10 + s); };
  const uint32_t p_full = bars + 8u * 12, p_empty = bars + 8u * 13;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.group, H = p.num_kv_heads;
  const int Tq = 128 / G;                                   // tokens per query tile
  const int b = blockIdx.y, h = blockIdx.z;
  const int tile = static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x);  // long tiles first

  // ---- this CTA's rows (uniform across the CTA; exits before any allocation)
  const int c_lo = __ldg(p.cu_new + b), c_hi = __ldg(p.cu_new + b + 1);
  const int n = c_hi - c_lo;
  const int t0 = tile * Tq;
  if (n <= 0 || t0 >= n) return;
  const int L = __ldg(p.seq_lens + b);
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

  // ---- setup: tensor memory (S buffers at columns 0 and 64, O at 128), barriers
  if (warp == 0) {
    tc05::tmem_alloc(tslot, 256);
    tc05::tmem_relinquish();
    tc05::fence_before_sync();
  }
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(stage_full(s), 1);
      mbar_init(stage_empty(s), kDqThreads);
      mbar_init(kv_full(s), kDqThreads);
      mbar_init(kv_empty(s), 1);
      mbar_init(s_full(s), 1);
      mbar_init(s_empty(s), 32 * kSoftmaxWarps);
    }
    mbar_init(p_full, 32 * kSoftmaxWarps);
    mbar_init(p_empty, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // ---- Q tile: row r = (token r / G, head r % G); rows >= rows are zero
  for (int ch = tid; ch < 128 * 16; ch += kThreadsP) {
    const int r = ch >> 4, c = ch & 15;
    const int tl = r / G, g = r - tl * G;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < rows)
      v = __ldg(reinterpret_cast<const uint4 *>(
                    p.q + (static_cast<long>(c_lo + t0 + tl) * p.num_q_heads + h * G + g) * kHeadDim) + c);
    sts128(sQ + tc05::sw128_offset(r, 8 * c, 128), v);
  }
  fence_proxy_async();
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = lds32_at(tslot);
  const uint32_t tO = tmem + 128;
  auto tS = [&](int s) { return tmem + 64u * s; };
  bool failed = false;
  auto fail = [&]() {
    failed = true;
    *abort_flag = 1;
  };

  if (warp == kProducerWarp) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      const int32_t *bt = p.block_tables + static_cast<long>(b) * p.max_pages;
      const uint8_t *head_pool = p.pool + static_cast<long>(h) * kBlockBytes;
      const long long page_stride = static_cast<long long>(H) * kBlockBytes;
      int issued = 0;
      for (int kt = 0; kt < n_ktiles && !failed; ++kt) {
        const int s = kt & 1;
        if (kt >= 2 && !wait_bounded(stage_empty(s), ((kt >> 1) - 1) & 1, abort_flag)) {
          fail();
          break;
        }
        ++issued;
        const int pg0 = kt * kPagesPerTile;
        const int q = max(0, min(kPagesPerTile, nfull - pg0));
        mbar_arrive_expect_tx(stage_full(s), static_cast<uint32_t>(q) * kBlockBytes);
        for (int k = 0; k < q; ++k) {
          int phys = __ldg(bt + pg0 + k);
          if (static_cast<unsigned>(phys) >= static_cast<unsigned>(p.num_pages)) {
            flag_error(p.err, S4KV_EFLAG_PAGE_RANGE);
            phys = 0;
          }
          bulk_copy_g2s(stage0 + s * kStageBytes + k * kBlockBytes, head_pool + phys * page_stride, kBlockBytes,
                        stage_full(s));
        }
      }
      // before the CTA exits, the copies in flight must have landed (bounded
      // by time only, also after an abort)
      const volatile int no_abort = 0;
      for (int kt = max(0, issued - 2); kt < issued; ++kt) wait_bounded(stage_full(kt & 1), (kt >> 1) & 1, &no_abort);
    }
  } else if (warp >= kSoftmaxWarps && warp < kSoftmaxWarps + kDequantWarps) {
    // -------------------------------------------------------- dequantizer
    const int t = tid - 32 * kSoftmaxWarps;  // 0 .. 255
    const int dpage = t >> 6, widx = t & 63;
    const int dq = widx & 3, dlane0 = widx >> 2;
    // swizzled store offsets of this thread's words (the same for every
    // tile): keys rows 16 dpage + dn (and + 8 rows = + 1024 bytes), channels
    // 32 di + 4 tt; values rows cb, cb + 1, keys 16 dpage + 2 di (+ 8)
    uint32_t kofs[4], vofs[4][4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int ln = dlane0 + 16 * (e & 1), tt = 4 * (e >> 1) + dq;
      const int dn = ln >> 2, di = ln & 3;
      kofs[e] = tc05::sw128_offset(dpage * 16 + dn, 32 * di + 4 * tt, 64);
      const int cb = 32 * (tt >> 1) + 4 * dn + 2 * (tt & 1);
      const int key = dpage * 16 + 2 * di;
      vofs[e][0] = tc05::sw128_offset(cb, key, 128);
      vofs[e][1] = tc05::sw128_offset(cb + 1, key, 128);
      vofs[e][2] = tc05::sw128_offset(cb, key + 8, 128);
      vofs[e][3] = tc05::sw128_offset(cb + 1, key + 8, 128);
    }
    const long res_base = (static_cast<long>(b) * H + h) * kPage * kHeadDim;
    for (int kt = 0; kt < n_ktiles; ++kt) {
      const int s = kt & 1;
      if (!wait_bounded(stage_full(s), (kt >> 1) & 1, abort_flag)) {
        fail();
        break;
      }
      if (kt >= 2 && !wait_bounded(kv_empty(s), ((kt >> 1) - 1) & 1, abort_flag)) {
        fail();
        break;
      }
      const uint32_t sKh = khi(s), sKl = klo(s), sV = vop(s);
      const int pg = kt * kPagesPerTile + dpage;
      const uint32_t blk = stage0 + s * kStageBytes + dpage * kBlockBytes;
      if (pg < nfull) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int w = widx + 64 * e;
          const int ln = dlane0 + 16 * (e & 1), tt = 4 * (e >> 1) + dq;
          const int di = ln & 3;
          // keys: tokens dn, dn + 8; channels c0 .. c0 + 3
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
            uint32_t hi0, lo0, hi1, lo1, hi2, lo2, hi3, lo3;
            split_key(a0, s01, zf01, hi0, lo0);
            split_key(a1, s01, zf01, hi1, lo1);
            split_key(a2, s23, zf23, hi2, lo2);
            split_key(a3, s23, zf23, hi3, lo3);
            sts64(sKh + kofs[e], hi0, hi2);
            sts64(sKh + kofs[e] + 1024, hi1, hi3);
            sts64(sKl + kofs[e], lo0, lo2);
            sts64(sKl + kofs[e] + 1024, lo1, lo3);
          }
          // values: channels cb, cb + 1; tokens 2 di, 2 di + 1 (+ 8)
          {
            uint32_t a0, a1, a2, a3;
            unpack_codes(lds32_at(blk + kVCodeOff + 4 * w), a0, a1, a2, a3);
            const int g = tt >> 1;
            const uint32_t sv_lo = lds32_at(blk + kVScaleOff + 2 * (16 * g + 2 * di));
            const uint32_t sv_hi = lds32_at(blk + kVScaleOff + 2 * (16 * g + 2 * di + 8));
            const uint32_t zv_lo = lds32_at(blk + kVZeroOff + 2 * (16 * g + 2 * di));
            const uint32_t zv_hi = lds32_at(blk + kVZeroOff + 2 * (16 * g + 2 * di + 8));
            sts32(sV + vofs[e][0], hfma2_u32(a0, sv_lo, zv_lo));
            sts32(sV + vofs[e][1], hfma2_u32(a1, sv_lo, zv_lo));
            sts32(sV + vofs[e][2], hfma2_u32(a2, sv_hi, zv_hi));
            sts32(sV + vofs[e][3], hfma2_u32(a3, sv_hi, zv_hi));
          }
        }
      } else {
        // the partial last page (fp16 residual rows < L % 16) or no page:
        // copy the valid rows, zero the rest, so masked keys hold finite values
        const int rres = (pg == nfull && pg < np) ? L - nfull * kPage : 0;
        const __half *rk = p.res_k + res_base;
        const __half *rv = p.res_v + res_base;
        for (int e = widx; e < kPage * kHeadDim / 2; e += 64) {
          const int tk = e >> 6, c = 2 * (e & 63);
          uint32_t kb = 0;
          if (tk < rres) kb = *reinterpret_cast<const uint32_t *>(rk + tk * kHeadDim + c);
          const uint32_t ko = tc05::sw128_offset(dpage * 16 + tk, c, 64);
          sts32(sKh + ko, kb);
          sts32(sKl + ko, 0u);
        }
        for (int e = widx; e < kPage * kHeadDim; e += 64) {
          const int tk = e >> 7, c = e & 127;
          uint16_t vb = 0;
          if (tk < rres) vb = __half_as_ushort(rv[tk * kHeadDim + c]);
          sts16(sV + tc05::sw128_offset(c, dpage * 16 + tk, 128), vb);
        }
      }
      fence_proxy_async();  // operand writes -> MMA reads; staging reads -> the next bulk copy
      mbar_arrive(kv_full(s));
      mbar_arrive(stage_empty(s));
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      auto issue_pv = [&](int k) {  // O += P(k) V(k)
        const int s = k & 1;
        if (!wait_bounded(p_full, k & 1, abort_flag)) return false;
        tc05::fence_after_sync();
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tc05::mma_f16_ss(tO, tc05::smem_desc_sw128(sP + 32 * j), tc05::smem_desc_sw128(vop(s) + 32 * j), kIdescO,
                           (k > 0 || j > 0) ? 1u : 0u);
        tc05::mma_commit(p_empty);
        tc05::mma_commit(kv_empty(s));
        return true;
      };
      for (int kt = 0; kt < n_ktiles; ++kt) {
        const int s = kt & 1;
        if (!wait_bounded(kv_full(s), (kt >> 1) & 1, abort_flag) ||
            (kt >= 2 && !wait_bounded(s_empty(s), ((kt >> 1) - 1) & 1, abort_flag))) {
          fail();
          break;
        }
        tc05::fence_after_sync();
        // S(kt) = Q K_hi^T + Q K_lo^T
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t qo = (j >> 2) * (kQBytes / 2) + (j & 3) * 32;
          const uint32_t ko = (j >> 2) * (kKBytes / 2) + (j & 3) * 32;
          tc05::mma_f16_ss(tS(s), tc05::smem_desc_sw128(sQ + qo), tc05::smem_desc_sw128(khi(s) + ko), kIdescS,
                           j > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t qo = (j >> 2) * (kQBytes / 2) + (j & 3) * 32;
          const uint32_t ko = (j >> 2) * (kKBytes / 2) + (j & 3) * 32;
          tc05::mma_f16_ss(tS(s), tc05::smem_desc_sw128(sQ + qo), tc05::smem_desc_sw128(klo(s) + ko), kIdescS, 1u);
        }
        tc05::mma_commit(s_full(s));
        // O += P(kt-1) V(kt-1) while the softmax of kt runs
        if (kt >= 1 && !issue_pv(kt - 1)) {
          fail();
          break;
        }
      }
      if (!failed && !issue_pv(n_ktiles - 1)) fail();
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
    for (int kt = 0; kt < n_ktiles; ++kt) {
      const int s = kt & 1;
      if (!wait_bounded(s_full(s), (kt >> 1) & 1, abort_flag)) {
        fail();
        break;
      }
      tc05::fence_after_sync();
      uint32_t v[64];
      {
        uint32_t (&v0)[32] = *reinterpret_cast<uint32_t (*)[32]>(&v[0]);
        uint32_t (&v1)[32] = *reinterpret_cast<uint32_t (*)[32]>(&v[32]);
        tc05::tmem_ld32(tS(s) + lane_base, v0);
        tc05::tmem_ld32(tS(s) + lane_base + 32, v1);
        tc05::tmem_wait_ld();
      }
      tc05::fence_before_sync();
      mbar_arrive(s_empty(s));
      // a key tile wholly before the tile's first query position needs no
      // mask (rows past the last row hold q = 0: finite logits, never written)
      const int key0 = kt * kKeyTile;
      const bool full = key0 + kKeyTile - 1 <= pos_first;
      float mx = -INFINITY;
      if (full) {
#pragma unroll
        for (int j = 0; j < 64; ++j) mx = fmaxf(mx, __uint_as_float(v[j]));
      } else {
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const bool ok = row_ok && key0 + j <= pos_row;
          const float x = ok ? __uint_as_float(v[j]) : -INFINITY;
          v[j] = __float_as_uint(x);
          mx = fmaxf(mx, x);
        }
      }
      mx *= sl2;
      // the reference moves only when the row maximum passes it by > 8
      const bool move = mx > ref + kSlack;
      const float new_ref = move ? mx : ref;
      const float alpha = move ? fast_exp2(ref - new_ref) : 1.0f;  // 0 when ref was -inf
      // O and P are free once O += P(kt-1) V(kt-1) has completed
      if (kt >= 1) {
        if (!wait_bounded(p_empty, (kt - 1) & 1, abort_flag)) {
          fail();
          break;
        }
        tc05::fence_after_sync();
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
          tc05::tmem_wait_st();
        }
      }
      lsum = mul2(lsum, make_float2(alpha, alpha));
      ref = new_ref;
      // weights exp2(s * scale - ref); masked logits are -inf and give 0 (a
      // row without a valid key keeps a -inf reference, replaced by 0 so that
      // no inf - inf appears)
      const float nref = ref == -INFINITY ? 0.f : -ref;
      const float2 sc = make_float2(sl2, sl2), nr = make_float2(nref, nref);
#pragma unroll
      for (int q8 = 0; q8 < 8; ++q8) {
        uint32_t hp[4];
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
          const int k = 8 * q8 + j;
          const float2 x = fma2(make_float2(__uint_as_float(v[k]), __uint_as_float(v[k + 1])), sc, nr);
          const __half2 ph = __floats2half2_rn(fast_exp2(x.x), fast_exp2(x.y));
          // the row sum takes the fp16 weights the MMA multiplies with
          lsum = add2(lsum, __half22float2(ph));
          hp[j >> 1] = h2_as_u32(ph);
        }
        sts128(sP + tc05::sw128_offset(row, 8 * q8, 128), make_uint4(hp[0], hp[1], hp[2], hp[3]));
      }
      fence_proxy_async();
      tc05::fence_before_sync();
      mbar_arrive(p_full);
    }
    // ---- out = O / l once the last O += P V has completed
    if (!failed && !wait_bounded(p_empty, (n_ktiles - 1) & 1, abort_flag)) fail();
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
    tc05::tmem_dealloc(tmem, 256);
  }
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
