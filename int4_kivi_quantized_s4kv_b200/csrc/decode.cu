// s4kv_decode_attention device side: GQA paged decode attention over int4
// KIVI pages plus the fp16 residual, split along the KV sequence.
//
// What it computes: for sequence b and query head j (kv head j / G, the GQA
// grouping of "KV-Cache-Optimierung -- PagedAttention, quantisierter KV,
// Speculative Cache", "Begriffe auf dieser Seite"),
//   out = softmax(sm_scale * q K^T) V
// over the sequence's tokens, where the keys and values of full pages are
// the dequantized int4 codes (code * scale + zero; "S4 KV -- int4
// KV-Cache-Kompression fuer vLLM", "Funktionsweise" step 1) and the tokens of
// the partial last page come from the fp16 residual.
//
// How (B200):
//  * Work split.  The pages of all (sequence, kv head) segments are laid end
//    to end and cut into one contiguous range per worker warp (all SMs, a
//    fixed number of resident warps each).  A segment cut between workers
//    produces partial (m, l, O) results; the worker that finishes a
//    segment's last piece (an atomic ticket per segment) merges them with a
//    log-sum-exp and writes the output, then resets the ticket.
//  * Staging.  Each warp owns a ring of shared-memory stages, one page block
//    each, filled by 1-D bulk copies (TMA engine, no multicast) gathered
//    through block_tables and completing on one mbarrier per stage.  The
//    consumer takes pages two at a time: one vote waits for both stages, and
//    lanes 0 and 1 refill both released stages with one copy instruction.
//    Waits are bounded and report a timeout through err_flag.
//  * Math.  Per page (16 tokens) and kv head, with tokens on the MMA's M, the
//    G <= 8 query heads on N and channels on K:
//      S = codes_K . (q * sK) + zK . q
//    and, with channels on M and tokens on K,
//      O += codes_V^T . (P * sV) + [zV rows] . P
//    The per-channel key scale and per-token value scale multiply the small
//    operand, so the 4-bit codes (exact in fp16) feed the tensor cores
//    directly; each scaled operand is split into fp16 hi + lo parts whose sum
//    is exact (q and sK, P-hi and sV are fp16, their product fits in two
//    halves), giving fp32-level accuracy.  A lane's packed 32-bit code word is
//    its own operand fragment: the low and high nibbles of its bytes are
//    masked apart and each byte pair converted as an fp8 e4m3 pair, which
//    yields code * 2^-9 exactly (1 shift, 2 LOP3 and 4 conversions per 8
//    codes); the factor 512 is restored in fp32.  The key zero-point terms of
//    a page pair come from one MMA per k-tile (rows 0-7 one page's zeros,
//    rows 8-15 the other's).  The softmax is an online update in the exp2
//    domain whose reference only moves when a maximum passes it (with a
//    headroom of 4, so every weight stays <= 1 and no fp16 operand can
//    overflow); P is moved from the QK accumulator layout to the PV operand
//    layout with movmatrix.
//  * Pipelining.  Within a warp, the softmax of page pair k, the QK MMAs of
//    pair k+1 and the PV MMAs of pair k are issued in one straight-line
//    block, so the softmax's latency overlaps tensor-core work.
#include <cfloat>

#include "kernels.cuh"
#include "quant.cuh"

namespace s4kv {

// Build-time tuning constants: stages per warp ring; worker warps per CTA,
// one CTA per SM so that all warps of an SM are equally old and the warp
// schedulers serve them alike (4- and 2-bit pages: 12 warps with 6 stages;
// 4864-byte int8 blocks: 8 warps with 5 stages); the fewest pages a worker
// is given, so that small batches are not cut into many short pieces.
#ifndef S4KV_DECODE_STAGES
#define S4KV_DECODE_STAGES 6
#endif
#ifndef S4KV_DECODE_WARPS
#define S4KV_DECODE_WARPS 12
#endif
#ifndef S4KV_DECODE_STAGES_INT8
#define S4KV_DECODE_STAGES_INT8 5
#endif
#ifndef S4KV_DECODE_WARPS_INT8
#define S4KV_DECODE_WARPS_INT8 8
#endif
#ifndef S4KV_DECODE_MIN_PAGES
#define S4KV_DECODE_MIN_PAGES 16
#endif
template <int kBits>
__host__ __device__ constexpr int stages_for() { return kBits == 8 ? S4KV_DECODE_STAGES_INT8 : S4KV_DECODE_STAGES; }
template <int kBits>
__host__ __device__ constexpr int warps_for() { return kBits == 8 ? S4KV_DECODE_WARPS_INT8 : S4KV_DECODE_WARPS; }
template <int kBits>
__host__ __device__ constexpr int threads_for() { return 32 * warps_for<kBits>(); }
// registers: the whole file of an SM for 12 warps, half of it for 4
template <int kBits>
__host__ __device__ constexpr int min_ctas_for() { return 12 / warps_for<kBits>() > 1 ? 12 / warps_for<kBits>() : 1; }
constexpr long long kWaitLimitCycles = 2000000000LL;  // about one second
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr float kHeadroom = 4.0f;  // log2 headroom of the softmax reference

template <int kBits>
constexpr size_t smem_bytes_for() {
  return static_cast<size_t>(warps_for<kBits>()) * stages_for<kBits>() * (Fmt<kBits>::kBlock + 8);
}

size_t decode_smem_bytes(int bits) {
  return bits == 8 ? smem_bytes_for<8>() : bits == 2 ? smem_bytes_for<2>() : smem_bytes_for<4>();
}

__device__ __forceinline__ int clamp_len(int L, int max_pages) {
  return min(max(L, 0), max_pages * kPage);
}

// Position in the flattened (sequence, kv head, page) order.
struct Cursor {
  long long start;    // flattened index of the segment's first page
  const int32_t *bt;  // block_tables row of sequence b
  int b, h;
  int len;            // tokens of sequence b
  int np;             // pages of b (full pages + a partial residual page)
  int nfull;          // full (quantized) pages of b
};

__device__ __forceinline__ void set_seq(Cursor &c, const DecodeParams &p, int b, int len) {
  c.b = b;
  c.len = len;
  c.np = (len + kPage - 1) / kPage;
  c.nfull = len / kPage;
  c.bt = p.block_tables + static_cast<long>(b) * p.max_pages;
}

__device__ __forceinline__ void next_segment(Cursor &c, const DecodeParams &p) {
  c.start += c.np;
  if (++c.h == p.num_kv_heads) {
    c.h = 0;
    int b = c.b + 1, L = 0;
    while (b < p.batch) {
      L = clamp_len(__ldg(p.seq_lens + b), p.max_pages);
      if (L > 0) break;
      ++b;
    }
    set_seq(c, p, b, b < p.batch ? L : 0);
  }
}

// Worker whose range [w*T/W, (w+1)*T/W) holds flattened page x (W <= T).
__device__ __forceinline__ long long worker_of(long long x, long long T, long long W) {
  return ((x + 1) * W + T - 1) / T - 1;
}

// Running softmax state of one lane: heads 2i, 2i+1 of the group.
struct Online {
  float2 nref;       // minus the log2-domain reference: weights are exp2(s - ref) <= 1
  float thr0, thr1;  // raw-logit threshold ref / scale (rounded down)
  float2 l;          // partial sums of weights over this lane's tokens
  float O[8][4];     // PV accumulators (M-tile, C fragment)
  float Z[4];        // value zero-point term: sum_t zV[g][t] P[t][h]
};

// Per-lane byte offsets inside a stage: the lane's 16 bytes of code words
// (16*lane), its key-scale run (64*i: channels 32i .. 32i+31), its value-scale
// run (32*i: token pairs 2i, 2i+8 of the four groups), its row of the value
// zero points for ldmatrix (row r of the operand holds group r % 4; lanes
// 16..31 read tokens 8..15) and its row of the key zero points (lanes 16..31
// read k columns 8..15).
struct LaneOff {
  uint32_t code, kmeta, vscale, vzero, kzero;
};

template <int kBits>
__device__ __forceinline__ LaneOff lane_offsets(int lane) {
  using F = Fmt<kBits>;
  const uint32_t i = lane & 3, half_k = (lane >> 4) ? 16u : 0u;
  return LaneOff{16u * lane, F::kKScale + 64u * i, F::kVScale + 32u * i, F::kVZero + 32u * (lane & 3) + half_k,
                 F::kKZero + half_k};
}

// Query fragments of this lane (B operand of the QK MMAs: channels 32i ..
// 32i + 31, head n).
struct QFrag {
  uint32_t w[16];
  __device__ __forceinline__ uint4 pair(int m) const { return make_uint4(w[4 * m], w[4 * m + 1], w[4 * m + 2], w[4 * m + 3]); }
};

// Key zero-point operand of k-tile kt (kt is a constant after unrolling, so
// the switch folds to one ldmatrix with an immediate offset).
__device__ __forceinline__ void ldmatrix_kzero(uint32_t base, int kt, uint32_t &z0, uint32_t &z1, uint32_t &z2,
                                               uint32_t &z3) {
  switch (kt) {
    case 0: ldmatrix_x4<0>(base, z0, z1, z2, z3); break;
    case 1: ldmatrix_x4<32>(base, z0, z1, z2, z3); break;
    case 2: ldmatrix_x4<64>(base, z0, z1, z2, z3); break;
    case 3: ldmatrix_x4<96>(base, z0, z1, z2, z3); break;
    case 4: ldmatrix_x4<128>(base, z0, z1, z2, z3); break;
    case 5: ldmatrix_x4<160>(base, z0, z1, z2, z3); break;
    case 6: ldmatrix_x4<192>(base, z0, z1, z2, z3); break;
    default: ldmatrix_x4<224>(base, z0, z1, z2, z3); break;
  }
}

// Operand fragment of key / value tile kt of a quantized page (kt constant
// after unrolling): one 4-bit code word (values code * 2^-9), or two 8-bit
// words of the chunk that holds tiles 2m, 2m + 1 of this lane, or the 2-bit
// word of tiles 2m, 2m + 1.
template <int kBits>
__device__ __forceinline__ void tile_fragment(const uint32_t (&w)[8], int kt, uint32_t &a0, uint32_t &a1,
                                              uint32_t &a2, uint32_t &a3) {
  if (kBits == 8) unpack_codes8(w[2 * (kt & 1)], w[2 * (kt & 1) + 1], a0, a1, a2, a3);
  else if (kBits == 2) {
    if (kt & 1) unpack_codes2<1>(w[kt >> 1], a0, a1, a2, a3);
    else unpack_codes2<0>(w[kt >> 1], a0, a1, a2, a3);
  } else unpack_codes_s9(w[kt], a0, a1, a2, a3);
}

// What the code operand's values must be multiplied by to give the codes:
// 4-bit codes enter the MMAs as code * 2^-9.
template <int kBits>
__host__ __device__ constexpr float code_unit_inv() { return kBits == 4 ? 512.0f : 1.0f; }

// The key code words of a page for the whole QK (4- and 2-bit codes; 8-bit
// codes are loaded per k-tile pair).
template <int kBits>
__device__ __forceinline__ void load_key_words(uint32_t code, uint32_t (&kw)[8]) {
  using F = Fmt<kBits>;
  if (kBits == 4) {
    const uint4 w0 = lds128<F::kKCode>(code), w1 = lds128<F::kKCode + 512>(code);
    kw[0] = w0.x; kw[1] = w0.y; kw[2] = w0.z; kw[3] = w0.w;
    kw[4] = w1.x; kw[5] = w1.y; kw[6] = w1.z; kw[7] = w1.w;
  } else if (kBits == 2) {
    const uint4 w0 = lds128<F::kKCode>(code);
    kw[0] = w0.x; kw[1] = w0.y; kw[2] = w0.z; kw[3] = w0.w;
  }
}

template <int kBits>
__device__ __forceinline__ void load_key_words8(uint32_t code, int m, uint32_t (&kw)[8]) {
  using F = Fmt<kBits>;
  if (kBits == 8) {
    const uint4 cw = m == 0 ? lds128<F::kKCode>(code) : m == 1 ? lds128<F::kKCode + 512>(code)
                   : m == 2 ? lds128<F::kKCode + 1024>(code) : lds128<F::kKCode + 1536>(code);
    kw[0] = cw.x; kw[1] = cw.y; kw[2] = cw.z; kw[3] = cw.w;
  }
}

// One k-tile of one page's codes against q * sK (hi and lo parts into their
// own accumulators).
template <int kBits>
__device__ __forceinline__ void qk_tile(const uint32_t (&kw)[8], int kt, uint32_t s0w, uint32_t s1w, uint32_t q0w,
                                        uint32_t q1w, float (&Sh)[4], float (&Sl)[4]) {
  uint32_t a0, a1, a2, a3;
  tile_fragment<kBits>(kw, kt, a0, a1, a2, a3);
  const __half2 qb0 = u32_as_h2(q0w), qb1 = u32_as_h2(q1w);
  const __half2 s0 = u32_as_h2(s0w), s1 = u32_as_h2(s1w);
  // q * sK split into fp16 hi + lo; the lo part is the exact remainder
  const __half2 h0 = __hmul2(qb0, s0), h1 = __hmul2(qb1, s1);
  const __half2 r0 = __hfma2(qb0, s0, __hneg2(h0));
  const __half2 r1 = __hfma2(qb1, s1, __hneg2(h1));
  mma16816(Sh, a0, a1, a2, a3, h2_as_u32(h0), h2_as_u32(h1));
  mma16816(Sl, a0, a1, a2, a3, h2_as_u32(r0), h2_as_u32(r1));
}

// Logits of two quantized pages A and B (stage byte addresses sa, sb; B may
// be A again): this lane's S^T[tokens n, n+8][heads 2i, 2i+1] of each page,
// before sm_scale.  zrow: this lane's key-zero row address (page A's stage for
// lanes 0-7 and 16-23, page B's for lanes 8-15 and 24-31), so that one MMA
// per k-tile gives page A's zero-point terms in rows 0-7 and page B's in rows
// 8-15.
template <int kBits>
__device__ __forceinline__ void qk_pair(uint32_t sa, uint32_t sb, uint32_t zrow, const LaneOff &lo, const QFrag &q,
                                        float (&SA)[4], float (&SB)[4]) {
  using F = Fmt<kBits>;
  float ShA[4] = {0.f, 0.f, 0.f, 0.f}, SlA[4] = {0.f, 0.f, 0.f, 0.f};
  float ShB[4] = {0.f, 0.f, 0.f, 0.f}, SlB[4] = {0.f, 0.f, 0.f, 0.f};
  float Sz[4] = {0.f, 0.f, 0.f, 0.f};
  const uint32_t ca = sa + lo.code, cb = sb + lo.code, ma = sa + lo.kmeta, mb = sb + lo.kmeta;
  uint32_t kwa[8], kwb[8];
  load_key_words<kBits>(ca, kwa);
  load_key_words<kBits>(cb, kwb);
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    load_key_words8<kBits>(ca, m, kwa);
    load_key_words8<kBits>(cb, m, kwb);
    // key scales and query words for k-tiles 2m, 2m+1 (four channel pairs)
    const uint4 sva = m == 0 ? lds128<0>(ma) : m == 1 ? lds128<16>(ma) : m == 2 ? lds128<32>(ma) : lds128<48>(ma);
    const uint4 svb = m == 0 ? lds128<0>(mb) : m == 1 ? lds128<16>(mb) : m == 2 ? lds128<32>(mb) : lds128<48>(mb);
    const uint4 qv = q.pair(m);
    const uint32_t ska[4] = {sva.x, sva.y, sva.z, sva.w}, skb[4] = {svb.x, svb.y, svb.z, svb.w};
    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int kt = 2 * m + h;
      qk_tile<kBits>(kwa, kt, ska[2 * h], ska[2 * h + 1], qw[2 * h], qw[2 * h + 1], ShA, SlA);
      qk_tile<kBits>(kwb, kt, skb[2 * h], skb[2 * h + 1], qw[2 * h], qw[2 * h + 1], ShB, SlB);
      // key zero points: A rows 0-7 are page A's zK, rows 8-15 page B's
      uint32_t z0, z1, z2, z3;
      ldmatrix_kzero(zrow, kt, z0, z1, z2, z3);
      mma16816(Sz, z0, z1, z2, z3, qw[2 * h], qw[2 * h + 1]);
    }
  }
  (void)F::kBlock;
  const float cs = code_unit_inv<kBits>();
  const float2 c2 = make_float2(cs, cs);
  const float2 za = make_float2(Sz[0], Sz[1]), zb = make_float2(Sz[2], Sz[3]);
  const float2 a01 = fma2(add2(make_float2(ShA[0], ShA[1]), make_float2(SlA[0], SlA[1])), c2, za);
  const float2 a23 = fma2(add2(make_float2(ShA[2], ShA[3]), make_float2(SlA[2], SlA[3])), c2, za);
  const float2 b01 = fma2(add2(make_float2(ShB[0], ShB[1]), make_float2(SlB[0], SlB[1])), c2, zb);
  const float2 b23 = fma2(add2(make_float2(ShB[2], ShB[3]), make_float2(SlB[2], SlB[3])), c2, zb);
  SA[0] = a01.x; SA[1] = a01.y; SA[2] = a23.x; SA[3] = a23.y;
  SB[0] = b01.x; SB[1] = b01.y; SB[2] = b23.x; SB[3] = b23.y;
}

// Move the softmax reference when a logit of the page pair passes it (for any
// lane of the warp): new reference = pair maximum + headroom, state rescaled.
// m0, m1: this lane's maxima of heads 2i, 2i+1.
__device__ __forceinline__ void softmax_reference(float m0, float m1, float scale_log2, Online &st) {
  // common case: no logit passes the reference (compared on the raw logits
  // against ref / scale, kept in thr), one vote and no shuffles
  if (!__any_sync(kFull, m0 > st.thr0 || m1 > st.thr1)) return;
  float pm0 = m0 * scale_log2, pm1 = m1 * scale_log2;
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    pm0 = fmaxf(pm0, __shfl_xor_sync(kFull, pm0, off));
    pm1 = fmaxf(pm1, __shfl_xor_sync(kFull, pm1, off));
  }
  const float r0 = -st.nref.x, r1 = -st.nref.y;
  const float n0 = pm0 > r0 ? pm0 + kHeadroom : r0;
  const float n1 = pm1 > r1 ? pm1 + kHeadroom : r1;
  const float2 a = make_float2(fast_exp2(r0 - n0), fast_exp2(r1 - n1));
  st.nref = make_float2(-n0, -n1);
  // largest raw logit whose weight stays <= 1 (rounded down: never above)
  st.thr0 = __fdiv_rd(n0, scale_log2);
  st.thr1 = __fdiv_rd(n1, scale_log2);
  st.l = mul2(st.l, a);
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const float2 o01 = mul2(make_float2(st.O[mt][0], st.O[mt][1]), a);
    const float2 o23 = mul2(make_float2(st.O[mt][2], st.O[mt][3]), a);
    st.O[mt][0] = o01.x;
    st.O[mt][1] = o01.y;
    st.O[mt][2] = o23.x;
    st.O[mt][3] = o23.y;
  }
  const float2 z01 = mul2(make_float2(st.Z[0], st.Z[1]), a);
  const float2 z23 = mul2(make_float2(st.Z[2], st.Z[3]), a);
  st.Z[0] = z01.x;
  st.Z[1] = z01.y;
  st.Z[2] = z23.x;
  st.Z[3] = z23.y;
}

// Weights of one page against the current reference: P^T fragments in the PV
// operand layout (head n; tokens 2i, 2i+1 and 2i+8, 2i+9) as fp16 hi (P[0],
// P[1]) and lo (P[2], P[3]) parts; their fp32 sum goes into l.
__device__ __forceinline__ void page_weights(const float (&S)[4], float scale_log2, Online &st, uint32_t (&P)[4]) {
  // exponents (S * scale - ref) for (heads 2i, 2i+1) of tokens n and n+8
  const float2 sc = make_float2(scale_log2, scale_log2);
  const float2 x01 = fma2(make_float2(S[0], S[1]), sc, st.nref);
  const float2 x23 = fma2(make_float2(S[2], S[3]), sc, st.nref);
  const float2 p01 = make_float2(fast_exp2(x01.x), fast_exp2(x01.y));
  const float2 p23 = make_float2(fast_exp2(x23.x), fast_exp2(x23.y));
  st.l = add2(st.l, add2(p01, p23));
  // P in fp16 hi + lo, rows = tokens, cols = heads; then transpose
  const __half2 h01 = __floats2half2_rn(p01.x, p01.y);
  const __half2 h23 = __floats2half2_rn(p23.x, p23.y);
  const float2 d01 = sub2(p01, __half22float2(h01));
  const float2 d23 = sub2(p23, __half22float2(h23));
  const __half2 l01 = __floats2half2_rn(d01.x, d01.y);
  const __half2 l23 = __floats2half2_rn(d23.x, d23.y);
  P[0] = movmatrix_trans(h2_as_u32(h01));
  P[1] = movmatrix_trans(h2_as_u32(h23));
  P[2] = movmatrix_trans(h2_as_u32(l01));
  P[3] = movmatrix_trans(h2_as_u32(l23));
}

// Online softmax of a page pair.
__device__ __forceinline__ void softmax_pair(const float (&SA)[4], const float (&SB)[4], float scale_log2, Online &st,
                                             uint32_t (&PA)[4], uint32_t (&PB)[4]) {
  const float m0 = fmaxf(fmaxf(SA[0], SA[2]), fmaxf(SB[0], SB[2]));
  const float m1 = fmaxf(fmaxf(SA[1], SA[3]), fmaxf(SB[1], SB[3]));
  softmax_reference(m0, m1, scale_log2, st);
  page_weights(SA, scale_log2, st, PA);
  page_weights(SB, scale_log2, st, PB);
}

// Online softmax of one page (the residual page).
__device__ __forceinline__ void softmax_page(const float (&S)[4], float scale_log2, Online &st, uint32_t (&P)[4]) {
  softmax_reference(fmaxf(S[0], S[2]), fmaxf(S[1], S[3]), scale_log2, st);
  page_weights(S, scale_log2, st, P);
}

// O += V^T P for the two M-tiles of value group G4 of one quantized page.
template <int kBits, int G4>
__device__ __forceinline__ void pv_group(uint32_t code, const uint32_t (&P)[4], uint32_t sv0w, uint32_t sv1w,
                                         uint32_t (&vws)[8], Online &st) {
  using F = Fmt<kBits>;
  if (kBits == 8) {  // M-tiles 2 G4, 2 G4 + 1 of this lane: one 16-byte chunk
    const uint4 cw = lds128<F::kVCode + 512 * G4>(code);
    vws[0] = cw.x; vws[1] = cw.y; vws[2] = cw.z; vws[3] = cw.w;
  }
  const __half2 sv0 = u32_as_h2(sv0w), sv1 = u32_as_h2(sv1w);
  // (P * sV) in fp16 hi + lo: P-hi * sV exactly as two halves, plus P-lo * sV
  const __half2 bh0 = __hmul2(u32_as_h2(P[0]), sv0);
  const __half2 bh1 = __hmul2(u32_as_h2(P[1]), sv1);
  const __half2 bl0 = __hfma2(u32_as_h2(P[2]), sv0, __hfma2(u32_as_h2(P[0]), sv0, __hneg2(bh0)));
  const __half2 bl1 = __hfma2(u32_as_h2(P[3]), sv1, __hfma2(u32_as_h2(P[1]), sv1, __hneg2(bh1)));
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int mt = 2 * G4 + j;
    uint32_t a0, a1, a2, a3;
    tile_fragment<kBits>(vws, mt, a0, a1, a2, a3);
    mma16816(st.O[mt], a0, a1, a2, a3, h2_as_u32(bh0), h2_as_u32(bh1));
    mma16816(st.O[mt], a0, a1, a2, a3, h2_as_u32(bl0), h2_as_u32(bl1));
  }
}

// O += V^T P for one quantized page at stage address s (O in code units:
// 2^-9 for 4-bit codes), Z += [zV rows] P.
template <int kBits>
__device__ __forceinline__ void pv_page(uint32_t s, const LaneOff &lo, const uint32_t (&P)[4], Online &st) {
  using F = Fmt<kBits>;
  const uint32_t code = s + lo.code;
  uint32_t vws[8];
  if (kBits == 4) {
    const uint4 vw0 = lds128<F::kVCode>(code), vw1 = lds128<F::kVCode + 512>(code);
    vws[0] = vw0.x; vws[1] = vw0.y; vws[2] = vw0.z; vws[3] = vw0.w;
    vws[4] = vw1.x; vws[5] = vw1.y; vws[6] = vw1.z; vws[7] = vw1.w;
  } else if (kBits == 2) {
    const uint4 vw0 = lds128<F::kVCode>(code);
    vws[0] = vw0.x; vws[1] = vw0.y; vws[2] = vw0.z; vws[3] = vw0.w;
  }
  // this lane's value scales: token pairs 2i (.x-.w: groups 0-3) and 2i + 8
  const uint32_t vsa = s + lo.vscale;
  const uint4 s0 = lds128<0>(vsa), s1 = lds128<16>(vsa);
  pv_group<kBits, 0>(code, P, s0.x, s1.x, vws, st);
  pv_group<kBits, 1>(code, P, s0.y, s1.y, vws, st);
  pv_group<kBits, 2>(code, P, s0.z, s1.z, vws, st);
  pv_group<kBits, 3>(code, P, s0.w, s1.w, vws, st);
  // value zero points: A row r carries group r % 4's zV (one ldmatrix), B = P
  uint32_t z0, z1, z2, z3;
  ldmatrix_x4<0>(s + lo.vzero, z0, z1, z2, z3);
  mma16816(st.Z, z0, z1, z2, z3, P[0], P[1]);
  mma16816(st.Z, z0, z1, z2, z3, P[2], P[3]);
}

// The partial last page, read straight from the fp16 residual (r rows valid).
__device__ __forceinline__ void residual_page(const __half *rk, const __half *rv, int r,
                                              const QFrag &q, int lane, float scale_log2,
                                              Online &st) {
  const int n = lane >> 2, i = lane & 3;
  uint32_t kn[16], kn8[16];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint4 u = make_uint4(0, 0, 0, 0), w = make_uint4(0, 0, 0, 0);
    if (n < r) u = reinterpret_cast<const uint4 *>(rk + n * kHeadDim + 32 * i)[k];
    if (n + 8 < r) w = reinterpret_cast<const uint4 *>(rk + (n + 8) * kHeadDim + 32 * i)[k];
    kn[4 * k] = u.x; kn[4 * k + 1] = u.y; kn[4 * k + 2] = u.z; kn[4 * k + 3] = u.w;
    kn8[4 * k] = w.x; kn8[4 * k + 1] = w.y; kn8[4 * k + 2] = w.z; kn8[4 * k + 3] = w.w;
  }
  float S[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint4 qv = q.pair(m);
    mma16816(S, kn[4 * m], kn8[4 * m], kn[4 * m + 1], kn8[4 * m + 1], qv.x, qv.y);
    mma16816(S, kn[4 * m + 2], kn8[4 * m + 2], kn[4 * m + 3], kn8[4 * m + 3], qv.z, qv.w);
  }
  if (n >= r) S[0] = S[1] = -INFINITY;
  if (n + 8 >= r) S[2] = S[3] = -INFINITY;
  uint32_t P[4];
  softmax_page(S, scale_log2, st, P);
  // V^T fragments: rows = channels 32g + 4n + {0..3}, k = tokens
  const int tok[4] = {2 * i, 2 * i + 1, 2 * i + 8, 2 * i + 9};
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint2 vv[4];
#pragma unroll
    for (int tk = 0; tk < 4; ++tk) {
      vv[tk] = make_uint2(0, 0);
      if (tok[tk] < r) vv[tk] = *reinterpret_cast<const uint2 *>(rv + tok[tk] * kHeadDim + 32 * g + 4 * n);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t x0 = j ? vv[0].y : vv[0].x, x1 = j ? vv[1].y : vv[1].x;
      const uint32_t x2 = j ? vv[2].y : vv[2].x, x3 = j ? vv[3].y : vv[3].x;
      const uint32_t a0 = __byte_perm(x0, x1, 0x5410), a1 = __byte_perm(x0, x1, 0x7632);
      const uint32_t a2 = __byte_perm(x2, x3, 0x5410), a3 = __byte_perm(x2, x3, 0x7632);
      mma16816(st.O[2 * g + j], a0, a1, a2, a3, P[0], P[1]);
      mma16816(st.O[2 * g + j], a0, a1, a2, a3, P[2], P[3]);
    }
  }
}

// Slot of worker w's partial for the segment starting at flattened page
// seg_start: a worker whose range starts inside the segment stored it as its
// first piece (slot 2w), the segment's first worker as its last (2w + 1)
// unless its range starts exactly at the segment.
__device__ __forceinline__ long long piece_slot(long long w, long long wf, long long seg_start, long long T,
                                                long long W) {
  return 2 * w + ((w == wf && w * T / W < seg_start) ? 1 : 0);
}

__device__ __forceinline__ void merge_pieces(const DecodeParams &p, long obase, int G, long long wf, long long wl,
                                          long long seg_start, long long T, long long W, int lane) {
  const int npieces = static_cast<int>(wl - wf + 1);
  float acc[8][4];
  float M[8], Ls[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    M[h] = -INFINITY;
    Ls[h] = 0.f;
    acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
  }
  // pass 1: maxima per head, pieces spread over lanes
  for (int k0 = 0; k0 < npieces; k0 += 32) {
    const int k = k0 + lane;
    if (k < npieces) {
      const long long sl = piece_slot(wf + k, wf, seg_start, T, W);
#pragma unroll
      for (int h = 0; h < 8; ++h)
        if (h < G) M[h] = fmaxf(M[h], __ldcg(p.part_ml + sl * 8 + h).x);
    }
  }
#pragma unroll
  for (int h = 0; h < 8; ++h)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M[h] = fmaxf(M[h], __shfl_xor_sync(kFull, M[h], off));
  // pass 2: weighted sums; each lane owns channels 4*lane..4*lane+3
#pragma unroll 2
  for (int k = 0; k < npieces; ++k) {
    const long long sl = piece_slot(wf + k, wf, seg_start, T, W);
    const float2 *ml = p.part_ml + sl * 8;
    const float4 *o = reinterpret_cast<const float4 *>(p.part + sl * 8 * kHeadDim) + lane;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      if (h < G) {
        const float2 m_l = __ldcg(ml + h);
        const float4 ov = __ldcg(o + h * (kHeadDim / 4));
        const float wt = fast_exp2(m_l.x - M[h]);
        Ls[h] += wt * m_l.y;
        acc[h][0] += wt * ov.x;
        acc[h][1] += wt * ov.y;
        acc[h][2] += wt * ov.z;
        acc[h][3] += wt * ov.w;
      }
    }
  }
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    if (h < G) {
      const float inv = 1.0f / Ls[h];
      const __half2 u = __floats2half2_rn(acc[h][0] * inv, acc[h][1] * inv);
      const __half2 v = __floats2half2_rn(acc[h][2] * inv, acc[h][3] * inv);
      *reinterpret_cast<uint2 *>(p.out + obase + h * kHeadDim + 4 * lane) = make_uint2(h2_as_u32(u), h2_as_u32(v));
    }
  }
}

// Append of one decode step (s4kv_append_decode) for (sequence b, kv head h)
// whose length after the append is L >= 1: the new token (row b of k_new /
// v_new) is position L - 1, row (L - 1) % 16 of the sequence's last page.
//  * If that row is not the page's last, one warp writes the token into the
//    residual (lane l: channels 4l .. 4l + 3).
//  * Otherwise the token completes the page, which is quantized from the
//    residual rows 0..14 plus the token by the whole CTA (quantize_page_cta,
//    the routine s4kv_append uses, so the bytes are the same).

__device__ __forceinline__ void residual_row_write(const DecodeParams &p, const FusedAppend &f, int b, int h, int L,
                                                   int lane) {
  const int H = p.num_kv_heads;
  const long rbase = (static_cast<long>(b) * H + h) * kPage * kHeadDim + 4 * lane;
  const long nbase = (static_cast<long>(b) * H + h) * kHeadDim + 4 * lane;
  const int r = (L - 1) % kPage;
  // the cache is written only by the step's append (the parameters carry it
  // read-only for the attention)
  __half *res_k = const_cast<__half *>(p.res_k), *res_v = const_cast<__half *>(p.res_v);
  *reinterpret_cast<uint2 *>(res_k + rbase + r * kHeadDim) = *reinterpret_cast<const uint2 *>(f.k_new + nbase);
  *reinterpret_cast<uint2 *>(res_v + rbase + r * kHeadDim) = *reinterpret_cast<const uint2 *>(f.v_new + nbase);
}

// One completed page (job = sequence, kv head, physical page) quantized by
// all threads of the CTA, with `scratch` (12 KB of shared memory) as staging.
template <int kBits, int kThreads>
__device__ __forceinline__ void cta_quantize_job(const DecodeParams &p, const FusedAppend &f, int4 job, uint8_t *scratch,
                                                 int tid) {
  const int b = job.x, h = job.y, phys = job.w;
  const int H = p.num_kv_heads;
  auto ks = reinterpret_cast<__half (*)[kHeadDim]>(scratch);
  auto vs = reinterpret_cast<__half (*)[kHeadDim]>(scratch + kPage * kHeadDim * 2);
  auto kc = reinterpret_cast<uint8_t (*)[kHeadDim]>(scratch + 2 * kPage * kHeadDim * 2);
  auto vc = reinterpret_cast<uint8_t (*)[kHeadDim]>(scratch + 2 * kPage * kHeadDim * 2 + kPage * kHeadDim);
  const long res_base = (static_cast<long>(b) * H + h) * kPage * kHeadDim;
  const long new_base = (static_cast<long>(b) * H + h) * kHeadDim;
  for (int ch = tid; ch < kPage * (kHeadDim / 8); ch += kThreads) {
    const int t = ch / (kHeadDim / 8), c8 = (ch % (kHeadDim / 8)) * 8;
    const __half *sk = t < kPage - 1 ? p.res_k + res_base + t * kHeadDim + c8 : f.k_new + new_base + c8;
    const __half *sv = t < kPage - 1 ? p.res_v + res_base + t * kHeadDim + c8 : f.v_new + new_base + c8;
    *reinterpret_cast<uint4 *>(&ks[t][c8]) = *reinterpret_cast<const uint4 *>(sk);
    *reinterpret_cast<uint4 *>(&vs[t][c8]) = *reinterpret_cast<const uint4 *>(sv);
  }
  __syncthreads();
  quantize_page_cta<kBits>(ks, vs, kc, vc,
                           const_cast<uint8_t *>(p.pool) + (static_cast<long>(phys) * H + h) * Fmt<kBits>::kBlock,
                    tid);
  __syncthreads();  // the scratch is reused by the next job
}

// The step's append grid: one 128-thread CTA per (sequence, kv head), as in
// s4kv_append, so that the pages completed in one step (all kv heads of a
// sequence complete together) are quantized side by side.  Warp 0 writes a
// row that completes nothing; the whole CTA quantizes a completed page.
constexpr int kStepThreads = 128;
constexpr int kQuantScratch = 2 * kPage * kHeadDim * 2 + 2 * kPage * kHeadDim;

template <int kBits>
__global__ void __launch_bounds__(kStepThreads) step_append_kernel(const DecodeParams p, const FusedAppend f) {
  // the dependent decode grid may start now: it plans its split while this
  // grid runs and waits for this grid's completion before it reads the cache
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ __align__(16) uint8_t scratch[kQuantScratch];
  const int H = p.num_kv_heads;
  const int b = static_cast<int>(blockIdx.x / H), h = static_cast<int>(blockIdx.x % H);
  const int L = __ldg(p.seq_lens + b);
  // no token (L == 0), or a length the decode grid flags as out of range
  if (L <= 0 || L > p.max_pages * kPage) return;
  if (L % kPage != 0) {
    if (threadIdx.x < 32) residual_row_write(p, f, b, h, L, threadIdx.x);
    return;
  }
  const int phys = __ldg(p.block_tables + static_cast<long>(b) * p.max_pages + (L - 1) / kPage);
  if (static_cast<unsigned>(phys) >= static_cast<unsigned>(p.num_pages)) {
    if (threadIdx.x == 0) flag_error(p.err, S4KV_EFLAG_PAGE_RANGE);
    return;
  }
  cta_quantize_job<kBits, kStepThreads>(p, f, make_int4(b, h, L, phys), scratch, threadIdx.x);
  // the pool writes are read next by the decode grid's bulk copies (async proxy)
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

template <int kBits>
__global__ void __launch_bounds__(threads_for<kBits>(), min_ctas_for<kBits>())
    decode_kernel(const DecodeParams p) {
  constexpr int kStages = stages_for<kBits>();
  constexpr int kWarpsPerCta = warps_for<kBits>();
  constexpr int kThreads = threads_for<kBits>();
  constexpr int kBlockBytes = Fmt<kBits>::kBlock;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = lane >> 2, i = lane & 3;
  const uint32_t ring0 = smem_addr(smem) + warp * kStages * kBlockBytes;
  const uint32_t bar0 = smem_addr(smem) + kWarpsPerCta * kStages * kBlockBytes + warp * kStages * 8;
  // worker ids run over the CTAs first, so that a launch with fewer workers
  // than warps spreads them over the SMs
  const long long worker = static_cast<long long>(warp) * gridDim.x + blockIdx.x;
  const int B = p.batch, H = p.num_kv_heads, G = p.group;
  const LaneOff lo = lane_offsets<kBits>(lane);

  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < kStages; ++st) mbar_init(bar0 + 8 * st, 1);
    fence_barrier_init();
  }
  __syncthreads();

  // ---- plan: pages per kv head of each lane's block of sequences, scanned
  const int per = (B + 31) >> 5;
  const int b_lo = min(B, lane * per), b_hi = min(B, b_lo + per);
  long long lsum = 0;
  bool bad_len = false;
  for (int b = b_lo; b < b_hi; ++b) {
    const int raw = __ldg(p.seq_lens + b);
    const int L = clamp_len(raw, p.max_pages);
    bad_len |= (L != raw);
    lsum += (L + kPage - 1) / kPage;
  }
  long long incl = lsum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const long long t = __shfl_up_sync(kFull, incl, off);
    if (lane >= off) incl += t;
  }
  const long long excl = incl - lsum;
  const long long total = __shfl_sync(kFull, incl, 31);
  const long long T = total * H;
  // workers: all resident warps, or fewer so that each gets at least
  // S4KV_DECODE_MIN_PAGES pages
  const long long W = max(1LL, min(static_cast<long long>(p.num_workers),
                                   (T + S4KV_DECODE_MIN_PAGES - 1) / S4KV_DECODE_MIN_PAGES));
  if (worker == 0) {
    if (__any_sync(kFull, bad_len) && lane == 0) flag_error(p.err, S4KV_EFLAG_SEQ_LEN);
    // sequences with no tokens get zeros
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      const bool empty = b < B && clamp_len(__ldg(p.seq_lens + b), p.max_pages) == 0;
      unsigned m = __ballot_sync(kFull, empty);
      while (m) {
        const int eb = b0 + __ffs(m) - 1;
        m &= m - 1;
        uint2 *o = reinterpret_cast<uint2 *>(p.out + static_cast<long>(eb) * p.num_q_heads * kHeadDim);
        for (int k = lane; k < p.num_q_heads * kHeadDim / 4; k += 32) o[k] = make_uint2(0, 0);
      }
    }
  }
  if (T == 0) return;
  const bool active = worker < W;
  const long long s = active ? worker * T / W : 0;
  const long long e = active ? (worker + 1) * T / W : 0;

  // ---- locate the segment holding page s
  const unsigned hit = __ballot_sync(kFull, H * excl <= s && s < H * incl);
  const int src = __ffs(hit) - 1;
  int bs = 0;
  long long pre = 0;
  if (lane == src) {
    long long acc = excl;
    for (int b = b_lo; b < b_hi; ++b) {
      const int np = (clamp_len(__ldg(p.seq_lens + b), p.max_pages) + kPage - 1) / kPage;
      if (s < H * (acc + np)) {
        bs = b;
        break;
      }
      acc += np;
    }
    pre = acc;
  }
  bs = __shfl_sync(kFull, bs, src);
  pre = __shfl_sync(kFull, pre, src);
  Cursor cc;
  set_seq(cc, p, bs, clamp_len(__ldg(p.seq_lens + bs), p.max_pages));
  cc.h = static_cast<int>((s - H * pre) / cc.np);
  cc.start = H * pre + static_cast<long long>(cc.h) * cc.np;
  const int range = static_cast<int>(e - s);
  const int p_first = static_cast<int>(s - cc.start);

  // s4kv_append_decode launches this grid as the programmatic dependent of
  // its append grid: everything above (the plan, the zeroed outputs) reads
  // nothing that grid writes, and here every thread waits for that grid's
  // completion and its writes before the cache is read.  Launched plainly
  // (no dependency), the wait returns at once.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (active) {
  // ---- producer: issue the next quantized pages of [s, e) into the ring.
  // It walks the same pieces as the consumer.  The page ids of a piece are
  // read 32 at a time into a window (lane l holds the l-th) with one
  // coalesced load, and taken with a shuffle, so no per-page global load
  // sits on the warp's critical path.
  const long long page_stride = static_cast<long long>(H) * kBlockBytes;
  Cursor pc = cc;
  int p_page = p_first;       // page index of the producer's current piece start
  int p_left = range;         // pages of [s, e) from the current piece on
  int p_q = 0;                // quantized pages left in the current piece
  const int32_t *p_bt = nullptr;
  const uint8_t *p_head = nullptr;
  int p_win = 0, p_widx = 0;  // window of page ids, next index into it
  int issued = 0;
  auto p_window = [&]() {     // the next (up to) 32 page ids of the piece
    p_win = lane < p_q ? __ldg(p_bt + lane) : 0;
    p_widx = 0;
  };
  auto p_piece = [&]() {      // set up the piece starting at p_page
    const int take = min(p_left, pc.np - p_page);
    p_q = max(0, min(p_page + take, pc.nfull) - p_page);
    p_bt = pc.bt + p_page;
    p_head = p.pool + static_cast<long long>(pc.h) * kBlockBytes;
    p_left -= take;
    p_window();
  };
  p_piece();
  // issue one copy into `stage` (barrier `bar`)
  auto produce = [&](uint32_t stage, uint32_t bar) {
    while (p_q == 0) {
      if (p_left == 0) return;
      next_segment(pc, p);
      p_page = 0;
      p_piece();
    }
    if (p_widx == 32) {
      p_bt += 32;
      p_window();
    }
    int phys = __shfl_sync(kFull, p_win, p_widx);
    ++p_widx;
    --p_q;
    if (static_cast<unsigned>(phys) >= static_cast<unsigned>(p.num_pages)) {
      if (lane == 0) flag_error(p.err, S4KV_EFLAG_PAGE_RANGE);
      phys = 0;
    }
    if (lane == 0) {
      mbar_arrive_expect_tx(bar, kBlockBytes);
      bulk_copy_g2s(ring0 + stage, p_head + phys * page_stride, kBlockBytes, bar);
    }
    ++issued;
  };
  // issue copies into two stages: lanes 0 and 1 take one each when both
  // pages are in the current window, otherwise one after the other
  auto produce2 = [&](uint32_t st_a, uint32_t bar_a, uint32_t st_b, uint32_t bar_b) {
    if (p_q >= 2 && p_widx <= 30) {
      int phys = __shfl_sync(kFull, p_win, p_widx + (lane & 1));
      p_widx += 2;
      p_q -= 2;
      const bool bad = static_cast<unsigned>(phys) >= static_cast<unsigned>(p.num_pages);
      if (bad) phys = 0;
      if (lane < 2) {
        if (bad) flag_error(p.err, S4KV_EFLAG_PAGE_RANGE);
        const uint32_t bar = lane ? bar_b : bar_a;
        mbar_arrive_expect_tx(bar, kBlockBytes);
        bulk_copy_g2s(ring0 + (lane ? st_b : st_a), p_head + phys * page_stride, kBlockBytes, bar);
      }
      issued += 2;
    } else {
      produce(st_a, bar_a);
      produce(st_b, bar_b);
    }
  };
  static_assert(kStages >= 5, "the pipeline holds four stages at once");
#pragma unroll 1
  for (int k = 0; k < kStages; ++k) produce(static_cast<uint32_t>(k) * kBlockBytes, bar0 + 8u * k);

  // ---- consumer.  A ring position: stage offset, barrier address, parity.
  struct Pos {
    uint32_t off, bar, phase;
  };
  auto next_pos = [&](Pos q) {
    const bool wrap = (q.off == (kStages - 1) * kBlockBytes);
    q.off = wrap ? 0u : q.off + kBlockBytes;
    q.bar = wrap ? bar0 : q.bar + 8;
    q.phase ^= wrap ? 1u : 0u;
    return q;
  };
  int consumed = 0;
  bool failed = false;
  Pos c0{0u, bar0, 0u};
  // wait for the copies of stages a and (when `two`) b: lane 1 watches b
  auto wait_pair = [&](const Pos &a, const Pos &b, bool two) {
    const bool mine_b = two && (lane & 1);
    const uint32_t bar = mine_b ? b.bar : a.bar, ph = mine_b ? b.phase : a.phase;
    if (__all_sync(kFull, mbar_try_wait(bar, ph))) return true;
    const bool ok = mbar_wait_bounded(bar, ph, kWaitLimitCycles);
    return !__any_sync(kFull, !ok);
  };
  // the key-zero row of this lane for the page pair (a, b)
  auto zero_row = [&](const Pos &a, const Pos &b) { return ring0 + ((lane & 8) ? b.off : a.off) + lo.kzero; };
  // the pages at c0 (and the next stage when `two`) have been read completely
  auto release = [&](bool two) {
    fence_proxy_async();
    __syncwarp();
    const Pos a = c0, b = next_pos(c0);
    if (two) {
      consumed += 2;
      c0 = next_pos(b);
      produce2(a.off, a.bar, b.off, b.bar);
    } else {
      ++consumed;
      c0 = b;
      produce(a.off, a.bar);
    }
  };

  int page = p_first, rem = range;
  bool first = true;
  while (rem > 0 && !failed) {
    if (page == cc.np) {
      next_segment(cc, p);
      page = 0;
    }
    const int take = min(rem, cc.np - page);
    const int p1 = page + take;
    const bool complete = (page == 0) && (p1 == cc.np);
    const int nq = max(0, min(p1, cc.nfull) - page);

    QFrag qf;
    {
      uint4 qv[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0),
                     make_uint4(0, 0, 0, 0)};
      if (n < G) {
        const uint4 *qp = reinterpret_cast<const uint4 *>(
            p.q + (static_cast<long>(cc.b) * p.num_q_heads + cc.h * G + n) * kHeadDim + 32 * i);
#pragma unroll
        for (int k = 0; k < 4; ++k) qv[k] = __ldg(qp + k);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        qf.w[4 * k] = qv[k].x; qf.w[4 * k + 1] = qv[k].y; qf.w[4 * k + 2] = qv[k].z; qf.w[4 * k + 3] = qv[k].w;
      }
    }
    Online st;
    st.nref = make_float2(INFINITY, INFINITY);
    st.thr0 = st.thr1 = -INFINITY;
    st.l = make_float2(0.f, 0.f);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) st.O[mt][0] = st.O[mt][1] = st.O[mt][2] = st.O[mt][3] = 0.f;
    st.Z[0] = st.Z[1] = st.Z[2] = st.Z[3] = 0.f;

    if (nq > 0) {
      // software pipeline over the piece's quantized pages, two at a time:
      // step k turns the logits of pair k into weights, issues the QK MMAs
      // of pair k+1 (independent of that softmax, so they hide its latency)
      // and then the PV MMAs of pair k.  A pair whose second page is missing
      // (odd count, last pair only) reads its first page twice and gives the
      // copy zero weight.
      float SA[4], SB[4];
      {
        const bool two = nq >= 2;
        const Pos cb = next_pos(c0);
        if (!wait_pair(c0, cb, two)) {
          failed = true;
          break;
        }
        const Pos pb = two ? cb : c0;
        qk_pair<kBits>(ring0 + c0.off, ring0 + pb.off, zero_row(c0, pb), lo, qf, SA, SB);
        if (!two) SB[0] = SB[1] = SB[2] = SB[3] = -INFINITY;
      }
      int done = 0;  // pages before the current pair
#pragma unroll 1
      while (done + 2 < nq) {
        const Pos cb = next_pos(c0), cn = next_pos(cb), cnb = next_pos(cn);
        const bool two = done + 3 < nq;
        if (!wait_pair(cn, cnb, two)) {
          failed = true;
          break;
        }
        uint32_t PA[4], PB[4];
        softmax_pair(SA, SB, p.scale_log2, st, PA, PB);
        const Pos pb = two ? cnb : cn;
        qk_pair<kBits>(ring0 + cn.off, ring0 + pb.off, zero_row(cn, pb), lo, qf, SA, SB);
        if (!two) SB[0] = SB[1] = SB[2] = SB[3] = -INFINITY;
        pv_page<kBits>(ring0 + c0.off, lo, PA, st);
        pv_page<kBits>(ring0 + cb.off, lo, PB, st);
        release(true);
        done += 2;
      }
      if (failed) break;
      // the last pair
      {
        const bool two = done + 1 < nq;
        uint32_t PA[4], PB[4];
        softmax_pair(SA, SB, p.scale_log2, st, PA, PB);
        pv_page<kBits>(ring0 + c0.off, lo, PA, st);
        if (two) pv_page<kBits>(ring0 + next_pos(c0).off, lo, PB, st);
        release(two);
      }
      // the code unit back to codes (4-bit codes entered as code * 2^-9)
      if (code_unit_inv<kBits>() != 1.0f) {
        const float2 cs = make_float2(code_unit_inv<kBits>(), code_unit_inv<kBits>());
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const float2 o01 = mul2(make_float2(st.O[mt][0], st.O[mt][1]), cs);
          const float2 o23 = mul2(make_float2(st.O[mt][2], st.O[mt][3]), cs);
          st.O[mt][0] = o01.x;
          st.O[mt][1] = o01.y;
          st.O[mt][2] = o23.x;
          st.O[mt][3] = o23.y;
        }
      }
    }
    if (p1 == cc.np && cc.np > cc.nfull) {
      const long rbase = (static_cast<long>(cc.b) * H + cc.h) * kPage * kHeadDim;
      residual_page(p.res_k + rbase, p.res_v + rbase, cc.len % kPage, qf, lane, p.scale_log2, st);
    }

    // ---- finish the piece
    float l0 = st.l.x, l1 = st.l.y;
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(kFull, l0, off);
      l1 += __shfl_xor_sync(kFull, l1, off);
    }
    float za[4], zb[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      za[g] = __shfl_sync(kFull, st.Z[0], 4 * g + i);
      zb[g] = __shfl_sync(kFull, st.Z[1], 4 * g + i);
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      st.O[mt][0] += za[mt >> 1];
      st.O[mt][2] += za[mt >> 1];
      st.O[mt][1] += zb[mt >> 1];
      st.O[mt][3] += zb[mt >> 1];
    }
    const long obase = (static_cast<long>(cc.b) * p.num_q_heads + cc.h * G) * kHeadDim;
    if (complete) {
      const float inv0 = 1.0f / l0, inv1 = 1.0f / l1;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int ch = 32 * g + 4 * n;
        if (2 * i < G) {
          const __half2 u = __floats2half2_rn(st.O[2 * g][0] * inv0, st.O[2 * g][2] * inv0);
          const __half2 v = __floats2half2_rn(st.O[2 * g + 1][0] * inv0, st.O[2 * g + 1][2] * inv0);
          *reinterpret_cast<uint2 *>(p.out + obase + (2 * i) * kHeadDim + ch) = make_uint2(h2_as_u32(u), h2_as_u32(v));
        }
        if (2 * i + 1 < G) {
          const __half2 u = __floats2half2_rn(st.O[2 * g][1] * inv1, st.O[2 * g][3] * inv1);
          const __half2 v = __floats2half2_rn(st.O[2 * g + 1][1] * inv1, st.O[2 * g + 1][3] * inv1);
          *reinterpret_cast<uint2 *>(p.out + obase + (2 * i + 1) * kHeadDim + ch) = make_uint2(h2_as_u32(u), h2_as_u32(v));
        }
      }
    } else {
      const long long slot = 2 * worker + (first ? 0 : 1);
      float *dst = p.part + slot * 8 * kHeadDim;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int ch = 32 * g + 4 * n;
        *reinterpret_cast<float4 *>(dst + (2 * i) * kHeadDim + ch) =
            make_float4(st.O[2 * g][0], st.O[2 * g][2], st.O[2 * g + 1][0], st.O[2 * g + 1][2]);
        *reinterpret_cast<float4 *>(dst + (2 * i + 1) * kHeadDim + ch) =
            make_float4(st.O[2 * g][1], st.O[2 * g][3], st.O[2 * g + 1][1], st.O[2 * g + 1][3]);
      }
      if (n == 0) {
        p.part_ml[slot * 8 + 2 * i] = make_float2(-st.nref.x, l0);
        p.part_ml[slot * 8 + 2 * i + 1] = make_float2(-st.nref.y, l1);
      }
      __threadfence();
      __syncwarp();
      const long long seg_end = cc.start + cc.np;
      const long long wf = worker_of(cc.start, T, W), wl = worker_of(seg_end - 1, T, W);
      uint32_t last = 0;
      if (lane == 0) {
        const uint32_t old = atomicAdd(p.tickets + static_cast<long>(cc.b) * H + cc.h, 1u);
        last = (old + 1 == static_cast<uint32_t>(wl - wf + 1));
      }
      last = __shfl_sync(kFull, last, 0);
      if (last) {
        // merge every piece of this (sequence, kv head): log-sum-exp.  Lanes
        // take pieces for (m, l) (warp reductions); for O each lane owns 4
        // channels of every head and loads the pieces independently.
        __threadfence();
        merge_pieces(p, obase, G, wf, wl, cc.start, T, W, lane);
        if (lane == 0) p.tickets[static_cast<long>(cc.b) * H + cc.h] = 0u;
      }
    }
    rem -= take;
    page = p1;
    first = false;
  }

  if (failed) {
    if (lane == 0) flag_error(p.err, S4KV_EFLAG_TIMEOUT);
    // wait (bounded) for the copies still in flight before the CTA exits
    for (int j = consumed; j < issued; ++j) {
      mbar_wait_bounded(c0.bar, c0.phase, kWaitLimitCycles);
      c0 = next_pos(c0);
    }
  }
  }  // active
}

// One CTA per SM by design for every code width: its ring takes more than
// half of an SM's shared memory, so no second CTA fits.
static_assert(2 * smem_bytes_for<4>() > 228 * 1024 && 2 * smem_bytes_for<8>() > 228 * 1024 &&
                  2 * smem_bytes_for<2>() > 228 * 1024,
              "one decode CTA per SM");

int decode_warps_per_cta(int bits) {
  return bits == 8 ? warps_for<8>() : bits == 2 ? warps_for<2>() : warps_for<4>();
}

template <int kBits>
cudaError_t prepare_for() {
  return cudaFuncSetAttribute(decode_kernel<kBits>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(smem_bytes_for<kBits>()));
}

template <int kBits>
cudaError_t launch_for(const DecodeParams &p, const FusedAppend &f, int num_ctas, cudaStream_t stream) {
  // the kernel's shared-memory allowance, set at every launch (the library
  // keeps no record of what it configured)
  cudaError_t pe = prepare_for<kBits>();
  if (pe != cudaSuccess) return pe;
  if (f.k_new == nullptr) {
    decode_kernel<kBits><<<num_ctas, threads_for<kBits>(), smem_bytes_for<kBits>(), stream>>>(p);
    return cudaGetLastError();
  }
  // one decode step: the append grid, then the decode grid as its
  // programmatic dependent (launched while the append runs; it waits for the
  // append's completion before reading the cache)
  step_append_kernel<kBits><<<static_cast<unsigned>(p.batch * p.num_kv_heads), kStepThreads, 0, stream>>>(p, f);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_ctas));
  cfg.blockDim = dim3(threads_for<kBits>());
  cfg.dynamicSmemBytes = smem_bytes_for<kBits>();
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<kBits>, p);
}

cudaError_t launch_decode(const DecodeParams &p, const FusedAppend &f, int bits, int num_ctas, cudaStream_t stream) {
  return bits == 8 ? launch_for<8>(p, f, num_ctas, stream)
                   : bits == 2 ? launch_for<2>(p, f, num_ctas, stream) : launch_for<4>(p, f, num_ctas, stream);
}

}  // namespace s4kv
