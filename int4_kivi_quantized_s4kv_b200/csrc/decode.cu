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
//  * Staging.  Each warp owns a ring of shared-memory stages; lane 0 issues
//    one 1-D bulk copy (TMA engine, no multicast) of a whole 2816-byte page
//    block per stage, gathered through block_tables, completing on an
//    mbarrier.  Waits are bounded and report a timeout through err_flag.
//  * Math.  Per page (16 tokens) and kv head, with tokens on the MMA's M, the
//    G <= 8 query heads on N and channels on K:
//      S = codes_K . (q * sK) + zK . q              (3 m16n8k16 per k-tile)
//    and, with channels on M and tokens on K,
//      O += codes_V^T . (P * sV) + [zV rows] . P    (per M-tile, plus 2 for z)
//    The per-channel key scale and per-token value scale multiply the small
//    operand, so the 4-bit codes (exact in fp16) feed the tensor cores
//    directly; each scaled operand is split into fp16 hi + lo parts whose sum
//    is exact (q and sK, P-hi and sV are fp16, their product fits in two
//    halves), giving fp32-level accuracy.  The packed page layout makes each
//    lane's 32-bit code word its own operand fragment (one 16-byte shared
//    load per 4 tiles, 1 shift + 4 LOP3 + 4 fp16 ops to unpack 8 codes).
//    The softmax is the usual online update in the exp2 domain; P is moved
//    from the QK accumulator layout to the PV operand layout with movmatrix.
#include <cfloat>

#include "kernels.cuh"

namespace s4kv {

constexpr int kStages = 4;
constexpr int kWarpsPerCta = 4;
constexpr int kThreads = 32 * kWarpsPerCta;
constexpr long long kWaitLimitCycles = 2000000000LL;  // about one second
constexpr unsigned kFull = 0xFFFFFFFFu;

size_t decode_smem_bytes() {
  return static_cast<size_t>(kWarpsPerCta) * kStages * (kBlockBytes + 8);
}

struct Segment {
  long long start;  // flattened index of the segment's first page
  int b, h;
  int len;          // tokens of sequence b
  int np;           // pages of b (full pages + a partial residual page)
  int nfull;        // full (quantized) pages of b
};

__device__ __forceinline__ int clamp_len(int L, int max_pages) {
  return min(max(L, 0), max_pages * kPage);
}

__device__ __forceinline__ void set_seq(Segment &c, int len) {
  c.len = len;
  c.np = (len + kPage - 1) / kPage;
  c.nfull = len / kPage;
}

__device__ __forceinline__ void next_segment(Segment &c, const DecodeParams &p) {
  c.start += c.np;
  if (++c.h == p.num_kv_heads) {
    c.h = 0;
    int b = c.b + 1, L = 0;
    while (b < p.batch) {
      L = clamp_len(__ldg(p.seq_lens + b), p.max_pages);
      if (L > 0) break;
      ++b;
    }
    c.b = b;
    set_seq(c, b < p.batch ? L : 0);
  }
}

// Worker whose range [w*T/W, (w+1)*T/W) holds flattened page x (W <= T).
__device__ __forceinline__ long long worker_of(long long x, long long T, long long W) {
  return ((x + 1) * W + T - 1) / T - 1;
}

// Online-softmax update for one 16-token page.  S: this lane's logits
// (tokens n, n+8; heads 2i, 2i+1).  Produces P^T fragments (hi, lo) in the
// PV operand layout: head n, tokens 2i, 2i+1 (t0) and 2i+8, 2i+9 (t1).
__device__ __forceinline__ void softmax_page(const float (&S)[4], float scale_log2, float &m0,
                                             float &m1, float &l0, float &l1, float (&O)[8][4],
                                             float (&Z)[4], uint32_t &t0h, uint32_t &t1h,
                                             uint32_t &t0l, uint32_t &t1l) {
  const float s0 = S[0] * scale_log2, s1 = S[1] * scale_log2;
  const float s2 = S[2] * scale_log2, s3 = S[3] * scale_log2;
  float pm0 = fmaxf(s0, s2), pm1 = fmaxf(s1, s3);
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    pm0 = fmaxf(pm0, __shfl_xor_sync(kFull, pm0, off));
    pm1 = fmaxf(pm1, __shfl_xor_sync(kFull, pm1, off));
  }
  const float mn0 = fmaxf(m0, pm0), mn1 = fmaxf(m1, pm1);
  const float a0 = fast_exp2(m0 - mn0), a1 = fast_exp2(m1 - mn1);
  m0 = mn0;
  m1 = mn1;
  const float p0 = fast_exp2(s0 - mn0), p2 = fast_exp2(s2 - mn0);
  const float p1 = fast_exp2(s1 - mn1), p3 = fast_exp2(s3 - mn1);
  l0 = l0 * a0 + (p0 + p2);
  l1 = l1 * a1 + (p1 + p3);
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    O[mt][0] *= a0;
    O[mt][1] *= a1;
    O[mt][2] *= a0;
    O[mt][3] *= a1;
  }
  Z[0] *= a0;
  Z[1] *= a1;
  Z[2] *= a0;
  Z[3] *= a1;
  // P in fp16 hi + lo, rows = tokens, cols = heads; then transpose
  const __half2 h01 = __floats2half2_rn(p0, p1);
  const __half2 h23 = __floats2half2_rn(p2, p3);
  const float2 b01 = __half22float2(h01);
  const float2 b23 = __half22float2(h23);
  const __half2 l01 = __floats2half2_rn(p0 - b01.x, p1 - b01.y);
  const __half2 l23 = __floats2half2_rn(p2 - b23.x, p3 - b23.y);
  t0h = movmatrix_trans(h2_as_u32(h01));
  t1h = movmatrix_trans(h2_as_u32(h23));
  t0l = movmatrix_trans(h2_as_u32(l01));
  t1l = movmatrix_trans(h2_as_u32(l23));
}

// One quantized page from shared memory (stage at shared address `blk`).
__device__ __forceinline__ void page_step(uint32_t blk, const uint32_t (&qf)[16], int lane,
                                          float scale_log2, float &m0, float &m1, float &l0,
                                          float &l1, float (&O)[8][4], float (&Z)[4]) {
  const int n = lane >> 2, i = lane & 3;
  float S[4] = {0.f, 0.f, 0.f, 0.f};
  const uint4 kw0 = lds128(blk + kKCodeOff + 16 * lane);
  const uint4 kw1 = lds128(blk + kKCodeOff + 512 + 16 * lane);
  const uint32_t kws[8] = {kw0.x, kw0.y, kw0.z, kw0.w, kw1.x, kw1.y, kw1.z, kw1.w};
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const uint4 sa = lds128(blk + kKScaleOff + 64 * i + 32 * hf);
    const uint4 sb = lds128(blk + kKScaleOff + 64 * i + 32 * hf + 16);
    const uint4 za = lds128(blk + kKZeroOff + 64 * i + 32 * hf);
    const uint4 zb = lds128(blk + kKZeroOff + 64 * i + 32 * hf + 16);
    const uint32_t sk[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
    const uint32_t zk[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      const int kt = 4 * hf + q4;
      uint32_t a0, a1, a2, a3;
      unpack_codes(kws[kt], a0, a1, a2, a3);
      const __half2 qb0 = u32_as_h2(qf[2 * kt]), qb1 = u32_as_h2(qf[2 * kt + 1]);
      const __half2 s0 = u32_as_h2(sk[2 * q4]), s1 = u32_as_h2(sk[2 * q4 + 1]);
      const __half2 h0 = __hmul2(qb0, s0), h1 = __hmul2(qb1, s1);
      const __half2 r0 = __hfma2(qb0, s0, __hneg2(h0));
      const __half2 r1 = __hfma2(qb1, s1, __hneg2(h1));
      mma16816(S, a0, a1, a2, a3, h2_as_u32(h0), h2_as_u32(h1));
      mma16816(S, a0, a1, a2, a3, h2_as_u32(r0), h2_as_u32(r1));
      // key zero point: every A row is zK, so each row gets sum_c zK q
      mma16816(S, zk[2 * q4], zk[2 * q4], zk[2 * q4 + 1], zk[2 * q4 + 1], qf[2 * kt], qf[2 * kt + 1]);
    }
  }
  uint32_t t0h, t1h, t0l, t1l;
  softmax_page(S, scale_log2, m0, m1, l0, l1, O, Z, t0h, t1h, t0l, t1l);

  const uint4 vw0 = lds128(blk + kVCodeOff + 16 * lane);
  const uint4 vw1 = lds128(blk + kVCodeOff + 512 + 16 * lane);
  const uint32_t vws[8] = {vw0.x, vw0.y, vw0.z, vw0.w, vw1.x, vw1.y, vw1.z, vw1.w};
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const __half2 sv0 = u32_as_h2(lds32(blk + kVScaleOff + 32 * g + 4 * i));
    const __half2 sv1 = u32_as_h2(lds32(blk + kVScaleOff + 32 * g + 4 * i + 16));
    const __half2 bh0 = __hmul2(u32_as_h2(t0h), sv0);
    const __half2 bh1 = __hmul2(u32_as_h2(t1h), sv1);
    const __half2 bl0 = __hfma2(u32_as_h2(t0l), sv0, __hfma2(u32_as_h2(t0h), sv0, __hneg2(bh0)));
    const __half2 bl1 = __hfma2(u32_as_h2(t1l), sv1, __hfma2(u32_as_h2(t1h), sv1, __hneg2(bh1)));
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int mt = 2 * g + j;
      uint32_t a0, a1, a2, a3;
      unpack_codes(vws[mt], a0, a1, a2, a3);
      mma16816(O[mt], a0, a1, a2, a3, h2_as_u32(bh0), h2_as_u32(bh1));
      mma16816(O[mt], a0, a1, a2, a3, h2_as_u32(bl0), h2_as_u32(bl1));
    }
  }
  // value zero points: A row r carries group r % 4's zV, B = P
  const uint32_t zv0 = lds32(blk + kVZeroOff + 32 * (n & 3) + 4 * i);
  const uint32_t zv1 = lds32(blk + kVZeroOff + 32 * (n & 3) + 4 * i + 16);
  mma16816(Z, zv0, zv0, zv1, zv1, t0h, t1h);
  mma16816(Z, zv0, zv0, zv1, zv1, t0l, t1l);
}

// The partial last page, read straight from the fp16 residual (r rows valid).
__device__ __forceinline__ void residual_step(const __half *rk, const __half *rv, int r,
                                              const uint32_t (&qf)[16], int lane, float scale_log2,
                                              float &m0, float &m1, float &l0, float &l1,
                                              float (&O)[8][4], float (&Z)[4]) {
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
  for (int kt = 0; kt < 8; ++kt)
    mma16816(S, kn[2 * kt], kn8[2 * kt], kn[2 * kt + 1], kn8[2 * kt + 1], qf[2 * kt], qf[2 * kt + 1]);
  if (n >= r) S[0] = S[1] = -INFINITY;
  if (n + 8 >= r) S[2] = S[3] = -INFINITY;
  uint32_t t0h, t1h, t0l, t1l;
  softmax_page(S, scale_log2, m0, m1, l0, l1, O, Z, t0h, t1h, t0l, t1l);
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
      mma16816(O[2 * g + j], a0, a1, a2, a3, t0h, t1h);
      mma16816(O[2 * g + j], a0, a1, a2, a3, t0l, t1l);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 4) decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = lane >> 2, i = lane & 3;
  const uint32_t ring0 = smem_addr(smem) + warp * kStages * kBlockBytes;
  const uint32_t bar0 = smem_addr(smem) + kWarpsPerCta * kStages * kBlockBytes + warp * kStages * 8;
  const long long worker = static_cast<long long>(blockIdx.x) * kWarpsPerCta + warp;
  const int B = p.batch, H = p.num_kv_heads, G = p.group;

  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < kStages; ++st) mbar_init(bar0 + 8 * st, 1);
    fence_barrier_init();
  }
  __syncwarp();

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
  const long long W = max(1LL, min(static_cast<long long>(p.num_workers), T));
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
  if (worker >= W || T == 0) return;
  const long long s = worker * T / W, e = (worker + 1) * T / W;

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
  Segment cc;
  cc.b = bs;
  set_seq(cc, clamp_len(__ldg(p.seq_lens + bs), p.max_pages));
  cc.h = static_cast<int>((s - H * pre) / cc.np);
  cc.start = H * pre + static_cast<long long>(cc.h) * cc.np;

  // ---- producer: issue the next quantized page of [s, e) into the ring
  Segment pc = cc;
  long long px = s;
  int issued = 0;
  auto produce = [&]() {
    while (px < e) {
      if (px >= pc.start + pc.np) next_segment(pc, p);
      const int pp = static_cast<int>(px - pc.start);
      ++px;
      if (pp < pc.nfull) {
        int phys = __ldg(p.block_tables + static_cast<long>(pc.b) * p.max_pages + pp);
        if (phys < 0 || phys >= p.num_pages) {
          if (lane == 0) flag_error(p.err, S4KV_EFLAG_PAGE_RANGE);
          phys = 0;
        }
        const int st = issued % kStages;
        if (lane == 0) {
          mbar_arrive_expect_tx(bar0 + 8 * st, kBlockBytes);
          bulk_copy_g2s(ring0 + st * kBlockBytes,
                        p.pool + (static_cast<long>(phys) * H + pc.h) * kBlockBytes, kBlockBytes,
                        bar0 + 8 * st);
        }
        ++issued;
        return;
      }
    }
  };
#pragma unroll 1
  for (int k = 0; k < kStages; ++k) produce();

  // ---- consumer
  long long x = s;
  int consumed = 0;
  bool failed = false;
  while (x < e) {
    if (x >= cc.start + cc.np) next_segment(cc, p);
    const long long seg_end = cc.start + cc.np;
    const long long piece_end = min(e, seg_end);
    const bool complete = cc.start >= s && seg_end <= e;
    const bool first_piece = (x == s);

    uint32_t qf[16];
    if (n < G) {
      const uint4 *qp = reinterpret_cast<const uint4 *>(
          p.q + (static_cast<long>(cc.b) * p.num_q_heads + cc.h * G + n) * kHeadDim + 32 * i);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint4 v = __ldg(qp + k);
        qf[4 * k] = v.x; qf[4 * k + 1] = v.y; qf[4 * k + 2] = v.z; qf[4 * k + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) qf[k] = 0u;
    }
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float O[8][4], Z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) O[mt][0] = O[mt][1] = O[mt][2] = O[mt][3] = 0.f;

#pragma unroll 1
    for (; x < piece_end; ++x) {
      const int pp = static_cast<int>(x - cc.start);
      if (pp < cc.nfull) {
        const int st = consumed % kStages;
        const uint32_t par = (consumed / kStages) & 1;
        const bool ok = mbar_wait_bounded(bar0 + 8 * st, par, kWaitLimitCycles);
        if (__any_sync(kFull, !ok)) {
          failed = true;
          break;
        }
        page_step(ring0 + st * kBlockBytes, qf, lane, p.scale_log2, m0, m1, l0, l1, O, Z);
        fence_proxy_async();
        __syncwarp();
        ++consumed;
        produce();
      } else {
        const long rbase = (static_cast<long>(cc.b) * H + cc.h) * kPage * kHeadDim;
        residual_step(p.res_k + rbase, p.res_v + rbase, cc.len % kPage, qf, lane, p.scale_log2, m0,
                      m1, l0, l1, O, Z);
      }
    }
    if (failed) break;

    // ---- finish the piece
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(kFull, l0, off);
      l1 += __shfl_xor_sync(kFull, l1, off);
    }
    float za[4], zb[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      za[g] = __shfl_sync(kFull, Z[0], 4 * g + i);
      zb[g] = __shfl_sync(kFull, Z[1], 4 * g + i);
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      O[mt][0] += za[mt >> 1];
      O[mt][2] += za[mt >> 1];
      O[mt][1] += zb[mt >> 1];
      O[mt][3] += zb[mt >> 1];
    }
    const long obase = (static_cast<long>(cc.b) * p.num_q_heads + cc.h * G) * kHeadDim;
    if (complete) {
      const float inv0 = 1.0f / l0, inv1 = 1.0f / l1;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int ch = 32 * g + 4 * n;
        if (2 * i < G) {
          const __half2 u = __floats2half2_rn(O[2 * g][0] * inv0, O[2 * g][2] * inv0);
          const __half2 v = __floats2half2_rn(O[2 * g + 1][0] * inv0, O[2 * g + 1][2] * inv0);
          *reinterpret_cast<uint2 *>(p.out + obase + (2 * i) * kHeadDim + ch) = make_uint2(h2_as_u32(u), h2_as_u32(v));
        }
        if (2 * i + 1 < G) {
          const __half2 u = __floats2half2_rn(O[2 * g][1] * inv1, O[2 * g][3] * inv1);
          const __half2 v = __floats2half2_rn(O[2 * g + 1][1] * inv1, O[2 * g + 1][3] * inv1);
          *reinterpret_cast<uint2 *>(p.out + obase + (2 * i + 1) * kHeadDim + ch) = make_uint2(h2_as_u32(u), h2_as_u32(v));
        }
      }
    } else {
      const long long slot = 2 * worker + (first_piece ? 0 : 1);
      float *dst = p.part + slot * 8 * kHeadDim;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int ch = 32 * g + 4 * n;
        *reinterpret_cast<float4 *>(dst + (2 * i) * kHeadDim + ch) =
            make_float4(O[2 * g][0], O[2 * g][2], O[2 * g + 1][0], O[2 * g + 1][2]);
        *reinterpret_cast<float4 *>(dst + (2 * i + 1) * kHeadDim + ch) =
            make_float4(O[2 * g][1], O[2 * g][3], O[2 * g + 1][1], O[2 * g + 1][3]);
      }
      if (n == 0) {
        p.part_ml[slot * 8 + 2 * i] = make_float2(m0, l0);
        p.part_ml[slot * 8 + 2 * i + 1] = make_float2(m1, l1);
      }
      __threadfence();
      __syncwarp();
      const long long wf = worker_of(cc.start, T, W), wl = worker_of(seg_end - 1, T, W);
      uint32_t last = 0;
      if (lane == 0) {
        const uint32_t old = atomicAdd(p.tickets + static_cast<long>(cc.b) * H + cc.h, 1u);
        last = (old + 1 == static_cast<uint32_t>(wl - wf + 1));
      }
      last = __shfl_sync(kFull, last, 0);
      if (last) {
        __threadfence();
        for (int hh = 0; hh < G; ++hh) {
          float M = -INFINITY;
          for (long long w = wf; w <= wl; ++w) {
            const long long sl = 2 * w + ((w == wf && w * T / W < cc.start) ? 1 : 0);
            M = fmaxf(M, __ldcg(p.part_ml + sl * 8 + hh).x);
          }
          float Ls = 0.f;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          for (long long w = wf; w <= wl; ++w) {
            const long long sl = 2 * w + ((w == wf && w * T / W < cc.start) ? 1 : 0);
            const float2 ml = __ldcg(p.part_ml + sl * 8 + hh);
            const float wt = fast_exp2(ml.x - M);
            Ls += wt * ml.y;
            const float4 o = __ldcg(reinterpret_cast<const float4 *>(p.part + sl * 8 * kHeadDim + hh * kHeadDim) + lane);
            acc.x += wt * o.x;
            acc.y += wt * o.y;
            acc.z += wt * o.z;
            acc.w += wt * o.w;
          }
          const float inv = 1.0f / Ls;
          const __half2 u = __floats2half2_rn(acc.x * inv, acc.y * inv);
          const __half2 v = __floats2half2_rn(acc.z * inv, acc.w * inv);
          *reinterpret_cast<uint2 *>(p.out + obase + hh * kHeadDim + 4 * lane) = make_uint2(h2_as_u32(u), h2_as_u32(v));
        }
        if (lane == 0) p.tickets[static_cast<long>(cc.b) * H + cc.h] = 0u;
      }
    }
  }

  if (failed) {
    if (lane == 0) flag_error(p.err, S4KV_EFLAG_TIMEOUT);
    // wait (bounded) for the copies still in flight before the CTA exits
    for (int j = consumed; j < issued; ++j)
      mbar_wait_bounded(bar0 + 8 * (j % kStages), (j / kStages) & 1, kWaitLimitCycles);
  }
}

int decode_ctas_per_sm() {
  int n = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel, kThreads, decode_smem_bytes());
  return n;
}

int decode_warps_per_cta() { return kWarpsPerCta; }

cudaError_t prepare_decode_kernel() {
  return cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(decode_smem_bytes()));
}

void launch_decode(const DecodeParams &p, int num_ctas, cudaStream_t stream) {
  decode_kernel<<<num_ctas, kThreads, decode_smem_bytes(), stream>>>(p);
}

}  // namespace s4kv
