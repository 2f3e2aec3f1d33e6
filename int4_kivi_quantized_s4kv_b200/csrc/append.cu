// s4kv_append device side: write new tokens' fp16 K/V into the sequence's
// residual page, and quantize every page the call completes.
//
// KIVI split ("S4 KV -- int4 KV-Cache-Kompression fuer vLLM", "Funktionsweise"
// step 1): keys asymmetric int4 per channel (one group = one channel over the
// page's 16 tokens), values int4 per token (groups of 32 channels).  Pages are
// the 16-token blocks of "PagedAttention reduziert den KV-Cache-Speicherbedarf
// beim LLM-Serving erheblich" ("Wichtigste Kernpunkte & Evidenz"), addressed
// through block_tables.
//
// Grid: (page slot, sequence, kv head), 128 threads.  Slot s handles the
// s-th page the call touches for that (sequence, kv head).  A completed page
// is gathered into shared memory (earlier tokens from the residual, new ones
// from k/v), quantized and written as one 2816-byte block.  Slot 0 also owns
// the partial tail page: it writes the tail's new rows into the residual
// after its own page has read the residual rows it needed, so one call can
// complete a page and start the next one without a race.
#include "kernels.cuh"
#include "quant.cuh"

namespace s4kv {

__global__ void __launch_bounds__(128) append_kernel(const AppendParams p) {
  const int slot = blockIdx.x;
  const int b = blockIdx.y;
  const int h = blockIdx.z;
  const int tid = threadIdx.x;
  const int H = p.num_kv_heads;

  const int c0 = p.cu_new[b];
  const int n_b = p.cu_new[b + 1] - c0;
  if (n_b <= 0) return;
  const int L = p.seq_lens[b];
  const int L0 = L - n_b;
  if (L0 < 0 || n_b > p.max_new || (L + kPage - 1) / kPage > p.max_pages || c0 < 0 ||
      c0 + n_b > p.n_tokens) {
    if (slot == 0 && h == 0 && tid == 0) flag_error(p.err, S4KV_EFLAG_SEQ_LEN);
    return;
  }
  const int pf = L0 / kPage;        // first page touched
  const int pl = (L - 1) / kPage;   // last page touched
  const int pg = pf + slot;
  if (pg > pl) return;
  const bool full = (pg + 1) * kPage <= L;
  if (!full && slot != 0) return;   // the partial tail belongs to slot 0

  const long res_base = (static_cast<long>(b) * H + h) * kPage * kHeadDim;

  __shared__ __align__(16) __half ks[kPage][kHeadDim];
  __shared__ __align__(16) __half vs[kPage][kHeadDim];
  __shared__ uint8_t kc[kPage][kHeadDim];
  __shared__ uint8_t vc[kPage][kHeadDim];

  if (full) {
    const int phys = p.block_tables[static_cast<long>(b) * p.max_pages + pg];
    const bool phys_ok = phys >= 0 && phys < p.num_pages;
    // gather the page's 16 rows: residual rows for positions < L0, else k/v
    for (int ch = tid; ch < kPage * (kHeadDim / 8); ch += 128) {
      const int t = ch / (kHeadDim / 8);
      const int c8 = (ch % (kHeadDim / 8)) * 8;
      const int pos = pg * kPage + t;
      const __half *sk, *sv;
      if (pos < L0) {
        sk = p.res_k + res_base + t * kHeadDim + c8;
        sv = p.res_v + res_base + t * kHeadDim + c8;
      } else {
        const long tok = c0 + (pos - L0);
        sk = p.k + (tok * H + h) * kHeadDim + c8;
        sv = p.v + (tok * H + h) * kHeadDim + c8;
      }
      *reinterpret_cast<uint4 *>(&ks[t][c8]) = *reinterpret_cast<const uint4 *>(sk);
      *reinterpret_cast<uint4 *>(&vs[t][c8]) = *reinterpret_cast<const uint4 *>(sv);
    }
    if (tid < kPage && h == 0) {
      const int pos = pg * kPage + tid;
      if (pos >= L0 && phys_ok) {
        const long tok = c0 + (pos - L0);
        if (p.slot_mapping[tok] != static_cast<int64_t>(phys) * kPage + tid)
          flag_error(p.err, S4KV_EFLAG_SLOT);
      }
    }
    if (!phys_ok && tid == 0) flag_error(p.err, S4KV_EFLAG_PAGE_RANGE);
    __syncthreads();

    if (phys_ok) {
      if (p.bits == 8)
        quantize_page_cta<8>(ks, vs, kc, vc, p.pool + (static_cast<long>(phys) * H + h) * Fmt<8>::kBlock, tid);
      else if (p.bits == 2)
        quantize_page_cta<2>(ks, vs, kc, vc, p.pool + (static_cast<long>(phys) * H + h) * Fmt<2>::kBlock, tid);
      else
        quantize_page_cta<4>(ks, vs, kc, vc, p.pool + (static_cast<long>(phys) * H + h) * Fmt<4>::kBlock, tid);
    }
    if (slot != 0) return;
    __syncthreads();  // residual rows read above before the tail overwrites them
  }

  // slot 0: write the new rows of a partial tail page into the residual
  if (L % kPage != 0) {
    const int tail0 = max(L0, pl * kPage);
    const int rows = L - tail0;
    const int tphys = p.block_tables[static_cast<long>(b) * p.max_pages + pl];
    const bool tphys_ok = tphys >= 0 && tphys < p.num_pages;
    for (int ch = tid; ch < rows * (kHeadDim / 8); ch += 128) {
      const int rr = ch / (kHeadDim / 8);
      const int c8 = (ch % (kHeadDim / 8)) * 8;
      const int pos = tail0 + rr;
      const long tok = c0 + (pos - L0);
      const int row = pos % kPage;
      *reinterpret_cast<uint4 *>(p.res_k + res_base + row * kHeadDim + c8) =
          *reinterpret_cast<const uint4 *>(p.k + (tok * H + h) * kHeadDim + c8);
      *reinterpret_cast<uint4 *>(p.res_v + res_base + row * kHeadDim + c8) =
          *reinterpret_cast<const uint4 *>(p.v + (tok * H + h) * kHeadDim + c8);
    }
    if (h == 0 && tid < rows) {
      const int pos = tail0 + tid;
      const long tok = c0 + (pos - L0);
      if (!tphys_ok) {
        flag_error(p.err, S4KV_EFLAG_PAGE_RANGE);
      } else if (p.slot_mapping[tok] != static_cast<int64_t>(tphys) * kPage + pos % kPage) {
        flag_error(p.err, S4KV_EFLAG_SLOT);
      }
    }
  }
}

void launch_append(const AppendParams &p, int batch, int max_new, cudaStream_t stream) {
  // pages one sequence can touch: its partial first page plus the new tokens
  const int slots = (kPage - 1 + max_new + kPage - 1) / kPage;
  dim3 grid(slots, batch, p.num_kv_heads);
  append_kernel<<<grid, 128, 0, stream>>>(p);
}

}  // namespace s4kv
