/*
 * s4kv -- int4 KIVI-quantized paged KV cache and GQA decode attention
 * for NVIDIA B200 (sm_100a).  Plain C ABI: no CUDA, PyTorch or C++ types
 * cross this boundary.  Device memory is passed as untyped pointers and
 * streams as `void *` holding a cudaStream_t (NULL = the legacy default
 * stream).
 *
 * What is computed (sources: web pages on the subject, cited by title and
 * section):
 *  - "S4 KV -- int4 KV-Cache-Kompression fuer vLLM" (intro, "Funktionsweise"
 *    step 1, "Lieferumfang"): the paged KV cache is held in int4, KIVI
 *    style -- keys asymmetric int4 per channel, values int4 per token;
 *    models with head_dim 128 only, refused at start-up otherwise.
 *  - "PagedAttention reduziert den KV-Cache-Speicherbedarf beim
 *    LLM-Serving erheblich" ("Wichtigste Kernpunkte & Evidenz") and
 *    "KV-Cache und PagedAttention: Warum Ihr LLM-Server langsamer wird"
 *    ("Wie PagedAttention das loest"): fixed 16-token pages addressed
 *    through per-sequence page tables, physical pages shareable between
 *    sequences (shared prefixes).
 *  - "KV-Cache-Optimierung -- PagedAttention, quantisierter KV, Speculative
 *    Cache" ("Begriffe auf dieser Seite", GQA): a group of query heads
 *    shares one K/V head.
 * The pages print no quantizer formula; this library defines it as: over
 * a group of fp16 values x, in IEEE fp32,
 *     mn = min x, mx = max x (IEEE total order: -0 below +0),
 *     s  = (mx - mn) / 15,
 *     code = (s == 0) ? 0 : clamp(rint((x - mn) / s), 0, 15),
 * with rint rounding half to even; stored scale = fp16_rne(s), stored zero
 * = fp16(mn) (exact); dequantized value = code * scale + zero in fp32.
 * Key groups: one channel over the 16 tokens of a page.  Value groups:
 * 32 consecutive channels of one token.  A page's keys and values are
 * quantized together when its 16th token is appended; until then the
 * page's tokens stay in an fp16 residual buffer of the sequence.
 *
 * Memory layout (all device memory is owned and allocated by the caller;
 * the library allocates nothing and keeps no per-cache state):
 *  pool     uint8 [num_pages][num_kv_heads][S4KV_BLOCK_BYTES], 128-byte
 *           aligned.  One block per (physical page, kv head):
 *             [   0,1024) key codes   : 256 little-endian 32-bit words
 *             [1024,2048) value codes : 256 little-endian 32-bit words
 *             [2048,2304) key scale   : fp16 [128 channels]
 *             [2304,2560) key zero    : fp16 [8 k-tiles][16 k-slots]:
 *                                       channel c at k-tile (c%32)/4, slot
 *                                       2*(c/32) + (c%2) + 8*((c%4)/2)
 *             [2560,2688) value scale : fp16 [4 groups][16 tokens]
 *             [2688,2816) value zero  : fp16 [4 groups][16 tokens]
 *           Code word w = 128*h + 4*lane + q, lane = 4*n + i (n < 8,
 *           i < 4, q < 4); nibble j (bits 4j..4j+3) of the word holds
 *             keys  : token 8*(j&1) + n,
 *                     channel 32*i + 4*(4*h+q) + 2*((j>>1)&1) + (j>>2)
 *             values: token 2*i + (j>>2) + 8*((j>>1)&1),
 *                     channel 32*((4*h+q)>>1) + 4*n + 2*((4*h+q)&1) + (j&1)
 *           (each 32-bit word is one lane's tensor-core operand fragment,
 *           and the key zero points follow the same k order, so one
 *           ldmatrix row is a lane quad's k columns; s4kv_dequant_page
 *           returns the natural [token][channel] order).
 *           With 8-bit codes (s4kv_cache_t.bits == 8, the INT8 variant of the
 *           same KIVI split: 255 levels, s = (mx - mn) / 255, codes clamped
 *           to [0, 255]) the block is S4KV_BLOCK_BYTES_INT8 = 4864 bytes:
 *             [   0,2048) key codes, [2048,4096) value codes, then the
 *             same fp16 metadata at [4096,4864) in the order above.
 *           A code keeps the 4-bit layout's place in the operand fragments,
 *           with bytes for nibbles: the 8 codes of tile 4*h+q of lane l are
 *           bytes ((32*m + l)*16 + 8*(tile%2) + 2*(j&3) + (j>>2)), m =
 *           tile/2, j the 4-bit nibble index of that (token, channel).
 *           With 2-bit codes (bits == 2, 3 levels: s = (mx - mn) / 3, codes
 *           clamped to [0, 3]) the block is S4KV_BLOCK_BYTES_INT2 = 1792
 *           bytes: [0,512) key codes, [512,1024) value codes, metadata at
 *           [1024,1792).  The 16 codes of tiles 2m, 2m+1 of lane l are the
 *           32-bit word 4*l + m: code (register r = j&3, half j>>2) of tile
 *           2m+p at bit 16*(j>>2) + 2*(4*p + r).
 *  res_k,   fp16 [max_seqs][num_kv_heads][16][128] each.  Row r of batch
 *  res_v    row b holds token 16*floor(L/16) + r of that sequence for
 *           r < L mod 16 (L = its current length); other rows are
 *           unspecified.
 *  err_flag one uint32 word (may be NULL).  Kernels OR S4KV_EFLAG_* bits
 *           into it instead of faulting; read it with s4kv_get_error.
 *
 * Calls are asynchronous on the given stream, do no host<->device copies
 * (except s4kv_get_error) and validate every host-visible argument before
 * launching anything: an invalid call returns a status and launches
 * nothing.  Device-side inconsistencies (page ids out of range, a
 * slot_mapping that disagrees with block_tables) set err_flag bits and the
 * offending element is skipped or clamped; no kernel traps or faults on
 * purpose.  Distinct caches may be used from different host threads.
 */
#ifndef S4KV_H
#define S4KV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define S4KV_API __attribute__((visibility("default")))
#else
#define S4KV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define S4KV_VERSION 3
#define S4KV_HEAD_DIM 128
#define S4KV_PAGE_TOKENS 16
#define S4KV_VALUE_GROUP 32
#define S4KV_BLOCK_BYTES 2816      /* 4-bit codes */
#define S4KV_BLOCK_BYTES_INT8 4864 /* 8-bit codes */
#define S4KV_BLOCK_BYTES_INT2 1792 /* 2-bit codes */
#define S4KV_MAX_GQA_GROUP 8

/* status codes returned by every call */
#define S4KV_OK 0
#define S4KV_ERR_INVALID_ARG 1  /* NULL pointer, bad size, misalignment */
#define S4KV_ERR_UNSUPPORTED 2  /* head_dim != 128, page != 16, group > 8 */
#define S4KV_ERR_CUDA 3         /* a CUDA runtime call failed */
#define S4KV_ERR_DEVICE_CHECK 4 /* s4kv_get_error found err_flag bits */
#define S4KV_ERR_WORKSPACE 5    /* workspace NULL or smaller than required */

/* err_flag bits (device side) */
#define S4KV_EFLAG_PAGE_RANGE 1u /* a block_tables entry outside [0, num_pages) */
#define S4KV_EFLAG_SLOT 2u       /* slot_mapping != block_tables[b][pos/16]*16 + pos%16 */
#define S4KV_EFLAG_SEQ_LEN 4u    /* seq_lens / cu_new inconsistent with the call */
#define S4KV_EFLAG_TIMEOUT 8u    /* a bounded pipeline wait gave up */

/* Caller-owned description of one layer's cache.  Plain data; the library
 * never frees or retains it. */
typedef struct s4kv_cache {
    void *pool;         /* device, see layout above */
    void *res_k;        /* device, fp16 */
    void *res_v;        /* device, fp16 */
    uint32_t *err_flag; /* device, optional */
    int32_t num_pages;
    int32_t num_kv_heads;
    int32_t max_seqs;
    int32_t head_dim;    /* must be S4KV_HEAD_DIM */
    int32_t page_tokens; /* must be S4KV_PAGE_TOKENS */
    int32_t bits;        /* code width: 4 (or 0, meaning 4), 8 or 2 */
} s4kv_cache_t;

/* Library version (S4KV_VERSION). */
S4KV_API int s4kv_version(void);

/* Human-readable text of a status code (static storage). */
S4KV_API const char *s4kv_status_string(int status);

/* Fail-fast model check ("S4 KV", "Lieferumfang": unsupported models are
 * refused at start-up): OK for head_dim 128, 16-token pages and
 * num_q_heads = G * num_kv_heads with 1 <= G <= 8; S4KV_ERR_UNSUPPORTED
 * otherwise; S4KV_ERR_INVALID_ARG for non-positive sizes. Host only. */
S4KV_API int s4kv_check_model(int head_dim, int page_tokens, int num_q_heads,
                     int num_kv_heads);

/* Bytes the caller must allocate for a cache of num_pages physical pages
 * ("KV-Cache-Quantisierung: Kapazitaet und Qualitaetspruefung", "Gewichte,
 * laufenden Zustand und reservierten Speicher trennen": the payload
 * formula 2 x kv_heads x head_dim x tokens x bytes, here with int4 codes
 * plus scale/zero metadata).  Host only; either output may be NULL. */
S4KV_API int s4kv_cache_layout(int num_pages, int num_kv_heads, int max_seqs,
                      size_t *pool_bytes, size_t *residual_bytes);

/* The same for a code width of `bits` (2, 4 or 8; pages then take
 * S4KV_BLOCK_BYTES_INT2 / S4KV_BLOCK_BYTES / S4KV_BLOCK_BYTES_INT8 bytes per
 * kv head). */
S4KV_API int s4kv_cache_layout_bits(int num_pages, int num_kv_heads, int max_seqs, int bits,
                                    size_t *pool_bytes, size_t *residual_bytes);

/* Append new tokens' K/V and quantize every page they complete: keys per
 * channel and values per token, asymmetric ("S4 KV -- int4
 * KV-Cache-Kompression fuer vLLM", "Funktionsweise" step 1), into 16-token
 * pages reached through block_tables ("PagedAttention reduziert den
 * KV-Cache-Speicherbedarf beim LLM-Serving erheblich", "Wichtigste
 * Kernpunkte & Evidenz").
 *  k, v          device fp16 [n_tokens][num_kv_heads][128], 16-B aligned,
 *                sequence b's new tokens at rows cu_new[b]..cu_new[b+1]-1
 *                in position order.
 *  slot_mapping  device int64 [n_tokens]: block_tables[b][pos/16]*16 +
 *                pos%16 for each new token (checked; mismatch -> flag).
 *  cu_new        device int32 [batch+1], cu_new[0] = 0, nondecreasing,
 *                cu_new[batch] = n_tokens.
 *  seq_lens      device int32 [batch]: lengths AFTER the append.
 *  block_tables  device int32 [batch][max_pages_per_seq].
 *  max_new_per_seq  host bound on any sequence's new-token count (sizes
 *                the launch; a larger count sets S4KV_EFLAG_SEQ_LEN).
 * The residual rows a page needs are read before any are overwritten, so a
 * single call may both complete a page and start the next one.  Full pages
 * are written once; pages not completed by this call are not touched (a
 * shared-prefix page is never rewritten).  Re-running an identical call is
 * idempotent. */
S4KV_API int s4kv_append(const s4kv_cache_t *cache, const void *k, const void *v,
                int n_tokens, const int64_t *slot_mapping,
                const int32_t *cu_new, const int32_t *seq_lens,
                const int32_t *block_tables, int batch,
                int max_pages_per_seq, int max_new_per_seq, void *stream);

/* Bytes of device workspace s4kv_decode_attention needs on the CURRENT
 * device for this batch and kv head count.  The workspace must be
 * zero-filled once after allocation; every completed decode call leaves
 * its counters at zero again.  A workspace sized for a batch serves every
 * smaller batch too (its per-sequence counters come last).  After a call
 * that set S4KV_EFLAG_TIMEOUT some counters may be left nonzero: zero-fill
 * the workspace again before reusing it.  Needs a CUDA device
 * (S4KV_ERR_CUDA if none). */
S4KV_API int s4kv_decode_workspace_size(int batch, int num_kv_heads, size_t *bytes);

/* GQA paged decode attention over the quantized pages plus the residual
 * (a group of query heads shares one kv head: "KV-Cache-Optimierung --
 * PagedAttention, quantisierter KV, Speculative Cache", "Begriffe auf dieser
 * Seite"; keys and values of full pages are the dequantized int4 codes of
 * "S4 KV -- int4 KV-Cache-Kompression fuer vLLM", "Funktionsweise" step 1).
 *  q       device fp16 [batch][num_q_heads][128], 16-B aligned; query head
 *          j reads kv head j / (num_q_heads / num_kv_heads).
 *  seq_lens, block_tables as for s4kv_append (lengths including the tokens
 *          already appended for this step).
 *  sm_scale  logit scale (1/sqrt(128) for standard attention).
 *  out     device fp16 [batch][num_q_heads][128], 8-B aligned:
 *          softmax(sm_scale * q.K^T) V over the sequence's tokens, with
 *          dequantized full pages and fp16 residual rows; a sequence of
 *          length 0 gets zeros.
 *  workspace  device, >= s4kv_decode_workspace_size bytes, 16-B aligned.
 * Work is split along the KV sequence over all SMs; the last split of a
 * (sequence, kv head) to finish merges the partial results (log-sum-exp).
 * Calls sharing one workspace must not overlap on the device. */
S4KV_API int s4kv_decode_attention(const s4kv_cache_t *cache, const void *q,
                          int num_q_heads, const int32_t *seq_lens,
                          const int32_t *block_tables, int batch,
                          int max_pages_per_seq, float sm_scale, void *out,
                          void *workspace, size_t workspace_bytes,
                          void *stream);

/* One decode step in one call: the append of one new token per sequence
 * (row (L-1) % 16 of the last page; a page completed by it is quantized), then
 * s4kv_decode_attention over the grown cache.  The append runs as its own
 * grid and the decode grid is launched as its programmatic dependent: the
 * decode grid's launch and split plan overlap the append, and it reads the
 * cache only after the append grid has completed.
 *  k_new, v_new  device fp16 [batch][num_kv_heads][128], 16-B aligned: the
 *          token of sequence b at position seq_lens[b] - 1.  A sequence with
 *          seq_lens[b] == 0 has no token and gets zeros.
 *  seq_lens  lengths AFTER the append (each sequence grows by exactly one).
 *  All other arguments, the output and the workspace: as
 *  s4kv_decode_attention.  The cache afterwards is byte-identical to what
 *  s4kv_append with the same tokens writes, and the output is that of
 *  s4kv_decode_attention after it. */
S4KV_API int s4kv_append_decode(const s4kv_cache_t *cache, const void *k_new, const void *v_new,
                                const void *q, int num_q_heads, const int32_t *seq_lens,
                                const int32_t *block_tables, int batch, int max_pages_per_seq,
                                float sm_scale, void *out, void *workspace, size_t workspace_bytes,
                                void *stream);

/* Size of the fixed scratch array behind s4kv_decode_attention_noalloc. */
#define S4KV_NOALLOC_SCRATCH_BYTES (24u * 1024u * 1024u)

/* Decode attention that allocates nothing and takes no workspace.  The source
 * pages have no counterpart to this call: it exists for callers that cannot
 * call cudaMalloc, such as a plugin inside a host engine that owns the
 * device's whole memory pool, or a latency-critical path that cannot afford
 * cudaMalloc's implicit device-wide synchronisation.
 *  Arguments and result: as s4kv_decode_attention, without the workspace.
 *  Scratch: one device array of S4KV_NOALLOC_SCRATCH_BYTES (24 MiB) inside
 *          the library; every GPU that loads the library holds it until the
 *          process exits.  A batch whose decode workspace
 *          (s4kv_decode_workspace_size) would exceed it is rejected with
 *          S4KV_ERR_WORKSPACE and nothing is launched.
 *  Set-up: the first call on a device looks up the array's device address
 *          (make that first call before any stream capture).
 *  Sharing: each call clears, on `stream`, the part of the array that must
 *          start at zero; all calls on a device share the array and it keeps
 *          the last call's contents, so calls whose kernels overlap on the
 *          GPU race.
 * No cudaMalloc, cudaFree or other allocating routine is called. */
S4KV_API int s4kv_decode_attention_noalloc(const s4kv_cache_t *cache, const void *q,
                                           int num_q_heads, const int32_t *seq_lens,
                                           const int32_t *block_tables, int batch,
                                           int max_pages_per_seq, float sm_scale,
                                           void *out, void *stream);

/* Causal attention of a chunk of new query tokens over the cache (the
 * prefill / chunked-append side of the same paged int4 cache; GQA map of
 * "KV-Cache-Optimierung -- PagedAttention, quantisierter KV, Speculative
 * Cache", "Begriffe auf dieser Seite"; dequantization of "S4 KV -- int4
 * KV-Cache-Kompression fuer vLLM", "Funktionsweise" step 1).  Call it after
 * s4kv_append has written the chunk (same cu_new, seq_lens, block_tables).
 *  q       device fp16 [n_tokens][num_q_heads][128], 16-B aligned, token
 *          major like the appended k and v: sequence b owns rows
 *          cu_new[b] .. cu_new[b+1]-1.
 *  cu_new, seq_lens (lengths AFTER the append), block_tables: as for
 *          s4kv_append; n = cu_new[b+1] - cu_new[b] must not exceed
 *          seq_lens[b] (else S4KV_EFLAG_SEQ_LEN and the sequence is skipped).
 *  max_new_per_seq  host bound on any n (sizes the launch; rows beyond it
 *          are not computed).
 *  out     device fp16 [n_tokens][num_q_heads][128], 16-B aligned: row j of
 *          sequence b (position L - n + j) gets softmax(sm_scale * q.K^T) V
 *          over the cache's tokens 0 .. L - n + j; rows of no sequence are
 *          left untouched.
 *  workspace, workspace_bytes  device scratch owned by the caller, 16-B
 *          aligned, at least s4kv_prefill_workspace_size(num_kv_heads, batch,
 *          max_pages_per_seq) bytes (else S4KV_ERR_WORKSPACE and nothing is
 *          launched).  Its contents are overwritten and mean nothing after the
 *          call; it must not be shared with work that runs concurrently.
 * Two launches on `stream`: the first dequantizes every 128-key tile of each
 * (sequence, kv head) once into the workspace as MMA operands (keys as an
 * fp16 hi part plus the e5m2 rounding of the remainder, which carries them
 * to about 2^-14 relative; values correctly rounded to fp16); the second runs
 * the attention on the tcgen05 tensor cores with those operands and the fp16
 * softmax weights (fp32 accumulation), so results agree with exact attention
 * to about fp16 precision of the values and the weights.  Allocates nothing;
 * the attention launch needs about 178 KB of shared memory per CTA.  Any code width of
 * the cache (4, 8 or 2 bits): only the first launch reads the codes. */
S4KV_API int s4kv_prefill_attention(const s4kv_cache_t *cache, const void *q,
                                    int num_q_heads, int n_tokens,
                                    const int32_t *cu_new, const int32_t *seq_lens,
                                    const int32_t *block_tables, int batch,
                                    int max_pages_per_seq, int max_new_per_seq,
                                    float sm_scale, void *out, void *workspace,
                                    size_t workspace_bytes, void *stream);

/* Bytes of workspace s4kv_prefill_attention needs: 80 KB per 128-key tile
 * of max_pages_per_seq pages (rounded up to whole tiles of 8 pages), per
 * sequence slot and kv head.  S4KV_ERR_INVALID_ARG for non-positive sizes or a total above
 * 2^40 bytes. */
S4KV_API int s4kv_prefill_workspace_size(int num_kv_heads, int batch, int max_pages_per_seq,
                                         size_t *bytes);

/* Dequantize one physical page for all kv heads into natural order (the
 * inverse of the KIVI step of "S4 KV -- int4 KV-Cache-Kompression fuer
 * vLLM", "Funktionsweise" step 1, on one 16-token page of "PagedAttention
 * reduziert den KV-Cache-Speicherbedarf beim LLM-Serving erheblich",
 * "Wichtigste Kernpunkte & Evidenz"):
 * out_k, out_v device [num_kv_heads][16][128], fp32 if out_fp32 != 0
 * (x = code*scale + zero, exact product, one rounding) else fp16 (the fp32
 * value rounded to nearest even).  16-B aligned. */
S4KV_API int s4kv_dequant_page(const s4kv_cache_t *cache, int physical_page,
                      void *out_k, void *out_v, int out_fp32, void *stream);

/* Dequantize a list of physical pages at once: pages is a device int32
 * [n] list (n <= 65535); page i goes to out_k / out_v slot i, each
 * [n][num_kv_heads][16][128] in the format of s4kv_dequant_page.  A page id
 * outside the pool sets S4KV_EFLAG_PAGE_RANGE and its slot is left as is. */
S4KV_API int s4kv_dequant_pages(const s4kv_cache_t *cache, const int32_t *pages, int n,
                                void *out_k, void *out_v, int out_fp32, void *stream);

/* ---- page movement: swap-out / swap-in and copy-on-write fork.  A paged
 * cache allocates pages on demand, lets sequences share them through their
 * page tables and copies a page only when it is written ("KV-Cache und
 * PagedAttention: Warum Ihr LLM-Server langsamer wird", "Wie PagedAttention
 * das loest").  A page RECORD is all kv heads' blocks of one physical page:
 * num_kv_heads * block bytes (1792 / 2816 / 4864 with 2- / 4- / 8-bit codes)
 * contiguous bytes, the unit these calls move.  All page
 * and row lists are device int32 arrays; an id out of range sets
 * S4KV_EFLAG_PAGE_RANGE (rows: S4KV_EFLAG_SLOT) and that item is skipped.
 * Every call is asynchronous on `stream`. */

/* Bytes of one page record of this cache (num_kv_heads * block bytes). */
S4KV_API int s4kv_page_record_bytes(const s4kv_cache_t *cache, size_t *bytes);

/* dst (device, 16-B aligned, [n][page record]) slot i = page record
 * pages[i]. */
S4KV_API int s4kv_gather_pages(const s4kv_cache_t *cache, const int32_t *pages, int n,
                               void *dst, void *stream);

/* Page record pages[i] = src slot i (src: device, 16-B aligned).  The pages
 * must be distinct. */
S4KV_API int s4kv_scatter_pages(const s4kv_cache_t *cache, const int32_t *pages, int n,
                                const void *src, void *stream);

/* Page record dst_pages[i] = page record src_pages[i], inside the pool (the
 * copy-on-write copy of a shared full page).  No dst page may appear among
 * the src pages or twice among the dst pages. */
S4KV_API int s4kv_copy_pages(const s4kv_cache_t *cache, const int32_t *src_pages,
                             const int32_t *dst_pages, int n, void *stream);

/* Residual rows (the fp16 keys and values of the partial last page, all kv
 * heads) of batch row src_rows[i] copied to batch row dst_rows[i]: the fork
 * of a sequence whose last page is shared and partial.  The full pages are
 * shared by pointing the new row's page table at them; the next page the
 * fork fills must be a page of its own.  No dst row may be a src row. */
S4KV_API int s4kv_fork_residual(const s4kv_cache_t *cache, const int32_t *src_rows,
                                const int32_t *dst_rows, int n, void *stream);

/* Swap-out: s4kv_gather_pages into `staging` (device, n records), then one
 * device-to-host copy of the n records into host_dst (page-locked host
 * memory for an asynchronous copy). */
S4KV_API int s4kv_swap_out(const s4kv_cache_t *cache, const int32_t *pages, int n,
                           void *staging, void *host_dst, void *stream);

/* Swap-in: one host-to-device copy of n records from host_src into
 * `staging`, then s4kv_scatter_pages into `pages` (any free pages: the
 * caller points the sequence's page table at them). */
S4KV_API int s4kv_swap_in(const s4kv_cache_t *cache, const int32_t *pages, int n,
                          void *staging, const void *host_src, void *stream);

/* Synchronize `stream`, read the cache's err_flag into *flags and clear it
 * when `clear` != 0.  Returns S4KV_ERR_DEVICE_CHECK when bits were set. */
S4KV_API int s4kv_get_error(const s4kv_cache_t *cache, uint32_t *flags, int clear,
                   void *stream);

#ifdef __cplusplus
}
#endif

#endif /* S4KV_H */
