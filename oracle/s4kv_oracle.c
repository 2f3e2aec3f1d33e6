/*
 * s4kv CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded restatement of what the int4 KIVI paged
 * KV cache computes.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this file; the CUDA library never does, and the
 * two share no code, header, table or constant.
 *
 * Sources (web pages on the subject; cited by title and section):
 *   [S4KV]  "S4 KV -- int4 KV-Cache-Kompression fuer vLLM", intro,
 *           "Funktionsweise" step 1, "Lieferumfang": keys are quantized to
 *           asymmetric int4 per channel, values to int4 per token (KIVI
 *           style); head_dim 128 only, with fail-fast otherwise.
 *   [KVOPT] "KV-Cache-Optimierung -- PagedAttention, quantisierter KV,
 *           Speculative Cache", "Kernpunkte" and "Begriffe auf dieser
 *           Seite" (GQA: a group of query heads shares one K/V head;
 *           PagedAttention: fixed-size blocks addressed like OS pages).
 *   [PAGED] "PagedAttention reduziert den KV-Cache-Speicherbedarf beim
 *           LLM-Serving erheblich", "Wichtigste Kernpunkte & Evidenz":
 *           16-token pages addressed through page tables.
 *   [CAP]   adechristanto.de, "KV-Cache-Quantisierung: Kapazitaet und
 *           Qualitaetspruefung", section "Gewichte, laufenden Zustand und
 *           reservierten Speicher trennen": KV payload bytes =
 *           2 x layers x kv_heads x head_dim x tokens x bytes per element.
 *
 * The pages fix the KIVI axis split but print no formula.  This library
 * states the quantizer as: over a group of fp16 values x, in fp32,
 *   mn = min x, mx = max x, s = (mx - mn) / 15,
 *   code = (s == 0) ? 0 : clamp(rint((x - mn) / s), 0, 15),
 * stored scale = fp16_rne(s), stored zero = fp16(mn) (exact); the
 * dequantized value is code * scale + zero, evaluated in fp32.  A key group
 * is one channel over the 16 tokens of a page; a value group is 32
 * consecutive channels of one token.  Minimum and maximum are taken in IEEE
 * total order, so -0 counts below +0.
 *
 * Page block layout (2816 bytes per (physical page, kv head)):
 *   [   0,1024) key codes   : 256 little-endian 32-bit words
 *   [1024,2048) value codes : 256 little-endian 32-bit words
 *   [2048,2304) key scale   : fp16 [128 channels]
 *   [2304,2560) key zero    : fp16 [8 k-tiles][16 k-slots], channel c at
 *                             k-tile (c%32)/4, slot 2*(c/32) + (c%2) + 8*((c%4)/2)
 *   [2560,2688) value scale : fp16, (token t, group g) at half
 *                             16*((t%8)/2) + 8*(t/8) + 2*g + t%2
 *   [2688,2816) value zero  : fp16 [4 groups][16 tokens]
 * Code word w (0..255) splits as w = 128*h + 4*lane + q with lane = 4*n + i
 * (n 0..7, i 0..3, q 0..3).  Nibble j (bits 4j..4j+3) of the word is
 * register r = (j&1) + 2*(j>>2), half e = (j>>1)&1 of the lane's operand
 * fragment and holds
 *   keys  : token 8*(r&1) + n,
 *           channel 32*i + 4*(4*h + q) + 2*(r>>1) + e;
 *   values: token 2*i + e + 8*(r>>1),
 *           channel 32*((4*h+q)>>1) + 4*n + 2*((4*h+q)&1) + (r&1).
 * Residual buffers hold fp16 [max_seqs][kv_heads][16][128] each for keys
 * and values: row r of sequence b is its token 16*floor(L/16) + r while
 * r < L mod 16; other rows are unspecified.
 *
 * Parity status of every function here is pinned by tests in
 * tests/test_oracle.py (see the header of that file for which pin covers
 * which function).  Build: gcc -O2 -ffp-contract=off -fno-fast-math.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define HEAD_DIM 128
#define PAGE 16
#define VGROUP 32

/* Block regions for `bits`-bit codes (2, 4 or 8): K codes, V codes, then the
 * fp16 metadata (K scale [128], K zero [128], V scale [4][16], V zero
 * [4][16]); with 4-bit codes this is the 2816-byte block. */
static long code_bytes(int bits) { return (long)PAGE * HEAD_DIM * bits / 8; }
static long kcode_off(int bits) { (void)bits; return 0; }
static long vcode_off(int bits) { return code_bytes(bits); }
static long kscale_off(int bits) { return 2 * code_bytes(bits); }
static long kzero_off(int bits) { return kscale_off(bits) + 2 * HEAD_DIM; }
static long vscale_off(int bits) { return kzero_off(bits) + 2 * HEAD_DIM; }
static long vzero_off(int bits) { return vscale_off(bits) + 2 * PAGE * (HEAD_DIM / VGROUP); }
static long block_bytes_of(int bits) { return vzero_off(bits) + 2 * PAGE * (HEAD_DIM / VGROUP); }

/* ---------------------------------------------------------------- fp16 -- */

/* IEEE binary16 -> binary32, exact.  Textbook decoding of the bit fields. */
float s4kv_ref_half_to_float(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    float v;
    if (e == 0) {
        v = ldexpf((float)m, -24); /* subnormal: m * 2^-24 */
    } else if (e == 31) {
        v = m ? NAN : INFINITY;
    } else {
        v = ldexpf((float)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* binary32 -> binary16 with round-to-nearest-even.  The magnitude is scaled
 * to an integer count of units in the last place of the target format
 * (exact: a power-of-two scaling), rounded with nearbyint (ties to even
 * under the default rounding mode), and the bit fields are assembled. */
uint16_t s4kv_ref_float_to_half(float f) {
    uint16_t sign = signbit(f) ? 0x8000 : 0;
    if (isnan(f)) return sign | 0x7e00;
    double a = fabs((double)f);
    if (isinf(f)) return sign | 0x7c00;
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: unit is 2^-24; a count of 1024 is the smallest
         * normal, whose bit pattern 0x0400 is the count itself */
        double q = nearbyint(ldexp(a, 24));
        return sign | (uint16_t)q;
    }
    int e2;
    frexp(a, &e2);        /* a = mant * 2^e2, mant in [0.5, 1) */
    int E = e2 - 1;       /* a = (2*mant) * 2^E, 2*mant in [1, 2) */
    double q = nearbyint(ldexp(a, 10 - E)); /* in [1024, 2048] */
    if (q == 2048.0) {
        q = 1024.0;
        E += 1;
    }
    if (E + 15 >= 31) return sign | 0x7c00; /* overflow to infinity */
    return sign | (uint16_t)(((E + 15) << 10) | ((int)q - 1024));
}

/* ----------------------------------------------------------- quantizer -- */

/* a < b in IEEE total order restricted to non-NaN values (-0 < +0). */
static int total_less(float a, float b) {
    if (a < b) return 1;
    if (a == b && signbit(a) && !signbit(b)) return 1;
    return 0;
}

/* Asymmetric quantization of one group of n fp16 values to `levels` + 1
 * codes (the KIVI step of [S4KV] "Funktionsweise" 1: levels = 15 for int4,
 * 255 for int8).  x[k*stride] are the fp16 inputs; codes[k*code_stride]
 * receive the codes.  Returns the fp32 scale so that tests can check the
 * rounding bound against it. */
static float quantize_group_levels(const uint16_t *x, int n, int stride,
                                   uint8_t *codes, int code_stride, int levels,
                                   uint16_t *scale_h, uint16_t *zero_h) {
    float mn = s4kv_ref_half_to_float(x[0]);
    float mx = mn;
    for (int k = 1; k < n; ++k) {
        float xv = s4kv_ref_half_to_float(x[k * stride]);
        if (total_less(xv, mn)) mn = xv;
        if (total_less(mx, xv)) mx = xv;
    }
    volatile float range = mx - mn; /* one fp32 rounding */
    volatile float s = range / (float)levels; /* one fp32 rounding */
    for (int k = 0; k < n; ++k) {
        float xv = s4kv_ref_half_to_float(x[k * stride]);
        int code = 0;
        if (s != 0.0f) {
            volatile float d = xv - mn;
            volatile float t = d / s;
            float r = nearbyintf(t); /* ties to even */
            if (r < 0.0f) r = 0.0f;
            if (r > (float)levels) r = (float)levels;
            code = (int)r;
        }
        codes[k * code_stride] = (uint8_t)code;
    }
    *scale_h = s4kv_ref_float_to_half(s);
    *zero_h = s4kv_ref_float_to_half(mn);
    return s;
}

/* ------------------------------------------------------------- packing -- */

float s4kv_ref_quantize_group(const uint16_t *x, int n, int stride,
                              uint8_t *codes, int code_stride,
                              uint16_t *scale_h, uint16_t *zero_h) {
    return quantize_group_levels(x, n, stride, codes, code_stride, 15, scale_h, zero_h);
}

/* The same with (1 << bits) - 1 levels (bits = 4 or 8). */
float s4kv_ref_quantize_group_bits(const uint16_t *x, int n, int stride,
                                   uint8_t *codes, int code_stride, int bits,
                                   uint16_t *scale_h, uint16_t *zero_h) {
    return quantize_group_levels(x, n, stride, codes, code_stride, (1 << bits) - 1, scale_h, zero_h);
}

/* Position (in halves) of channel c's key zero point: the zero points are
 * stored in the order in which the MMA k axis visits the channels. */
int s4kv_ref_key_zero_slot(int c) {
    int i = c / 32, kt = (c % 32) / 4, e = c % 4;
    return 16 * kt + 2 * i + (e % 2) + 8 * (e / 2);
}

/* A code's place in a lane's tensor-core operand fragment -- register r
 * (0..3) and half e (0: low 16 bits) -- is held by nibble r%2 + 2e + 4(r/2)
 * of the lane's 32-bit word: the even nibbles of the word's four bytes, then
 * the odd ones, are registers 0 and 2 (byte pairs 0-1 and 2-3 of the even
 * nibbles) and 1 and 3 (the same of the odd nibbles), the lower byte of a
 * pair in the lower half. */
static int nibble_of(int reg, int half) { return reg % 2 + 2 * half + 4 * (reg / 2); }
static int reg_of(int nibble) { return nibble % 2 + 2 * (nibble / 4); }
static int half_of(int nibble) { return (nibble / 2) % 2; }

/* (token, channel) -> (word, nibble) of the key code region: tile kt =
 * (c%32)/4 of lane 4n + i (n = t%8, i = c/32); rows are tokens (register
 * bit 0: row n + 8), the k axis is the channel (register bit 1: k + 8, half:
 * k + 1). */
void s4kv_ref_key_code_slot(int t, int c, int *word, int *nibble) {
    int i = c / 32, kt = (c % 32) / 4, e = c % 4;
    int n = t % 8;
    *nibble = nibble_of((t / 8) + 2 * (e / 2), e % 2);
    *word = 128 * (kt / 4) + 4 * (4 * n + i) + (kt % 4);
}

/* (token, channel) -> (word, nibble) of the value code region: M-tile m =
 * 2(c/32) + (c%4)/2 of lane 4n + i (n = (c%32)/4, i = (t%8)/2); rows are
 * channels (register bit 0: row + 8 = channel + 1), the k axis is the token
 * (register bit 1: k + 8, half: k + 1). */
void s4kv_ref_value_code_slot(int t, int c, int *word, int *nibble) {
    int grp = c / 32, n = (c % 32) / 4, e = c % 4;
    int m = 2 * grp + e / 2;
    int i = (t % 8) / 2;
    *nibble = nibble_of((e % 2) + 2 * (t / 8), t % 2);
    *word = 128 * (m / 4) + 4 * (4 * n + i) + (m % 4);
}

/* Position (in halves) of the value scale of (token t, group g) in its
 * region: lane quad i = (t%8)/2 owns 16 consecutive halves -- for k half
 * e = t/8, the token pair 2i + 8e, 2i + 8e + 1 of groups 0..3 -- so that one
 * lane reads all the scales it multiplies with two 16-byte loads. */
int s4kv_ref_value_scale_slot(int t, int g) {
    return 16 * ((t % 8) / 2) + 8 * (t / 8) + 2 * g + t % 2;
}

/* 8-bit codes keep the 4-bit layout's assignment of (token, channel) to MMA
 * operand fragments -- tile 4*(word/128) + word%4, lane (word/4)%32, and
 * within the lane's fragment register r and half e of the nibble -- with
 * bytes for nibbles: a lane's 8 codes of a tile are 8 consecutive bytes,
 * register r at bytes 2r (half 0) and 2r + 1 (half 1), and the 16 bytes of
 * tiles 2m and 2m+1 of one lane sit together, lanes in order. */
static long byte_offset8(int word, int nibble) {
    int tile = 4 * (word / 128) + word % 4, lane = (word / 4) % 32;
    return ((long)(tile / 2) * 32 + lane) * 16 + (tile % 2) * 8 + 2 * reg_of(nibble) + half_of(nibble);
}

/* 2-bit codes keep the same assignment with two bits per code: the 16 codes
 * of tiles 2m and 2m+1 of one lane form one 32-bit word, word 4*lane + m of
 * the region (a lane's four words sit together); half 0 of every register
 * is in the low 16 bits and half 1 in the high 16 bits, register r of tile
 * 2m+p at bits 2*(4*p + r) of its half. */
static void bit_position2(int word, int nibble, long *word2, int *bit) {
    int tile = 4 * (word / 128) + word % 4, lane = (word / 4) % 32;
    *word2 = 4L * lane + tile / 2;
    *bit = 16 * half_of(nibble) + 2 * (4 * (tile % 2) + reg_of(nibble));
}

/* Word index and bit of the 2-bit code of (token t, channel c) inside the
 * key (is_value = 0) or value (1) code region. */
void s4kv_ref_code_position2(int is_value, int t, int c, long *word, int *bit) {
    int w, nb;
    if (is_value) s4kv_ref_value_code_slot(t, c, &w, &nb);
    else s4kv_ref_key_code_slot(t, c, &w, &nb);
    bit_position2(w, nb, word, bit);
}

/* Byte offset of the 8-bit code of (token t, channel c) inside the key
 * (is_value = 0) or value (1) code region. */
long s4kv_ref_code_offset8(int is_value, int t, int c) {
    int w, nb;
    if (is_value) s4kv_ref_value_code_slot(t, c, &w, &nb);
    else s4kv_ref_key_code_slot(t, c, &w, &nb);
    return byte_offset8(w, nb);
}

static void put_nibble(uint8_t *region, int word, int nibble, int code) {
    uint8_t *byte = region + 4 * word + nibble / 2; /* little-endian word */
    int sh = 4 * (nibble % 2);
    *byte = (uint8_t)((*byte & ~(0xf << sh)) | ((code & 0xf) << sh));
}

static int get_nibble(const uint8_t *region, int word, int nibble) {
    const uint8_t *byte = region + 4 * word + nibble / 2;
    return (*byte >> (4 * (nibble % 2))) & 0xf;
}

static void put_code(uint8_t *region, int is_value, int t, int c, int code, int bits) {
    int w, nb;
    if (is_value) s4kv_ref_value_code_slot(t, c, &w, &nb);
    else s4kv_ref_key_code_slot(t, c, &w, &nb);
    if (bits == 8) {
        region[byte_offset8(w, nb)] = (uint8_t)code;
    } else if (bits == 2) {
        long w2;
        int bit;
        bit_position2(w, nb, &w2, &bit);
        uint32_t word;
        memcpy(&word, region + 4 * w2, 4); /* little-endian words */
        word = (word & ~(3u << bit)) | ((uint32_t)(code & 3) << bit);
        memcpy(region + 4 * w2, &word, 4);
    } else {
        put_nibble(region, w, nb, code);
    }
}

static int get_code(const uint8_t *region, int is_value, int t, int c, int bits) {
    int w, nb;
    if (is_value) s4kv_ref_value_code_slot(t, c, &w, &nb);
    else s4kv_ref_key_code_slot(t, c, &w, &nb);
    if (bits == 8) return region[byte_offset8(w, nb)];
    if (bits == 2) {
        long w2;
        int bit;
        bit_position2(w, nb, &w2, &bit);
        uint32_t word;
        memcpy(&word, region + 4 * w2, 4);
        return (int)((word >> bit) & 3u);
    }
    return get_nibble(region, w, nb);
}

static void put_half(uint8_t *p, uint16_t h) { memcpy(p, &h, 2); }
static uint16_t get_half(const uint8_t *p) {
    uint16_t h;
    memcpy(&h, p, 2);
    return h;
}

/* Quantize one full page of one kv head with `bits`-bit codes.  kp, vp:
 * fp16 [16][128] rows.  Writes the block_bytes_of(bits) block. */
void s4kv_ref_quantize_page_bits(const uint16_t *kp, const uint16_t *vp,
                                 uint8_t *block, int bits) {
    uint8_t kc[PAGE][HEAD_DIM], vc[PAGE][HEAD_DIM];
    int levels = (1 << bits) - 1;
    memset(block, 0, (size_t)block_bytes_of(bits));
    /* keys: one group per channel, over the page's 16 tokens */
    for (int c = 0; c < HEAD_DIM; ++c) {
        uint16_t sh, zh;
        quantize_group_levels(kp + c, PAGE, HEAD_DIM, &kc[0][c], HEAD_DIM, levels, &sh, &zh);
        put_half(block + kscale_off(bits) + 2 * c, sh);
        put_half(block + kzero_off(bits) + 2 * s4kv_ref_key_zero_slot(c), zh);
    }
    /* values: one group per token and 32-channel slice */
    for (int t = 0; t < PAGE; ++t) {
        for (int g = 0; g < HEAD_DIM / VGROUP; ++g) {
            uint16_t sh, zh;
            quantize_group_levels(vp + t * HEAD_DIM + g * VGROUP, VGROUP, 1,
                                  &vc[t][g * VGROUP], 1, levels, &sh, &zh);
            put_half(block + vscale_off(bits) + 2 * s4kv_ref_value_scale_slot(t, g), sh);
            put_half(block + vzero_off(bits) + 2 * (g * PAGE + t), zh);
        }
    }
    for (int t = 0; t < PAGE; ++t) {
        for (int c = 0; c < HEAD_DIM; ++c) {
            put_code(block + kcode_off(bits), 0, t, c, kc[t][c], bits);
            put_code(block + vcode_off(bits), 1, t, c, vc[t][c], bits);
        }
    }
}

void s4kv_ref_quantize_page(const uint16_t *kp, const uint16_t *vp,
                            uint8_t *block) {
    s4kv_ref_quantize_page_bits(kp, vp, block, 4);
}

/* Read back the codes of one block in natural [token][channel] order. */
void s4kv_ref_unpack_codes_bits(const uint8_t *block, uint8_t *kcodes,
                                uint8_t *vcodes, int bits) {
    for (int t = 0; t < PAGE; ++t) {
        for (int c = 0; c < HEAD_DIM; ++c) {
            kcodes[t * HEAD_DIM + c] = (uint8_t)get_code(block + kcode_off(bits), 0, t, c, bits);
            vcodes[t * HEAD_DIM + c] = (uint8_t)get_code(block + vcode_off(bits), 1, t, c, bits);
        }
    }
}

void s4kv_ref_unpack_codes(const uint8_t *block, uint8_t *kcodes,
                           uint8_t *vcodes) {
    s4kv_ref_unpack_codes_bits(block, kcodes, vcodes, 4);
}

/* Dequantize one block: x = code * scale + zero, in fp32 (the product of a
 * 4- or 8-bit code and an fp16 scale is exact in fp32, so this is one
 * rounding).  kout, vout: fp32 [16][128]. */
void s4kv_ref_dequant_block_bits(const uint8_t *block, float *kout, float *vout, int bits) {
    uint8_t kc[PAGE * HEAD_DIM], vc[PAGE * HEAD_DIM];
    s4kv_ref_unpack_codes_bits(block, kc, vc, bits);
    for (int t = 0; t < PAGE; ++t) {
        for (int c = 0; c < HEAD_DIM; ++c) {
            float ks = s4kv_ref_half_to_float(get_half(block + kscale_off(bits) + 2 * c));
            float kz = s4kv_ref_half_to_float(get_half(block + kzero_off(bits) + 2 * s4kv_ref_key_zero_slot(c)));
            int g = c / VGROUP;
            float vs = s4kv_ref_half_to_float(get_half(block + vscale_off(bits) + 2 * s4kv_ref_value_scale_slot(t, g)));
            float vz = s4kv_ref_half_to_float(get_half(block + vzero_off(bits) + 2 * (g * PAGE + t)));
            volatile float kprod = (float)kc[t * HEAD_DIM + c] * ks;
            volatile float vprod = (float)vc[t * HEAD_DIM + c] * vs;
            kout[t * HEAD_DIM + c] = kprod + kz;
            vout[t * HEAD_DIM + c] = vprod + vz;
        }
    }
}

void s4kv_ref_dequant_block(const uint8_t *block, float *kout, float *vout) {
    s4kv_ref_dequant_block_bits(block, kout, vout, 4);
}

/* --------------------------------------------------------------- cache -- */

/* Return codes shared with the tests (values of the library's header are
 * not included here on purpose; the tests compare meanings, not numbers). */
#define REF_OK 0
#define REF_BAD_ARG 1
#define REF_BAD_SLOT 2

/* Bytes of one (page, kv head) block of this layout, derived from its
 * parts: 4-bit codes for K and V plus fp16 scale/zero metadata. */
long s4kv_ref_block_bytes_bits(int bits) { return block_bytes_of(bits); }

long s4kv_ref_block_bytes(void) {
    long codes = 2L * PAGE * HEAD_DIM / 2;                   /* K + V, 4 bits */
    long kmeta = 2L * HEAD_DIM * 2;                          /* scale + zero */
    long vmeta = 2L * PAGE * (HEAD_DIM / VGROUP) * 2;        /* scale + zero */
    return codes + kmeta + vmeta;
}

/* The KV payload formula of [CAP]: 2 x layers x kv_heads x head_dim x
 * tokens x bytes per element (no metadata, no block rounding). */
double s4kv_ref_kv_payload_bytes(long layers, long kv_heads, long head_dim,
                                 long tokens, double bytes_per_elem) {
    return 2.0 * (double)layers * (double)kv_heads * (double)head_dim *
           (double)tokens * bytes_per_elem;
}

/* Append new fp16 K/V tokens (token-major [n_tokens][kv_heads][128]) to the
 * cache, one token at a time in sequence order: each token is written to its
 * sequence's residual row pos mod 16; when that row is 15 the page is
 * complete and is quantized from the residual into the physical page
 * block_tables[b][pos/16] ([PAGED] page tables; [S4KV] per-channel keys and
 * per-token values, keys quantized once the page is full).
 * cu_new[b]..cu_new[b+1] are sequence b's new tokens; seq_lens[b] is its
 * length after the append.  slot_mapping[tok] must equal
 * block_tables[b][pos/16] * 16 + pos % 16. */
int s4kv_ref_append_bits(uint8_t *pool, uint16_t *res_k, uint16_t *res_v,
                         int num_pages, int num_kv_heads, int max_seqs,
                         const uint16_t *k, const uint16_t *v, int n_tokens,
                         const int64_t *slot_mapping, const int32_t *cu_new,
                         const int32_t *seq_lens, const int32_t *block_tables,
                         int batch, int max_pages_per_seq, int bits) {
    if (batch < 0 || batch > max_seqs || n_tokens < 0) return REF_BAD_ARG;
    if (cu_new[0] != 0 || cu_new[batch] != n_tokens) return REF_BAD_ARG;
    const long row = HEAD_DIM;
    for (int b = 0; b < batch; ++b) {
        int n_b = cu_new[b + 1] - cu_new[b];
        int L = seq_lens[b];
        int L0 = L - n_b;
        if (n_b < 0 || L0 < 0 || (L + PAGE - 1) / PAGE > max_pages_per_seq)
            return REF_BAD_ARG;
        for (int j = 0; j < n_b; ++j) {
            int pos = L0 + j;
            int tok = cu_new[b] + j;
            int page = block_tables[(long)b * max_pages_per_seq + pos / PAGE];
            if (page < 0 || page >= num_pages) return REF_BAD_SLOT;
            if (slot_mapping[tok] != (int64_t)page * PAGE + pos % PAGE)
                return REF_BAD_SLOT;
            int r = pos % PAGE;
            for (int h = 0; h < num_kv_heads; ++h) {
                uint16_t *rk = res_k + (((long)b * num_kv_heads + h) * PAGE) * row;
                uint16_t *rv = res_v + (((long)b * num_kv_heads + h) * PAGE) * row;
                memcpy(rk + r * row, k + ((long)tok * num_kv_heads + h) * row, 2 * row);
                memcpy(rv + r * row, v + ((long)tok * num_kv_heads + h) * row, 2 * row);
                if (r == PAGE - 1) {
                    uint8_t *blk = pool + ((long)page * num_kv_heads + h) * block_bytes_of(bits);
                    s4kv_ref_quantize_page_bits(rk, rv, blk, bits);
                }
            }
        }
    }
    return REF_OK;
}

int s4kv_ref_append(uint8_t *pool, uint16_t *res_k, uint16_t *res_v,
                    int num_pages, int num_kv_heads, int max_seqs,
                    const uint16_t *k, const uint16_t *v, int n_tokens,
                    const int64_t *slot_mapping, const int32_t *cu_new,
                    const int32_t *seq_lens, const int32_t *block_tables,
                    int batch, int max_pages_per_seq) {
    return s4kv_ref_append_bits(pool, res_k, res_v, num_pages, num_kv_heads, max_seqs, k, v, n_tokens,
                                slot_mapping, cu_new, seq_lens, block_tables, batch, max_pages_per_seq, 4);
}

/* Dequantize one physical page for all kv heads.  out_k, out_v: fp32
 * [kv_heads][16][128]. */
int s4kv_ref_dequant_page_bits(const uint8_t *pool, int num_pages, int num_kv_heads,
                               int physical_page, float *out_k, float *out_v, int bits) {
    if (physical_page < 0 || physical_page >= num_pages) return REF_BAD_ARG;
    for (int h = 0; h < num_kv_heads; ++h) {
        const uint8_t *blk = pool + ((long)physical_page * num_kv_heads + h) * block_bytes_of(bits);
        s4kv_ref_dequant_block_bits(blk, out_k + (long)h * PAGE * HEAD_DIM,
                                    out_v + (long)h * PAGE * HEAD_DIM, bits);
    }
    return REF_OK;
}

int s4kv_ref_dequant_page(const uint8_t *pool, int num_pages, int num_kv_heads,
                          int physical_page, float *out_k, float *out_v) {
    return s4kv_ref_dequant_page_bits(pool, num_pages, num_kv_heads, physical_page, out_k, out_v, 4);
}

/* ------------------------------------------------ page movement ---- */
/* Moving whole pages between the pool and other memory, as a paged cache
 * does when it swaps sequences out and back in or forks one copy-on-write
 * ("KV-Cache und PagedAttention: Warum Ihr LLM-Server langsamer wird", "Wie
 * PagedAttention das loest": pages are allocated on demand, shared between
 * sequences and copied only when written).  A page record is all kv heads'
 * blocks of one physical page: num_kv_heads * 2816 contiguous bytes. */

/* dst[i] = page record pages[i], i < n (dst: [n][num_kv_heads][block bytes];
 * the block bytes follow the code width `bits`). */
int s4kv_ref_gather_pages(const uint8_t *pool, int num_pages, int num_kv_heads,
                          const int32_t *pages, int n, uint8_t *dst, int bits) {
    long rec = (long)num_kv_heads * block_bytes_of(bits);
    for (int i = 0; i < n; ++i)
        if (pages[i] < 0 || pages[i] >= num_pages) return REF_BAD_SLOT;
    for (int i = 0; i < n; ++i) memcpy(dst + i * rec, pool + pages[i] * rec, (size_t)rec);
    return REF_OK;
}

/* page record pages[i] = src[i], i < n (pages must be distinct). */
int s4kv_ref_scatter_pages(uint8_t *pool, int num_pages, int num_kv_heads,
                           const int32_t *pages, int n, const uint8_t *src, int bits) {
    long rec = (long)num_kv_heads * block_bytes_of(bits);
    for (int i = 0; i < n; ++i)
        if (pages[i] < 0 || pages[i] >= num_pages) return REF_BAD_SLOT;
    for (int i = 0; i < n; ++i) memcpy(pool + pages[i] * rec, src + i * rec, (size_t)rec);
    return REF_OK;
}

/* page record dst_pages[i] = page record src_pages[i] (a copy-on-write copy
 * of a shared full page); no dst page may also be a src page. */
int s4kv_ref_copy_pages(uint8_t *pool, int num_pages, int num_kv_heads,
                        const int32_t *src_pages, const int32_t *dst_pages, int n, int bits) {
    long rec = (long)num_kv_heads * block_bytes_of(bits);
    for (int i = 0; i < n; ++i)
        if (src_pages[i] < 0 || src_pages[i] >= num_pages || dst_pages[i] < 0 || dst_pages[i] >= num_pages)
            return REF_BAD_SLOT;
    for (int i = 0; i < n; ++i) memcpy(pool + dst_pages[i] * rec, pool + src_pages[i] * rec, (size_t)rec);
    return REF_OK;
}

/* The partial last page lives in the residual of its batch row: a fork
 * copies batch row src_rows[i]'s residual keys and values (all kv heads, all
 * 16 rows) to batch row dst_rows[i]. */
int s4kv_ref_fork_residual(uint16_t *res_k, uint16_t *res_v, int max_seqs, int num_kv_heads,
                           const int32_t *src_rows, const int32_t *dst_rows, int n) {
    long rec = (long)num_kv_heads * PAGE * HEAD_DIM;
    for (int i = 0; i < n; ++i)
        if (src_rows[i] < 0 || src_rows[i] >= max_seqs || dst_rows[i] < 0 || dst_rows[i] >= max_seqs)
            return REF_BAD_SLOT;
    for (int i = 0; i < n; ++i) {
        memcpy(res_k + dst_rows[i] * rec, res_k + src_rows[i] * rec, 2 * (size_t)rec);
        memcpy(res_v + dst_rows[i] * rec, res_v + src_rows[i] * rec, 2 * (size_t)rec);
    }
    return REF_OK;
}

/* Gather the K and V rows (fp32 [L][128]) of sequence b, kv head h: full
 * pages are dequantized page by page, the tail comes from the fp16
 * residual. */
static void sequence_kv(const uint8_t *pool, const uint16_t *res_k,
                        const uint16_t *res_v, int num_kv_heads,
                        const int32_t *bt_row, int L, int b, int h,
                        float *K, float *V, int bits) {
    int full = L / PAGE;
    for (int p = 0; p < full; ++p) {
        const uint8_t *blk = pool + ((long)bt_row[p] * num_kv_heads + h) * block_bytes_of(bits);
        s4kv_ref_dequant_block_bits(blk, K + (long)p * PAGE * HEAD_DIM,
                                    V + (long)p * PAGE * HEAD_DIM, bits);
    }
    for (int t = full * PAGE; t < L; ++t) {
        int r = t % PAGE;
        const uint16_t *rk = res_k + (((long)b * num_kv_heads + h) * PAGE + r) * HEAD_DIM;
        const uint16_t *rv = res_v + (((long)b * num_kv_heads + h) * PAGE + r) * HEAD_DIM;
        for (int c = 0; c < HEAD_DIM; ++c) {
            K[(long)t * HEAD_DIM + c] = s4kv_ref_half_to_float(rk[c]);
            V[(long)t * HEAD_DIM + c] = s4kv_ref_half_to_float(rv[c]);
        }
    }
}

/* GQA decode attention over the cache ([KVOPT] GQA: query head j reads kv
 * head j / (num_q_heads / num_kv_heads)).  For each sequence b and query
 * head: logits_t = sm_scale * sum_c q_c * k_tc over the L_b tokens, a
 * two-pass softmax (max, then exp and sum) and out = sum_t p_t v_t / sum p.
 * q: fp16 [batch][num_q_heads][128]; out: fp64 [batch][num_q_heads][128].
 * use_double selects fp64 (1) or fp32 (0) for every step after the fp32
 * dequantization.  Sequences of length 0 give an all-zero output. */
int s4kv_ref_decode_attention(const uint8_t *pool, const uint16_t *res_k,
                              const uint16_t *res_v, int num_pages,
                              int num_kv_heads, const uint16_t *q,
                              int num_q_heads, const int32_t *seq_lens,
                              const int32_t *block_tables, int batch,
                              int max_pages_per_seq, double sm_scale,
                              int use_double, double *out, int bits) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return REF_BAD_ARG;
    int G = num_q_heads / num_kv_heads;
    for (int b = 0; b < batch; ++b) {
        int L = seq_lens[b];
        const int32_t *bt_row = block_tables + (long)b * max_pages_per_seq;
        if (L < 0 || (L + PAGE - 1) / PAGE > max_pages_per_seq) return REF_BAD_ARG;
        for (int p = 0; p < L / PAGE; ++p)
            if (bt_row[p] < 0 || bt_row[p] >= num_pages) return REF_BAD_SLOT;
        for (int h = 0; h < num_kv_heads; ++h) {
            /* rounded up to whole pages: sequence_kv fills full pages */
            size_t rows = (size_t)((L + PAGE - 1) / PAGE + 1) * PAGE;
            float *K = (float *)malloc(sizeof(float) * rows * HEAD_DIM);
            float *V = (float *)malloc(sizeof(float) * rows * HEAD_DIM);
            double *logit = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
            if (!K || !V || !logit) { free(K); free(V); free(logit); return REF_BAD_ARG; }
            sequence_kv(pool, res_k, res_v, num_kv_heads, bt_row, L, b, h, K, V, bits);
            for (int g = 0; g < G; ++g) {
                int qh = h * G + g;
                const uint16_t *qv = q + ((long)b * num_q_heads + qh) * HEAD_DIM;
                double *o = out + ((long)b * num_q_heads + qh) * HEAD_DIM;
                if (L == 0) {
                    for (int c = 0; c < HEAD_DIM; ++c) o[c] = 0.0;
                    continue;
                }
                if (use_double) {
                    double mx = -INFINITY;
                    for (int t = 0; t < L; ++t) {
                        double acc = 0.0;
                        for (int c = 0; c < HEAD_DIM; ++c)
                            acc += (double)s4kv_ref_half_to_float(qv[c]) * (double)K[(long)t * HEAD_DIM + c];
                        logit[t] = sm_scale * acc;
                        if (logit[t] > mx) mx = logit[t];
                    }
                    double sum = 0.0;
                    for (int t = 0; t < L; ++t) {
                        logit[t] = exp(logit[t] - mx);
                        sum += logit[t];
                    }
                    for (int c = 0; c < HEAD_DIM; ++c) {
                        double acc = 0.0;
                        for (int t = 0; t < L; ++t) acc += logit[t] * (double)V[(long)t * HEAD_DIM + c];
                        o[c] = acc / sum;
                    }
                } else {
                    float mx = -INFINITY;
                    float sc = (float)sm_scale;
                    for (int t = 0; t < L; ++t) {
                        float acc = 0.0f;
                        for (int c = 0; c < HEAD_DIM; ++c)
                            acc += s4kv_ref_half_to_float(qv[c]) * K[(long)t * HEAD_DIM + c];
                        logit[t] = (double)(sc * acc);
                        if ((float)logit[t] > mx) mx = (float)logit[t];
                    }
                    float sum = 0.0f;
                    for (int t = 0; t < L; ++t) {
                        float e = expf((float)logit[t] - mx);
                        logit[t] = (double)e;
                        sum += e;
                    }
                    for (int c = 0; c < HEAD_DIM; ++c) {
                        float acc = 0.0f;
                        for (int t = 0; t < L; ++t) acc += (float)logit[t] * V[(long)t * HEAD_DIM + c];
                        o[c] = (double)(acc / sum);
                    }
                }
            }
            free(K);
            free(V);
            free(logit);
        }
    }
    return REF_OK;
}

/* Causal attention of a chunk of new query tokens over the cache after the
 * chunk was appended (the prefill / chunked-append side of the same cache).
 * Sequence b owns query rows cu_new[b] .. cu_new[b+1]-1 of q (fp16
 * [n_tokens][num_q_heads][128]); with n = cu_new[b+1] - cu_new[b] and
 * L = seq_lens[b] (after the append), query row j of b sits at position
 * L - n + j and attends to the cache's tokens 0 .. L - n + j: full pages
 * dequantized, the partial last page from the fp16 residual, exactly the
 * keys and values decode attention reads.  Per query head, fp64 logits
 * sm_scale * q.k, a two-pass softmax and the weighted sum of values.
 * out: fp64 [n_tokens][num_q_heads][128]; rows of no sequence are left
 * untouched. */
/* Softmax attention of one query head over tokens 0..pos of the dequantized
 * K, V (fp64 logits, two-pass softmax); w: scratch of pos + 1 doubles. */
static void attend_row(const float *K, const float *V, int pos, const uint16_t *qv, double sm_scale, double *w,
                       double *o) {
    double mx = -INFINITY;
    for (int t = 0; t <= pos; ++t) {
        double acc = 0.0;
        for (int c = 0; c < HEAD_DIM; ++c)
            acc += (double)s4kv_ref_half_to_float(qv[c]) * (double)K[(long)t * HEAD_DIM + c];
        w[t] = sm_scale * acc;
        if (w[t] > mx) mx = w[t];
    }
    double sum = 0.0;
    for (int t = 0; t <= pos; ++t) {
        w[t] = exp(w[t] - mx);
        sum += w[t];
    }
    for (int c = 0; c < HEAD_DIM; ++c) {
        double acc = 0.0;
        for (int t = 0; t <= pos; ++t) acc += w[t] * (double)V[(long)t * HEAD_DIM + c];
        o[c] = acc / sum;
    }
}

int s4kv_ref_prefill_attention(const uint8_t *pool, const uint16_t *res_k,
                               const uint16_t *res_v, int num_pages,
                               int num_kv_heads, const uint16_t *q,
                               int num_q_heads, const int32_t *cu_new,
                               const int32_t *seq_lens,
                               const int32_t *block_tables, int batch,
                               int max_pages_per_seq, double sm_scale,
                               double *out, int bits) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return REF_BAD_ARG;
    int G = num_q_heads / num_kv_heads;
    for (int b = 0; b < batch; ++b) {
        int L = seq_lens[b];
        int n = cu_new[b + 1] - cu_new[b];
        const int32_t *bt_row = block_tables + (long)b * max_pages_per_seq;
        if (L < 0 || n < 0 || n > L || (L + PAGE - 1) / PAGE > max_pages_per_seq) return REF_BAD_ARG;
        if (n == 0) continue;
        for (int p = 0; p < L / PAGE; ++p)
            if (bt_row[p] < 0 || bt_row[p] >= num_pages) return REF_BAD_SLOT;
        size_t rows = (size_t)((L + PAGE - 1) / PAGE + 1) * PAGE;
        float *K = (float *)malloc(sizeof(float) * rows * HEAD_DIM);
        float *V = (float *)malloc(sizeof(float) * rows * HEAD_DIM);
        double *w = (double *)malloc(sizeof(double) * (size_t)L);
        if (!K || !V || !w) { free(K); free(V); free(w); return REF_BAD_ARG; }
        for (int h = 0; h < num_kv_heads; ++h) {
            sequence_kv(pool, res_k, res_v, num_kv_heads, bt_row, L, b, h, K, V, bits);
            for (int j = 0; j < n; ++j) {
                int pos = L - n + j;
                long row = cu_new[b] + j;
                for (int g = 0; g < G; ++g) {
                    int qh = h * G + g;
                    attend_row(K, V, pos, q + (row * num_q_heads + qh) * HEAD_DIM, sm_scale, w,
                               out + (row * num_q_heads + qh) * HEAD_DIM);
                }
            }
        }
        free(K);
        free(V);
        free(w);
    }
    return REF_OK;
}

/* One query row (all q heads, [num_q_heads][128]) of sequence b at position
 * pos < L, over the cache as it stands with L tokens: tokens 0..pos, full
 * pages dequantized and the partial last page from the residual -- the view
 * of row pos - (L - n) of a chunk of n rows in s4kv_ref_prefill_attention,
 * without computing the chunk's other rows. */
int s4kv_ref_attention_at(const uint8_t *pool, const uint16_t *res_k, const uint16_t *res_v, int num_pages,
                          int num_kv_heads, const uint16_t *q, int num_q_heads, int L, int pos,
                          const int32_t *bt_row, int max_pages_per_seq, int b, double sm_scale, double *out,
                          int bits) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return REF_BAD_ARG;
    if (L <= 0 || pos < 0 || pos >= L || (L + PAGE - 1) / PAGE > max_pages_per_seq) return REF_BAD_ARG;
    for (int p = 0; p < L / PAGE; ++p)
        if (bt_row[p] < 0 || bt_row[p] >= num_pages) return REF_BAD_SLOT;
    int G = num_q_heads / num_kv_heads;
    size_t rows = (size_t)((L + PAGE - 1) / PAGE + 1) * PAGE;
    float *K = (float *)malloc(sizeof(float) * rows * HEAD_DIM);
    float *V = (float *)malloc(sizeof(float) * rows * HEAD_DIM);
    double *w = (double *)malloc(sizeof(double) * (size_t)L);
    if (!K || !V || !w) { free(K); free(V); free(w); return REF_BAD_ARG; }
    for (int h = 0; h < num_kv_heads; ++h) {
        sequence_kv(pool, res_k, res_v, num_kv_heads, bt_row, L, b, h, K, V, bits);
        for (int g = 0; g < G; ++g) {
            int qh = h * G + g;
            attend_row(K, V, pos, q + (long)qh * HEAD_DIM, sm_scale, w, out + (long)qh * HEAD_DIM);
        }
    }
    free(K);
    free(V);
    free(w);
    return REF_OK;
}

/* Attention on unquantized fp16 K/V rows given directly ([n][128] per
 * (sequence, kv head)); used only to report the quantization error.
 * k, v: fp16 [total_tokens][num_kv_heads][128] with sequence b occupying
 * rows cu[b]..cu[b+1]. */
int s4kv_ref_attention_fp16(const uint16_t *k, const uint16_t *v,
                            const int32_t *cu, int num_kv_heads,
                            const uint16_t *q, int num_q_heads, int batch,
                            double sm_scale, double *out) {
    int G = num_q_heads / num_kv_heads;
    for (int b = 0; b < batch; ++b) {
        int L = cu[b + 1] - cu[b];
        double *logit = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        if (!logit) return REF_BAD_ARG;
        for (int qh = 0; qh < num_q_heads; ++qh) {
            int h = qh / G;
            const uint16_t *qv = q + ((long)b * num_q_heads + qh) * HEAD_DIM;
            double *o = out + ((long)b * num_q_heads + qh) * HEAD_DIM;
            if (L == 0) {
                for (int c = 0; c < HEAD_DIM; ++c) o[c] = 0.0;
                continue;
            }
            double mx = -INFINITY;
            for (int t = 0; t < L; ++t) {
                const uint16_t *kr = k + ((long)(cu[b] + t) * num_kv_heads + h) * HEAD_DIM;
                double acc = 0.0;
                for (int c = 0; c < HEAD_DIM; ++c)
                    acc += (double)s4kv_ref_half_to_float(qv[c]) * (double)s4kv_ref_half_to_float(kr[c]);
                logit[t] = sm_scale * acc;
                if (logit[t] > mx) mx = logit[t];
            }
            double sum = 0.0;
            for (int t = 0; t < L; ++t) {
                logit[t] = exp(logit[t] - mx);
                sum += logit[t];
            }
            for (int c = 0; c < HEAD_DIM; ++c) {
                double acc = 0.0;
                for (int t = 0; t < L; ++t) {
                    const uint16_t *vr = v + ((long)(cu[b] + t) * num_kv_heads + h) * HEAD_DIM;
                    acc += logit[t] * (double)s4kv_ref_half_to_float(vr[c]);
                }
                o[c] = acc / sum;
            }
        }
        free(logit);
    }
    return REF_OK;
}
