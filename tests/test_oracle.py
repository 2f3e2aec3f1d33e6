"""Pins for the CPU oracle: each test ties an oracle function to something other
than the oracle itself -- a figure the pages print, a closed form, a textbook
or library routine, an invariant, or brute force on tiny inputs.

Which pin covers which oracle function:
  half_to_float / float_to_half : numpy's IEEE binary16 conversion (exhaustive
                                   and on rounding ties)
  quantize_group                : closed forms (exact grids, all-equal groups,
                                   signed zeros) and the exact-rational rounding
                                   bound |x - (code*s + min)| <= s*(1/2 + 2e-6)
  key/value code slots, packing : bijection over all (token, channel); the
                                   per-channel / per-token closed forms read back;
                                   the PTX mma.m16n8k16 fragment table (codes and
                                   the k order of the key zero points)
  block_bytes, kv_payload_bytes : the pages' worked sizes (tests/golden/kv_bytes.txt)
                                   and the ~3x density claim
  append                        : chunking invariance; closed-form page contents;
                                   slot_mapping check
  dequant                       : closed-form grids dequantize exactly
  decode_attention              : textbook softmax attention (numpy) on inputs the
                                   quantizer represents exactly; single key; uniform
                                   weights; page permutation and shared-prefix
                                   invariance; GQA identical queries; fp32 vs fp64
  int2 codes (code_position2, OracleCache(bits=2)) : 4-level closed forms,
                                   the rounding bound, the bit-pair layout
                                   against the int4 fragment map, exact-grid
                                   attention, chunking invariance
  int8 codes (quantize_group_bits, code_offset8, OracleCache(bits=8)) :
                                   256-level closed forms and the rounding bound;
                                   the byte layout against the int4 fragment map;
                                   textbook attention on exact 256-level grids;
                                   chunking invariance
  prefill_attention             : textbook causal softmax attention (numpy) on
                                   inputs the quantizer represents exactly, per
                                   query position; the chunk's last row equals
                                   decode attention
  attention_at                  : the same textbook attention for one row at a
                                   given position, and the chunk's row there
"""
import os
from fractions import Fraction

import numpy as np
import pytest

HD, PAGE = 128, 16
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f16bits(x):
    return np.asarray(x, np.float16).view(np.uint16)


# ------------------------------------------------------------------ fp16 --

def test_half_to_float_exhaustive(oracle_mod):
    bits = np.arange(65536, dtype=np.uint32)
    ref = bits.astype(np.uint16).view(np.float16).astype(np.float32)
    got = np.array([oracle_mod.half_to_float(int(b)) for b in bits], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_float_to_half_matches_numpy_including_ties(oracle_mod):
    rng = np.random.default_rng(7)
    vals = [rng.standard_normal(4000).astype(np.float32) * s for s in (1e-7, 1e-5, 1e-3, 1, 100, 3e4)]
    vals.append(np.array([0.0, -0.0, 65504, 65519.99, 65520, 65536, 1e10, -1e10,
                          2 ** -24, 2 ** -25, 3 * 2 ** -26, 2 ** -14, np.inf, -np.inf], np.float32))
    # exact ties halfway between neighbouring halves (exact in fp32)
    h = rng.integers(0, 0x7BFF, 4000).astype(np.uint16)
    lo = h.view(np.float16).astype(np.float32)
    hi = (h + 1).view(np.float16).astype(np.float32)
    vals.append(((lo.astype(np.float64) + hi) / 2).astype(np.float32))
    x = np.concatenate(vals).astype(np.float32)
    ref = x.astype(np.float16).view(np.uint16)
    got = np.array([oracle_mod.float_to_half(float(v)) for v in x], np.uint16)
    assert np.array_equal(got, ref)


# ------------------------------------------------------------- quantizer --

def test_quantize_group_integer_grid(oracle_mod):
    x = np.arange(16, dtype=np.float16)
    codes, sh, zh, s = oracle_mod.quantize_group(x)
    assert list(codes) == list(range(16))
    assert s == 1.0 and sh == 0x3C00 and zh == 0


def test_quantize_group_shifted_progression(oracle_mod):
    d, a = 2.0 ** -3, -1.5
    k = np.array([3, 0, 15, 7, 9, 1, 14, 2, 5, 6, 8, 10, 4, 11, 12, 13])
    x = (a + k * d).astype(np.float16)
    codes, sh, zh, s = oracle_mod.quantize_group(x)
    assert list(codes) == list(k)
    assert s == d and sh == f16bits(d) and zh == f16bits(a)


def test_quantize_group_all_equal_and_signed_zero(oracle_mod):
    codes, sh, zh, s = oracle_mod.quantize_group(np.full(32, 0.7, np.float16))
    assert s == 0.0 and sh == 0 and (codes == 0).all() and zh == f16bits(0.7)
    z = np.array([0.0, -0.0] * 8, np.float16)
    codes, sh, zh, s = oracle_mod.quantize_group(z)
    assert s == 0.0 and (codes == 0).all() and zh == 0x8000  # min in total order is -0


def _half_to_even(t):
    """Round to the nearest integer, ties to the even neighbour: the IEEE
    default rounding that rint names, restated with Python's exact rationals
    (independent of the C library the oracle calls)."""
    t = Fraction(t)
    f = t.numerator // t.denominator
    rem = t - f
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and f % 2 == 1):
        f += 1
    return f


@pytest.mark.parametrize("bits,n,lo,step", [(4, 16, 0.0, 1.0), (4, 32, -4.0, 0.5), (4, 16, 2.0, 0.25),
                                            (8, 32, 0.0, 1.0), (8, 16, -8.0, 0.125), (2, 16, 0.0, 1.0),
                                            (2, 32, -1.0, 0.5)])
def test_quantize_group_ties_round_half_to_even(oracle_mod, bits, n, lo, step):
    """Groups whose quotients (x - min) / s are exact half-integers (a grid of
    spacing s/2 from min to min + levels*s, every point exact in fp16 and in
    fp32): rint sends k + 1/2 to the even one of k and k + 1, so 0.5 -> 0,
    1.5 -> 2, 2.5 -> 2, 3.5 -> 4.  Rounding ties away from zero (roundf), or
    up (floor(t + 1/2)), gives odd codes here and fails."""
    levels = (1 << bits) - 1
    rng = np.random.default_rng(bits * 100 + n)
    halves = (np.arange(levels) + 0.5)                     # every tie the grid has
    t = np.concatenate([[0.0, float(levels)], rng.choice(halves, n - 2, replace=levels < n - 2)])
    t = t[rng.permutation(n)]
    x = (lo + t * step).astype(np.float16)
    assert np.array_equal(x.astype(np.float64), lo + t * step)   # exact in fp16
    codes, sh, zh, s = oracle_mod.quantize_group_bits(x, bits)
    assert s == step and zh == f16bits(lo)
    want = [_half_to_even(Fraction(v)) for v in t]
    assert list(codes) == want
    assert any(int(v * 2) % 4 == 1 for v in t) and any(int(v * 2) % 4 == 3 for v in t)  # both tie parities occur


def _bound_ok(x16, codes, s32, zero_bits):
    mn = Fraction(float(np.uint16(zero_bits).view(np.float16)))
    S = Fraction(s32)
    for xv, c in zip(x16.astype(np.float64), codes):
        err = abs(Fraction(float(xv)) - (c * S + mn))
        if err > S * Fraction(1, 2) + S * Fraction(2, 10 ** 6):
            return False
    return True


@pytest.mark.parametrize("kind", ["normal", "subnormal", "large", "outlier", "two-level"])
def test_quantize_group_rounding_bound(oracle_mod, kind):
    rng = np.random.default_rng(11)
    for trial in range(60):
        n = 16 if trial % 2 else 32
        if kind == "normal":
            x = rng.standard_normal(n)
        elif kind == "subnormal":
            x = rng.integers(-40, 40, n) * 2.0 ** -24
        elif kind == "large":
            x = rng.uniform(-60000, 60000, n)
        elif kind == "outlier":
            x = rng.standard_normal(n)
            x[rng.integers(n)] *= 300
        else:
            x = rng.choice([-2.5, 3.25], n)
        x16 = np.asarray(x).astype(np.float16)
        codes, sh, zh, s = oracle_mod.quantize_group(x16)
        assert codes.min() >= 0 and codes.max() <= 15
        assert zh == x16[np.argmin(x16)].view(np.uint16) or float(x16.min()) == 0.0
        if s > 0:
            assert codes[np.argmin(x16)] == 0 and codes[np.argmax(x16)] == 15
            assert _bound_ok(x16, codes, s, zh)
        assert sh == np.float32(s).astype(np.float16).view(np.uint16)


# ---------------------------------------------------------------- layout --

def test_code_slots_are_a_bijection(oracle_mod):
    for slot in (oracle_mod.key_code_slot, oracle_mod.value_code_slot):
        seen = set()
        for t in range(PAGE):
            for c in range(HD):
                w, nb = slot(t, c)
                assert 0 <= w < 256 and 0 <= nb < 8
                seen.add((w, nb))
        assert len(seen) == PAGE * HD


def _fragment_position(word, nibble):
    """Where a nibble lands in the warp-level MMA operand, per the PTX ISA's
    fragment table for mma.m16n8k16 (row-major A, f16): lane = 4*g + t holds
    a0 = (row g, cols 2t, 2t+1), a1 = (row g+8, same cols), a2 = (row g,
    cols 2t+8, 2t+9), a3 = (row g+8, cols 2t+8, 2t+9), the lower column in the
    low half.  The library unpacks a lane's word by keeping the low nibble of
    every byte (bytes 0-1 -> register 0, bytes 2-3 -> register 2) and the high
    nibble of every byte (-> registers 1 and 3), each byte pair converted to
    an f16x2 with the lower byte in the low half: nibble j is register
    (j & 1) + 2 (j >> 2), half (j >> 1) & 1.  Returns (tile, lane, row, col)."""
    tile = 4 * (word // 128) + word % 4
    lane = (word % 128) // 4
    g, t = lane // 4, lane % 4
    r, e = (nibble & 1) + 2 * (nibble >> 2), (nibble >> 1) & 1
    return tile, lane, g + 8 * (r & 1), 2 * t + e + 8 * (r >> 1)


def test_code_layout_is_the_mma_operand_order(oracle_mod):
    """Each 32-bit code word is one lane's tensor-core A fragment: for keys,
    rows are tokens and the k axis of tile kt is lane t's channels
    32t + 4kt + {0,1} (cols 2t, 2t+1) and + {2,3} (cols 2t+8, 2t+9), matching
    a B fragment that holds channels 32t..32t+31; for values, rows of M-tile m
    are channels 32*(m//2) + 4*(row%8) + 2*(m%2) + row//8 and the k axis is the
    token index."""
    for t in range(PAGE):
        for c in range(HD):
            tile, lane, row, col = _fragment_position(*oracle_mod.key_code_slot(t, c))
            tq = lane % 4
            k_slot_channel = 32 * tq + 4 * tile + ((col - 2 * tq) if col < 8 else 2 + (col - 2 * tq - 8))
            assert (row, k_slot_channel) == (t, c)
            tile, lane, row, col = _fragment_position(*oracle_mod.value_code_slot(t, c))
            ch = 32 * (tile // 2) + 4 * (row % 8) + 2 * (tile % 2) + row // 8
            assert (col, ch) == (t, c)


def test_value_scales_are_lane_major(oracle_mod):
    """Value scales are stored so that the lane quad whose B-operand k rows
    are tokens 2i, 2i+1 (and 2i+8, 2i+9) finds the scales of those tokens, for
    all four channel groups, in one 32-byte run: quad i owns halves 16i ..
    16i + 15, k half e (tokens + 8e) the 8 halves from 16i + 8e, group g the
    token pair at 16i + 8e + 2g.  A bijection onto the 64 slots."""
    seen = set()
    for t in range(PAGE):
        for g in range(4):
            pos = oracle_mod.value_scale_slot(t, g)
            i, e = (t % 8) // 2, t // 8
            assert 16 * i + 8 * e <= pos < 16 * i + 8 * e + 8
            assert pos == 16 * i + 8 * e + 2 * g + t % 2
            seen.add(pos)
    assert seen == set(range(64))


def test_key_zero_order_is_the_mma_k_order(oracle_mod):
    """Key zero points are stored in the order the m16n8k16 k axis visits
    channels: k-tile kt, slot s holds the channel whose code sits in k column
    s of tile kt (same map as the code layout), so one ldmatrix row of 8
    halves is a lane quad's k columns."""
    seen = set()
    for c in range(HD):
        pos = oracle_mod.key_zero_slot(c)
        kt, slot = divmod(pos, 16)
        seen.add(pos)
        # the key code of channel c, token 0, sits in tile kt at column `slot`
        tile, lane, row, col = _fragment_position(*oracle_mod.key_code_slot(0, c))
        assert (tile, col) == (kt, slot)
    assert seen == set(range(HD))


def _grid_page(rng, per="key"):
    """fp16 [16][128] whose groups are exact 16-level grids: returns the page,
    expected codes, and per-group (scale, zero)."""
    if per == "key":   # group = channel over the 16 tokens
        d = 2.0 ** rng.integers(-6, 0, HD)
        a = rng.integers(-64, 64, HD) * d
        codes = np.stack([rng.permutation(16) for _ in range(HD)], axis=1)  # [t][c]
        x = (a[None, :] + codes * d[None, :]).astype(np.float16)
        return x, codes, d, a
    # value: group = 32 channels of one token; two copies of a 16-level grid
    d = 2.0 ** rng.integers(-6, 0, (PAGE, 4))
    a = rng.integers(-64, 64, (PAGE, 4)) * d
    codes = np.zeros((PAGE, HD), np.int64)
    for t in range(PAGE):
        for g in range(4):
            codes[t, 32 * g:32 * g + 32] = np.concatenate([rng.permutation(16), rng.permutation(16)])
    x = (a.repeat(32, axis=1) + codes * d.repeat(32, axis=1)).astype(np.float16)
    return x, codes, d, a


def test_page_axis_split_closed_form(oracle_mod):
    """Keys are quantized per channel and values per token in 32-channel
    groups ("S4 KV", "Funktionsweise" 1): on exact grids the stored scale is
    the grid step of exactly that group and the codes are the grid indices."""
    rng = np.random.default_rng(3)
    k, kc_ref, kd, ka = _grid_page(rng, "key")
    v, vc_ref, vd, va = _grid_page(rng, "value")
    blk = oracle_mod.quantize_page(k, v)
    assert blk.size == 2816
    kc, vc = oracle_mod.unpack_codes(blk)
    assert np.array_equal(kc, kc_ref) and np.array_equal(vc, vc_ref)
    ks = blk[2048:2304].view(np.float16).astype(np.float64)
    kz_slots = blk[2304:2560].view(np.float16).astype(np.float64)
    kz = np.array([kz_slots[oracle_mod.key_zero_slot(c)] for c in range(HD)])
    vs_slots = blk[2560:2688].view(np.float16).astype(np.float64)
    vs = np.array([[vs_slots[oracle_mod.value_scale_slot(t, g)] for t in range(PAGE)] for g in range(4)])
    vz = blk[2688:2816].view(np.float16).astype(np.float64).reshape(4, 16)
    assert np.array_equal(ks, kd) and np.array_equal(kz, ka)
    assert np.array_equal(vs, vd.T) and np.array_equal(vz, va.T)
    kdq, vdq = oracle_mod.dequant_block(blk)
    assert np.array_equal(kdq, k.astype(np.float32)) and np.array_equal(vdq, v.astype(np.float32))


# ------------------------------------------------------------ byte model --

def test_kv_byte_formula_reproduces_page_figures(oracle_mod):
    rows = [l.split() for l in open(os.path.join(GOLDEN, "kv_bytes.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 4
    for r in rows:
        L, H, D, T, by, lo, hi = int(r[0]), int(r[1]), int(r[2]), int(r[3]), float(r[4]), float(r[5]), float(r[6])
        got = oracle_mod.kv_payload_bytes(L, H, D, T, by)
        assert lo <= got <= hi, (r, got)
    assert oracle_mod.kv_payload_bytes(80, 8, 128, 4096, 2) == 1342177280


def test_density_about_three_times(oracle_mod):
    """"S4 KV" intro and "Highlights": about 3x more KV density than fp16;
    "KV-Cache-Optimierung", "Warum es zaehlt": INT4 quarters the payload."""
    fp16 = oracle_mod.kv_payload_bytes(1, 1, 128, 16, 2.0)
    assert fp16 == 8192
    blk = oracle_mod.block_bytes()
    assert blk == 2816
    assert 2.75 <= fp16 / blk <= 3.25
    assert fp16 / oracle_mod.kv_payload_bytes(1, 1, 128, 16, 0.5) == 4.0


# ---------------------------------------------------------------- append --

def _append_all(oracle_mod, cache, k, v, lens_before, lens_after, bt, chunk=None):
    """Append tokens lens_before..lens_after for every sequence (k, v are the
    per-sequence full streams) in chunks of `chunk` tokens per call."""
    B = len(lens_after)
    cur = np.array(lens_before, np.int64)
    tgt = np.array(lens_after, np.int64)
    while (cur < tgt).any():
        take = tgt - cur if chunk is None else np.minimum(tgt - cur, chunk)
        ks, vs, pos_list = [], [], []
        for b in range(B):
            pos = np.arange(cur[b], cur[b] + take[b])
            pos_list.append(pos)
            ks.append(k[b][pos])
            vs.append(v[b][pos])
        from int4_kivi_quantized_s4kv_b200 import workloads
        sm = workloads.slot_mapping(bt, pos_list)
        cu = np.concatenate([[0], np.cumsum(take)]).astype(np.int32)
        rc = cache.append(np.concatenate(ks), np.concatenate(vs), sm, cu,
                          (cur + take).astype(np.int32), bt)
        assert rc == 0
        cur = cur + take


def _rand_kv(rng, B, H, lens):
    k = [rng.standard_normal((L, H, HD)).astype(np.float16) for L in lens]
    v = [rng.standard_normal((L, H, HD)).astype(np.float16) for L in lens]
    return k, v


def _tables(rng, lens, extra=3):
    need = [(L + PAGE - 1) // PAGE for L in lens]
    NP = sum(need) + extra
    perm = rng.permutation(NP).astype(np.int32)
    bt = np.full((len(lens), max(need)), -1, np.int32)
    c = 0
    for b, n in enumerate(need):
        bt[b, :n] = perm[c:c + n]
        c += n
    return bt, NP


def test_append_chunking_invariance(oracle_mod):
    rng = np.random.default_rng(5)
    lens = [37, 50, 16, 5]
    H = 2
    k, v = _rand_kv(rng, 4, H, lens)
    bt, NP = _tables(rng, lens)
    caches = []
    for chunk in (None, 1, 7, 16, 23):
        c = oracle_mod.OracleCache(NP, H, 4)
        _append_all(oracle_mod, c, k, v, [0] * 4, lens, bt, chunk)
        caches.append(c)
    for c in caches[1:]:
        assert np.array_equal(c.pool, caches[0].pool)
        for b, L in enumerate(lens):
            r = L % PAGE
            assert np.array_equal(c.res_k[b, :, :r], caches[0].res_k[b, :, :r])
            assert np.array_equal(c.res_v[b, :, :r], caches[0].res_v[b, :, :r])
    # residual rows are the sequence's tail tokens, bit for bit
    for b, L in enumerate(lens):
        r = L % PAGE
        tail = k[b][L - r:L].transpose(1, 0, 2)
        assert np.array_equal(caches[0].res_k[b, :, :r], tail.view(np.uint16))


def test_append_page_contents_closed_form(oracle_mod):
    rng = np.random.default_rng(9)
    kp, kcodes, kd, ka = _grid_page(rng, "key")
    vp, vcodes, vd, va = _grid_page(rng, "value")
    k = [kp[:, None, :]]
    v = [vp[:, None, :]]
    bt = np.array([[2]], np.int32)
    c = oracle_mod.OracleCache(4, 1, 1)
    _append_all(oracle_mod, c, k, v, [0], [16], bt, chunk=5)
    kc, vc = oracle_mod.unpack_codes(c.pool[2, 0])
    assert np.array_equal(kc, kcodes) and np.array_equal(vc, vcodes)
    assert (c.pool[[0, 1, 3]] == 0).all()


def test_append_rejects_inconsistent_slot(oracle_mod):
    c = oracle_mod.OracleCache(4, 1, 1)
    k = np.zeros((3, 1, HD), np.float16)
    bt = np.array([[1]], np.int32)
    sm = np.array([16, 17, 19], np.int64)  # third token should be slot 18
    rc = c.append(k, k, sm, np.array([0, 3], np.int32), np.array([3], np.int32), bt)
    assert rc != 0


# ------------------------------------------------------- decode attention --

def _textbook_attention(q, K, V, scale):
    """softmax(scale * q K^T) V in float64 with numpy, per (b, q head)."""
    s = scale * (K.astype(np.float64) @ q.astype(np.float64))
    s -= s.max()
    p = np.exp(s)
    return (p[:, None] * V.astype(np.float64)).sum(0) / p.sum()


def _build_cache(oracle_mod, k, v, lens, bt, NP, H, chunk=None):
    c = oracle_mod.OracleCache(NP, H, len(lens))
    _append_all(oracle_mod, c, k, v, [0] * len(lens), lens, bt, chunk)
    return c


def test_decode_matches_textbook_attention_on_exact_grids(oracle_mod):
    """On K/V the quantizer represents exactly, decode attention must equal
    plain softmax attention (numpy, float64) on the original fp16 values: this
    pins page addressing, GQA head mapping, the residual and the softmax."""
    rng = np.random.default_rng(21)
    H, G = 2, 4
    lens = [37, 64, 3, 50]
    k, v = [], []
    for L in lens:
        npg = (L + PAGE - 1) // PAGE
        kk = np.zeros((npg * PAGE, H, HD), np.float16)
        vv = np.zeros((npg * PAGE, H, HD), np.float16)
        for p in range(npg):
            for h in range(H):
                kk[p * PAGE:(p + 1) * PAGE, h] = _grid_page(rng, "key")[0]
                vv[p * PAGE:(p + 1) * PAGE, h] = _grid_page(rng, "value")[0]
        k.append(kk[:L])
        v.append(vv[:L])
    bt, NP = _tables(rng, lens)
    c = _build_cache(oracle_mod, k, v, lens, bt, NP, H, chunk=9)
    q = rng.standard_normal((len(lens), H * G, HD)).astype(np.float16)
    out = c.decode_attention(q, np.array(lens, np.int32), bt)
    scale = 1 / np.sqrt(HD)
    for b, L in enumerate(lens):
        for qh in range(H * G):
            ref = _textbook_attention(q[b, qh], k[b][:, qh // G], v[b][:, qh // G], scale)
            assert np.allclose(out[b, qh], ref, rtol=1e-12, atol=1e-12)


def test_single_key_returns_its_value(oracle_mod):
    rng = np.random.default_rng(1)
    k, v = _rand_kv(rng, 3, 1, [1, 1, 1])
    bt, NP = _tables(rng, [1, 1, 1])
    c = _build_cache(oracle_mod, k, v, [1, 1, 1], bt, NP, 1)
    q = rng.standard_normal((3, 4, HD)).astype(np.float16)
    out = c.decode_attention(q, np.array([1, 1, 1], np.int32), bt)
    for b in range(3):
        for qh in range(4):
            assert np.array_equal(out[b, qh], v[b][0, 0].astype(np.float64))


def test_zero_query_gives_mean_of_values(oracle_mod):
    """q = 0 makes every weight equal; with values constant inside each
    quantization group the dequantized values are exact, so the output is the
    plain mean of the fp16 inputs."""
    rng = np.random.default_rng(2)
    lens = [37, 16]
    H = 1
    k, _ = _rand_kv(rng, 2, H, lens)
    v = []
    for L in lens:
        base = rng.standard_normal((L, H, 4)).astype(np.float16)
        v.append(np.repeat(base, 32, axis=2))
    bt, NP = _tables(rng, lens)
    c = _build_cache(oracle_mod, k, v, lens, bt, NP, H)
    q = np.zeros((2, 2, HD), np.float16)
    out = c.decode_attention(q, np.array(lens, np.int32), bt)
    for b in range(2):
        ref = v[b][:, 0].astype(np.float64).mean(0)
        assert np.allclose(out[b, 0], ref, rtol=0, atol=1e-12)


def test_page_permutation_and_shared_prefix_invariance(oracle_mod):
    rng = np.random.default_rng(4)
    H, lens = 2, [64, 70]
    prefix = 32
    k0, v0 = _rand_kv(rng, 1, H, [70])
    k1, v1 = _rand_kv(rng, 1, H, [70])
    k1[0][:prefix], v1[0][:prefix] = k0[0][:prefix], v0[0][:prefix]
    k, v = [k0[0][:64], k1[0]], [v0[0][:64], v1[0]]
    q = rng.standard_normal((2, 2 * H, HD)).astype(np.float16)
    sl = np.array(lens, np.int32)
    outs = []
    for seed in (0, 1):
        bt, NP = _tables(np.random.default_rng(seed), lens)
        c = _build_cache(oracle_mod, k, v, lens, bt, NP, H)
        outs.append(c.decode_attention(q, sl, bt))
    assert np.array_equal(outs[0], outs[1])
    # shared: sequence 1 points its first two pages at sequence 0's pages
    bt, NP = _tables(np.random.default_rng(2), lens)
    c = _build_cache(oracle_mod, k, v, lens, bt, NP, H)
    bt_shared = bt.copy()
    bt_shared[1, :2] = bt[0, :2]
    out_shared = c.decode_attention(q, sl, bt_shared)
    assert np.array_equal(out_shared, outs[0])


def test_gqa_identical_queries_identical_outputs(oracle_mod):
    rng = np.random.default_rng(6)
    lens = [45]
    k, v = _rand_kv(rng, 1, 2, lens)
    bt, NP = _tables(rng, lens)
    c = _build_cache(oracle_mod, k, v, lens, bt, NP, 2)
    q = rng.standard_normal((1, 8, HD)).astype(np.float16)
    q[0, 4:8] = q[0, 4]
    out = c.decode_attention(q, np.array(lens, np.int32), bt)
    for j in range(5, 8):
        assert np.array_equal(out[0, j], out[0, 4])
    assert not np.array_equal(out[0, 0], out[0, 4])


def test_fp32_oracle_close_to_fp64(oracle_mod):
    from int4_kivi_quantized_s4kv_b200 import workloads as W
    spec = W.SPECS["tiny"]
    lens = W.final_lens(spec)
    plan = W.page_plan(spec)
    k = [W.kv_sequence_np(spec, 0, b, int(L))[0] for b, L in enumerate(lens)]
    v = [W.kv_sequence_np(spec, 0, b, int(L))[1] for b, L in enumerate(lens)]
    c = _build_cache(oracle_mod, k, v, list(lens), plan.block_tables, plan.num_pages, 1)
    q = W.queries_np(spec, 0)
    o64 = c.decode_attention(q, lens, plan.block_tables, use_double=True)
    o32 = c.decode_attention(q, lens, plan.block_tables, use_double=False)
    assert np.abs(o64 - o32).max() < 1e-4
    # quantization error against unquantized fp16 attention: information only
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    ref = oracle_mod.attention_fp16(np.concatenate(k), np.concatenate(v), cu, 1, q)
    err = np.abs(o64 - ref).max()
    assert np.isfinite(err) and err < 1.0


# ------------------------------------------------------------ prefill --

def _grid_streams(rng, lens, H, bits=4):
    """Key/value streams whose every page is an exact grid of the code width
    (the grid pages of each width are defined further down; looked up at
    call time)."""
    page = {4: lambda per: _grid_page(rng, per)[0], 8: lambda per: _grid_page8(rng, per),
            2: lambda per: _grid_page2(rng, per)}[bits]
    k, v = [], []
    for L in lens:
        npg = (L + PAGE - 1) // PAGE
        kk = np.zeros((npg * PAGE, H, HD), np.float16)
        vv = np.zeros((npg * PAGE, H, HD), np.float16)
        for p in range(npg):
            for h in range(H):
                kk[p * PAGE:(p + 1) * PAGE, h] = page("key")
                vv[p * PAGE:(p + 1) * PAGE, h] = page("value")
        k.append(kk[:L])
        v.append(vv[:L])
    return k, v


@pytest.mark.parametrize("bits", [4, 8, 2])
def test_prefill_matches_textbook_causal_attention_on_exact_grids(oracle_mod, bits):
    """A chunk of n new tokens appended to a context of L - n tokens: every
    query row at position pos must equal plain softmax attention (numpy,
    float64) over the original fp16 keys and values 0..pos.  On exact grids
    of the code width the dequantized cache is the input itself, so this
    pins the causal limit, the position of each chunk row, the GQA map and
    the page walk, for every width."""
    rng = np.random.default_rng(31 + bits)
    H, G = 2, 3
    before = [21, 0, 32, 5]
    after = [40, 17, 50, 37]
    k, v = _grid_streams(rng, after, H, bits)
    bt, NP = _tables(rng, after)
    c = oracle_mod.OracleCache(NP, H, len(after), bits=bits)
    _append_all(oracle_mod, c, k, v, [0] * 4, before, bt)
    _append_all(oracle_mod, c, k, v, before, after, bt)
    n = np.array(after) - np.array(before)
    cu = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    q = rng.standard_normal((int(cu[-1]), H * G, HD)).astype(np.float16)
    out = c.prefill_attention(q, cu, np.array(after, np.int32), bt)
    scale = 1 / np.sqrt(HD)
    for b in range(4):
        for j in range(n[b]):
            pos = before[b] + j
            row = cu[b] + j
            for qh in range(H * G):
                ref = _textbook_attention(q[row, qh], k[b][:pos + 1, qh // G], v[b][:pos + 1, qh // G], scale)
                assert np.allclose(out[row, qh], ref, rtol=1e-12, atol=1e-12), (b, j, qh)


def test_prefill_last_row_is_decode(oracle_mod):
    """The last row of a chunk sits at position L - 1 and sees the whole
    sequence: it must be exactly what decode attention gives for that query."""
    rng = np.random.default_rng(32)
    H, G = 2, 4
    before = [30, 16, 1]
    after = [47, 33, 20]
    k, v = _rand_kv(rng, 3, H, after)
    bt, NP = _tables(rng, after)
    c = oracle_mod.OracleCache(NP, H, 3)
    _append_all(oracle_mod, c, k, v, [0] * 3, after, bt)
    n = np.array(after) - np.array(before)
    cu = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    q = rng.standard_normal((int(cu[-1]), H * G, HD)).astype(np.float16)
    out = c.prefill_attention(q, cu, np.array(after, np.int32), bt, sm_scale=0.07)
    last = q[cu[1:] - 1]
    dec = c.decode_attention(last, np.array(after, np.int32), bt, sm_scale=0.07)
    assert np.array_equal(out[cu[1:] - 1], dec)


@pytest.mark.parametrize("bits", [4, 8])
def test_attention_at_matches_textbook_and_the_chunk_rows(oracle_mod, bits):
    """One query row at position pos over the cache as it stands: plain
    softmax attention (numpy, float64) over the fp16 keys and values 0..pos on
    exact grids, and exactly the row a chunk whose row sits at pos gets.
    Positions on both sides of page boundaries, inside the partial last
    page, and 0."""
    rng = np.random.default_rng(33 + bits)
    H, G = 2, 3
    after = [45, 33]
    k, v = _grid_streams(rng, after, H, bits)
    bt, NP = _tables(rng, after)
    c = oracle_mod.OracleCache(NP, H, len(after), bits=bits)
    _append_all(oracle_mod, c, k, v, [0, 0], after, bt)
    n = np.array(after)
    cu = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    q = rng.standard_normal((int(cu[-1]), H * G, HD)).astype(np.float16)
    chunk = c.prefill_attention(q, cu, np.array(after, np.int32), bt)
    scale = 1 / np.sqrt(HD)
    for b, positions in ((0, [0, 15, 16, 31, 32, 40, 44]), (1, [0, 17, 31, 32])):
        for pos in positions:
            row = cu[b] + pos
            got = c.attention_at(q[row], b, after[b], pos, bt[b])
            assert np.array_equal(got, chunk[row]), (b, pos)
            for qh in range(H * G):
                ref = _textbook_attention(q[row, qh], k[b][:pos + 1, qh // G], v[b][:pos + 1, qh // G], scale)
                assert np.allclose(got[qh], ref, rtol=1e-12, atol=1e-12), (b, pos, qh)


# ------------------------------------------------------ page movement --

def test_swap_out_and_in_elsewhere_preserves_attention(oracle_mod):
    """Swap a sequence's pages out (gather), wipe them, swap them back into
    other physical pages (scatter) and point its page table there: decode
    attention must come out bit-identical, and the gathered records must be
    the same bytes as before."""
    rng = np.random.default_rng(41)
    H, G = 2, 4
    lens = [37, 70, 16]
    k, v = _rand_kv(rng, 3, H, lens)
    bt, NP = _tables(rng, lens, extra=8)
    c = _build_cache(oracle_mod, k, v, lens, bt, NP, H, chunk=13)
    q = rng.standard_normal((3, H * G, HD)).astype(np.float16)
    before = c.decode_attention(q, np.array(lens, np.int32), bt)
    full = [int(p) for p in bt[1, :lens[1] // PAGE]]
    rec = c.gather_pages(full)
    c.scatter_pages(full, np.zeros_like(rec))
    used = set(int(p) for p in bt[bt >= 0].ravel())
    free = [p for p in range(NP) if p not in used][:len(full)]
    c.scatter_pages(free, rec)
    bt2 = bt.copy()
    bt2[1, :len(full)] = free
    after = c.decode_attention(q, np.array(lens, np.int32), bt2)
    assert np.array_equal(before, after)
    assert np.array_equal(c.gather_pages(free), rec)
    # the wiped pages really were read before: with the old table the output changes
    assert not np.array_equal(c.decode_attention(q, np.array(lens, np.int32), bt)[1], before[1])


def test_fork_shares_full_pages_and_copies_the_partial_page(oracle_mod):
    """Fork sequence 0 into batch row 2: the full pages are shared through the
    page table, the partial page is copied (fork_residual).  Both rows then
    give the same attention; appending to the fork fills its own page and
    leaves the original untouched, and the fork equals a cache built from its
    whole token stream directly."""
    rng = np.random.default_rng(42)
    H, G = 2, 3
    L0, extra = 37, 20
    k, v = _rand_kv(rng, 1, H, [L0 + extra])
    k2 = [k[0][:L0], k[0][:L0], k[0]]
    v2 = [v[0][:L0], v[0][:L0], v[0]]
    NP = 16
    bt = np.full((3, 4), -1, np.int32)
    bt[0, :3] = [5, 9, 2]
    bt[1, :3] = [7, 1, 12]
    c = oracle_mod.OracleCache(NP, H, 3)
    _append_all(oracle_mod, c, k2, v2, [0, 0, 0], [L0, L0, 0], bt)
    # fork 0 -> 2: share the two full pages, copy the partial page's residual
    bt[2, :2] = bt[0, :2]
    bt[2, 2:4] = [3, 14]
    c.fork_residual([0], [2])
    q = rng.standard_normal((3, H * G, HD)).astype(np.float16)
    q[2] = q[0]
    out = c.decode_attention(q, np.array([L0, L0, L0], np.int32), bt)
    assert np.array_equal(out[2], out[0])
    ref0 = out[0].copy()
    # the fork diverges: 20 more tokens complete its page 2 and start page 3
    _append_all(oracle_mod, c, k2, v2, [L0, L0, L0], [L0, L0, L0 + extra], bt)
    out = c.decode_attention(q, np.array([L0, L0, L0 + extra], np.int32), bt)
    assert np.array_equal(out[0], ref0)
    direct = oracle_mod.OracleCache(NP, H, 1)
    btd = bt[2:3].copy()
    _append_all(oracle_mod, direct, [k[0]], [v[0]], [0], [L0 + extra], btd)
    assert np.array_equal(direct.decode_attention(q[2:3], np.array([L0 + extra], np.int32), btd)[0], out[2])


def test_copy_pages_then_remap_preserves_attention(oracle_mod):
    rng = np.random.default_rng(43)
    H = 1
    lens = [64, 33]
    k, v = _rand_kv(rng, 2, H, lens)
    bt, NP = _tables(rng, lens, extra=6)
    c = _build_cache(oracle_mod, k, v, lens, bt, NP, H)
    q = rng.standard_normal((2, 4, HD)).astype(np.float16)
    before = c.decode_attention(q, np.array(lens, np.int32), bt)
    used = set(int(p) for p in bt[bt >= 0].ravel())
    free = [p for p in range(NP) if p not in used][:4]
    c.copy_pages(bt[0, :4], free)
    bt2 = bt.copy()
    bt2[0, :4] = free
    assert np.array_equal(c.decode_attention(q, np.array(lens, np.int32), bt2), before)


# ------------------------------------------------------------- int8 codes --

def test_int8_group_closed_forms(oracle_mod):
    """255 levels: an exact 256-level grid gives its indices and step; the
    all-equal group gives scale 0."""
    x = np.arange(256, dtype=np.float16)
    codes, sh, zh, s = oracle_mod.quantize_group_bits(x, 8)
    assert list(codes) == list(range(256)) and s == 1.0 and sh == 0x3C00 and zh == 0
    d, a = 2.0 ** -6, -2.0
    k = np.random.default_rng(3).permutation(256)[:32]
    k[0], k[1] = 0, 255
    codes, sh, zh, s = oracle_mod.quantize_group_bits((a + k * d).astype(np.float16), 8)
    assert list(codes) == list(k) and s == d and zh == f16bits(a)
    codes, sh, zh, s = oracle_mod.quantize_group_bits(np.full(32, -1.25, np.float16), 8)
    assert s == 0.0 and (codes == 0).all()


def test_int8_group_rounding_bound(oracle_mod):
    rng = np.random.default_rng(12)
    for trial in range(80):
        n = 16 if trial % 2 else 32
        x = rng.standard_normal(n) * (1 if trial % 3 else 300)
        x16 = x.astype(np.float16)
        codes, sh, zh, s = oracle_mod.quantize_group_bits(x16, 8)
        assert codes.max() <= 255
        if s > 0:
            assert _bound_ok(x16, codes, s, zh)
            assert codes[np.argmin(x16)] == 0 and codes[np.argmax(x16)] == 255


def test_int8_layout_is_the_int4_fragment_map_in_bytes(oracle_mod):
    """8-bit codes sit where the 4-bit layout's MMA fragment assignment says,
    with bytes for nibbles: a lane's 8 codes of one tile are consecutive
    bytes (register r at bytes 2r, 2r + 1), tiles 2m and 2m+1 of a lane form
    one 16-byte chunk, chunks in lane order.  Together with the fragment-table
    pin of the 4-bit layout this ties the 8-bit layout to the PTX table; it
    must also be a bijection onto the 2048-byte region."""
    for is_value, slot in ((False, oracle_mod.key_code_slot), (True, oracle_mod.value_code_slot)):
        seen = set()
        for t in range(PAGE):
            for c in range(HD):
                off = oracle_mod.code_offset8(is_value, t, c)
                chunk, within = divmod(off, 16)
                m, lane = divmod(chunk, 32)
                tile = 2 * m + within // 8
                r, half = divmod(within % 8, 2)
                word, nib = slot(t, c)
                assert (tile, lane) == (4 * (word // 128) + word % 4, (word % 128) // 4)
                assert (r, half) == ((nib & 1) + 2 * (nib >> 2), (nib >> 1) & 1)
                seen.add(off)
        assert seen == set(range(2048))


def test_int8_block_size(oracle_mod):
    # 16 x 128 one-byte codes for K and V plus the same 768 bytes of fp16
    # metadata as the int4 block
    assert oracle_mod.block_bytes(8) == 2 * 2048 + 768 == 4864
    assert oracle_mod.block_bytes(4) == 2816


def _grid_page8(rng, per):
    if per == "key":
        d = 2.0 ** rng.integers(-8, -4, HD)
        a = rng.integers(-8, 8, HD) * 0.25
        codes = np.stack([rng.permutation(256)[:16] for _ in range(HD)], axis=1)
        codes[0], codes[1] = 0, 255
        return (a[None, :] + codes * d[None, :]).astype(np.float16)
    d = 2.0 ** rng.integers(-8, -4, (PAGE, 4))
    a = rng.integers(-8, 8, (PAGE, 4)) * 0.25
    codes = np.stack([np.stack([rng.permutation(256)[:32] for _ in range(4)]) for _ in range(PAGE)])
    codes[:, :, 0], codes[:, :, 1] = 0, 255
    return (a[:, :, None] + codes * d[:, :, None]).reshape(PAGE, HD).astype(np.float16)


def test_int8_decode_matches_textbook_on_exact_grids(oracle_mod):
    """Pages whose key channels and value groups are exact 256-level grids
    dequantize to themselves, so int8 decode attention equals numpy's."""
    rng = np.random.default_rng(44)
    H, G = 2, 4
    lens = [40, 64, 9]
    k, v = [], []
    for L in lens:
        npg = (L + PAGE - 1) // PAGE
        kk = np.zeros((npg * PAGE, H, HD), np.float16)
        vv = np.zeros((npg * PAGE, H, HD), np.float16)
        for p in range(npg):
            for h in range(H):
                kk[p * PAGE:(p + 1) * PAGE, h] = _grid_page8(rng, "key")
                vv[p * PAGE:(p + 1) * PAGE, h] = _grid_page8(rng, "value")
        k.append(kk[:L])
        v.append(vv[:L])
    bt, NP = _tables(rng, lens)
    c = oracle_mod.OracleCache(NP, H, len(lens), bits=8)
    _append_all(oracle_mod, c, k, v, [0] * 3, lens, bt, 11)
    q = rng.standard_normal((3, H * G, HD)).astype(np.float16)
    out = c.decode_attention(q, np.array(lens, np.int32), bt)
    for b, L in enumerate(lens):
        for qh in range(H * G):
            ref = _textbook_attention(q[b, qh], k[b][:, qh // G], v[b][:, qh // G], 1 / np.sqrt(HD))
            assert np.allclose(out[b, qh], ref, rtol=1e-12, atol=1e-12)
    # and int8 attention is closer to unquantized attention than int4 on random data
    kr, vr = _rand_kv(rng, 2, 1, [96, 64])
    btr, NPr = _tables(rng, [96, 64])
    errs = []
    for bits in (4, 8):
        cc = oracle_mod.OracleCache(NPr, 1, 2, bits=bits)
        _append_all(oracle_mod, cc, kr, vr, [0, 0], [96, 64], btr)
        qq = rng.standard_normal((2, 4, HD)).astype(np.float16) if bits == 4 else qq
        o = cc.decode_attention(qq, np.array([96, 64], np.int32), btr)
        ref = np.stack([np.stack([_textbook_attention(qq[b, j], kr[b][:, 0], vr[b][:, 0], 1 / np.sqrt(HD))
                                  for j in range(4)]) for b in range(2)])
        errs.append(np.abs(o - ref).max())
    assert errs[1] < errs[0] / 4


def test_int8_append_chunking_invariance(oracle_mod):
    rng = np.random.default_rng(45)
    lens = [37, 50]
    k, v = _rand_kv(rng, 2, 2, lens)
    bt, NP = _tables(rng, lens)
    pools = []
    for chunk in (None, 1, 16, 23):
        c = oracle_mod.OracleCache(NP, 2, 2, bits=8)
        _append_all(oracle_mod, c, k, v, [0, 0], lens, bt, chunk)
        pools.append((c.pool.copy(), c.res_k.copy()))
    for p_, r_ in pools[1:]:
        assert np.array_equal(p_, pools[0][0])
        for b, L in enumerate(lens):
            assert np.array_equal(r_[b, :, :L % 16], pools[0][1][b, :, :L % 16])


# ------------------------------------------------------------- int2 codes --

def test_int2_group_closed_forms_and_bound(oracle_mod):
    """3 levels: a 4-level grid gives its indices and step; random groups
    stay within half a step of their dequantized values."""
    d, a = 0.5, -1.0
    k = np.array([0, 3, 1, 2, 2, 1, 0, 3] * 4)
    codes, sh, zh, s = oracle_mod.quantize_group_bits((a + k * d).astype(np.float16), 2)
    assert list(codes) == list(k) and s == d and zh == f16bits(a)
    rng = np.random.default_rng(13)
    for trial in range(60):
        x16 = (rng.standard_normal(16 if trial % 2 else 32) * 3).astype(np.float16)
        codes, sh, zh, s = oracle_mod.quantize_group_bits(x16, 2)
        assert codes.max() <= 3
        if s > 0:
            assert _bound_ok(x16, codes, s, zh)
            assert codes[np.argmin(x16)] == 0 and codes[np.argmax(x16)] == 3


def test_int2_layout_is_the_int4_fragment_map_in_bit_pairs(oracle_mod):
    """2-bit codes keep the 4-bit fragment assignment: word 4*lane + m holds
    tiles 2m, 2m+1 of that lane, half h of register r of tile 2m+p at bits
    16h + 2(4p + r); every (word, bit pair) of the 512-byte region is used
    exactly once."""
    for is_value, slot in ((False, oracle_mod.key_code_slot), (True, oracle_mod.value_code_slot)):
        seen = set()
        for t in range(PAGE):
            for c in range(HD):
                w2, bit = oracle_mod.code_position2(is_value, t, c)
                lane, m = divmod(w2, 4)
                half, rest = divmod(bit, 16)
                p, r = divmod(rest // 2, 4)
                word, nib = slot(t, c)
                assert (2 * m + p, lane) == (4 * (word // 128) + word % 4, (word % 128) // 4)
                assert (r, half) == ((nib & 1) + 2 * (nib >> 2), (nib >> 1) & 1) and bit % 2 == 0
                seen.add((w2, bit))
        assert seen == {(w, b) for w in range(128) for b in range(0, 32, 2)}
    assert oracle_mod.block_bytes(2) == 2 * 512 + 768


def _grid_page2(rng, per):
    if per == "key":
        d = 2.0 ** rng.integers(-4, 0, HD)
        a = rng.integers(-8, 8, HD) * 0.25
        codes = np.stack([rng.permutation(np.arange(16) % 4) for _ in range(HD)], axis=1)
        return (a[None, :] + codes * d[None, :]).astype(np.float16)
    d = 2.0 ** rng.integers(-4, 0, (PAGE, 4))
    a = rng.integers(-8, 8, (PAGE, 4)) * 0.25
    codes = np.stack([np.stack([rng.permutation(np.arange(32) % 4) for _ in range(4)]) for _ in range(PAGE)])
    return (a[:, :, None] + codes * d[:, :, None]).reshape(PAGE, HD).astype(np.float16)


def test_int2_decode_matches_textbook_on_exact_grids(oracle_mod):
    rng = np.random.default_rng(46)
    H, G = 1, 4
    lens = [33, 48, 5]
    k, v = [], []
    for L in lens:
        npg = (L + PAGE - 1) // PAGE
        kk = np.zeros((npg * PAGE, H, HD), np.float16)
        vv = np.zeros((npg * PAGE, H, HD), np.float16)
        for p in range(npg):
            kk[p * PAGE:(p + 1) * PAGE, 0] = _grid_page2(rng, "key")
            vv[p * PAGE:(p + 1) * PAGE, 0] = _grid_page2(rng, "value")
        k.append(kk[:L])
        v.append(vv[:L])
    bt, NP = _tables(rng, lens)
    c = oracle_mod.OracleCache(NP, H, len(lens), bits=2)
    _append_all(oracle_mod, c, k, v, [0] * 3, lens, bt, 7)
    q = rng.standard_normal((3, H * G, HD)).astype(np.float16)
    out = c.decode_attention(q, np.array(lens, np.int32), bt)
    for b, L in enumerate(lens):
        for qh in range(H * G):
            ref = _textbook_attention(q[b, qh], k[b][:, 0], v[b][:, 0], 1 / np.sqrt(HD))
            assert np.allclose(out[b, qh], ref, rtol=1e-12, atol=1e-12)
    # chunking invariance of the 2-bit append
    pools = []
    for chunk in (None, 3, 16):
        cc = oracle_mod.OracleCache(NP, H, len(lens), bits=2)
        _append_all(oracle_mod, cc, k, v, [0] * 3, lens, bt, chunk)
        pools.append(cc.pool.copy())
    assert all(np.array_equal(p_, pools[0]) for p_ in pools[1:])
