"""The C-ABI library without a GPU: it loads, exports every function the
header declares, and its host-side checks answer before anything is launched
(the fail-fast model check of "S4 KV -- int4 KV-Cache-Kompression fuer vLLM",
"Lieferumfang": unsupported shapes are refused up front)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def S():
    from int4_kivi_quantized_s4kv_b200 import build
    build.build()
    import int4_kivi_quantized_s4kv_b200 as S
    return S


def header_functions():
    text = open(os.path.join(ROOT, "include", "s4kv.h")).read()
    return sorted(set(re.findall(r"S4KV_API\s+[\w\s\*]*?\b(s4kv_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    fns = header_functions()
    for name in ("s4kv_append", "s4kv_decode_attention", "s4kv_dequant_page"):
        assert name in fns


def test_library_exports_every_declared_symbol(S):
    lib = ctypes.CDLL(S.LIB_PATH)
    for name in header_functions():
        assert hasattr(lib, name), name
    assert set(header_functions()) <= set(S.EXPORTED)


def test_constants_match_header(S):
    text = open(os.path.join(ROOT, "include", "s4kv.h")).read()
    defs = dict(re.findall(r"#define\s+(S4KV_\w+)\s+(\d+)u?\b", text))
    assert int(defs["S4KV_BLOCK_BYTES"]) == S.BLOCK_BYTES
    assert int(defs["S4KV_HEAD_DIM"]) == S.HEAD_DIM
    assert int(defs["S4KV_PAGE_TOKENS"]) == S.PAGE_TOKENS
    for k, v in [("S4KV_OK", S.OK), ("S4KV_ERR_INVALID_ARG", S.ERR_INVALID_ARG),
                 ("S4KV_ERR_UNSUPPORTED", S.ERR_UNSUPPORTED), ("S4KV_ERR_CUDA", S.ERR_CUDA),
                 ("S4KV_ERR_DEVICE_CHECK", S.ERR_DEVICE_CHECK), ("S4KV_ERR_WORKSPACE", S.ERR_WORKSPACE),
                 ("S4KV_EFLAG_PAGE_RANGE", S.EFLAG_PAGE_RANGE), ("S4KV_EFLAG_SLOT", S.EFLAG_SLOT),
                 ("S4KV_EFLAG_SEQ_LEN", S.EFLAG_SEQ_LEN), ("S4KV_EFLAG_TIMEOUT", S.EFLAG_TIMEOUT)]:
        assert int(defs[k]) == v, k


def test_model_check_fail_fast(S):
    assert S.s4kv_check_model(128, 16, 32, 8) == S.OK
    assert S.s4kv_check_model(128, 16, 28, 4) == S.OK
    assert S.s4kv_check_model(128, 16, 64, 8) == S.OK
    assert S.s4kv_check_model(64, 16, 32, 8) == S.ERR_UNSUPPORTED
    assert S.s4kv_check_model(256, 16, 32, 8) == S.ERR_UNSUPPORTED
    assert S.s4kv_check_model(128, 32, 32, 8) == S.ERR_UNSUPPORTED
    assert S.s4kv_check_model(128, 16, 30, 8) == S.ERR_UNSUPPORTED
    assert S.s4kv_check_model(128, 16, 72, 8) == S.ERR_UNSUPPORTED  # group 9
    assert S.s4kv_check_model(0, 16, 32, 8) == S.ERR_INVALID_ARG
    for st in range(6):
        assert isinstance(S.s4kv_status_string(st), str)


def test_cache_layout_matches_block_size(S, oracle_mod):
    pool, res = S.s4kv_cache_layout(1000, 8, 256)
    assert pool == 1000 * 8 * oracle_mod.block_bytes()
    assert res == 256 * 8 * 16 * 128 * 2
    pool8, res8 = S.s4kv_cache_layout(1000, 8, 256, bits=8)
    assert pool8 == 1000 * 8 * oracle_mod.block_bytes(8) and res8 == res
    pool2, _ = S.s4kv_cache_layout(1000, 8, 256, bits=2)
    assert pool2 == 1000 * 8 * oracle_mod.block_bytes(2)
    with pytest.raises(S.S4KVError):
        S.s4kv_cache_layout(10, 8, 1, bits=3)
    with pytest.raises(S.S4KVError):
        S.s4kv_cache_layout(0, 8, 1)


def test_invalid_calls_rejected_before_launch(S):
    L = S.lib()
    P = ctypes.c_void_p
    fake = 0x100000  # a non-null, 128-B aligned address that is never dereferenced
    c = S.s4kv_cache_t(fake, fake, fake, None, 10, 2, 4, 128, 16)
    bad_dim = S.s4kv_cache_t(fake, fake, fake, None, 10, 2, 4, 64, 16)
    null_pool = S.s4kv_cache_t(None, fake, fake, None, 10, 2, 4, 128, 16)
    st = P(0)
    # append
    assert L.s4kv_append(None, P(fake), P(fake), 1, P(fake), P(fake), P(fake), P(fake), 1, 1, 1, st) == S.ERR_INVALID_ARG
    assert L.s4kv_append(ctypes.byref(bad_dim), P(fake), P(fake), 1, P(fake), P(fake), P(fake), P(fake), 1, 1, 1, st) == S.ERR_UNSUPPORTED
    assert L.s4kv_append(ctypes.byref(null_pool), P(fake), P(fake), 1, P(fake), P(fake), P(fake), P(fake), 1, 1, 1, st) == S.ERR_INVALID_ARG
    assert L.s4kv_append(ctypes.byref(c), None, P(fake), 1, P(fake), P(fake), P(fake), P(fake), 1, 1, 1, st) == S.ERR_INVALID_ARG
    assert L.s4kv_append(ctypes.byref(c), P(fake + 2), P(fake), 1, P(fake), P(fake), P(fake), P(fake), 1, 1, 1, st) == S.ERR_INVALID_ARG
    assert L.s4kv_append(ctypes.byref(c), P(fake), P(fake), 1, P(fake), P(fake), P(fake), P(fake), 5, 1, 1, st) == S.ERR_INVALID_ARG  # batch > max_seqs
    assert L.s4kv_append(ctypes.byref(c), P(fake), P(fake), 0, P(fake), P(fake), P(fake), P(fake), 1, 1, 1, st) == S.OK  # nothing to do
    # decode
    dec = L.s4kv_decode_attention
    assert dec(ctypes.byref(c), P(fake), 18, P(fake), P(fake), 1, 1, 0.088, P(fake), P(fake), 1 << 30, st) == S.ERR_UNSUPPORTED
    assert dec(ctypes.byref(c), P(fake), 7, P(fake), P(fake), 1, 1, 0.088, P(fake), P(fake), 1 << 30, st) == S.ERR_UNSUPPORTED
    assert dec(ctypes.byref(c), P(fake), 8, P(fake), P(fake), 1, 1, float("nan"), P(fake), P(fake), 1 << 30, st) == S.ERR_INVALID_ARG
    assert dec(ctypes.byref(c), P(fake), 8, P(fake), P(fake), 1, 1, -1.0, P(fake), P(fake), 1 << 30, st) == S.ERR_INVALID_ARG
    assert dec(ctypes.byref(c), None, 8, P(fake), P(fake), 1, 1, 0.088, P(fake), P(fake), 1 << 30, st) == S.ERR_INVALID_ARG
    assert dec(ctypes.byref(c), P(fake), 8, P(fake), P(fake), 0, 1, 0.088, P(fake), P(fake), 1 << 30, st) == S.OK
    # the one-call decode step: missing or unaligned new tokens, and an append grid (one CTA per
    # sequence and kv head) beyond the launch limit, are refused before anything runs
    step = L.s4kv_append_decode
    assert step(ctypes.byref(c), None, P(fake), P(fake), 8, P(fake), P(fake), 1, 1, 0.088, P(fake), P(fake),
                1 << 30, st) == S.ERR_INVALID_ARG
    assert step(ctypes.byref(c), P(fake), P(fake + 8), P(fake), 8, P(fake), P(fake), 1, 1, 0.088, P(fake), P(fake),
                1 << 30, st) == S.ERR_INVALID_ARG
    wide = S.s4kv_cache_t(fake, fake, fake, None, 10, 65536, 40000, 128, 16)
    assert step(ctypes.byref(wide), P(fake), P(fake), P(fake), 65536, P(fake), P(fake), 40000, 1, 0.088, P(fake),
                P(fake), 1 << 30, st) == S.ERR_INVALID_ARG
    # prefill
    pre = L.s4kv_prefill_attention
    args = lambda **kw: dict(dict(cache=ctypes.byref(c), q=P(fake), hq=8, n=4, cu=P(fake), sl=P(fake), bt=P(fake),
                                  batch=1, maxp=1, maxnew=4, scale=0.088, out=P(fake), ws=P(fake),
                                  wsb=1 << 30), **kw)
    call = lambda a: pre(a["cache"], a["q"], a["hq"], a["n"], a["cu"], a["sl"], a["bt"], a["batch"], a["maxp"],
                         a["maxnew"], a["scale"], a["out"], a["ws"], a["wsb"], st)
    assert call(args(hq=18)) == S.ERR_UNSUPPORTED
    assert call(args(cache=ctypes.byref(bad_dim))) == S.ERR_UNSUPPORTED
    assert call(args(scale=float("nan"))) == S.ERR_INVALID_ARG
    assert call(args(q=None)) == S.ERR_INVALID_ARG
    assert call(args(out=P(fake + 8))) == S.ERR_INVALID_ARG
    assert call(args(maxnew=0)) == S.ERR_INVALID_ARG
    assert call(args(maxnew=5)) == S.ERR_INVALID_ARG  # more than n_tokens
    assert call(args(batch=5)) == S.ERR_INVALID_ARG   # batch > max_seqs
    assert call(args(n=0)) == S.OK and call(args(batch=0)) == S.OK  # nothing to do
    # workspace: 80 KB per 128-key tile (8 pages) per (sequence slot, kv head)
    tile = 2 * 128 * 128 + 128 * 128 + 2 * 128 * 128  # K_hi fp16, K_lo e5m2, V^T fp16
    assert S.prefill_workspace_bytes(2, 1, 1) == 2 * tile
    assert S.prefill_workspace_bytes(8, 4, 512) == 4 * 8 * 64 * tile
    assert S.prefill_workspace_bytes(1, 1, 9) == 2 * tile  # 9 pages round up to 2 tiles
    n = ctypes.c_size_t(0)
    assert L.s4kv_prefill_workspace_size(0, 1, 1, ctypes.byref(n)) == S.ERR_INVALID_ARG
    assert L.s4kv_prefill_workspace_size(1, 1, 0, ctypes.byref(n)) == S.ERR_INVALID_ARG
    assert L.s4kv_prefill_workspace_size(1, 1, 1, None) == S.ERR_INVALID_ARG
    assert L.s4kv_prefill_workspace_size(65535, 65535, 1 << 30, ctypes.byref(n)) == S.ERR_INVALID_ARG
    assert call(args(ws=None)) == S.ERR_WORKSPACE
    assert call(args(ws=P(fake + 8))) == S.ERR_WORKSPACE  # not 16-B aligned
    assert call(args(wsb=2 * tile - 1)) == S.ERR_WORKSPACE
    # dequant
    assert L.s4kv_dequant_page(ctypes.byref(c), 10, P(fake), P(fake), 1, st) == S.ERR_INVALID_ARG
    assert L.s4kv_dequant_page(ctypes.byref(c), -1, P(fake), P(fake), 1, st) == S.ERR_INVALID_ARG
    assert L.s4kv_dequant_page(ctypes.byref(bad_dim), 0, P(fake), P(fake), 1, st) == S.ERR_UNSUPPORTED
    # code width: 4 (or 0), 8 and 2 only
    bad_bits = S.s4kv_cache_t(fake, fake, fake, None, 10, 2, 4, 128, 16, 3)
    assert L.s4kv_dequant_page(ctypes.byref(bad_bits), 0, P(fake), P(fake), 1, st) == S.ERR_UNSUPPORTED
    c8 = S.s4kv_cache_t(fake, fake, fake, None, 10, 2, 4, 128, 16, 8)
    # prefill takes 8- and 2-bit caches too: its host checks still run first
    # (these calls stop at them, before any launch)
    assert pre(ctypes.byref(c8), P(fake), 18, 4, P(fake), P(fake), P(fake), 1, 1, 4, 0.088, P(fake), P(fake), 1 << 30,
               st) == S.ERR_UNSUPPORTED
    assert pre(ctypes.byref(c8), P(fake), 8, 4, P(fake), P(fake), P(fake), 1, 1, 4, 0.088, P(fake), None, 1 << 30,
               st) == S.ERR_WORKSPACE
    n = ctypes.c_size_t(0)
    assert L.s4kv_page_record_bytes(ctypes.byref(c8), ctypes.byref(n)) == S.OK and n.value == 2 * 4864
    assert L.s4kv_page_record_bytes(ctypes.byref(c), ctypes.byref(n)) == S.OK and n.value == 2 * 2816
    # error read with no flag word needs no device
    flags = ctypes.c_uint32(7)
    assert L.s4kv_get_error(ctypes.byref(c), ctypes.byref(flags), 1, st) == S.OK and flags.value == 0
