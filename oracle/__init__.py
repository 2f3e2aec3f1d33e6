"""CPU oracle for the int4 (and int8) KIVI paged KV cache -- TEST INFRASTRUCTURE ONLY.

Thin ctypes/numpy wrapper around ``s4kv_oracle.c`` (plain C, single thread).
Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library and its Python
binding never do; the two implementations share no code.

What each function computes, and the page it restates, is documented in
``s4kv_oracle.c``.  The pins that tie each function to the pages and to
mathematics (not to itself) live in ``tests/test_oracle.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HEAD_DIM = 128
PAGE = 16
VGROUP = 32
BLOCK_BYTES = 2816

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "s4kv_oracle.c")
_LIB = os.path.join(_HERE, "libs4kv_oracle.so")
_CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-Wall",
           "-shared", "-fPIC"]

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libs4kv_oracle.so`` (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, f32, f64 = ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_double
        L.s4kv_ref_half_to_float.argtypes = [ctypes.c_uint16]
        L.s4kv_ref_half_to_float.restype = f32
        L.s4kv_ref_float_to_half.argtypes = [f32]
        L.s4kv_ref_float_to_half.restype = ctypes.c_uint16
        L.s4kv_ref_quantize_group.argtypes = [P, i32, i32, P, i32, P, P]
        L.s4kv_ref_quantize_group.restype = f32
        L.s4kv_ref_key_code_slot.argtypes = [i32, i32, P, P]
        L.s4kv_ref_value_code_slot.argtypes = [i32, i32, P, P]
        L.s4kv_ref_key_zero_slot.argtypes = [i32]
        L.s4kv_ref_key_zero_slot.restype = i32
        L.s4kv_ref_value_scale_slot.argtypes = [i32, i32]
        L.s4kv_ref_value_scale_slot.restype = i32
        L.s4kv_ref_quantize_page.argtypes = [P, P, P]
        L.s4kv_ref_unpack_codes.argtypes = [P, P, P]
        L.s4kv_ref_dequant_block.argtypes = [P, P, P]
        L.s4kv_ref_block_bytes.restype = ctypes.c_long
        L.s4kv_ref_kv_payload_bytes.argtypes = [ctypes.c_long] * 4 + [f64]
        L.s4kv_ref_kv_payload_bytes.restype = f64
        L.s4kv_ref_append.argtypes = [P, P, P, i32, i32, i32, P, P, i32, P, P, P, P, i32, i32]
        L.s4kv_ref_append.restype = i32
        L.s4kv_ref_dequant_page.argtypes = [P, i32, i32, i32, P, P]
        L.s4kv_ref_dequant_page.restype = i32
        L.s4kv_ref_decode_attention.argtypes = [P, P, P, i32, i32, P, i32, P, P, i32, i32, f64, i32, P, i32]
        L.s4kv_ref_decode_attention.restype = i32
        L.s4kv_ref_attention_fp16.argtypes = [P, P, P, i32, P, i32, i32, f64, P]
        L.s4kv_ref_prefill_attention.argtypes = [P, P, P, i32, i32, P, i32, P, P, P, i32, i32, f64, P, i32]
        L.s4kv_ref_prefill_attention.restype = i32
        L.s4kv_ref_attention_at.argtypes = [P, P, P, i32, i32, P, i32, i32, i32, P, i32, i32, f64, P, i32]
        L.s4kv_ref_attention_at.restype = i32
        L.s4kv_ref_gather_pages.argtypes = [P, i32, i32, P, i32, P, i32]
        L.s4kv_ref_gather_pages.restype = i32
        L.s4kv_ref_scatter_pages.argtypes = [P, i32, i32, P, i32, P, i32]
        L.s4kv_ref_scatter_pages.restype = i32
        L.s4kv_ref_copy_pages.argtypes = [P, i32, i32, P, P, i32, i32]
        L.s4kv_ref_copy_pages.restype = i32
        L.s4kv_ref_fork_residual.argtypes = [P, P, i32, i32, P, P, i32]
        L.s4kv_ref_fork_residual.restype = i32
        L.s4kv_ref_attention_fp16.restype = i32
        L.s4kv_ref_quantize_group_bits.argtypes = [P, i32, i32, P, i32, i32, P, P]
        L.s4kv_ref_quantize_group_bits.restype = f32
        L.s4kv_ref_code_offset8.argtypes = [i32, i32, i32]
        L.s4kv_ref_code_offset8.restype = ctypes.c_long
        L.s4kv_ref_code_position2.argtypes = [i32, i32, i32, P, P]
        L.s4kv_ref_quantize_page_bits.argtypes = [P, P, P, i32]
        L.s4kv_ref_unpack_codes_bits.argtypes = [P, P, P, i32]
        L.s4kv_ref_dequant_block_bits.argtypes = [P, P, P, i32]
        L.s4kv_ref_block_bytes_bits.argtypes = [i32]
        L.s4kv_ref_block_bytes_bits.restype = ctypes.c_long
        L.s4kv_ref_append_bits.argtypes = [P, P, P, i32, i32, i32, P, P, i32, P, P, P, P, i32, i32, i32]
        L.s4kv_ref_append_bits.restype = i32
        L.s4kv_ref_dequant_page_bits.argtypes = [P, i32, i32, i32, P, P, i32]
        L.s4kv_ref_dequant_page_bits.restype = i32
        _lib = L
        del i64
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    """fp16 array (or its raw uint16 bits) -> contiguous uint16 bit view."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    assert a.dtype == np.uint16
    return a


# ------------------------------------------------------------------ fp16 --

def half_to_float(bits: int) -> float:
    return float(lib().s4kv_ref_half_to_float(int(bits)))


def float_to_half(x: float) -> int:
    return int(lib().s4kv_ref_float_to_half(float(x)))


# ------------------------------------------------------------- quantizer --

def quantize_group(x) -> tuple[np.ndarray, int, int, float]:
    """Quantize one group of fp16 values -> (codes u8, scale bits, zero bits, fp32 scale)."""
    xb = _u16(np.asarray(x, dtype=np.float16) if not isinstance(x, np.ndarray) or x.dtype != np.uint16 else x)
    n = xb.size
    codes = np.zeros(n, np.uint8)
    sh = np.zeros(1, np.uint16)
    zh = np.zeros(1, np.uint16)
    s = lib().s4kv_ref_quantize_group(_p(xb), n, 1, _p(codes), 1, _p(sh), _p(zh))
    return codes, int(sh[0]), int(zh[0]), float(s)


def key_code_slot(t: int, c: int) -> tuple[int, int]:
    w = np.zeros(1, np.int32)
    nb = np.zeros(1, np.int32)
    lib().s4kv_ref_key_code_slot(t, c, _p(w), _p(nb))
    return int(w[0]), int(nb[0])


def value_code_slot(t: int, c: int) -> tuple[int, int]:
    w = np.zeros(1, np.int32)
    nb = np.zeros(1, np.int32)
    lib().s4kv_ref_value_code_slot(t, c, _p(w), _p(nb))
    return int(w[0]), int(nb[0])


def key_zero_slot(c: int) -> int:
    """Position (in halves, within the key-zero region) of channel c."""
    return int(lib().s4kv_ref_key_zero_slot(int(c)))


def value_scale_slot(t: int, g: int) -> int:
    """Position (in halves, within the value-scale region) of token t's scale
    for channel group g."""
    return int(lib().s4kv_ref_value_scale_slot(int(t), int(g)))


def quantize_group_bits(x, bits: int) -> tuple[np.ndarray, int, int, float]:
    """As quantize_group with (1 << bits) - 1 levels (bits = 4 or 8)."""
    xb = _u16(np.asarray(x, dtype=np.float16) if not isinstance(x, np.ndarray) or x.dtype != np.uint16 else x)
    n = xb.size
    codes = np.zeros(n, np.uint8)
    sh = np.zeros(1, np.uint16)
    zh = np.zeros(1, np.uint16)
    s = lib().s4kv_ref_quantize_group_bits(_p(xb), n, 1, _p(codes), 1, int(bits), _p(sh), _p(zh))
    return codes, int(sh[0]), int(zh[0]), float(s)


def code_offset8(is_value: bool, t: int, c: int) -> int:
    """Byte offset of (token t, channel c) in an 8-bit code region."""
    return int(lib().s4kv_ref_code_offset8(1 if is_value else 0, int(t), int(c)))


def code_position2(is_value: bool, t: int, c: int) -> tuple[int, int]:
    """(word, bit) of (token t, channel c) in a 2-bit code region."""
    w = np.zeros(1, np.int64)
    b = np.zeros(1, np.int32)
    lib().s4kv_ref_code_position2(1 if is_value else 0, int(t), int(c), _p(w), _p(b))
    return int(w[0]), int(b[0])


def quantize_page(kp, vp, bits: int = 4) -> np.ndarray:
    """fp16 K, V [16][128] of one page and kv head -> block (2816 bytes for
    4-bit codes)."""
    kb = _u16(kp).reshape(PAGE, HEAD_DIM)
    vb = _u16(vp).reshape(PAGE, HEAD_DIM)
    blk = np.zeros(block_bytes(bits), np.uint8)
    lib().s4kv_ref_quantize_page_bits(_p(np.ascontiguousarray(kb)), _p(np.ascontiguousarray(vb)), _p(blk), bits)
    return blk


def unpack_codes(block: np.ndarray, bits: int = 4) -> tuple[np.ndarray, np.ndarray]:
    block = np.ascontiguousarray(block, dtype=np.uint8)
    kc = np.zeros((PAGE, HEAD_DIM), np.uint8)
    vc = np.zeros((PAGE, HEAD_DIM), np.uint8)
    lib().s4kv_ref_unpack_codes_bits(_p(block), _p(kc), _p(vc), bits)
    return kc, vc


def dequant_block(block: np.ndarray, bits: int = 4) -> tuple[np.ndarray, np.ndarray]:
    block = np.ascontiguousarray(block, dtype=np.uint8)
    k = np.zeros((PAGE, HEAD_DIM), np.float32)
    v = np.zeros((PAGE, HEAD_DIM), np.float32)
    lib().s4kv_ref_dequant_block_bits(_p(block), _p(k), _p(v), bits)
    return k, v


def block_bytes(bits: int = 4) -> int:
    return int(lib().s4kv_ref_block_bytes_bits(int(bits)))


def kv_payload_bytes(layers, kv_heads, head_dim, tokens, bytes_per_elem) -> float:
    return float(lib().s4kv_ref_kv_payload_bytes(layers, kv_heads, head_dim, tokens, bytes_per_elem))


# ----------------------------------------------------------------- cache --

class OracleCache:
    """Host copy of the paged cache: pool u8 [NP][Hkv][block bytes] (1792 for
    2-bit codes, 2816 for 4-bit, 4864 for 8-bit), residual fp16 bits
    [max_seqs][Hkv][16][128] for K and V."""

    def __init__(self, num_pages: int, num_kv_heads: int, max_seqs: int, bits: int = 4):
        assert bits in (2, 4, 8)
        self.bits = bits
        self.num_pages = num_pages
        self.num_kv_heads = num_kv_heads
        self.max_seqs = max_seqs
        self.pool = np.zeros((num_pages, num_kv_heads, block_bytes(bits)), np.uint8)
        self.res_k = np.zeros((max_seqs, num_kv_heads, PAGE, HEAD_DIM), np.uint16)
        self.res_v = np.zeros((max_seqs, num_kv_heads, PAGE, HEAD_DIM), np.uint16)

    def append(self, k, v, slot_mapping, cu_new, seq_lens, block_tables) -> int:
        kb = np.ascontiguousarray(_u16(k))
        vb = np.ascontiguousarray(_u16(v))
        sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        cu = np.ascontiguousarray(cu_new, dtype=np.int32)
        sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        batch, max_pages = bt.shape
        n_tokens = int(cu[-1]) if cu.size else 0
        return int(lib().s4kv_ref_append_bits(
            _p(self.pool), _p(self.res_k), _p(self.res_v), self.num_pages,
            self.num_kv_heads, self.max_seqs, _p(kb), _p(vb), n_tokens, _p(sm),
            _p(cu), _p(sl), _p(bt), batch, max_pages, self.bits))

    def dequant_page(self, physical_page: int) -> tuple[np.ndarray, np.ndarray]:
        ok = np.zeros((self.num_kv_heads, PAGE, HEAD_DIM), np.float32)
        ov = np.zeros((self.num_kv_heads, PAGE, HEAD_DIM), np.float32)
        rc = lib().s4kv_ref_dequant_page_bits(_p(self.pool), self.num_pages, self.num_kv_heads,
                                              physical_page, _p(ok), _p(ov), self.bits)
        if rc != 0:
            raise ValueError(f"dequant_page rc={rc}")
        return ok, ov

    def decode_attention(self, q, seq_lens, block_tables, sm_scale=None,
                         use_double=True) -> np.ndarray:
        qb = np.ascontiguousarray(_u16(q))
        batch, num_q_heads, d = qb.shape
        assert d == HEAD_DIM
        sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        if sm_scale is None:
            sm_scale = 1.0 / np.sqrt(HEAD_DIM)
        out = np.zeros((batch, num_q_heads, HEAD_DIM), np.float64)
        rc = lib().s4kv_ref_decode_attention(
            _p(self.pool), _p(self.res_k), _p(self.res_v), self.num_pages,
            self.num_kv_heads, _p(qb), num_q_heads, _p(sl), _p(bt), batch,
            bt.shape[1], float(sm_scale), 1 if use_double else 0, _p(out), self.bits)
        if rc != 0:
            raise ValueError(f"decode_attention rc={rc}")
        return out

    def gather_pages(self, pages) -> np.ndarray:
        """Page records of the listed physical pages: u8 [n][kv_heads][block bytes]."""
        pg = np.ascontiguousarray(pages, dtype=np.int32)
        out = np.zeros((len(pg), self.num_kv_heads, block_bytes(self.bits)), np.uint8)
        rc = lib().s4kv_ref_gather_pages(_p(self.pool), self.num_pages, self.num_kv_heads, _p(pg), len(pg), _p(out),
                                        self.bits)
        if rc != 0:
            raise ValueError(f"gather_pages rc={rc}")
        return out

    def scatter_pages(self, pages, records) -> None:
        pg = np.ascontiguousarray(pages, dtype=np.int32)
        rec = np.ascontiguousarray(records, dtype=np.uint8)
        rc = lib().s4kv_ref_scatter_pages(_p(self.pool), self.num_pages, self.num_kv_heads, _p(pg), len(pg), _p(rec),
                                         self.bits)
        if rc != 0:
            raise ValueError(f"scatter_pages rc={rc}")

    def copy_pages(self, src_pages, dst_pages) -> None:
        s_ = np.ascontiguousarray(src_pages, dtype=np.int32)
        d_ = np.ascontiguousarray(dst_pages, dtype=np.int32)
        rc = lib().s4kv_ref_copy_pages(_p(self.pool), self.num_pages, self.num_kv_heads, _p(s_), _p(d_), len(s_),
                                      self.bits)
        if rc != 0:
            raise ValueError(f"copy_pages rc={rc}")

    def fork_residual(self, src_rows, dst_rows) -> None:
        s_ = np.ascontiguousarray(src_rows, dtype=np.int32)
        d_ = np.ascontiguousarray(dst_rows, dtype=np.int32)
        rc = lib().s4kv_ref_fork_residual(_p(self.res_k), _p(self.res_v), self.max_seqs, self.num_kv_heads,
                                         _p(s_), _p(d_), len(s_))
        if rc != 0:
            raise ValueError(f"fork_residual rc={rc}")

    def prefill_attention(self, q, cu_new, seq_lens, block_tables, sm_scale=None) -> np.ndarray:
        """Causal attention of the appended chunk's query rows (q: fp16
        [n_tokens][num_q_heads][128], sequence b owning rows cu_new[b]..)
        over the cache after the append; fp64 [n_tokens][num_q_heads][128]."""
        qb = np.ascontiguousarray(_u16(q))
        n_tokens, num_q_heads, d = qb.shape
        assert d == HEAD_DIM
        cu = np.ascontiguousarray(cu_new, dtype=np.int32)
        sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        if sm_scale is None:
            sm_scale = 1.0 / np.sqrt(HEAD_DIM)
        out = np.zeros((n_tokens, num_q_heads, HEAD_DIM), np.float64)
        rc = lib().s4kv_ref_prefill_attention(
            _p(self.pool), _p(self.res_k), _p(self.res_v), self.num_pages,
            self.num_kv_heads, _p(qb), num_q_heads, _p(cu), _p(sl), _p(bt),
            len(sl), bt.shape[1], float(sm_scale), _p(out), self.bits)
        if rc != 0:
            raise ValueError(f"prefill_attention rc={rc}")
        return out

    def attention_at(self, q_row, b: int, L: int, pos: int, bt_row, sm_scale=None) -> np.ndarray:
        """One query row (fp16 [num_q_heads][128]) of batch row b at position
        pos < L over the cache with L tokens (tokens 0..pos): the view that
        row has inside a chunked prefill; fp64 [num_q_heads][128]."""
        qb = np.ascontiguousarray(_u16(q_row))
        num_q_heads, d = qb.shape
        assert d == HEAD_DIM
        bt = np.ascontiguousarray(bt_row, dtype=np.int32).ravel()
        if sm_scale is None:
            sm_scale = 1.0 / np.sqrt(HEAD_DIM)
        out = np.zeros((num_q_heads, HEAD_DIM), np.float64)
        rc = lib().s4kv_ref_attention_at(
            _p(self.pool), _p(self.res_k), _p(self.res_v), self.num_pages, self.num_kv_heads, _p(qb),
            num_q_heads, int(L), int(pos), _p(bt), bt.size, int(b), float(sm_scale), _p(out), self.bits)
        if rc != 0:
            raise ValueError(f"attention_at rc={rc}")
        return out


def attention_fp16(k, v, cu, num_kv_heads, q, sm_scale=None) -> np.ndarray:
    """Attention on unquantized fp16 K/V (token-major, sequences by ``cu``)."""
    kb = np.ascontiguousarray(_u16(k))
    vb = np.ascontiguousarray(_u16(v))
    qb = np.ascontiguousarray(_u16(q))
    cu = np.ascontiguousarray(cu, dtype=np.int32)
    batch, num_q_heads, _ = qb.shape
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(HEAD_DIM)
    out = np.zeros((batch, num_q_heads, HEAD_DIM), np.float64)
    rc = lib().s4kv_ref_attention_fp16(_p(kb), _p(vb), _p(cu), num_kv_heads, _p(qb),
                                       num_q_heads, batch, float(sm_scale), _p(out))
    if rc != 0:
        raise ValueError(f"attention_fp16 rc={rc}")
    return out
