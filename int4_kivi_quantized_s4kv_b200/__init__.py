"""Python binding of the s4kv C ABI (``include/s4kv.h``).

Argument marshalling only: every step of the path runs in the CUDA kernels
of ``libs4kv.so``.  PyTorch provides device memory and streams.  There is no
CPU fallback: the first call raises if the library is missing.

    cache = S4KVCache(num_pages, num_kv_heads, max_seqs, device="cuda")
    s4kv_append(cache, k, v, slot_mapping, cu_new, seq_lens, block_tables, max_new)
    ws = decode_workspace(batch, num_kv_heads, device)
    s4kv_decode_attention(cache, q, seq_lens, block_tables, out, ws)
"""
from __future__ import annotations

import ctypes
import os

HEAD_DIM = 128
PAGE_TOKENS = 16
VALUE_GROUP = 32
BLOCK_BYTES = 2816
BLOCK_BYTES_INT8 = 4864
BLOCK_BYTES_INT2 = 1792
MAX_GQA_GROUP = 8
NOALLOC_SCRATCH_BYTES = 24 * 1024 * 1024

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_DEVICE_CHECK, ERR_WORKSPACE = range(6)
EFLAG_PAGE_RANGE, EFLAG_SLOT, EFLAG_SEQ_LEN, EFLAG_TIMEOUT = 1, 2, 4, 8

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libs4kv.so")

class s4kv_cache_t(ctypes.Structure):
    _fields_ = [("pool", ctypes.c_void_p), ("res_k", ctypes.c_void_p), ("res_v", ctypes.c_void_p),
                ("err_flag", ctypes.c_void_p), ("num_pages", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("max_seqs", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_tokens", ctypes.c_int32), ("bits", ctypes.c_int32)]


_P, _I, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_CP = ctypes.POINTER(s4kv_cache_t)
_SIGS = {
    "s4kv_version": ([], _I),
    "s4kv_status_string": ([_I], ctypes.c_char_p),
    "s4kv_check_model": ([_I, _I, _I, _I], _I),
    "s4kv_cache_layout": ([_I, _I, _I, ctypes.POINTER(_SZ), ctypes.POINTER(_SZ)], _I),
    "s4kv_cache_layout_bits": ([_I, _I, _I, _I, ctypes.POINTER(_SZ), ctypes.POINTER(_SZ)], _I),
    "s4kv_append": ([_CP, _P, _P, _I, _P, _P, _P, _P, _I, _I, _I, _P], _I),
    "s4kv_decode_workspace_size": ([_I, _I, ctypes.POINTER(_SZ)], _I),
    "s4kv_decode_attention": ([_CP, _P, _I, _P, _P, _I, _I, ctypes.c_float, _P, _P, _SZ, _P], _I),
    "s4kv_decode_attention_noalloc": ([_CP, _P, _I, _P, _P, _I, _I, ctypes.c_float, _P, _P], _I),
    "s4kv_append_decode": ([_CP, _P, _P, _P, _I, _P, _P, _I, _I, ctypes.c_float, _P, _P, _SZ, _P], _I),
    "s4kv_prefill_attention": ([_CP, _P, _I, _I, _P, _P, _P, _I, _I, _I, ctypes.c_float, _P, _P, _SZ, _P], _I),
    "s4kv_prefill_workspace_size": ([_I, _I, _I, ctypes.POINTER(_SZ)], _I),
    "s4kv_dequant_page": ([_CP, _I, _P, _P, _I, _P], _I),
    "s4kv_dequant_pages": ([_CP, _P, _I, _P, _P, _I, _P], _I),
    "s4kv_page_record_bytes": ([_CP, ctypes.POINTER(_SZ)], _I),
    "s4kv_gather_pages": ([_CP, _P, _I, _P, _P], _I),
    "s4kv_scatter_pages": ([_CP, _P, _I, _P, _P], _I),
    "s4kv_copy_pages": ([_CP, _P, _P, _I, _P], _I),
    "s4kv_fork_residual": ([_CP, _P, _P, _I, _P], _I),
    "s4kv_swap_out": ([_CP, _P, _I, _P, _P, _P], _I),
    "s4kv_swap_in": ([_CP, _P, _I, _P, _P, _P], _I),
    "s4kv_get_error": ([_CP, ctypes.POINTER(ctypes.c_uint32), _I, _P], _I),
}
EXPORTED = tuple(_SIGS)
_lib = None


def lib():
    """The loaded libs4kv.so; raises if it was not built (no CPU fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m int4_kivi_quantized_s4kv_b200.build` "
                "(there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


class S4KVError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {s4kv_status_string(status)} (status {status})")


def _check(status: int, what: str):
    if status != OK:
        raise S4KVError(status, what)


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t, dtype=None, name="tensor"):
    if t is None:
        return None
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


# ------------------------------------------------------------ host calls --

def s4kv_version() -> int:
    return lib().s4kv_version()


def s4kv_status_string(status: int) -> str:
    return lib().s4kv_status_string(status).decode()


def s4kv_check_model(head_dim: int, page_tokens: int, num_q_heads: int, num_kv_heads: int) -> int:
    return lib().s4kv_check_model(head_dim, page_tokens, num_q_heads, num_kv_heads)


def s4kv_cache_layout(num_pages: int, num_kv_heads: int, max_seqs: int, bits: int = 4) -> tuple[int, int]:
    pb, rb = _SZ(0), _SZ(0)
    _check(lib().s4kv_cache_layout_bits(num_pages, num_kv_heads, max_seqs, bits, ctypes.byref(pb),
                                        ctypes.byref(rb)), "s4kv_cache_layout_bits")
    return pb.value, rb.value


def s4kv_decode_workspace_size(batch: int, num_kv_heads: int) -> int:
    n = _SZ(0)
    _check(lib().s4kv_decode_workspace_size(batch, num_kv_heads, ctypes.byref(n)), "s4kv_decode_workspace_size")
    return n.value


# ----------------------------------------------------------------- cache --

class S4KVCache:
    """Caller-owned device memory of one layer's cache (torch tensors) and the
    plain C descriptor the library reads."""

    def __init__(self, num_pages: int, num_kv_heads: int, max_seqs: int, device="cuda", bits: int = 4):
        import torch
        pool_bytes, res_bytes = s4kv_cache_layout(num_pages, num_kv_heads, max_seqs, bits)
        self.num_pages, self.num_kv_heads, self.max_seqs, self.bits = num_pages, num_kv_heads, max_seqs, bits
        block = {4: BLOCK_BYTES, 8: BLOCK_BYTES_INT8, 2: BLOCK_BYTES_INT2}[bits]
        self.pool = torch.zeros((num_pages, num_kv_heads, block), dtype=torch.uint8, device=device)
        self.res_k = torch.zeros((max_seqs, num_kv_heads, PAGE_TOKENS, HEAD_DIM), dtype=torch.float16, device=device)
        self.res_v = torch.zeros_like(self.res_k)
        self.err_flag = torch.zeros(1, dtype=torch.int32, device=device)
        assert self.pool.numel() == pool_bytes and self.res_k.numel() * 2 == res_bytes
        self.c = s4kv_cache_t(self.pool.data_ptr(), self.res_k.data_ptr(), self.res_v.data_ptr(),
                              self.err_flag.data_ptr(), num_pages, num_kv_heads, max_seqs,
                              HEAD_DIM, PAGE_TOKENS, bits)

    @property
    def ref(self):
        return ctypes.byref(self.c)


def decode_workspace(batch: int, num_kv_heads: int, device="cuda"):
    """Zero-filled workspace of the size s4kv_decode_attention needs."""
    import torch
    n = s4kv_decode_workspace_size(batch, num_kv_heads)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device)


# ----------------------------------------------------------- device calls --

def s4kv_append(cache: S4KVCache, k, v, slot_mapping, cu_new, seq_lens, block_tables,
                max_new_per_seq: int, stream=None):
    import torch
    batch, max_pages = block_tables.shape
    n_tokens = k.shape[0]
    st = lib().s4kv_append(cache.ref, _ptr(k, torch.float16, "k"), _ptr(v, torch.float16, "v"), n_tokens,
                          _ptr(slot_mapping, torch.int64, "slot_mapping"), _ptr(cu_new, torch.int32, "cu_new"),
                          _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(block_tables, torch.int32, "block_tables"),
                          batch, max_pages, int(max_new_per_seq), _stream(stream))
    _check(st, "s4kv_append")


def s4kv_decode_attention(cache: S4KVCache, q, seq_lens, block_tables, out, workspace,
                          sm_scale: float | None = None, stream=None):
    import torch
    batch, num_q_heads, _ = q.shape
    if sm_scale is None:
        sm_scale = HEAD_DIM ** -0.5
    st = lib().s4kv_decode_attention(cache.ref, _ptr(q, torch.float16, "q"), num_q_heads,
                                    _ptr(seq_lens, torch.int32, "seq_lens"),
                                    _ptr(block_tables, torch.int32, "block_tables"), batch,
                                    block_tables.shape[1], float(sm_scale), _ptr(out, torch.float16, "out"),
                                    _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                                    _stream(stream))
    _check(st, "s4kv_decode_attention")


def s4kv_append_decode(cache: S4KVCache, k_new, v_new, q, seq_lens, block_tables, out, workspace,
                       sm_scale: float | None = None, stream=None):
    """One decode step in one call: append each sequence's new token
    (k_new, v_new fp16 [batch][kv_heads][128]) and attend over the result
    (an append grid, then the decode grid as its programmatic dependent)."""
    import torch
    batch, num_q_heads, _ = q.shape
    if sm_scale is None:
        sm_scale = HEAD_DIM ** -0.5
    st = lib().s4kv_append_decode(cache.ref, _ptr(k_new, torch.float16, "k_new"), _ptr(v_new, torch.float16, "v_new"),
                                 _ptr(q, torch.float16, "q"), num_q_heads,
                                 _ptr(seq_lens, torch.int32, "seq_lens"),
                                 _ptr(block_tables, torch.int32, "block_tables"), batch, block_tables.shape[1],
                                 float(sm_scale), _ptr(out, torch.float16, "out"),
                                 _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream))
    _check(st, "s4kv_append_decode")


def s4kv_decode_attention_noalloc(cache: S4KVCache, q, seq_lens, block_tables, out,
                                  sm_scale: float | None = None, stream=None):
    """Decode attention for callers that cannot allocate device memory: the
    scratch is a fixed 24 MiB array inside the library (shared by all calls
    on a device; overlapping calls race)."""
    import torch
    batch, num_q_heads, _ = q.shape
    if sm_scale is None:
        sm_scale = HEAD_DIM ** -0.5
    st = lib().s4kv_decode_attention_noalloc(cache.ref, _ptr(q, torch.float16, "q"), num_q_heads,
                                            _ptr(seq_lens, torch.int32, "seq_lens"),
                                            _ptr(block_tables, torch.int32, "block_tables"), batch,
                                            block_tables.shape[1], float(sm_scale),
                                            _ptr(out, torch.float16, "out"), _stream(stream))
    _check(st, "s4kv_decode_attention_noalloc")


def prefill_workspace_bytes(num_kv_heads: int, batch: int, max_pages_per_seq: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().s4kv_prefill_workspace_size(num_kv_heads, batch, max_pages_per_seq, ctypes.byref(n)),
           "s4kv_prefill_workspace_size")
    return n.value


def prefill_workspace(num_kv_heads: int, batch: int, max_pages_per_seq: int, device="cuda"):
    """Device scratch for s4kv_prefill_attention (uint8)."""
    import torch
    return torch.empty(prefill_workspace_bytes(num_kv_heads, batch, max_pages_per_seq), dtype=torch.uint8,
                       device=device)


def s4kv_prefill_attention(cache: S4KVCache, q, cu_new, seq_lens, block_tables, out,
                           max_new_per_seq: int, sm_scale: float | None = None, workspace=None, stream=None):
    """Causal attention of the appended chunk's query rows (q: fp16
    [n_tokens][num_q_heads][128], sequence b owning rows cu_new[b]..) over the
    cache after s4kv_append wrote the chunk; fills out [n_tokens][num_q_heads][128].
    `workspace` (from prefill_workspace) is allocated per call when omitted."""
    import torch
    n_tokens, num_q_heads, _ = q.shape
    if sm_scale is None:
        sm_scale = HEAD_DIM ** -0.5
    batch, max_pages = seq_lens.shape[0], block_tables.shape[1]
    if workspace is None:
        workspace = prefill_workspace(cache.num_kv_heads, max(batch, 1), max_pages, q.device)
    st = lib().s4kv_prefill_attention(cache.ref, _ptr(q, torch.float16, "q"), num_q_heads, n_tokens,
                                     _ptr(cu_new, torch.int32, "cu_new"),
                                     _ptr(seq_lens, torch.int32, "seq_lens"),
                                     _ptr(block_tables, torch.int32, "block_tables"), batch,
                                     max_pages, int(max_new_per_seq), float(sm_scale),
                                     _ptr(out, torch.float16, "out"), _ptr(workspace, torch.uint8, "workspace"),
                                     workspace.numel(), _stream(stream))
    _check(st, "s4kv_prefill_attention")


def s4kv_dequant_page(cache: S4KVCache, physical_page: int, out_k, out_v, out_fp32: bool = True,
                      stream=None):
    st = lib().s4kv_dequant_page(cache.ref, int(physical_page), _ptr(out_k), _ptr(out_v),
                                1 if out_fp32 else 0, _stream(stream))
    _check(st, "s4kv_dequant_page")


def s4kv_dequant_pages(cache: S4KVCache, pages, out_k, out_v, out_fp32: bool = True, stream=None):
    import torch
    st = lib().s4kv_dequant_pages(cache.ref, _ptr(pages, torch.int32, "pages"), pages.numel(), _ptr(out_k),
                                 _ptr(out_v), 1 if out_fp32 else 0, _stream(stream))
    _check(st, "s4kv_dequant_pages")


def s4kv_page_record_bytes(cache: S4KVCache) -> int:
    n = _SZ(0)
    _check(lib().s4kv_page_record_bytes(cache.ref, ctypes.byref(n)), "s4kv_page_record_bytes")
    return n.value


def s4kv_gather_pages(cache: S4KVCache, pages, dst, stream=None):
    import torch
    st = lib().s4kv_gather_pages(cache.ref, _ptr(pages, torch.int32, "pages"), pages.numel(),
                                _ptr(dst, torch.uint8, "dst"), _stream(stream))
    _check(st, "s4kv_gather_pages")


def s4kv_scatter_pages(cache: S4KVCache, pages, src, stream=None):
    import torch
    st = lib().s4kv_scatter_pages(cache.ref, _ptr(pages, torch.int32, "pages"), pages.numel(),
                                 _ptr(src, torch.uint8, "src"), _stream(stream))
    _check(st, "s4kv_scatter_pages")


def s4kv_copy_pages(cache: S4KVCache, src_pages, dst_pages, stream=None):
    import torch
    st = lib().s4kv_copy_pages(cache.ref, _ptr(src_pages, torch.int32, "src_pages"),
                              _ptr(dst_pages, torch.int32, "dst_pages"), src_pages.numel(), _stream(stream))
    _check(st, "s4kv_copy_pages")


def s4kv_fork_residual(cache: S4KVCache, src_rows, dst_rows, stream=None):
    import torch
    st = lib().s4kv_fork_residual(cache.ref, _ptr(src_rows, torch.int32, "src_rows"),
                                 _ptr(dst_rows, torch.int32, "dst_rows"), src_rows.numel(), _stream(stream))
    _check(st, "s4kv_fork_residual")


def s4kv_swap_out(cache: S4KVCache, pages, staging, host_dst, stream=None):
    """Gather the pages' records into `staging` (device) and copy them to
    `host_dst` (pinned host uint8 tensor of the same size)."""
    import torch
    st = lib().s4kv_swap_out(cache.ref, _ptr(pages, torch.int32, "pages"), pages.numel(),
                            _ptr(staging, torch.uint8, "staging"), ctypes.c_void_p(host_dst.data_ptr()),
                            _stream(stream))
    _check(st, "s4kv_swap_out")


def s4kv_swap_in(cache: S4KVCache, pages, staging, host_src, stream=None):
    import torch
    st = lib().s4kv_swap_in(cache.ref, _ptr(pages, torch.int32, "pages"), pages.numel(),
                           _ptr(staging, torch.uint8, "staging"), ctypes.c_void_p(host_src.data_ptr()),
                           _stream(stream))
    _check(st, "s4kv_swap_in")


def s4kv_get_error(cache: S4KVCache, clear: bool = True, stream=None) -> int:
    flags = ctypes.c_uint32(0)
    st = lib().s4kv_get_error(cache.ref, ctypes.byref(flags), 1 if clear else 0, _stream(stream))
    if st not in (OK, ERR_DEVICE_CHECK):
        raise S4KVError(st, "s4kv_get_error")
    return flags.value
