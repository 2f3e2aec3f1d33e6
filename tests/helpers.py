"""Shared test plumbing: build the same cache through the CUDA path and the
oracle from identical seeded inputs, and compare.

Parity bars:
  * pool bytes, residual rows and dequantized fp32 pages: bit-exact;
  * decode attention: |gpu - oracle| <= ATOL + RTOL * |oracle| element-wise
    against the fp64 oracle on the same dequantized cache.
"""
from __future__ import annotations

import numpy as np

from int4_kivi_quantized_s4kv_b200 import workloads as W

ATOL = 2e-3
RTOL = 1e-3
PAGE = 16


def assert_attention_close(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                           f"max abs {err.max():.3g}, worst excess {(err - bound).max():.3g}")
    return float(err.max())


def append_batches(positions_before, positions_after, k_streams, v_streams, block_tables, chunk=None):
    """Yield (k, v, slot_mapping, cu_new, seq_lens, max_new) for appending
    tokens [before, after) of every sequence, `chunk` tokens per call."""
    cur = np.array(positions_before, np.int64)
    tgt = np.array(positions_after, np.int64)
    while (cur < tgt).any():
        take = tgt - cur if chunk is None else np.minimum(tgt - cur, chunk)
        ks, vs, pos_list = [], [], []
        for b in range(len(cur)):
            pos = np.arange(cur[b], cur[b] + take[b])
            pos_list.append(pos)
            ks.append(k_streams[b][pos])
            vs.append(v_streams[b][pos])
        H = k_streams[0].shape[1]
        k = np.concatenate(ks) if ks else np.zeros((0, H, 128), np.float16)
        v = np.concatenate(vs) if vs else np.zeros((0, H, 128), np.float16)
        sm = W.slot_mapping(block_tables, pos_list)
        cu = np.concatenate([[0], np.cumsum(take)]).astype(np.int32)
        yield k, v, sm, cu, (cur + take).astype(np.int32), int(take.max())
        cur = cur + take


class Pair:
    """One layer's cache built on the GPU and in the oracle from the same
    inputs (numpy backend)."""

    def __init__(self, spec: W.Spec, layer: int = 0, prefill_chunk=None, device="cuda",
                 with_gpu=True, bits: int = 4):
        import oracle
        self.spec, self.layer = spec, layer
        self.ctx = W.context_lens(spec)
        self.lens = W.final_lens(spec)
        self.plan = W.page_plan(spec)
        B, H = spec.batch, spec.num_kv_heads
        self.k = []
        self.v = []
        for b in range(B):
            kk, vv = W.kv_sequence_np(spec, layer, b, int(self.lens[b]))
            self.k.append(kk)
            self.v.append(vv)
        self.q = W.queries_np(spec, layer)
        self.bits = bits
        self.oc = oracle.OracleCache(self.plan.num_pages, H, B, bits=bits)
        self.gpu = None
        self.device = device
        if with_gpu:
            import int4_kivi_quantized_s4kv_b200 as S
            self.S = S
            self.gpu = S.S4KVCache(self.plan.num_pages, H, B, device=device, bits=bits)
            self.bt_dev = self._dev(self.plan.block_tables)
        self.append(np.zeros(B, np.int64), self.ctx, prefill_chunk)
        self.append(self.ctx, self.lens, None)

    def _dev(self, a):
        import torch
        return torch.from_numpy(np.ascontiguousarray(a)).to(self.device)

    def append(self, before, after, chunk):
        for k, v, sm, cu, sl, mx in append_batches(before, after, self.k, self.v,
                                                    self.plan.block_tables, chunk):
            rc = self.oc.append(k, v, sm, cu, sl, self.plan.block_tables)
            assert rc == 0
            if self.gpu is not None:
                self.S.s4kv_append(self.gpu, self._dev(k), self._dev(v), self._dev(sm), self._dev(cu),
                                   self._dev(sl), self.bt_dev, mx)

    def gpu_decode(self, q=None, sm_scale=None):
        import torch
        S = self.S
        q = self.q if q is None else q
        qd = self._dev(q)
        out = torch.empty_like(qd)
        ws = S.decode_workspace(self.spec.batch, self.spec.num_kv_heads, self.device)
        S.s4kv_decode_attention(self.gpu, qd, self._dev(self.lens), self.bt_dev, out, ws, sm_scale)
        torch.cuda.synchronize()
        return out.float().cpu().numpy()

    def oracle_decode(self, q=None, sm_scale=None):
        q = self.q if q is None else q
        return self.oc.decode_attention(q, self.lens, self.plan.block_tables, sm_scale)

    def assert_cache_bit_exact(self):
        import torch
        torch.cuda.synchronize()
        pool = self.gpu.pool.cpu().numpy()
        assert np.array_equal(pool, self.oc.pool), "pool bytes differ"
        rk = self.gpu.res_k.cpu().numpy().view(np.uint16)
        rv = self.gpu.res_v.cpu().numpy().view(np.uint16)
        for b, L in enumerate(self.lens):
            r = int(L) % PAGE
            assert np.array_equal(rk[b, :, :r], self.oc.res_k[b, :, :r]), f"res_k seq {b}"
            assert np.array_equal(rv[b, :, :r], self.oc.res_v[b, :, :r]), f"res_v seq {b}"
        assert self.S.s4kv_get_error(self.gpu) == 0
