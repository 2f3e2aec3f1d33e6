"""GPU parity of s4kv_append_decode (one decode step in one call: the
append of one token per sequence, then decode attention as a grid that
depends on the append's) against the oracle's append-then-decode, through
the C ABI.  The cache after the step must
be byte-identical to the oracle's, the output within the decode tolerance,
and the output bit-identical to the GPU's own two-launch path."""
import dataclasses

import numpy as np
import pytest

from helpers import append_batches, assert_attention_close
from int4_kivi_quantized_s4kv_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _run(spec, context_chunk=64):
    import torch
    import oracle
    import int4_kivi_quantized_s4kv_b200 as S
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    ctx = W.context_lens(spec)
    lens = W.final_lens(spec)
    plan = W.page_plan(spec)
    B, H = spec.batch, spec.num_kv_heads
    k, v = [], []
    for b in range(B):
        kk, vv = W.kv_sequence_np(spec, 0, b, int(lens[b]))
        k.append(kk)
        v.append(vv)
    q = W.queries_np(spec, 0)
    bt = plan.block_tables
    oc = oracle.OracleCache(plan.num_pages, H, B)
    fused = S.S4KVCache(plan.num_pages, H, B)
    plain = S.S4KVCache(plan.num_pages, H, B)
    bt_dev = dev(bt)
    for kk, vv, sm, cu, sl, mx in append_batches(np.zeros(B, np.int64), ctx, k, v, bt, context_chunk):
        assert oc.append(kk, vv, sm, cu, sl, bt) == 0
        for c in (fused, plain):
            S.s4kv_append(c, dev(kk), dev(vv), dev(sm), dev(cu), dev(sl), bt_dev, mx)
    # the step: one token per sequence
    for kk, vv, sm, cu, sl, mx in append_batches(ctx, lens, k, v, bt, None):
        assert oc.append(kk, vv, sm, cu, sl, bt) == 0
        S.s4kv_append(plain, dev(kk), dev(vv), dev(sm), dev(cu), dev(sl), bt_dev, mx)
    k_new = np.stack([k[b][int(lens[b]) - 1] for b in range(B)])
    v_new = np.stack([v[b][int(lens[b]) - 1] for b in range(B)])
    ws = S.decode_workspace(B, H)
    qd = dev(q)
    out_f = torch.empty_like(qd)
    out_p = torch.empty_like(qd)
    S.s4kv_append_decode(fused, dev(k_new), dev(v_new), qd, dev(lens), bt_dev, out_f, ws)
    S.s4kv_decode_attention(plain, qd, dev(lens), bt_dev, out_p, ws)
    torch.cuda.synchronize()
    assert S.s4kv_get_error(fused) == 0 and S.s4kv_get_error(plain) == 0
    assert np.array_equal(fused.pool.cpu().numpy(), oc.pool), "pool bytes differ from the oracle"
    rk = fused.res_k.cpu().numpy().view(np.uint16)
    rv = fused.res_v.cpu().numpy().view(np.uint16)
    for b, L in enumerate(lens):
        r = int(L) % 16
        assert np.array_equal(rk[b, :, :r], oc.res_k[b, :, :r]), f"res_k row {b}"
        assert np.array_equal(rv[b, :, :r], oc.res_v[b, :, :r]), f"res_v row {b}"
    got = out_f.float().cpu().numpy()
    assert np.array_equal(got, out_p.float().cpu().numpy())
    assert_attention_close(got, oc.decode_attention(q, lens, bt), spec.name)


def test_fused_step_completes_and_starts_pages():
    # after the step: 16, 32 and 48 tokens complete a page inside the kernel;
    # 1 is a sequence's very first token; 17, 101, 201 land in the residual
    spec = dataclasses.replace(W.SPECS["llama3.2-3b-step"], name="fused-mix", layers=1, batch=7,
                               ctx_kind="fixed", ctx_fixed=(15, 31, 16, 100, 47, 200, 0), step_new=(1,))
    _run(spec)


def test_fused_step_every_segment_completes_a_page():
    # every (sequence, kv head) completes a page: each append CTA quantizes
    # the most pages it can hold, one after the other
    ctx = tuple(16 * (1 + (b * 7) % 9) - 1 for b in range(40))
    spec = dataclasses.replace(W.SPECS["llama3.2-3b-step"], name="fused-fills", layers=1, batch=len(ctx),
                               ctx_kind="fixed", ctx_fixed=ctx, step_new=(1,))
    _run(spec)


def test_fused_step_many_sequences():
    # many short segments per worker: the fused appends are spread over workers
    spec = W.scaled(W.SPECS["llama3.2-3b-step"], batch=96, layers=1, ctx_scale=0.05)
    _run(spec, context_chunk=512)


def test_fused_step_long_contexts():
    spec = W.scaled(W.SPECS["llama3.1-8b"], batch=6, ctx_scale=0.5)
    spec = dataclasses.replace(spec, ctx_fixed=(4095, 4096, 4111, 1023, 2047, 3000))
    _run(spec, context_chunk=1024)


def test_rounding_ties_through_both_append_paths():
    """Groups whose quotients (x - min) / scale are exact half-integers: the
    code is then decided by round-half-to-even on the exact quotient.  Both
    the append kernel and the fused step must write the oracle's bytes."""
    spec = dataclasses.replace(W.SPECS["llama3.2-3b-step"], name="ties", layers=1, batch=3,
                               ctx_kind="fixed", ctx_fixed=(15, 47, 31), step_new=(1,), outlier_frac=0.0)
    import torch
    import oracle
    import int4_kivi_quantized_s4kv_b200 as S
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    rng = np.random.default_rng(77)
    lens = W.final_lens(spec)
    ctx = W.context_lens(spec)
    plan = W.page_plan(spec)
    B, H = spec.batch, spec.num_kv_heads
    k, v = [], []
    for b in range(B):
        L = int(lens[b])
        # per page and channel: the scale is exactly 1 (values 0 and 15 present)
        # and the other values sit on k + 1/2, with a random offset and sign
        grid = np.concatenate([[0.0, 15.0], np.arange(14) + 0.5])
        kk = np.empty((L, H, 128), np.float64)
        vv = np.empty((L, H, 128), np.float64)
        for p0 in range(0, L, 16):
            n = min(16, L - p0)
            for h in range(H):
                for c in range(128):
                    kk[p0:p0 + n, h, c] = rng.permutation(grid)[:n] + rng.integers(-8, 8)
                for t in range(n):
                    row = np.concatenate([rng.permutation(np.concatenate([[0.0, 15.0], (np.arange(30) % 14) + 0.5]))
                                          for _ in range(4)])
                    vv[p0 + t, h] = row - rng.integers(0, 4)
        k.append(kk.astype(np.float16))
        v.append(vv.astype(np.float16))
    bt = plan.block_tables
    oc = oracle.OracleCache(plan.num_pages, H, B)
    plain = S.S4KVCache(plan.num_pages, H, B)
    fused = S.S4KVCache(plan.num_pages, H, B)
    bt_dev = dev(bt)
    for kk, vv, sm, cu, sl, mx in append_batches(np.zeros(B, np.int64), ctx, k, v, bt, 7):
        assert oc.append(kk, vv, sm, cu, sl, bt) == 0
        for c in (plain, fused):
            S.s4kv_append(c, dev(kk), dev(vv), dev(sm), dev(cu), dev(sl), bt_dev, mx)
    for kk, vv, sm, cu, sl, mx in append_batches(ctx, lens, k, v, bt, None):
        assert oc.append(kk, vv, sm, cu, sl, bt) == 0
        S.s4kv_append(plain, dev(kk), dev(vv), dev(sm), dev(cu), dev(sl), bt_dev, mx)
    k_new = np.stack([k[b][int(lens[b]) - 1] for b in range(B)])
    v_new = np.stack([v[b][int(lens[b]) - 1] for b in range(B)])
    q = W.queries_np(spec, 0)
    out = torch.empty((B, spec.num_q_heads, 128), dtype=torch.float16, device="cuda")
    S.s4kv_append_decode(fused, dev(k_new), dev(v_new), dev(q), dev(lens), bt_dev, out, S.decode_workspace(B, H))
    torch.cuda.synchronize()
    assert np.array_equal(plain.pool.cpu().numpy(), oc.pool)
    assert np.array_equal(fused.pool.cpu().numpy(), oc.pool)
