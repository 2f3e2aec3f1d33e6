"""GPU parity of the INT8 and 2-bit variants (8- and 2-bit KIVI codes on the
same layout machinery) against the oracle, through the C ABI: cache bytes and
fp32 dequantization bit-exact, decode attention (plain and fused with the
step's append) within 2e-3 + 1e-3 |ref|."""
import dataclasses

import numpy as np
import pytest

from helpers import Pair, assert_attention_close
from int4_kivi_quantized_s4kv_b200 import workloads as W

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": dict(),
    "qwen2.5-7b": dict(batch=6, ctx_scale=0.1),
    "llama3-70b": dict(batch=3, ctx_scale=0.06),
    "llama3.2-3b-step": dict(batch=10, layers=1, ctx_scale=0.05),
}


BLOCK = {8: 4864, 2: 1792}


@pytest.mark.parametrize("bits", [8, 2])
@pytest.mark.parametrize("name", list(CASES))
def test_cache_and_decode_match_oracle(name, bits):
    import torch
    spec = W.SPECS[name] if not CASES[name] else W.scaled(W.SPECS[name], **CASES[name])
    p = Pair(spec, prefill_chunk=33, bits=bits)
    p.assert_cache_bit_exact()
    err = assert_attention_close(p.gpu_decode(), p.oracle_decode(), f"int{bits} {name}")
    # fp32 dequantization of a few pages, bit-exact
    S = p.S
    pages = np.unique(p.plan.block_tables[p.plan.block_tables >= 0])[:5].astype(np.int32)
    H = spec.num_kv_heads
    ok = torch.empty((len(pages), H, 16, 128), dtype=torch.float32, device="cuda")
    ov = torch.empty_like(ok)
    S.s4kv_dequant_pages(p.gpu, p._dev(pages), ok, ov, True)
    torch.cuda.synchronize()
    for i, pg in enumerate(pages):
        rk, rv = p.oc.dequant_page(int(pg))
        if p.plan.block_tables.size and (p.lens // 16).sum() > 0:
            full = any(int(pg) in p.plan.block_tables[b, :int(p.lens[b]) // 16] for b in range(spec.batch))
            if full:
                assert np.array_equal(ok[i].cpu().numpy(), rk) and np.array_equal(ov[i].cpu().numpy(), rv)
    print(f"int{bits} {name}: max abs err {err:.3g}")


@pytest.mark.parametrize("bits", [8, 2])
def test_fused_step_and_page_records(bits):
    """One fused decode step on an 8- or 2-bit cache (tokens that complete
    pages included) writes the oracle's bytes; gathered page records have
    that width's record size."""
    import torch
    import oracle
    import int4_kivi_quantized_s4kv_b200 as S
    from helpers import append_batches
    spec = dataclasses.replace(W.SPECS["llama3.2-3b-step"], name="int8-fused", layers=1, batch=5,
                               ctx_kind="fixed", ctx_fixed=(15, 31, 100, 47, 0), step_new=(1,))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    ctx, lens, plan = W.context_lens(spec), W.final_lens(spec), W.page_plan(spec)
    B, H = spec.batch, spec.num_kv_heads
    k, v = [], []
    for b in range(B):
        kk, vv = W.kv_sequence_np(spec, 0, b, int(lens[b]))
        k.append(kk)
        v.append(vv)
    bt = plan.block_tables
    oc = oracle.OracleCache(plan.num_pages, H, B, bits=bits)
    g = S.S4KVCache(plan.num_pages, H, B, bits=bits)
    bt_dev = dev(bt)
    for kk, vv, sm, cu, sl, mx in append_batches(np.zeros(B, np.int64), ctx, k, v, bt, 16):
        assert oc.append(kk, vv, sm, cu, sl, bt) == 0
        S.s4kv_append(g, dev(kk), dev(vv), dev(sm), dev(cu), dev(sl), bt_dev, mx)
    for kk, vv, sm, cu, sl, mx in append_batches(ctx, lens, k, v, bt, None):
        assert oc.append(kk, vv, sm, cu, sl, bt) == 0
    k_new = np.stack([k[b][int(lens[b]) - 1] for b in range(B)])
    v_new = np.stack([v[b][int(lens[b]) - 1] for b in range(B)])
    q = W.queries_np(spec, 0)
    out = torch.empty((B, spec.num_q_heads, 128), dtype=torch.float16, device="cuda")
    S.s4kv_append_decode(g, dev(k_new), dev(v_new), dev(q), dev(lens), bt_dev, out, S.decode_workspace(B, H))
    torch.cuda.synchronize()
    assert S.s4kv_get_error(g) == 0
    assert np.array_equal(g.pool.cpu().numpy(), oc.pool)
    assert_attention_close(out.float().cpu().numpy(), oc.decode_attention(q, lens, bt), f"int{bits} fused")
    rec = S.s4kv_page_record_bytes(g)
    assert rec == H * BLOCK[bits]
    pages = np.array(bt[2, :int(lens[2]) // 16], np.int32)
    dst = torch.empty((len(pages), rec), dtype=torch.uint8, device="cuda")
    S.s4kv_gather_pages(g, dev(pages), dst)
    torch.cuda.synchronize()
    assert np.array_equal(dst.cpu().numpy().reshape(len(pages), H, -1), oc.gather_pages(pages))
