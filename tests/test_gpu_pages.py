"""GPU parity of page movement (swap-out / swap-in, copy-on-write copy and
fork, batched dequantization) against the oracle, through the C ABI.  Every
byte that moves must be bit-exact; attention after a move is compared with
the oracle within the decode tolerance and, where the page ids are all that
changed, bit-for-bit with the GPU's own result before the move."""
import dataclasses

import numpy as np
import pytest

from helpers import Pair, assert_attention_close
from int4_kivi_quantized_s4kv_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _pair():
    spec = W.scaled(W.SPECS["qwen2.5-7b"], batch=5, ctx_scale=0.06)
    spec = dataclasses.replace(spec, step_new=(1,))
    return Pair(spec)


def _free_pages(p, count):
    used = set(int(x) for x in p.plan.block_tables[p.plan.block_tables >= 0].ravel())
    free = [x for x in range(p.plan.num_pages) if x not in used]
    assert len(free) >= count
    return free[:count]


def test_gather_matches_oracle_and_dequant_pages():
    import torch
    p = _pair()
    S = p.S
    pages = np.array(p.plan.block_tables[1, :int(p.lens[1]) // 16], np.int32)
    rec = S.s4kv_page_record_bytes(p.gpu)
    dst = torch.empty((len(pages), rec), dtype=torch.uint8, device="cuda")
    S.s4kv_gather_pages(p.gpu, p._dev(pages), dst)
    torch.cuda.synchronize()
    assert np.array_equal(dst.cpu().numpy().reshape(len(pages), p.spec.num_kv_heads, -1), p.oc.gather_pages(pages))
    # batched dequantization, fp32 bit-exact and fp16 the RNE of it
    H = p.spec.num_kv_heads
    ok = torch.empty((len(pages), H, 16, 128), dtype=torch.float32, device="cuda")
    ov = torch.empty_like(ok)
    S.s4kv_dequant_pages(p.gpu, p._dev(pages), ok, ov, True)
    hk = torch.empty((len(pages), H, 16, 128), dtype=torch.float16, device="cuda")
    hv = torch.empty_like(hk)
    S.s4kv_dequant_pages(p.gpu, p._dev(pages), hk, hv, False)
    torch.cuda.synchronize()
    for i, pg in enumerate(pages):
        rk, rv = p.oc.dequant_page(int(pg))
        assert np.array_equal(ok[i].cpu().numpy(), rk)
        assert np.array_equal(ov[i].cpu().numpy(), rv)
        assert np.array_equal(hk[i].cpu().numpy().view(np.uint16), rk.astype(np.float16).view(np.uint16))
        assert np.array_equal(hv[i].cpu().numpy().view(np.uint16), rv.astype(np.float16).view(np.uint16))
    assert S.s4kv_get_error(p.gpu) == 0


def test_swap_out_and_back_in_elsewhere():
    """Swap sequence 2's full pages out to pinned host memory, wipe them, swap
    them into free pages and remap: the pool equals the oracle after the same
    moves, and decode attention is bit-identical to before."""
    import torch
    p = _pair()
    S = p.S
    # rows 3 and 4 give up their pages (they become empty sequences)
    lens = p.lens.copy()
    lens[3:] = 0
    p.lens = lens
    p.plan.block_tables[3:] = -1
    p.bt_dev = p._dev(p.plan.block_tables)
    before = p.gpu_decode()
    nfull = int(p.lens[2]) // 16
    pages = np.array(p.plan.block_tables[2, :nfull], np.int32)
    rec = S.s4kv_page_record_bytes(p.gpu)
    staging = torch.empty((nfull, rec), dtype=torch.uint8, device="cuda")
    host = torch.empty((nfull, rec), dtype=torch.uint8, pin_memory=True)
    S.s4kv_swap_out(p.gpu, p._dev(pages), staging, host)
    torch.cuda.synchronize()
    oracle_rec = p.oc.gather_pages(pages)
    assert np.array_equal(host.numpy().reshape(oracle_rec.shape), oracle_rec)
    # wipe the old pages on both sides
    zeros = torch.zeros_like(staging)
    S.s4kv_scatter_pages(p.gpu, p._dev(pages), zeros)
    p.oc.scatter_pages(pages, np.zeros_like(oracle_rec))
    # swap in elsewhere and remap
    free = np.array(_free_pages(p, nfull), np.int32)
    staging.zero_()
    S.s4kv_swap_in(p.gpu, p._dev(free), staging, host)
    p.oc.scatter_pages(free, oracle_rec)
    p.plan.block_tables[2, :nfull] = free
    p.bt_dev = p._dev(p.plan.block_tables)
    torch.cuda.synchronize()
    assert np.array_equal(p.gpu.pool.cpu().numpy(), p.oc.pool)
    after = p.gpu_decode()
    assert np.array_equal(after, before)
    assert_attention_close(after, p.oracle_decode(), "decode after swap")
    assert S.s4kv_get_error(p.gpu) == 0


def test_copy_on_write_fork():
    """Fork sequence 0 into batch row 4 (full pages shared, the partial page's
    residual copied, a private copy of one full page made with copy_pages),
    then let the fork diverge by appending tokens: the cache stays bit-exact
    with the oracle, the original's attention is unchanged, and the fork's
    attention matches the oracle.  Rows 3 and 4 give up their pages to the
    fork (row 3 ends up empty)."""
    import torch
    p = _pair()
    S = p.S
    bt = p.plan.block_tables
    keep = set(int(x) for x in bt[:3][bt[:3] >= 0].ravel())
    free = [x for x in range(p.plan.num_pages) if x not in keep]
    cap = bt.shape[1]
    L0 = int(p.lens[0])
    nfull, np0 = L0 // 16, (L0 + 15) // 16
    L_after = min(16 * cap, 16 * np0 + 5)
    need = (L_after + 15) // 16
    assert len(free) >= need - nfull + 1 + 1
    bt[3, :] = -1
    bt[4, :] = -1
    bt[4, 0] = free[0]                       # private copy of page 0
    bt[4, 1:nfull] = bt[0, 1:nfull]          # shared full pages
    bt[4, nfull:need] = free[1:1 + need - nfull]  # the fork's own partial and later pages
    S.s4kv_copy_pages(p.gpu, p._dev(np.array([bt[0, 0]], np.int32)), p._dev(np.array([free[0]], np.int32)))
    p.oc.copy_pages([bt[0, 0]], [free[0]])
    S.s4kv_fork_residual(p.gpu, p._dev(np.array([0], np.int32)), p._dev(np.array([4], np.int32)))
    p.oc.fork_residual([0], [4])
    p.bt_dev = p._dev(bt)
    lens = p.lens.copy()
    lens[3] = 0
    lens[4] = L0
    p.lens = lens
    q = p.q.copy()
    q[4] = q[0]
    out = p.gpu_decode(q)
    # same pages and query: the same attention (the two rows sit at different
    # places of the split along the sequence, so the merges may round apart)
    assert_attention_close(out[4], out[0], "fork before diverging")
    assert not out[3].any()
    ref0 = out[0].copy()
    # the fork diverges: its own continuation completes the partial page
    extra = L_after - L0
    rng = np.random.default_rng(9)
    H = p.spec.num_kv_heads
    p.k[4] = np.concatenate([p.k[0][:L0], rng.standard_normal((extra, H, 128)).astype(np.float16)])
    p.v[4] = np.concatenate([p.v[0][:L0], rng.standard_normal((extra, H, 128)).astype(np.float16)])
    after = lens.copy()
    after[4] = L_after
    p.append(lens, after, None)
    p.lens = after
    out2 = p.gpu_decode(q)
    # the original is untouched (its pages are compared bit for bit below);
    # its attention may round differently where the split along the
    # sequence moved with the fork's new length
    assert_attention_close(out2[0], ref0, "original after the fork diverged")
    assert_attention_close(out2, p.oracle_decode(q), "decode after fork")
    torch.cuda.synchronize()
    assert np.array_equal(p.gpu.pool.cpu().numpy(), p.oc.pool)
    assert S.s4kv_get_error(p.gpu) == 0


def test_bad_page_ids_flag_instead_of_faulting():
    import torch
    p = _pair()
    S = p.S
    rec = S.s4kv_page_record_bytes(p.gpu)
    pages = np.array([0, p.plan.num_pages + 3, -1, 1], np.int32)
    dst = torch.full((4, rec), 7, dtype=torch.uint8, device="cuda")
    S.s4kv_gather_pages(p.gpu, p._dev(pages), dst)
    flags = S.s4kv_get_error(p.gpu)
    assert flags & 1  # S4KV_EFLAG_PAGE_RANGE
    got = dst.cpu().numpy()
    assert np.array_equal(got[0].reshape(p.spec.num_kv_heads, -1), p.oc.gather_pages([0])[0])
    assert (got[1] == 7).all() and (got[2] == 7).all()
    rows = np.array([0, 99], np.int32)
    S.s4kv_fork_residual(p.gpu, p._dev(rows), p._dev(np.array([1, 2], np.int32)))
    assert S.s4kv_get_error(p.gpu) & 2  # S4KV_EFLAG_SLOT
