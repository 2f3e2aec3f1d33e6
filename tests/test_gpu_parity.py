"""GPU parity: the CUDA path through the C ABI against the oracle, on the same
seeded inputs.  Cache bytes (codes, scales, zeros, residual rows) and fp32
page dequantization are compared bit for bit; decode attention within
|gpu - oracle| <= 2e-3 + 1e-3 |oracle| (fp64 oracle on the same dequantized
cache).  Sizes span several MMA tiles, many workers and ragged tails."""
import dataclasses

import numpy as np
import pytest

from int4_kivi_quantized_s4kv_b200 import workloads as W
from tests.helpers import Pair, assert_attention_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
    oracle.build()
    from int4_kivi_quantized_s4kv_b200 import build
    build.build()


def _spec(name, **kw):
    base = dict(layers=1, seed=1234, ctx_kind="fixed", outlier_frac=0.02, outlier_scale=8.0)
    base.update(kw)
    return W.Spec(name, **base)


# ------------------------------------------------------------------ tiny --

def test_tiny_append_bit_exact_and_decode():
    p = Pair(W.SPECS["tiny"])
    p.assert_cache_bit_exact()
    assert_attention_close(p.gpu_decode(), p.oracle_decode(), "tiny")


@pytest.mark.parametrize("chunk", [1, 7, 16, 23])
def test_tiny_chunked_prefill_bit_exact(chunk):
    spec = dataclasses.replace(W.SPECS["tiny"], ctx_fixed=(30, 41), step_new=(7, 9))
    p = Pair(spec, prefill_chunk=chunk)
    p.assert_cache_bit_exact()
    assert_attention_close(p.gpu_decode(), p.oracle_decode(), f"tiny chunk {chunk}")


def test_dequant_page_bit_exact():
    import torch
    import int4_kivi_quantized_s4kv_b200 as S
    p = Pair(dataclasses.replace(W.SPECS["tiny"], num_kv_heads=1))
    H = 1
    used = sorted(set(int(x) for x in p.plan.block_tables[:, :3].ravel() if x >= 0))
    for page in used:
        ok, ov = p.oc.dequant_page(page)
        k32 = torch.empty((H, 16, 128), dtype=torch.float32, device="cuda")
        v32 = torch.empty_like(k32)
        S.s4kv_dequant_page(p.gpu, page, k32, v32, out_fp32=True)
        k16 = torch.empty((H, 16, 128), dtype=torch.float16, device="cuda")
        v16 = torch.empty_like(k16)
        S.s4kv_dequant_page(p.gpu, page, k16, v16, out_fp32=False)
        torch.cuda.synchronize()
        assert np.array_equal(k32.cpu().numpy().view(np.uint32), ok.view(np.uint32))
        assert np.array_equal(v32.cpu().numpy().view(np.uint32), ov.view(np.uint32))
        assert np.array_equal(k16.cpu().numpy().view(np.uint16), ok.astype(np.float16).view(np.uint16))
        assert np.array_equal(v16.cpu().numpy().view(np.uint16), ov.astype(np.float16).view(np.uint16))


# ---------------------------------------------- scaled versions of configs --

SCALED = {
    "qwen2.5-7b": dict(batch=6, ctx_scale=0.1),
    "llama3.1-8b": dict(batch=4, ctx_scale=0.05),
    "llama3-70b": dict(batch=3, ctx_scale=0.03),
    "llama3.2-3b-step": dict(batch=5, layers=2),
}


@pytest.mark.parametrize("name", list(SCALED))
def test_scaled_config_parity(name):
    spec = W.scaled(W.SPECS[name], **SCALED[name])
    for layer in range(spec.layers):
        p = Pair(spec, layer=layer)
        p.assert_cache_bit_exact()
        assert_attention_close(p.gpu_decode(), p.oracle_decode(), f"{name} layer {layer}")


# ------------------------------------------------------------ edge cases --

@pytest.mark.parametrize("hq,hkv", [(16, 2), (4, 4), (9, 3), (10, 2), (14, 2)])
def test_edge_lengths_and_groups(hq, hkv):
    """Empty, single-token, page-aligned, one-past and ragged sequences; GQA
    groups 8, 1, 3, 5 and 7."""
    spec = _spec("edges", batch=9, num_q_heads=hq, num_kv_heads=hkv,
                 ctx_fixed=(0, 0, 14, 15, 16, 0, 31, 100, 47), step_new=(0, 1, 1, 1, 1, 17, 2, 3, 1))
    p = Pair(spec)
    p.assert_cache_bit_exact()
    got, ref = p.gpu_decode(), p.oracle_decode()
    assert (got[0] == 0).all()  # length-0 sequence
    assert_attention_close(got, ref, f"edges G={hq // hkv}")


def test_single_long_sequence_merges_many_splits():
    """One (sequence, kv head) spread over every worker: the log-sum-exp merge
    of many partial results."""
    spec = _spec("long1", batch=1, num_q_heads=8, num_kv_heads=1, ctx_fixed=(20000,), step_new=(5,))
    p = Pair(spec)
    assert_attention_close(p.gpu_decode(), p.oracle_decode(), "long single sequence")


def test_many_short_sequences_fewer_pages_than_workers():
    rng = np.random.default_rng(0)
    ctx = tuple(int(x) for x in rng.integers(0, 40, 60))
    spec = _spec("short", batch=60, num_q_heads=12, num_kv_heads=4, ctx_fixed=ctx, step_new=(1,))
    p = Pair(spec)
    p.assert_cache_bit_exact()
    assert_attention_close(p.gpu_decode(), p.oracle_decode(), "short sequences")


def test_large_batch_of_short_and_empty_sequences():
    """600 sequences (more than 8 per lane of the plan's scan), lengths 0..70
    with some empty: segments of a single page or only a residual, many
    segments per worker, and the floor on pages per worker."""
    rng = np.random.default_rng(5)
    ctx = rng.integers(0, 70, 600)
    ctx[rng.choice(600, 40, replace=False)] = 0
    step = tuple(int(x) for x in np.where(ctx == 0, 0, 1))
    spec = _spec("large-batch", batch=600, num_q_heads=16, num_kv_heads=2,
                 ctx_fixed=tuple(int(x) for x in ctx), step_new=step)
    p = Pair(spec)
    p.assert_cache_bit_exact()
    got = p.gpu_decode()
    assert not got[p.lens == 0].any()
    assert_attention_close(got[p.lens > 0], p.oracle_decode()[p.lens > 0], "600 short sequences")


def test_sm_scale_parameter():
    spec = _spec("scale", batch=3, num_q_heads=8, num_kv_heads=2, ctx_fixed=(50, 70, 90))
    p = Pair(spec)
    for sc in (0.02, 0.3):
        assert_attention_close(p.gpu_decode(sm_scale=sc), p.oracle_decode(sm_scale=sc), f"scale {sc}")


def test_repeated_decode_is_deterministic_and_workspace_resets():
    spec = _spec("repeat", batch=2, num_q_heads=16, num_kv_heads=2, ctx_fixed=(3000, 1000))
    p = Pair(spec)
    outs = [p.gpu_decode() for _ in range(3)]
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[1], outs[2])
    assert_attention_close(outs[0], p.oracle_decode(), "repeat")


def test_idempotent_step_append():
    """Re-running the same step append (same positions) leaves the cache unchanged."""
    spec = _spec("idem", batch=4, num_q_heads=8, num_kv_heads=2, ctx_fixed=(15, 31, 40, 16), step_new=(1,))
    p = Pair(spec)
    p.append(p.ctx, p.lens, None)   # the same append again, on both sides
    p.assert_cache_bit_exact()


# ------------------------------------------------------- error reporting --

def test_device_flags_instead_of_faults():
    import torch
    import int4_kivi_quantized_s4kv_b200 as S
    spec = _spec("flags", batch=2, num_q_heads=4, num_kv_heads=1, ctx_fixed=(40, 20))
    p = Pair(spec)
    assert S.s4kv_get_error(p.gpu) == 0
    bad = p.plan.block_tables.copy()
    bad[0, 1] = p.plan.num_pages + 5  # out of range
    qd = torch.from_numpy(p.q).cuda()
    out = torch.empty_like(qd)
    ws = S.decode_workspace(2, 1)
    S.s4kv_decode_attention(p.gpu, qd, torch.from_numpy(p.lens).cuda(), torch.from_numpy(bad).cuda(), out, ws)
    assert S.s4kv_get_error(p.gpu) & S.EFLAG_PAGE_RANGE
    assert S.s4kv_get_error(p.gpu) == 0  # cleared
    # slot_mapping disagreeing with block_tables
    k = torch.zeros((1, 1, 128), dtype=torch.float16, device="cuda")
    sl = torch.tensor([41, 20], dtype=torch.int32, device="cuda")
    cu = torch.tensor([0, 1, 1], dtype=torch.int32, device="cuda")
    sm = torch.tensor([12345], dtype=torch.int64, device="cuda")
    S.s4kv_append(p.gpu, k, k, sm, cu, sl, torch.from_numpy(p.plan.block_tables).cuda(), 1)
    assert S.s4kv_get_error(p.gpu) & S.EFLAG_SLOT


def test_host_validation_launches_nothing():
    import torch
    import int4_kivi_quantized_s4kv_b200 as S
    c = S.S4KVCache(4, 2, 2)
    q = torch.zeros((2, 6, 128), dtype=torch.float16, device="cuda")
    out = torch.empty_like(q)
    sl = torch.tensor([5, 5], dtype=torch.int32, device="cuda")
    bt = torch.zeros((2, 1), dtype=torch.int32, device="cuda")
    ws = S.decode_workspace(2, 2)
    with pytest.raises(S.S4KVError) as e:  # 6 q heads over 2 kv heads is fine; 5 is not
        S.s4kv_decode_attention(c, q[:, :5].contiguous(), sl, bt, out[:, :5].contiguous(), ws)
    assert e.value.status == S.ERR_UNSUPPORTED
    with pytest.raises(S.S4KVError) as e:
        S.s4kv_decode_attention(c, q, sl, bt, out, ws[:16])
    assert e.value.status == S.ERR_WORKSPACE
    big = torch.zeros((2, 18, 128), dtype=torch.float16, device="cuda")  # group 9 > 8
    with pytest.raises(S.S4KVError) as e:
        S.s4kv_decode_attention(c, big, sl, bt, torch.empty_like(big), ws)
    assert e.value.status == S.ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert S.s4kv_get_error(c) == 0


def test_workspace_sized_for_a_large_batch_serves_smaller_ones():
    """One zero-filled workspace sized for the largest batch, reused by calls
    with fewer sequences and then more: every call must read zero tickets and
    agree with the oracle (the partial results of a small call must never be
    read as tickets by a larger one)."""
    import torch
    import int4_kivi_quantized_s4kv_b200 as S
    spec = W.scaled(W.SPECS["llama3.1-8b"], batch=24, ctx_scale=1 / 16)   # 8 kv heads, 512+1 tokens
    p = Pair(spec)
    ref = p.oracle_decode()
    ws = S.decode_workspace(spec.batch, spec.num_kv_heads)
    q = p._dev(p.q)
    lens = p._dev(p.lens)
    for nb in (2, 24, 5, 24, 1):
        out = torch.full_like(q[:nb], float("nan"))
        S.s4kv_decode_attention(p.gpu, q[:nb].contiguous(), lens[:nb].contiguous(), p.bt_dev[:nb].contiguous(),
                                out, ws)
        torch.cuda.synchronize()
        assert_attention_close(out.float().cpu().numpy(), ref[:nb], f"batch {nb} on a batch-24 workspace")
    assert S.s4kv_get_error(p.gpu) == 0
