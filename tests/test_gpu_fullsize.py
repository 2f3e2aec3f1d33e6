"""Full-size parity in the launch configuration bench.py times: each workload
is built at its full shape by bench.DeviceWorkload (device-side seeded K/V,
appends through the C ABI), one step runs, and sampled (layer, sequence)
pairs are recomputed one by one by the oracle from the same K/V (copied back
from the device generator): their pool pages and residual rows bit-exact,
their decode outputs within 2e-3 + 1e-3 |ref|."""
import gc

import numpy as np
import pytest

from int4_kivi_quantized_s4kv_b200 import workloads as W
from tests.helpers import assert_attention_close

pytestmark = pytest.mark.gpu

PAGE = 16


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
    oracle.build()
    from int4_kivi_quantized_s4kv_b200 import build
    build.build()


def _check_sequence(wl, layer, b):
    import torch
    import oracle
    spec = wl.spec
    L = int(wl.lens[b])
    H = spec.num_kv_heads
    k, v = W.kv_sequence_torch(spec, layer, b, L, wl.device)
    k, v = k.cpu().numpy(), v.cpu().numpy()
    need = (L + PAGE - 1) // PAGE
    bt = np.arange(need, dtype=np.int32)[None, :]
    oc = oracle.OracleCache(need + 1, H, 1)
    sm = W.slot_mapping(bt, [np.arange(L)])
    assert oc.append(k, v, sm, np.array([0, L], np.int32), np.array([L], np.int32), bt) == 0
    # cache bytes of this sequence's pages and residual rows
    full = L // PAGE
    gpu_pages = wl.plan.block_tables[b, :full]
    pool = wl.caches[layer].pool[torch.from_numpy(gpu_pages.astype(np.int64)).to(wl.device)].cpu().numpy()
    assert np.array_equal(pool, oc.pool[:full]), f"pool pages of layer {layer} seq {b}"
    r = L % PAGE
    rk = wl.caches[layer].res_k[b, :, :r].cpu().numpy().view(np.uint16)
    assert np.array_equal(rk, oc.res_k[0, :, :r]), f"residual of layer {layer} seq {b}"
    q = wl.q[layer][b:b + 1].cpu().numpy()
    ref = oc.decode_attention(q, np.array([L], np.int32), bt)[0]
    got = wl.out[layer][b].float().cpu().numpy()
    return assert_attention_close(got, ref, f"{spec.name} layer {layer} seq {b} (L={L})")


SAMPLES = {
    "qwen2.5-7b": [(0, 0), (0, 31), (0, 63)],
    "llama3.1-8b": [(0, 0), (0, 128), (0, 255)],
    "llama3-70b": [(0, 0), (0, 15)],
    "llama3.2-3b-step": [(0, "longest"), (13, 5), (27, "shortest")],
}


@pytest.mark.parametrize("name", list(SAMPLES))
def test_full_size_sampled_parity(name):
    import torch
    import bench
    spec = W.SPECS[name]
    wl = bench.DeviceWorkload(spec, torch.device("cuda", 0))
    for _ in range(2):       # the step is idempotent: run it twice like warm-up
        wl.step()
    torch.cuda.synchronize()
    for c in wl.caches:
        assert wl.S.s4kv_get_error(c) == 0
    for layer, b in SAMPLES[name]:
        if b == "longest":
            b = int(np.argmax(wl.lens))
        elif b == "shortest":
            b = int(np.argmin(wl.lens))
        _check_sequence(wl, layer, b)
    del wl
    gc.collect()
    torch.cuda.empty_cache()


# chunked prefill: (sequence, rows) samples; the chunk's last rows see the
# whole sequence, so the oracle recomputes them from a one-sequence cache
PREFILL_SAMPLES = {
    "llama3.1-8b-prefill": [0, 3],
    "llama3-70b-prefill": [1],
}


@pytest.mark.parametrize("name", list(PREFILL_SAMPLES))
def test_full_size_prefill_sampled_parity(name):
    """The prefill workload at full shape in the launch configuration the
    bench times (the whole chunk of every sequence in one call): sampled
    sequences' pool pages bit-exact against the oracle's, and the last rows
    of their chunks and sampled interior rows within 2e-3 + 1e-3 |ref|."""
    import torch
    import oracle
    import bench
    spec = W.SPECS[name]
    dev = torch.device("cuda", 0)
    wl = bench.DeviceWorkload(spec, dev)
    S = wl.S
    cache = wl.caches[0]
    S.s4kv_append(cache, wl.k_new[0], wl.v_new[0], wl.step_slots, wl.step_cu, wl.seq_lens, wl.bt, wl.max_new)
    rows = int(wl.new.sum())
    q = W.chunk_queries_torch(spec, 0, rows, dev)
    out = torch.full_like(q, float("nan"))
    ws = S.prefill_workspace(spec.num_kv_heads, spec.batch, wl.bt.shape[1], dev)
    S.s4kv_prefill_attention(cache, q, wl.step_cu, wl.seq_lens, wl.bt, out, wl.max_new, workspace=ws)
    torch.cuda.synchronize()
    assert S.s4kv_get_error(cache) == 0
    assert bool(torch.isfinite(out.float()).all())
    cu = wl.step_cu.cpu().numpy()
    H = spec.num_kv_heads
    for b in PREFILL_SAMPLES[name]:
        L = int(wl.lens[b])
        k, v = W.kv_sequence_torch(spec, 0, b, L, dev)
        k, v = k.cpu().numpy(), v.cpu().numpy()
        need = (L + PAGE - 1) // PAGE
        bt = np.arange(need, dtype=np.int32)[None, :]
        oc = oracle.OracleCache(need + 1, H, 1)
        sm = W.slot_mapping(bt, [np.arange(L)])
        assert oc.append(k, v, sm, np.array([0, L], np.int32), np.array([L], np.int32), bt) == 0
        full = L // PAGE
        gpu_pages = wl.plan.block_tables[b, :full]
        pool = cache.pool[torch.from_numpy(gpu_pages.astype(np.int64)).to(dev)].cpu().numpy()
        assert np.array_equal(pool, oc.pool[:full]), f"pool pages of seq {b}"
        last = np.arange(int(cu[b + 1]) - 4, int(cu[b + 1]))
        ref = oc.prefill_attention(q[torch.from_numpy(last).to(dev)].cpu().numpy(), np.array([0, 4], np.int32),
                                   np.array([L], np.int32), bt)
        got = out[torch.from_numpy(last).to(dev)].float().cpu().numpy()
        assert_attention_close(got, ref, f"{spec.name} seq {b} last rows (L={L})")
        # interior rows of the chunk, where the causal limit cuts key tiles:
        # the first row, both sides of a query-tile and a key-tile boundary,
        # and one deep inside, each against the oracle's row at its position
        n = int(cu[b + 1] - cu[b])
        for j in (0, 127, 128, 1023):
            row = int(cu[b]) + j
            q_row = q[row].cpu().numpy()
            ref_row = oc.attention_at(q_row, 0, L, L - n + j, bt[0])
            got_row = out[row].float().cpu().numpy()
            assert_attention_close(got_row, ref_row, f"{spec.name} seq {b} chunk row {j} (L={L})")
    del wl
    gc.collect()
    torch.cuda.empty_cache()
