"""s4kv_decode_attention_noalloc, for callers that cannot call cudaMalloc
(for example a plugin inside an engine that owns the whole device memory
pool): called through the C ABI, it must give the same attention as the
workspace entry point, call after call, while its scratch is a fixed array
inside the library.  Collected last so that a failure here comes after every
other test has run."""
import ctypes

import numpy as np
import pytest

from int4_kivi_quantized_s4kv_b200 import workloads as W
from tests.helpers import ATOL, RTOL, Pair, assert_attention_close

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


def test_noalloc_matches_workspace_entry_point_twice():
    import torch
    import int4_kivi_quantized_s4kv_b200 as S
    spec = W.scaled(W.SPECS["llama3.2-3b-step"], batch=6, layers=1)
    p = Pair(spec)
    q = torch.from_numpy(p.q).cuda()
    sl = torch.from_numpy(p.lens).cuda()
    bt = p.bt_dev
    ref_out = torch.empty_like(q)
    ws = S.decode_workspace(spec.batch, spec.num_kv_heads)
    S.s4kv_decode_attention(p.gpu, q, sl, bt, ref_out, ws)
    outs = []
    for _ in range(2):
        o = torch.full_like(q, float("nan"))
        S.s4kv_decode_attention_noalloc(p.gpu, q, sl, bt, o)
        outs.append(o)
    torch.cuda.synchronize()
    ref = ref_out.float().cpu().numpy()
    for o in outs:
        got = o.float().cpu().numpy()
        assert np.isfinite(got).all()
        assert (np.abs(got - ref) <= ATOL + RTOL * np.abs(ref)).all()
    # and both against the oracle
    assert_attention_close(outs[1].float().cpu().numpy(), p.oracle_decode(), "noalloc vs oracle")
    assert S.s4kv_get_error(p.gpu) == 0


def test_noalloc_rejects_batches_beyond_its_scratch():
    """A batch whose decode workspace would not fit in the fixed scratch is
    refused by a size query alone; no call is made with addresses that are
    not real device memory."""
    import int4_kivi_quantized_s4kv_b200 as S
    huge = 10_000_000
    assert S.s4kv_decode_workspace_size(huge, 8) > S.NOALLOC_SCRATCH_BYTES
    assert S.s4kv_decode_workspace_size(64, 8) <= S.NOALLOC_SCRATCH_BYTES


def test_noalloc_checks_every_argument_before_touching_the_scratch():
    """An unsupported code width is refused before the scratch is cleared or
    anything is launched; the cache and the buffers are real, so nothing
    could read outside them even if the refusal were missing."""
    import torch
    import int4_kivi_quantized_s4kv_b200 as S
    spec = W.scaled(W.SPECS["llama3.2-3b-step"], batch=4, layers=1)
    p = Pair(spec)
    q = torch.from_numpy(p.q).cuda()
    out = torch.full_like(q, float("nan"))
    L = S.lib()
    P = ctypes.c_void_p
    bad = S.s4kv_cache_t.from_buffer_copy(p.gpu.c)
    bad.bits = 3
    rc = L.s4kv_decode_attention_noalloc(ctypes.byref(bad), P(q.data_ptr()), q.shape[1],
                                         P(torch.from_numpy(p.lens).cuda().data_ptr()), P(p.bt_dev.data_ptr()),
                                         spec.batch, p.bt_dev.shape[1], 0.088, P(out.data_ptr()), None)
    torch.cuda.synchronize()
    assert rc == S.ERR_UNSUPPORTED
    assert torch.isnan(out).all()
