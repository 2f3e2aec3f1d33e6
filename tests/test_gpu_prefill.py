"""GPU parity of s4kv_prefill_attention (causal attention of an appended
chunk over the int4 paged cache) against the fp64 oracle, through the C ABI.

The cache is built on both sides from the same seeded fp16 inputs (context
appended first, then the chunk) and must be bit-exact; the attention output
must be within |gpu - oracle| <= 2e-3 + 1e-3 |oracle| element-wise.  The
CUDA path feeds the tensor cores fp16 operands (dequantized keys and values,
softmax weights), which that bound covers with margin.
"""
import numpy as np
import pytest

from helpers import assert_attention_close

HD, PAGE = 128, 16

pytestmark = pytest.mark.gpu


class PrefillCase:
    def __init__(self, seed, H, G, before, after, outliers=8, context_chunk=64, bits=4):
        import torch
        import oracle
        import int4_kivi_quantized_s4kv_b200 as S
        rng = np.random.default_rng(seed)
        self.S, self.H, self.G = S, H, G
        self.before = np.array(before, np.int64)
        self.after = np.array(after, np.int64)
        B = len(after)
        # keys with a few outlier channels per kv head, values plain N(0, 1)
        scale = np.ones((H, HD))
        for h in range(H):
            scale[h, rng.choice(HD, outliers, replace=False)] = 10.0
        self.k = [(rng.standard_normal((L, H, HD)) * scale).astype(np.float16) for L in after]
        self.v = [rng.standard_normal((L, H, HD)).astype(np.float16) for L in after]
        need = [(L + PAGE - 1) // PAGE for L in after]
        NP = sum(need) + 5
        perm = rng.permutation(NP).astype(np.int32)
        self.bt = np.full((B, max(max(need), 1)), -1, np.int32)
        c = 0
        for b, m in enumerate(need):
            self.bt[b, :m] = perm[c:c + m]
            c += m
        self.oc = oracle.OracleCache(NP, H, B, bits=bits)
        self.gpu = S.S4KVCache(NP, H, B, device="cuda", bits=bits)
        self.dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
        self.bt_dev = self.dev(self.bt)
        self._append(np.zeros(B, np.int64), self.before, context_chunk)
        self.n = self.after - self.before
        self.cu = np.concatenate([[0], np.cumsum(self.n)]).astype(np.int32)
        self._append(self.before, self.after, None)
        self.q = rng.standard_normal((int(self.cu[-1]), H * G, HD)).astype(np.float16)

    def _append(self, before, after, chunk):
        from helpers import append_batches
        for k, v, sm, cu, sl, mx in append_batches(before, after, self.k, self.v, self.bt, chunk):
            if mx == 0:
                continue
            assert self.oc.append(k, v, sm, cu, sl, self.bt) == 0
            self.S.s4kv_append(self.gpu, self.dev(k), self.dev(v), self.dev(sm), self.dev(cu), self.dev(sl),
                               self.bt_dev, mx)

    def run(self, sm_scale=None, workspace=None):
        import torch
        qd = self.dev(self.q)
        out = torch.full_like(qd, float("nan"))
        self.S.s4kv_prefill_attention(self.gpu, qd, self.dev(self.cu), self.dev(self.after.astype(np.int32)),
                                      self.bt_dev, out, int(max(self.n.max(), 1)), sm_scale, workspace=workspace)
        torch.cuda.synchronize()
        assert self.S.s4kv_get_error(self.gpu) == 0
        got = out.float().cpu().numpy()
        ref = self.oc.prefill_attention(self.q, self.cu, self.after.astype(np.int32), self.bt, sm_scale)
        return got, ref


@pytest.mark.parametrize("G", [4, 1, 3, 8])
def test_prefill_matches_oracle(G):
    # chunks from position 0, across page and key-tile boundaries, a long
    # chunk spanning several query tiles, and a single new token
    case = PrefillCase(40 + G, 2, G, before=[0, 100, 5, 250], after=[37, 164, 300, 251])
    got, ref = case.run()
    err = assert_attention_close(got, ref, f"prefill G={G}")
    print(f"G={G} max abs err {err:.3g}")


def test_prefill_odd_groups_and_empty_chunk():
    # G = 7 (18-token query tiles, 126 rows) and G = 5; one sequence gets no
    # new tokens, one chunk ends exactly on a page boundary
    for G in (7, 5):
        case = PrefillCase(50 + G, 1, G, before=[16, 40, 0], after=[16, 64, 129])
        got, ref = case.run(sm_scale=0.05)
        assert_attention_close(got, ref, f"prefill G={G}")


def test_prefill_long_chunk_over_long_context():
    # 512-token chunks over 1.5K-token contexts: many key tiles, lazy
    # rescaling of the running output, sequence-level tiling of the grid
    case = PrefillCase(60, 2, 8, before=[1536, 1000], after=[2048, 1512], context_chunk=512)
    got, ref = case.run()
    assert_attention_close(got, ref, "prefill long")


def test_prefill_last_row_matches_decode():
    # the chunk's last row sees the whole sequence, as decode does
    import torch
    case = PrefillCase(70, 2, 4, before=[10, 60], after=[75, 200])
    got, ref = case.run()
    last = case.cu[1:] - 1
    S = case.S
    qd = case.dev(case.q[last])
    out = torch.empty_like(qd)
    ws = S.decode_workspace(2, 2)
    S.s4kv_decode_attention(case.gpu, qd, case.dev(case.after.astype(np.int32)), case.bt_dev, out, ws)
    torch.cuda.synchronize()
    assert_attention_close(out.float().cpu().numpy(), ref[last], "decode of the last rows")
    assert_attention_close(got[last], ref[last], "prefill of the last rows")


def test_prefill_ignores_stale_workspace_contents():
    """Every operand byte the attention reads is written by the same call:
    a workspace full of fp16 NaN patterns (0xFF bytes) gives the same output
    as a fresh one, also for keys past L inside the last tile (zero-filled)."""
    import torch
    case = PrefillCase(80, 2, 4, before=[3, 70], after=[45, 200])
    ws = case.S.prefill_workspace(2, 2, case.bt.shape[1])
    ws.fill_(0xFF)
    got, ref = case.run(workspace=ws)
    assert not np.isnan(got[:int(case.cu[-1])]).any()
    assert_attention_close(got, ref, "prefill, stale workspace")
    # the workspace reused for a second case of smaller sequences
    small = PrefillCase(81, 2, 4, before=[0, 17], after=[20, 33])
    ws2 = ws[:case.S.prefill_workspace_bytes(2, 2, small.bt.shape[1])]
    got2, ref2 = small.run(workspace=ws2)
    assert_attention_close(got2, ref2, "prefill, reused workspace")


@pytest.mark.parametrize("bits", [8, 2])
def test_prefill_8_and_2_bit_caches(bits):
    """The same attention over 8- and 2-bit pages: only the operand tiles'
    dequantization differs (every code through the code map); the cache
    bytes must match the oracle's and the output must be within the bound."""
    case = PrefillCase(90 + bits, 2, 4, before=[0, 100, 300], after=[37, 290, 301], bits=bits)
    assert np.array_equal(case.gpu.pool.cpu().numpy(), case.oc.pool)
    got, ref = case.run()
    assert_attention_close(got, ref, f"prefill int{bits}")
    case8 = PrefillCase(95 + bits, 1, 8, before=[1000], after=[1200], bits=bits, context_chunk=256)
    got, ref = case8.run(sm_scale=0.06)
    assert_attention_close(got, ref, f"prefill int{bits} G=8")


def test_prefill_leaves_rows_of_no_sequence_untouched():
    """q and out may hold more rows than cu_new[batch]: those rows belong to
    no sequence and are neither read nor written."""
    import torch
    case = PrefillCase(85, 2, 4, before=[5, 60], after=[40, 61])
    S = case.S
    n = int(case.cu[-1])
    extra = 7
    q = np.concatenate([case.q, np.random.default_rng(1).standard_normal((extra, 8, HD)).astype(np.float16)])
    qd = case.dev(q)
    out = torch.full_like(qd, float("nan"))
    S.s4kv_prefill_attention(case.gpu, qd, case.dev(case.cu), case.dev(case.after.astype(np.int32)), case.bt_dev,
                             out, int(case.n.max()))
    torch.cuda.synchronize()
    assert S.s4kv_get_error(case.gpu) == 0
    got = out.float().cpu().numpy()
    assert np.isnan(got[n:]).all()
    ref = case.oc.prefill_attention(case.q, case.cu, case.after.astype(np.int32), case.bt)
    assert_attention_close(got[:n], ref, "prefill with trailing rows")


def test_prefill_flags_a_chunk_longer_than_max_new_per_seq():
    """A chunk longer than the host bound max_new_per_seq (which sizes the
    grid) is reported through S4KV_EFLAG_SEQ_LEN; the rows the grid covers
    are still computed, the others are left untouched."""
    import torch
    case = PrefillCase(86, 1, 4, before=[10, 0], after=[50, 300])   # chunks of 40 and 300 rows
    S = case.S
    qd = case.dev(case.q)
    out = torch.full_like(qd, float("nan"))
    bound = 40                                    # one 32-row query tile at G = 4 covers 32 rows
    S.s4kv_prefill_attention(case.gpu, qd, case.dev(case.cu), case.dev(case.after.astype(np.int32)), case.bt_dev,
                             out, bound)
    torch.cuda.synchronize()
    flags = S.s4kv_get_error(case.gpu)
    assert flags & 4, flags                       # S4KV_EFLAG_SEQ_LEN
    got = out.float().cpu().numpy()
    ref = case.oc.prefill_attention(case.q, case.cu, case.after.astype(np.int32), case.bt)
    tiles = -(-bound // 32)
    covered = np.concatenate([np.arange(case.cu[b], case.cu[b] + min(int(case.n[b]), 32 * tiles))
                              for b in range(2)])
    assert_attention_close(got[covered], ref[covered], "prefill rows the grid covers")
    rest = np.setdiff1d(np.arange(int(case.cu[-1])), covered)
    assert rest.size > 0 and np.isnan(got[rest]).all()
