"""The bench's roofline numerators against closed forms of the workloads (no
GPU): the decode step's algorithmic bytes (pages read once per (page, kv
head), the partial page's fp16 residual rows, q; shared-prefix pages once on
the unique count and once per sequence on the logical one) and the causal
prefill's algorithmic FLOPs."""
import bench
from int4_kivi_quantized_s4kv_b200 import workloads as W

BLOCK = 2816  # one (page, kv head) block of the int4 pool


def _bytes(name):
    spec = W.SPECS[name]
    d, _ = bench.step_bytes(spec, W.page_plan(spec), W.final_lens(spec))
    return d


def test_llama31_8b_decode_bytes():
    # 256 sequences of 8193 tokens: 512 full pages and one residual row each,
    # 8 kv heads, 32 q heads
    d = _bytes("llama3.1-8b")
    pages = 256 * 512 * 8 * BLOCK
    residual = 256 * 8 * 1 * 128 * 2 * 2      # one row of K and V, fp16
    q = 256 * 32 * 128 * 2
    assert d["pages_unique"] == d["pages_logical"] == pages
    assert d["residual"] == residual and d["q"] == q
    assert d["algorithmic"] == pages + residual + q == 2_955_935_744


def test_llama3_70b_shared_prefix_counted_once():
    # 16 sequences of 32769 tokens, the first 2048 tokens (128 pages) shared
    d = _bytes("llama3-70b")
    per_seq = 32768 // 16
    assert d["pages_logical"] == 16 * per_seq * 8 * BLOCK
    assert d["pages_unique"] == (128 + 16 * (per_seq - 128)) * 8 * BLOCK
    assert d["algorithmic"] == d["pages_unique"] + d["residual"] + d["q"]
    assert d["logical"] == d["pages_logical"] + d["residual"] + d["q"]


def test_prefill_flops_closed_form():
    # 4 chunks of n = 2048 new tokens over L = 8192: row j sees L - n + j + 1
    # keys; q.k and p.v are 2 * 128 FLOP each per key and q head
    spec = W.SPECS["llama3.1-8b-prefill"]
    f = bench.prefill_flops(spec, W.final_lens(spec), W.step_new_tokens(spec))
    L, n = 8192, 2048
    keys = sum(L - n + j + 1 for j in range(n))
    assert f == 4 * 32 * 4 * 128 * keys == 962_139_783_168
