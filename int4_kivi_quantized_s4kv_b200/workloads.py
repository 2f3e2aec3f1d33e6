"""Seeded synthetic inputs for the s4kv decode path.

This module holds shapes, value distributions and page-table structure only:
none of the quantizer's or the attention's arithmetic.  Both the CUDA path
(tests, benchmark) and the CPU oracle consume what it produces, so it is the
one piece of code the two share.

The workloads stand in for the model shapes the pages name: Qwen2.5 and
Llama-3 families with head_dim 128 ("S4 KV -- int4 KV-Cache-Kompression fuer
vLLM", "Lieferumfang"), GQA with 8 KV heads ("KV-Cache-Optimierung --
PagedAttention, quantisierter KV, Speculative Cache", "Kernpunkte"), 4K-32K
contexts and shared system-prompt prefixes whose physical pages appear in
every page table ("KV-Cache und PagedAttention: Warum Ihr LLM-Server
langsamer wird", "Wie PagedAttention das loest").  No dataset is involved:
K, V and q are Gaussian, with outlier key channels (the KIVI observation
that keys have a few large channels) or a log-normal per-channel key scale.

Two backends draw the same distributions: ``numpy`` (PCG64, host) for the
sizes the oracle handles in seconds, and ``torch`` (a device generator) for
full-size benchmark inputs.  Each is deterministic on its own; the tests
always hand the *same* arrays to both implementations.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

HEAD_DIM = 128
PAGE = 16


@dataclasses.dataclass(frozen=True)
class Spec:
    name: str
    layers: int
    batch: int
    num_q_heads: int
    num_kv_heads: int
    seed: int
    # context length model (tokens already in the cache before the step)
    ctx_kind: str               # "fixed" | "uniform" | "lognormal"
    ctx_a: float = 0.0
    ctx_b: float = 0.0
    ctx_fixed: tuple = ()       # explicit per-sequence contexts ("fixed")
    # tokens appended by the step, per sequence (fixed list or one value)
    step_new: tuple = (1,)
    # key channel distribution
    outlier_channels: int = 0   # per (layer, kv head)
    outlier_frac: float = 0.0   # used when outlier_channels == 0
    outlier_scale: float = 1.0
    key_lognormal_sigma: float = 0.0
    shared_prefix_tokens: int = 0
    description: str = ""

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def n_outliers(self) -> int:
        if self.outlier_channels:
            return self.outlier_channels
        if self.outlier_frac > 0:
            return max(1, int(round(self.outlier_frac * HEAD_DIM)))
        return 0


SPECS = {
    "tiny": Spec(
        "tiny", layers=1, batch=2, num_q_heads=4, num_kv_heads=1, seed=0,
        ctx_kind="fixed", ctx_fixed=(0, 0), step_new=(37, 50),
        outlier_channels=4, outlier_scale=10.0,
        description="1 layer, 2 sequences of 37 and 50 tokens appended in one "
                    "call then one decode, 4 q heads / 1 kv head"),
    "qwen2.5-7b": Spec(
        "qwen2.5-7b", layers=1, batch=64, num_q_heads=28, num_kv_heads=4, seed=1,
        ctx_kind="uniform", ctx_a=512, ctx_b=4096,
        outlier_frac=0.02, outlier_scale=8.0,
        description="Qwen2.5-7B-shaped layer, batch 64, contexts U[512,4096]"),
    "llama3.1-8b": Spec(
        "llama3.1-8b", layers=1, batch=256, num_q_heads=32, num_kv_heads=8, seed=2,
        ctx_kind="fixed", ctx_a=8192,
        key_lognormal_sigma=0.75,
        description="Llama-3.1-8B-shaped layer, batch 256, context 8192, "
                    "1-token append starting a new page, then decode"),
    "llama3-70b": Spec(
        "llama3-70b", layers=1, batch=16, num_q_heads=64, num_kv_heads=8, seed=3,
        ctx_kind="fixed", ctx_a=32768, shared_prefix_tokens=2048,
        outlier_frac=0.01, outlier_scale=10.0,
        description="Llama-3-70B-shaped layer, batch 16, context 32768 with a "
                    "2048-token shared prefix"),
    "llama3.2-3b-step": Spec(
        "llama3.2-3b-step", layers=28, batch=128, num_q_heads=24, num_kv_heads=8, seed=4,
        ctx_kind="lognormal", ctx_a=math.log(2048.0), ctx_b=1.0,
        outlier_frac=0.02, outlier_scale=8.0,
        description="Llama-3.2-3B-shaped full decode step, 28 layers, batch 128, "
                    "contexts lognormal clipped to [128,16384]"),
    # chunked prefill: the step appends a chunk of new tokens per sequence and
    # runs causal attention of the chunk over the cache
    "llama3.1-8b-prefill": Spec(
        "llama3.1-8b-prefill", layers=1, batch=4, num_q_heads=32, num_kv_heads=8, seed=6,
        ctx_kind="fixed", ctx_a=6144, step_new=(2048,),
        key_lognormal_sigma=0.75,
        description="Llama-3.1-8B-shaped layer, 4 sequences, a 2048-token chunk "
                    "appended to a 6144-token context, causal attention of the chunk"),
    "llama3-70b-prefill": Spec(
        "llama3-70b-prefill", layers=1, batch=2, num_q_heads=64, num_kv_heads=8, seed=7,
        ctx_kind="fixed", ctx_a=14336, step_new=(2048,),
        outlier_frac=0.01, outlier_scale=10.0,
        description="Llama-3-70B-shaped layer, 2 sequences, a 2048-token chunk "
                    "appended to a 14336-token context, causal attention of the chunk"),
}
CONFIG_ORDER = ["tiny", "qwen2.5-7b", "llama3.1-8b", "llama3-70b", "llama3.2-3b-step"]
PREFILL_ORDER = ["llama3.1-8b-prefill", "llama3-70b-prefill"]


def scaled(spec: Spec, batch: int | None = None, ctx_scale: float | None = None,
           layers: int | None = None) -> Spec:
    """A smaller variant of a spec with the same distributions (for tests)."""
    kw = {}
    if batch is not None:
        kw["batch"] = batch
    if layers is not None:
        kw["layers"] = layers
    if ctx_scale is not None:
        if spec.ctx_kind == "fixed" and spec.ctx_fixed:
            kw["ctx_fixed"] = tuple(int(c * ctx_scale) for c in spec.ctx_fixed)
        kw["ctx_a"] = spec.ctx_a * ctx_scale if spec.ctx_kind != "lognormal" else spec.ctx_a + math.log(ctx_scale)
        if spec.ctx_kind == "uniform":
            kw["ctx_b"] = spec.ctx_b * ctx_scale
        if spec.shared_prefix_tokens:
            kw["shared_prefix_tokens"] = max(PAGE, int(spec.shared_prefix_tokens * ctx_scale) // PAGE * PAGE)
    return dataclasses.replace(spec, name=spec.name + "-scaled", **kw)


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng([int(k) & 0xFFFFFFFF for k in key])


# --------------------------------------------------------------- lengths --

def context_lens(spec: Spec) -> np.ndarray:
    """Tokens in each sequence's cache before the step (int32 [batch])."""
    rng = _rng(spec.seed, 101)
    B = spec.batch
    if spec.ctx_kind == "fixed":
        if spec.ctx_fixed:
            ctx = np.array(spec.ctx_fixed[:B], dtype=np.int64)
        else:
            ctx = np.full(B, int(spec.ctx_a), dtype=np.int64)
    elif spec.ctx_kind == "uniform":
        ctx = rng.integers(int(spec.ctx_a), int(spec.ctx_b) + 1, size=B)
    elif spec.ctx_kind == "lognormal":
        lo, hi = 128, 16384
        ctx = np.clip(np.rint(rng.lognormal(spec.ctx_a, spec.ctx_b, size=B)), lo, hi)
    else:
        raise ValueError(spec.ctx_kind)
    if spec.shared_prefix_tokens:
        ctx = np.maximum(ctx, spec.shared_prefix_tokens)
    return ctx.astype(np.int32)


def step_new_tokens(spec: Spec) -> np.ndarray:
    """Tokens each sequence appends in the step (int32 [batch])."""
    if len(spec.step_new) == 1:
        return np.full(spec.batch, spec.step_new[0], np.int32)
    return np.array(spec.step_new[: spec.batch], np.int32)


def final_lens(spec: Spec) -> np.ndarray:
    return (context_lens(spec) + step_new_tokens(spec)).astype(np.int32)


# ----------------------------------------------------------- page tables --

@dataclasses.dataclass
class PagePlan:
    block_tables: np.ndarray   # int32 [batch][max_pages]
    num_pages: int             # physical pages in the pool
    shared_pages: int          # leading logical pages shared by every sequence
    unique_pages: int          # physical pages referenced (per kv head)


def page_plan(spec: Spec) -> PagePlan:
    """Random physical-page assignment: a shuffled pool, the shared prefix's
    pages appearing in every table, one spare page per sequence, unused
    table entries set to -1."""
    lens = final_lens(spec)
    need = (lens + PAGE - 1) // PAGE
    max_pages = int(need.max()) if lens.size else 1
    max_pages = max(max_pages, 1)
    shared = spec.shared_prefix_tokens // PAGE
    private = need - shared if shared else need
    unique = int(shared + private.sum())
    num_pages = unique + spec.batch  # spare pages stay unreferenced
    rng = _rng(spec.seed, 202)
    perm = rng.permutation(num_pages).astype(np.int32)
    bt = np.full((spec.batch, max_pages), -1, np.int32)
    cur = 0
    shared_ids = perm[cur:cur + shared]
    cur += shared
    for b in range(spec.batch):
        if shared:
            bt[b, :shared] = shared_ids
        k = int(private[b])
        bt[b, shared:shared + k] = perm[cur:cur + k]
        cur += k
    return PagePlan(bt, num_pages, shared, unique)


def slot_mapping(block_tables: np.ndarray, positions_per_seq: list[np.ndarray]) -> np.ndarray:
    """Physical slot (page * 16 + offset) of each new token, in call order."""
    out = []
    for b, pos in enumerate(positions_per_seq):
        pos = np.asarray(pos, np.int64)
        out.append(block_tables[b, pos // PAGE].astype(np.int64) * PAGE + pos % PAGE)
    return np.concatenate(out) if out else np.zeros(0, np.int64)


# ------------------------------------------------------------ K, V and q --

def key_channel_scale(spec: Spec, layer: int) -> np.ndarray:
    """Per (kv head, channel) multiplier of the key distribution."""
    rng = _rng(spec.seed, 303, layer)
    sc = np.ones((spec.num_kv_heads, HEAD_DIM), np.float32)
    if spec.key_lognormal_sigma > 0:
        sc = rng.lognormal(0.0, spec.key_lognormal_sigma,
                           size=(spec.num_kv_heads, HEAD_DIM)).astype(np.float32)
    n_out = spec.n_outliers()
    for h in range(spec.num_kv_heads):
        if n_out:
            ch = rng.choice(HEAD_DIM, size=n_out, replace=False)
            sc[h, ch] *= spec.outlier_scale
    return sc


def _seq_seed(spec: Spec, layer: int, b: int, shared: bool) -> tuple:
    return (spec.seed, 404, layer, -1 if shared else b)


def kv_sequence_np(spec: Spec, layer: int, b: int, n_tokens: int):
    """fp16 K, V [n_tokens][kv_heads][128] for tokens [0, n_tokens) of
    sequence b (numpy; tokens inside the shared prefix are the same for every
    sequence)."""
    H = spec.num_kv_heads
    ks = key_channel_scale(spec, layer)
    P = min(spec.shared_prefix_tokens, n_tokens)
    parts_k, parts_v = [], []
    if P:
        r = _rng(*_seq_seed(spec, layer, b, True))
        x = r.standard_normal((2, spec.shared_prefix_tokens, H, HEAD_DIM), dtype=np.float32)[:, :P]
        parts_k.append(x[0] * ks)
        parts_v.append(x[1])
    if n_tokens > P:
        r = _rng(*_seq_seed(spec, layer, b, False))
        x = r.standard_normal((2, n_tokens, H, HEAD_DIM), dtype=np.float32)[:, P:n_tokens]
        parts_k.append(x[0] * ks)
        parts_v.append(x[1])
    if not parts_k:
        z = np.zeros((0, H, HEAD_DIM), np.float16)
        return z, z.copy()
    k = np.concatenate(parts_k).astype(np.float16)
    v = np.concatenate(parts_v).astype(np.float16)
    return k, v


def queries_np(spec: Spec, layer: int, step: int = 0) -> np.ndarray:
    r = _rng(spec.seed, 505, layer, step)
    return r.standard_normal((spec.batch, spec.num_q_heads, HEAD_DIM), dtype=np.float32).astype(np.float16)


def _torch_gen(device, key: tuple):
    import torch
    g = torch.Generator(device=device)
    h = 1469598103934665603
    for k in key:
        h = ((h ^ (int(k) & 0xFFFFFFFFFFFF)) * 1099511628211) & 0x7FFFFFFFFFFFFFFF
    g.manual_seed(h)
    return g


def kv_sequence_torch(spec: Spec, layer: int, b: int, n_tokens: int, device,
                      key_scale=None):
    """Device-side counterpart of kv_sequence_np (same distributions, torch
    generator): fp16 K, V [n_tokens][kv_heads][128] on ``device``."""
    import torch
    H = spec.num_kv_heads
    if key_scale is None:
        key_scale = torch.from_numpy(key_channel_scale(spec, layer)).to(device)
    P = min(spec.shared_prefix_tokens, n_tokens)
    ks_, vs_ = [], []
    if P:
        g = _torch_gen(device, _seq_seed(spec, layer, b, True))
        x = torch.randn((2, spec.shared_prefix_tokens, H, HEAD_DIM), generator=g,
                        device=device, dtype=torch.float32)[:, :P]
        ks_.append(x[0] * key_scale)
        vs_.append(x[1])
    if n_tokens > P:
        g = _torch_gen(device, _seq_seed(spec, layer, b, False))
        x = torch.randn((2, n_tokens, H, HEAD_DIM), generator=g, device=device,
                        dtype=torch.float32)[:, P:n_tokens]
        ks_.append(x[0] * key_scale)
        vs_.append(x[1])
    if not ks_:
        z = torch.zeros((0, H, HEAD_DIM), dtype=torch.float16, device=device)
        return z, z.clone()
    return torch.cat(ks_).half(), torch.cat(vs_).half()


def queries_torch(spec: Spec, layer: int, device, step: int = 0):
    import torch
    g = _torch_gen(device, (spec.seed, 505, layer, step))
    return torch.randn((spec.batch, spec.num_q_heads, HEAD_DIM), generator=g,
                       device=device, dtype=torch.float32).half()


# ------------------------------------------------------------- byte model --

def decode_bytes(spec: Spec, lens: np.ndarray | None = None, plan: PagePlan | None = None,
                 block_bytes: int = 2816) -> dict:
    """Algorithmic bytes one decode pass reads (per layer): every unique
    (physical page, kv head) block once, the fp16 residual rows (K and V) and
    q; plus the logical total that counts shared pages once per sequence."""
    if lens is None:
        lens = final_lens(spec)
    if plan is None:
        plan = page_plan(spec)
    full = lens // PAGE
    resid = lens % PAGE
    H = spec.num_kv_heads
    shared = plan.shared_pages
    unique_full = int(min(shared, int(full.min()) if full.size else 0) +
                      np.maximum(full - shared, 0).sum()) if shared else int(full.sum())
    pages_unique = unique_full * H * block_bytes
    pages_logical = int(full.sum()) * H * block_bytes
    residual = int(resid.sum()) * H * 2 * HEAD_DIM * 2
    q = spec.batch * spec.num_q_heads * HEAD_DIM * 2
    out = spec.batch * spec.num_q_heads * HEAD_DIM * 2
    return {"pages_unique": pages_unique, "pages_logical": pages_logical,
            "residual": residual, "q": q, "out": out,
            "algorithmic": pages_unique + residual + q,
            "logical": pages_logical + residual + q,
            "kv_tokens": int(lens.sum())}


def chunk_queries_np(spec: Spec, layer: int, n_rows: int, step: int = 0) -> np.ndarray:
    """fp16 q [n_rows][num_q_heads][128] for every appended token of a step."""
    r = _rng(spec.seed, 606, layer, step)
    return r.standard_normal((n_rows, spec.num_q_heads, HEAD_DIM), dtype=np.float32).astype(np.float16)


def chunk_queries_torch(spec: Spec, layer: int, n_rows: int, device, step: int = 0):
    import torch
    g = _torch_gen(device, (spec.seed, 606, layer, step))
    return torch.randn((n_rows, spec.num_q_heads, HEAD_DIM), generator=g,
                       device=device, dtype=torch.float32).half()
