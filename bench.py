#!/usr/bin/env python3
"""Benchmark of the int4 KIVI paged decode step on B200.

One step = for every layer of the workload: s4kv_append of the step's new
token(s) (quantizing every page it completes) followed by
s4kv_decode_attention over the whole cache.  Inputs are seeded synthetic
tensors shaped like the named model layer (see
int4_kivi_quantized_s4kv_b200/workloads.py), resident in HBM before timing.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Prints ONE JSON line (rank 0).  `value` is algorithmic bytes per step (pages
read once per unique physical page and kv head, residual rows, q, plus the
append's K/V in and residual out) divided by the device time of a step, over
all ranks.  Multi-GPU runs are independent replicas (weak scaling, no
collective on the data path); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from int4_kivi_quantized_s4kv_b200 import workloads as W  # noqa: E402

METRIC = "int4 paged decode attn: achieved HBM GB/s (% of B200 peak), tokens/s"
DEFAULT_WORKLOAD = "llama3.1-8b"
FALLBACK_HBM_GBS = 6650.0


def measured_hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------- traffic --

KERNEL_SOURCES = ["int4_kivi_quantized_s4kv_b200/csrc/decode.cu", "int4_kivi_quantized_s4kv_b200/csrc/common.cuh",
                  "int4_kivi_quantized_s4kv_b200/csrc/kernels.cuh", "include/s4kv.h"]


def kernel_sources_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(algorithmic_bytes: float, bits: int = 4):
    """DRAM bytes (read + write) per decode launch from the committed ncu
    capture of that code width, scaled from the captured case by algorithmic
    bytes; None when the decode kernel's sources changed since the capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "decode_traffic.json")) as f:
            recs = json.load(f)
    except Exception:
        return None
    rec = recs.get("widths", {}).get(str(bits))
    if rec is None or recs.get("kernel_sources_sha256") != kernel_sources_sha():
        return None
    return algorithmic_bytes * rec["dram_bytes"] / rec["algorithmic_bytes"]


# ----------------------------------------------------------------- clocks --

class ClockSampler:
    """Reads SM clocks and throttle reasons through NVML while running (read
    only; no GPU setting is changed)."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
        self.period = period_s

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                clk = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                util = nv.nvmlDeviceGetUtilizationRates(self._h).gpu
                self.samples.append((clk, rs, util))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self._nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        loaded = [s for s in self.samples if s[2] > 0] or self.samples
        reasons = set()
        for _, rs, _ in loaded:
            for name, bit in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": float(statistics.median(s[0] for s in loaded)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(loaded)}


# -------------------------------------------------------------- workload --

def step_bytes(spec, plan, lens, bits: int = 4):
    d = W.decode_bytes(spec, lens, plan, block_bytes={2: 1792, 4: 2816, 8: 4864}[bits])
    new = W.step_new_tokens(spec)
    kv_new = int(new.sum()) * spec.num_kv_heads * 128 * 2 * 2   # k and v read
    append = 2 * kv_new                                         # residual write (upper bound)
    return d, append


class DeviceWorkload:
    """All layers' caches of one workload on one GPU, filled through the C
    ABI, plus the step's inputs."""

    def __init__(self, spec: W.Spec, device, prefill_tokens_per_call=1 << 18, bits: int = 4):
        import torch
        import int4_kivi_quantized_s4kv_b200 as S
        self.S, self.torch = S, torch
        self.spec, self.device, self.bits = spec, device, bits
        self.ctx = W.context_lens(spec)
        self.lens = W.final_lens(spec)
        self.new = W.step_new_tokens(spec)
        self.plan = W.page_plan(spec)
        B, H = spec.batch, spec.num_kv_heads
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)  # noqa: E731
        self.bt = dev(self.plan.block_tables)
        self.seq_lens = dev(self.lens)
        pos = [np.arange(self.ctx[b], self.lens[b]) for b in range(B)]
        self.step_slots = dev(W.slot_mapping(self.plan.block_tables, pos))
        self.step_cu = dev(np.concatenate([[0], np.cumsum(self.new)]).astype(np.int32))
        self.max_new = int(self.new.max())
        self.one_token = bool((self.new == 1).all())
        self.caches, self.q, self.k_new, self.v_new = [], [], [], []
        for layer in range(spec.layers):
            cache = S.S4KVCache(self.plan.num_pages, H, B, device=device, bits=bits)
            ks = torch.from_numpy(W.key_channel_scale(spec, layer)).to(device)
            kn, vn = [], []
            b = 0
            # the shared prefix's pages are written once, by sequence 0; the
            # other sequences append from the prefix boundary (a page boundary)
            start = [0] + [spec.shared_prefix_tokens] * (B - 1)
            while b < B:
                # a batch of sequences per prefill call, bounded in tokens
                b1, tok = b, 0
                while b1 < B and (tok == 0 or tok + int(self.ctx[b1]) - start[b1] <= prefill_tokens_per_call):
                    tok += int(self.ctx[b1]) - start[b1]
                    b1 += 1
                kk, vv, slots, counts = [], [], [], []
                for bb in range(b, b1):
                    k_seq, v_seq = W.kv_sequence_torch(spec, layer, bb, int(self.lens[bb]), device, ks)
                    c, c0 = int(self.ctx[bb]), start[bb]
                    kk.append(k_seq[c0:c])
                    vv.append(v_seq[c0:c])
                    kn.append(k_seq[c:])
                    vn.append(v_seq[c:])
                    slots.append(W.slot_mapping(self.plan.block_tables[bb:bb + 1], [np.arange(c0, c)]))
                    counts.append(c - c0)
                cnt = np.zeros(B, np.int64)
                cnt[b:b1] = counts
                if cnt.sum() > 0:
                    # sequences outside [b, b1) append nothing: their lengths are not read
                    S.s4kv_append(cache, torch.cat(kk).contiguous(), torch.cat(vv).contiguous(),
                                  dev(np.concatenate(slots)), dev(np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32)),
                                  dev(self.ctx), self.bt, int(max(counts)))
                b = b1
            torch.cuda.synchronize(device)
            self.caches.append(cache)
            self.k_new.append(torch.cat(kn).contiguous())
            self.v_new.append(torch.cat(vn).contiguous())
            self.q.append(W.queries_torch(spec, layer, device))
        self.out = [torch.empty_like(q) for q in self.q]
        self.ws = S.decode_workspace(B, H, device)
        for c in self.caches:
            flags = S.s4kv_get_error(c)
            if flags:
                raise RuntimeError(f"device flags {flags} after prefill")

    def step(self, dec_events=None, one_call=False):
        """One decode step of every layer.  With `one_call` (and one new token
        per sequence) each layer is one s4kv_append_decode call; otherwise
        s4kv_append then s4kv_decode_attention, with `dec_events` (if given)
        recorded around the decode launch."""
        S = self.S
        if one_call and self.one_token and dec_events is None:
            B, H = self.spec.batch, self.spec.num_kv_heads
            for layer in range(self.spec.layers):
                S.s4kv_append_decode(self.caches[layer], self.k_new[layer].view(B, H, 128),
                                     self.v_new[layer].view(B, H, 128), self.q[layer], self.seq_lens, self.bt,
                                     self.out[layer], self.ws)
            return
        for layer in range(self.spec.layers):
            S.s4kv_append(self.caches[layer], self.k_new[layer], self.v_new[layer], self.step_slots,
                          self.step_cu, self.seq_lens, self.bt, self.max_new)
            if dec_events is not None:
                dec_events[0].append(self.torch.cuda.Event(enable_timing=True))
                dec_events[1].append(self.torch.cuda.Event(enable_timing=True))
                dec_events[0][-1].record()
            S.s4kv_decode_attention(self.caches[layer], self.q[layer], self.seq_lens, self.bt,
                                    self.out[layer], self.ws)
            if dec_events is not None:
                dec_events[1][-1].record()

    def launches_per_step(self):
        return 2 * self.spec.layers


# ------------------------------------------------------------ CPU oracle --

class OracleSample:
    """The oracle on a bounded sample of the workload: `n_units` (sequence, kv
    head) pairs of layer 0, prefilled untimed; one call of `run()` is the
    step (append of the new token(s) + decode) for the sampled sequences."""

    def __init__(self, spec: W.Spec, n_seqs: int, bits: int = 4, first: int = 0):
        import oracle
        oracle.build()
        first = max(0, min(first, spec.batch - 1))
        n_seqs = max(1, min(n_seqs, spec.batch - first))
        self.spec = spec
        ctx, lens = W.context_lens(spec), W.final_lens(spec)
        self.seqs = list(range(first, first + n_seqs))
        # compact page tables for the sample (shared pages become private)
        need = [(int(lens[b]) + 15) // 16 for b in self.seqs]
        bt = np.full((n_seqs, max(need)), -1, np.int32)
        c = 0
        for j, n in enumerate(need):
            bt[j, :n] = np.arange(c, c + n)
            c += n
        self.bt = bt
        self.cache = oracle.OracleCache(c + 1, spec.num_kv_heads, n_seqs, bits=bits)
        self.ctx = ctx[self.seqs]
        self.lens = lens[self.seqs]
        k, v = zip(*[W.kv_sequence_np(spec, 0, b, int(lens[b])) for b in self.seqs])
        cu = np.concatenate([[0], np.cumsum(self.ctx)]).astype(np.int32)
        sm = W.slot_mapping(bt, [np.arange(int(x)) for x in self.ctx])
        rc = self.cache.append(np.concatenate([k[j][:self.ctx[j]] for j in range(n_seqs)]),
                               np.concatenate([v[j][:self.ctx[j]] for j in range(n_seqs)]),
                               sm, cu, self.ctx, bt)
        assert rc == 0
        self.k_new = np.concatenate([k[j][self.ctx[j]:] for j in range(n_seqs)])
        self.v_new = np.concatenate([v[j][self.ctx[j]:] for j in range(n_seqs)])
        self.sm_new = W.slot_mapping(bt, [np.arange(self.ctx[j], self.lens[j]) for j in range(n_seqs)])
        self.cu_new = np.concatenate([[0], np.cumsum(self.lens - self.ctx)]).astype(np.int32)
        self.q = W.queries_np(spec, 0)[self.seqs]
        sub = W.Spec(**{**spec.__dict__, "batch": n_seqs, "shared_prefix_tokens": 0,
                        "ctx_kind": "fixed", "ctx_fixed": tuple(int(x) for x in self.ctx)})
        self.bytes = W.decode_bytes(sub, self.lens, W.PagePlan(bt, c + 1, 0, c),
                                    block_bytes={2: 1792, 4: 2816, 8: 4864}[bits])["algorithmic"]
        self.tokens = n_seqs

    def run(self):
        rc = self.cache.append(self.k_new, self.v_new, self.sm_new, self.cu_new, self.lens, self.bt)
        assert rc == 0
        return self.cache.decode_attention(self.q, self.lens, self.bt)


def _oracle_slice(args):
    """One process of the multi-core baseline: the unchanged oracle on a slice
    of sequences (prefilled untimed), one timed step after all processes are
    ready."""
    spec, first, n, bits, barrier = args
    samp = OracleSample(spec, n, bits, first=first)
    barrier.wait()
    t0 = time.perf_counter()
    samp.run()
    dt = time.perf_counter() - t0
    return samp.bytes, samp.tokens, dt


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline_multicore(spec, n_single: int, bits: int = 4):
    """The same oracle in one process per host core, each on its own slice of
    sequences (n_single of them per process, the single-threaded sample's
    size), started together: aggregate bytes over the slowest process's time.
    Processes are spawned (not forked) so that no CUDA state is inherited."""
    import multiprocessing as mp
    cores = cpu_cores()
    per = max(1, n_single)
    nproc = max(1, min(cores, spec.batch // per))
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        barrier = mgr.Barrier(nproc)
        with ctx.Pool(nproc) as pool:
            res = pool.map(_oracle_slice, [(spec, k * per, per, bits, barrier) for k in range(nproc)])
    total_bytes = sum(r[0] for r in res)
    total_tokens = sum(r[1] for r in res)
    dt = max(r[2] for r in res)
    return {"value": total_bytes / dt / 1e9, "unit": "GB/s", "cores": nproc, "host_cores": cores,
            "kind": "oracle",
            "sample": f"{nproc} processes x {per} sequences of layer 0 (all kv heads), one step "
                      f"(append + decode) each, started together; {dt:.1f} s for the slowest",
            "tokens_per_s": total_tokens / dt, "seconds": dt}


def cpu_baseline(spec, budget_s=12.0, bits: int = 4):
    probe = OracleSample(spec, 1, bits)
    t0 = time.perf_counter()
    probe.run()
    t1 = time.perf_counter() - t0
    n = int(max(1, min(spec.batch, budget_s / max(t1, 1e-3))))
    samp = OracleSample(spec, n, bits) if n > 1 else probe
    t0 = time.perf_counter()
    samp.run()
    dt = time.perf_counter() - t0
    single = {"value": samp.bytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
              "sample": f"{n} of {spec.batch} sequences of layer 0 (all kv heads), one step "
                        f"(append + decode), {dt:.1f} s single-threaded",
              "tokens_per_s": samp.tokens / dt, "seconds": dt}
    multi = cpu_baseline_multicore(spec, n, bits)
    out = dict(multi)
    out["single_core"] = single
    return out


# ------------------------------------------------------------------ main --

def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def replica_spec(spec, rank: int):
    """Rank r's replica of the workload: same shapes, its own seeds (each
    rank decodes its own batch; no data crosses GPUs)."""
    if rank == 0:
        return spec
    import dataclasses
    return dataclasses.replace(spec, seed=spec.seed + 1000 * rank)


def reduce_max(x: float, world: int, device) -> float:
    """Max over ranks of a per-rank time (the only collective in the bench)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(world: int, bytes_per_step_per_rank: float, step_ms: float) -> float:
    """Whole-job throughput: bytes all ranks processed per step / slowest step."""
    return world * bytes_per_step_per_rank / (step_ms * 1e-3) / 1e9


def config_dict(spec, extra=None):
    d = {"workload": spec.name, "model_shape": spec.description, "layers": spec.layers,
         "batch": spec.batch, "num_q_heads": spec.num_q_heads, "num_kv_heads": spec.num_kv_heads,
         "head_dim": 128, "page_tokens": 16}
    if extra:
        d.update(extra)
    return d


def measured_tensor_peak():
    """Dense fp16/bf16 tensor-core TFLOP/s measured on this machine (fp16 and bf16
    MMAs run at the same nominal rate)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (bf16 cuBLAS burst; fp16 has the same nominal rate)"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


def prefill_flops(spec, lens, new):
    """Algorithmic FLOPs of causal chunk attention: every q head of row j
    (position L - n + j) does 2 * 128 multiply-adds per key for q.k and as
    many for p.v over keys 0 .. L - n + j."""
    f = 0
    for L, n in zip(lens.tolist(), new.tolist()):
        f += spec.num_q_heads * 4 * 128 * (n * (L - n) + n * (n + 1) // 2)
    return f


def measure_prefill(device, steps: int, workload: str = "llama3.1-8b-prefill", bits: int = 4):
    """Chunked-prefill attention (the cache's prefill side) on its own
    workload: the chunk is appended once, then s4kv_prefill_attention is timed
    with CUDA events on the launching stream."""
    import torch
    spec = W.SPECS[workload]
    wl = DeviceWorkload(spec, device, bits=bits)
    S = wl.S
    cache = wl.caches[0]
    S.s4kv_append(cache, wl.k_new[0], wl.v_new[0], wl.step_slots, wl.step_cu, wl.seq_lens, wl.bt, wl.max_new)
    rows = int(wl.new.sum())
    q = W.chunk_queries_torch(spec, 0, rows, device)
    out = torch.empty_like(q)
    ws = S.prefill_workspace(spec.num_kv_heads, spec.batch, wl.bt.shape[1], device)

    def run():
        S.s4kv_prefill_attention(cache, q, wl.step_cu, wl.seq_lens, wl.bt, out, wl.max_new, workspace=ws)

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        run()
        b.record()
        times.append((a, b))
    torch.cuda.synchronize()
    ms = sum(x.elapsed_time(y) for x, y in times) / len(times)
    flags = S.s4kv_get_error(cache)
    if flags:
        raise RuntimeError(f"prefill device error flags {flags}")
    flops = prefill_flops(spec, wl.lens, wl.new)
    peak, kind = measured_tensor_peak()
    achieved = flops / (ms * 1e-3) / 1e12
    # a call is two launches: the operand tiles (each page dequantized once)
    # and the attention, whose MMAs per (query tile, key tile) are
    # Q K_hi^T + Q8 K_lo^T (keys carried to about 2^-14 relative; the K_lo
    # part on the e5m2 MMA at twice the fp16 rate) and P V: 1.5x the
    # algorithmic FLOPs
    return {"workload": spec.name, "model_shape": spec.description, "code_bits": bits, "calls": steps,
            "launches": 2 * steps,
            "avg_call_ms": ms, "tflops": achieved, "query_tokens": rows,
            "roofline": {"bound": "tensor", "kernel": "prefill_operands_kernel + prefill_kernel (one call)",
                         "achieved": achieved, "peak": peak, "peak_kind": kind, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": None, "flops_per_call": flops,
                         "mma_flops_per_call": 1.5 * flops}}


def measure_page_moves(wl, device, reps: int = 10):
    """Swap-side page movement on the decode workload's resident cache:
    gathering page records into a staging buffer (HBM read + write), and a
    whole swap-out / swap-in through pinned host memory (bound by the
    host link)."""
    import torch
    S = wl.S
    cache = wl.caches[0]
    H = wl.spec.num_kv_heads
    rec = S.s4kv_page_record_bytes(cache)
    nfull = (wl.lens // 16).astype(np.int64)
    # gather: as many whole sequences as make > 2x L2 of records
    rows, total = [], 0
    for b in range(wl.spec.batch):
        rows.append(wl.plan.block_tables[b, :nfull[b]])
        total += int(nfull[b]) * rec
        if total > 300e6:
            break
    pages = torch.from_numpy(np.ascontiguousarray(np.concatenate(rows).astype(np.int32))).to(device)
    n = pages.numel()
    staging = torch.empty((n, rec), dtype=torch.uint8, device=device)

    def timed(fn, k):
        fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(k):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / k

    g_ms = timed(lambda: S.s4kv_gather_pages(cache, pages, staging), reps)
    # swap-out / swap-in of one sequence's pages through pinned host memory
    sp = pages[: int(nfull[0])]
    host = torch.empty((sp.numel(), rec), dtype=torch.uint8, pin_memory=True)
    st = staging[: sp.numel()]
    o_ms = timed(lambda: S.s4kv_swap_out(cache, sp, st, host), 3)
    i_ms = timed(lambda: S.s4kv_swap_in(cache, sp, st, host), 3)   # writes the same bytes back
    if S.s4kv_get_error(cache):
        raise RuntimeError("page movement set device error flags")
    peak, kind = measured_hbm_peak()
    gbs = 2 * n * rec / (g_ms * 1e-3) / 1e9
    swap_bytes = sp.numel() * rec
    return {"gather": {"pages": n, "record_bytes": rec, "avg_launch_ms": g_ms,
                       "roofline": {"bound": "hbm", "kernel": "move_kernel", "achieved": gbs, "peak": peak,
                                    "peak_kind": kind, "unit": "GB/s", "frac": gbs / peak, "traffic": None,
                                    "bytes_per_launch": 2 * n * rec}},
            "swap_out": {"bytes": swap_bytes, "ms": o_ms, "GB_per_s": swap_bytes / (o_ms * 1e-3) / 1e9},
            "swap_in": {"bytes": swap_bytes, "ms": i_ms, "GB_per_s": swap_bytes / (i_ms * 1e-3) / 1e9}}


def measure_fused_step(wl, device, steps: int = 20):
    """One decode step as two independent calls (s4kv_append,
    s4kv_decode_attention) and as one s4kv_append_decode call (the step's
    append grid, then the decode grid as its programmatic dependent) on the
    same resident workload; both rewrite the same cache bytes each step."""
    import torch
    S = wl.S
    spec = wl.spec
    B, H = spec.batch, spec.num_kv_heads
    kn = [k.view(B, H, 128) for k in wl.k_new]
    vn = [v.view(B, H, 128) for v in wl.v_new]

    def fused():
        for layer in range(spec.layers):
            S.s4kv_append_decode(wl.caches[layer], kn[layer], vn[layer], wl.q[layer], wl.seq_lens, wl.bt,
                                 wl.out[layer], wl.ws)

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps

    two = timed(wl.step)
    one = timed(fused)
    if any(S.s4kv_get_error(c) for c in wl.caches):
        raise RuntimeError("fused step set device error flags")
    return {"workload": spec.name, "layers": spec.layers, "two_launch_ms": two, "fused_ms": one,
            "speedup": two / one, "launches_per_layer": {"two_launch": 2, "fused": 2},
            "fused_launch": "append grid + programmatically dependent decode grid"}


BLOCK_BYTES = {2: 1792, 4: 2816, 8: 4864}


def measure_decode_config(device, name: str, steps: int = 20):
    """Decode of one of the other large workloads (every layer): the average
    s4kv_decode_attention launch against the HBM roofline on its unique bytes
    (shared-prefix pages counted once), the logical bytes beside them, and the
    whole step (append + decode of every layer) as two independent calls per
    layer and as one s4kv_append_decode call per layer."""
    import torch
    spec = W.SPECS[name]
    wl = DeviceWorkload(spec, device)
    dbytes, abytes = step_bytes(wl.spec, wl.plan, wl.lens)
    for _ in range(3):
        wl.step()
    torch.cuda.synchronize()
    ev = ([], [])
    for _ in range(steps):
        wl.step(ev)
    torch.cuda.synchronize()
    dec_ms = sum(a.elapsed_time(b) for a, b in zip(*ev)) / len(ev[0])
    fused = measure_fused_step(wl, device, steps=max(3, min(steps, 10) if spec.layers > 1 else steps))
    if any(wl.S.s4kv_get_error(c) for c in wl.caches):
        raise RuntimeError(f"{name} decode set device error flags")
    peak, kind = measured_hbm_peak()
    gbs = dbytes["algorithmic"] / (dec_ms * 1e-3) / 1e9
    step_bytes_all = (dbytes["algorithmic"] + abytes) * spec.layers
    tokens = int(wl.new.sum())
    res = {"workload": name, "model_shape": spec.description, "layers": spec.layers, "batch": spec.batch,
           "num_q_heads": spec.num_q_heads, "num_kv_heads": spec.num_kv_heads,
           "context": {"min": int(wl.ctx.min()), "max": int(wl.ctx.max()), "mean": float(wl.ctx.mean())},
           "shared_prefix_tokens": spec.shared_prefix_tokens,
           "decode_launches": len(ev[0]), "avg_launch_ms": dec_ms,
           "unique_bytes_per_launch": dbytes["algorithmic"], "logical_bytes_per_launch": dbytes["logical"],
           "logical_GBs": dbytes["logical"] / (dec_ms * 1e-3) / 1e9,
           "tokens_per_s": tokens / (dec_ms * 1e-3 * spec.layers),
           "sequences_per_s": spec.batch / (dec_ms * 1e-3 * spec.layers),
           "roofline": {"bound": "hbm", "kernel": "decode_kernel<4>", "achieved": gbs, "peak": peak,
                        "peak_kind": kind, "unit": "GB/s", "frac": gbs / peak, "traffic": None,
                        "bytes_per_launch": dbytes["algorithmic"]},
           "step": {"two_launch_ms": fused["two_launch_ms"], "fused_ms": fused["fused_ms"],
                    "two_launch_GBs": step_bytes_all / (fused["two_launch_ms"] * 1e-3) / 1e9,
                    "fused_GBs": step_bytes_all / (fused["fused_ms"] * 1e-3) / 1e9,
                    "tokens_per_s_two_launch": tokens / (fused["two_launch_ms"] * 1e-3),
                    "tokens_per_s_fused": tokens / (fused["fused_ms"] * 1e-3),
                    "launches_per_step": {"two_launch": 2 * spec.layers, "fused": 2 * spec.layers}}}
    del wl
    torch.cuda.empty_cache()
    return res


def measure_width_decode(device, spec, bits: int, steps: int = 20):
    """The 8- or 2-bit variant's decode step (append + decode) on the same
    workload as the headline, against the HBM roofline."""
    import torch
    wl = DeviceWorkload(spec, device, bits=bits)
    dbytes, _ = step_bytes(wl.spec, wl.plan, wl.lens, bits=bits)
    for _ in range(3):
        wl.step()
    torch.cuda.synchronize()
    ev = ([], [])
    for _ in range(steps):
        wl.step(ev)
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in zip(*ev)) / steps
    if any(wl.S.s4kv_get_error(c) for c in wl.caches):
        raise RuntimeError(f"int{bits} decode set device error flags")
    peak, kind = measured_hbm_peak()
    gbs = dbytes["algorithmic"] / (ms * 1e-3) / 1e9
    return {"workload": spec.name, "bits": bits, "block_bytes": BLOCK_BYTES[bits], "avg_launch_ms": ms,
            "tokens_per_s": int(wl.new.sum()) / (ms * 1e-3),
            "roofline": {"bound": "hbm", "kernel": f"decode_kernel<{bits}>", "achieved": gbs, "peak": peak,
                         "peak_kind": kind, "unit": "GB/s", "frac": gbs / peak, "traffic": None,
                         "bytes_per_launch": dbytes["algorithmic"]}}


def run_reference(args, spec):
    world, rank, _ = _dist()
    if rank != 0:
        return 0
    total = args.steps + args.warmup
    probe = OracleSample(spec, 1)
    t0 = time.perf_counter()
    probe.run()
    t1 = time.perf_counter() - t0
    per_step_budget = max(0.05, 150.0 / max(total, 1))
    n = int(max(1, min(spec.batch, per_step_budget / max(t1, 1e-3))))
    samp = OracleSample(spec, n) if n > 1 else probe
    for _ in range(args.warmup):
        samp.run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        samp.run()
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    val = samp.bytes / dt / 1e9
    sample = f"{n} of {spec.batch} sequences of layer 0 per step (append + decode), single-threaded"
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(spec, {"sample": sample}),
            "cpu_baseline": {"value": val, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "tokens_per_s": samp.tokens / dt}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="s4kv", choices=["s4kv", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=W.CONFIG_ORDER)
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller profiling cases)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--bits", type=int, default=4, choices=[2, 4, 8],
                    help="code width of the cache (4: the int4 KIVI path; 8 / 2: its variants)")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the chunked-prefill attention measurement")
    args = ap.parse_args(argv)
    spec = W.SPECS[args.workload]
    if args.batch is not None:
        import dataclasses
        spec = dataclasses.replace(spec, batch=args.batch, name=f"{spec.name}-b{args.batch}")
    if args.impl == "reference":
        return run_reference(args, spec)
    if args.warmup < 3:
        args.warmup = 3

    import torch
    world, rank, local = _dist()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from int4_kivi_quantized_s4kv_b200 import build
    if rank == 0:
        build.build()
    if world > 1:
        torch.distributed.barrier()

    wl = DeviceWorkload(replica_spec(spec, rank), device, bits=args.bits)
    dbytes, abytes = step_bytes(wl.spec, wl.plan, wl.lens, bits=args.bits)
    bytes_per_step = (dbytes["algorithmic"] + abytes) * spec.layers
    decode_bytes_per_launch = dbytes["algorithmic"]

    # the step: one s4kv_append_decode call per layer (the append grid and
    # the decode grid as its programmatic dependent) when every sequence gets
    # one new token, else s4kv_append then s4kv_decode_attention
    for _ in range(args.warmup):
        wl.step(one_call=True)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                          else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local]))
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t_start.record()
    for _ in range(args.steps):
        wl.step(one_call=True)
    t_end.record()
    torch.cuda.synchronize()
    clocks.stop()
    step_ms = t_start.elapsed_time(t_end) / args.steps
    step_ms = reduce_max(step_ms, world, device)
    # the decode kernel on its own for the roofline: the same steps as two
    # calls, with events around each decode launch (a dependent grid of the
    # one-call step cannot be bracketed by events of its own)
    ev = ([], [])
    for _ in range(args.steps):
        wl.step(ev)
    torch.cuda.synchronize()
    dec_ms = [a.elapsed_time(b) for a, b in zip(*ev)]
    dec_avg_ms = sum(dec_ms) / len(dec_ms)

    # end to end through the public API: every step copies its inputs (q and
    # the new tokens' K/V) in from pinned host memory and its output back.
    # Two sets of device buffers let step i+1's inputs travel on a copy
    # stream while step i computes (the step reads only its own set).
    h_q = [q.cpu().pin_memory() for q in wl.q]
    h_k = [k.cpu().pin_memory() for k in wl.k_new]
    h_v = [v.cpu().pin_memory() for v in wl.v_new]
    h_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in wl.out]
    h2d = sum(t.numel() * t.element_size() for t in h_q + h_k + h_v)
    d2h = sum(t.numel() * t.element_size() for t in h_out)
    sets = [(wl.q, wl.k_new, wl.v_new, wl.out),
            ([torch.empty_like(t) for t in wl.q], [torch.empty_like(t) for t in wl.k_new],
             [torch.empty_like(t) for t in wl.v_new], [torch.empty_like(t) for t in wl.out])]
    comp = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    loaded = [torch.cuda.Event(), torch.cuda.Event()]
    done = [torch.cuda.Event(), torch.cuda.Event()]

    def h2d_copy(i):
        q_, k_, v_, _ = sets[i % 2]
        with torch.cuda.stream(copy):
            if i >= 2:
                copy.wait_event(done[i % 2])      # step i-2 finished with this set
            for layer in range(spec.layers):
                q_[layer].copy_(h_q[layer], non_blocking=True)
                k_[layer].copy_(h_k[layer], non_blocking=True)
                v_[layer].copy_(h_v[layer], non_blocking=True)
            loaded[i % 2].record(copy)

    def e2e_run(n):
        h2d_copy(0)
        for i in range(n):
            if i + 1 < n:
                h2d_copy(i + 1)
            comp.wait_event(loaded[i % 2])
            wl.q, wl.k_new, wl.v_new, wl.out = sets[i % 2]
            wl.step(one_call=True)
            done[i % 2].record(comp)
            with torch.cuda.stream(copy):
                copy.wait_event(done[i % 2])
                for layer in range(spec.layers):
                    h_out[layer].copy_(wl.out[layer], non_blocking=True)
        comp.wait_stream(copy)
        wl.q, wl.k_new, wl.v_new, wl.out = sets[0]

    e2e_run(3)
    torch.cuda.synchronize()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_steps = max(3, min(args.steps, 50))
    e_start.record()
    e2e_run(e_steps)
    e_end.record()
    torch.cuda.synchronize()
    e2e_ms = e_start.elapsed_time(e_end) / e_steps
    e2e_ms = reduce_max(e2e_ms, world, device)

    flags = [wl.S.s4kv_get_error(c) for c in wl.caches]
    if any(flags):
        raise RuntimeError(f"device error flags {flags}")

    peak, peak_kind = measured_hbm_peak()
    value = aggregate_gbs(world, bytes_per_step, step_ms)
    achieved = decode_bytes_per_launch / (dec_avg_ms * 1e-3) / 1e9
    tokens = int(wl.new.sum())
    prefill = moves = fused = int8 = int2 = configs = None
    extra_clocks = None
    if world == 1 and not args.no_prefill:
        # the HBM-bound measurements first: the tensor-bound prefill runs at
        # the power cap and leaves the clocks lower for a while afterwards
        extra = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                             else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local]))
        extra.start()
        fused = [measure_fused_step(wl, device)]
        moves = measure_page_moves(wl, device)
        configs = [measure_decode_config(device, name) for name in W.CONFIG_ORDER
                   if name not in ("tiny", spec.name.split("-b")[0] if args.batch else spec.name)]
        int8 = measure_width_decode(device, spec, 8)
        int2 = measure_width_decode(device, spec, 2)
        prefill = [measure_prefill(device, max(3, min(args.steps, 20)), w, args.bits) for w in W.PREFILL_ORDER]
        extra.stop()
        extra_clocks = extra.summary()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(spec, bits=args.bits)
    if world > 1:
        torch.distributed.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": f"int{args.bits} codes, f16 MMA operands, f32 accumulate",
            "data": "synthetic (seeded Gaussian K/V/q with outlier key channels; no dataset)",
            "config": config_dict(spec, {
                "code_bits": args.bits,
                "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                "context": {"min": int(wl.ctx.min()), "max": int(wl.ctx.max()), "mean": float(wl.ctx.mean())},
                "new_tokens_per_seq": int(wl.new.max()),
                "step_calls": ("s4kv_append_decode per layer" if wl.one_token
                               else "s4kv_append + s4kv_decode_attention per layer"),
                "shared_prefix_tokens": spec.shared_prefix_tokens,
                "decode_bytes_per_layer": dbytes, "append_bytes_per_layer": abytes,
                "l2": f"inputs larger than L2: {bytes_per_step / 1e9:.2f} GB read per step vs 126 MB L2"
                      if bytes_per_step > 2e8 else "inputs smaller than L2",
            }),
            "pct_of_peak": {"measured_hbm": value / world / peak, "spec_8tbs": value / world / 8000.0},
            "tokens_per_s": world * tokens / (step_ms * 1e-3),
            "sequences_per_s": world * spec.batch / (step_ms * 1e-3),
            "kv_tokens_per_s": world * spec.layers * int(wl.lens.sum()) / (step_ms * 1e-3),
            "roofline": {"bound": "hbm", "kernel": f"decode_kernel<{args.bits}>", "achieved": achieved, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": recorded_traffic(decode_bytes_per_launch, args.bits),
                         "bytes_per_launch": decode_bytes_per_launch, "avg_launch_ms": dec_avg_ms},
            "e2e": {"value": aggregate_gbs(world, bytes_per_step, e2e_ms), "unit": "GB/s",
                    "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps * wl.launches_per_step(),  # inside the timed region
            "clocks": clocks.summary(),
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        if prefill is not None:
            line["next_rows"] = {"decode_configs": configs, "fused_step": fused, "int8_decode": int8,
                                 "int2_decode": int2, "page_moves": moves, "prefill": prefill,
                                 "clocks": extra_clocks}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
