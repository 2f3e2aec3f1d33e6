"""The multi-process plumbing of bench.py on CPU (gloo, world size 2): each
rank builds its own replica (independent seeds, same shapes), the step time
is the max over ranks, and whole-job throughput counts every rank's bytes.
The decode path itself has no cross-GPU exchange, so no data collective is
tested because none exists."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import sys
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    import bench
    from int4_kivi_quantized_s4kv_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world)
    spec = bench.replica_spec(W.SPECS["qwen2.5-7b"], rank)
    step_ms = 2.0 + rank  # rank 1 is the slow one
    mx = bench.reduce_max(step_ms, world, "cpu")
    gbs = bench.aggregate_gbs(world, 1e9, mx)
    q.put((rank, spec.seed, int(W.context_lens(spec).sum()), mx, gbs))
    dist.destroy_process_group()


def test_replicas_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    (_, seed0, ctx0, mx0, gbs0), (_, seed1, ctx1, mx1, gbs1) = res
    assert seed0 != seed1 and ctx0 != ctx1          # independent replicas
    assert mx0 == mx1 == 3.0                         # slowest rank's time
    assert gbs0 == gbs1 == pytest.approx(2 * 1e9 / 3e-3 / 1e9)


def test_reference_arm_only_rank0_works(capsys):
    import bench
    os.environ["RANK"], os.environ["WORLD_SIZE"] = "1", "2"
    try:
        assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"]) == 0
    finally:
        os.environ.pop("RANK")
        os.environ.pop("WORLD_SIZE")
    assert capsys.readouterr().out == ""
