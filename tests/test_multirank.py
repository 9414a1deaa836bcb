"""The N > 1 host path of bench.py on CPU: two gloo ranks.

Each rank solves its own problem (its own seed, so different inputs), the
step time that counts is the maximum over ranks, and the job throughput is
every rank's FLOPs over that time.  The reference arm runs on rank 0 only.
"""
import datetime
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch
    import torch.distributed as dist
    import bench
    from attention_kl_divergence_attn_b200 import inputs
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        vals = bench.max_over_ranks([10.0 + rank, 5.0 - rank], world, "cpu")
        wr = bench.rank_workload(inputs.WORKLOADS["tiny_128"], rank)
        x = inputs.make_inputs(wr)[0].float().contiguous()
        got = [torch.zeros_like(x) for _ in range(world)]
        dist.all_gather(got, x)
        same = bool(torch.equal(got[0], got[1]))
        dist.barrier()
    finally:
        dist.destroy_process_group()
    q.put((rank, vals, wr.seed, same))


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, v0, s0, same0), (_, v1, s1, same1) = res
    assert v0 == v1 == [11.0, 5.0]          # element-wise maximum over the ranks
    assert s0 != s1                          # independent problems
    assert not same0 and not same1           # ... with different inputs


def test_job_throughput_counts_every_rank():
    import bench
    assert bench.job_throughput(1e12, 2, 1000.0) == pytest.approx(2.0)
    assert bench.job_throughput(2.2e12, 1, 2.2) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    import argparse
    import bench
    from attention_kl_divergence_attn_b200 import inputs
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(steps=1, warmup=3, gpus=2)
    assert bench.run_reference(args, inputs.WORKLOADS["tiny_128"]) == 0
    assert capsys.readouterr().out == ""
