"""Multi-rank plumbing of the benchmark on CPU: world_size 2 over gloo.

The layer runs as independent replicas (no data-path collective); the process
group only brackets the timed region and takes the max of the device times.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    from mixture_experts_ffn_expert_b200 import replicas
    info = replicas.init_from_env("gloo", timeout_s=30)
    try:
        replicas.barrier(info)
        mx = replicas.max_over_ranks(10.0 + rank, info)
        sm = replicas.sum_over_ranks(1.0, info)
        q.put((rank, info.world_size, info.initialized, mx, sm))
    finally:
        replicas.shutdown(info)


def test_two_rank_max_and_sum():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [r[0] for r in res] == [0, 1]
    for _, world, init, mx, sm in res:
        assert world == 2 and init and mx == 11.0 and sm == 2.0


def test_single_rank_needs_no_process_group(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    from mixture_experts_ffn_expert_b200 import replicas
    info = replicas.init_from_env("gloo")
    assert (info.rank, info.world_size, info.initialized) == (0, 1, False)
    assert replicas.max_over_ranks(3.5, info) == 3.5


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--gpus", "2"]) == 0
    assert capsys.readouterr().out == ""
