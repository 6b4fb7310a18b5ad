"""The benchmark's multi-rank bookkeeping, run as two gloo ranks on the CPU:
the job time is the slowest replica's, and only rank 0 runs the reference arm."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.slowest_rank(10.0 + 5.0 * rank, dist, device="cpu")
        dist.barrier()
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_slowest_rank_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, PORT, out))
                 for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs)
        assert dict(out) == {0: 15.0, 1: 15.0}


PORT = _free_port()


def test_slowest_rank_without_a_group_is_identity():
    import bench

    assert bench.slowest_rank(3.5, None) == 3.5


def test_reference_arm_runs_only_on_rank_zero(monkeypatch):
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    called = []
    monkeypatch.setattr(bench, "oracle_sample", lambda *a, **k: called.append(1))
    args = type("A", (), {"warmup": 1, "steps": 1, "head_dim": 96, "gpus": 2})()
    assert bench.run_reference(args) == 0
    assert not called


def test_streaming_placements():
    """The weight-streaming leg's two placements: "tail" streams the last
    L - k blocks; "spread" streams as many, spaced evenly, so that no two
    streamed blocks are adjacent while at least half the blocks stay
    resident, and no gap between streamed blocks exceeds one block more than
    the even spacing."""
    import bench

    L = bench.L
    for k in range(L + 1):
        tail = bench.streamed_set(k, "tail")
        spread = bench.streamed_set(k, "spread")
        assert tail == set(range(k, L))
        assert len(spread) == L - k and spread <= set(range(L))
        idx = sorted(spread)
        if 2 * k >= L:
            assert all(b - a >= 2 for a, b in zip(idx, idx[1:])), k
        if len(idx) > 1:
            gaps = [b - a for a, b in zip(idx, idx[1:])]
            assert max(gaps) - min(gaps) <= 1, (k, gaps)
