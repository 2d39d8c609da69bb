"""The N > 1 path of bench.py (independent replicas, max-over-ranks timing), as two gloo
ranks on the CPU."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w, local = bench.dist_setup(world)
    dist = bench.init_pg(local, w, backend="gloo")
    try:
        dist.barrier()
        # rank r took (r + 1) * 10 ms for 100 steps of 1 MB each
        ms = bench.max_over_ranks((r + 1) * 10.0, dist, torch.device("cpu"))
        out[r] = (r, w, ms, bench.job_gbs(1 << 20, w, ms, 100))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank_and_the_whole_job():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                           join=True, start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r, (rank, w, ms, gbs) in res.items():
        assert rank == r and w == world
        assert ms == pytest.approx(20.0)  # max over ranks, on every rank
        # 2 ranks x 1 MB per step over 0.2 ms per step (the slowest rank's time)
        assert gbs == pytest.approx(2 * (1 << 20) / 0.2e-3 / 1e9)


def test_world_size_must_match_gpus(monkeypatch):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "0")
    with pytest.raises(SystemExit):
        bench.dist_setup(4)
    monkeypatch.setenv("WORLD_SIZE", "1")
    assert bench.dist_setup(1) == (0, 1, 0)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.init_pg(0, 1) is None
    assert bench.max_over_ranks(3.5, None, None) == 3.5
    assert bench.job_gbs(1e9, 1, 1000.0, 1) == pytest.approx(1.0)
