"""Multi-rank host logic of bench.py on CPU: two gloo ranks (127.0.0.1).

bench.py --gpus N runs one process per GPU, each on its own data (the
channel-sequences are independent: weak scaling, no data-path collective);
the ranks only line up the timed region and take the max time over ranks.
The same Ranks class runs here over gloo.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import bench
    r = bench.Ranks("gloo")
    r.barrier()
    m = r.max(10.0 * (rank + 1))            # each rank's own "time"
    r.close()
    q.put((rank, r.world, m))


def test_two_gloo_ranks_take_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 2, 20.0), (1, 2, 20.0)]


def test_single_rank_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import bench
    r = bench.Ranks("gloo")
    assert (r.world, r.rank) == (1, 0)
    assert r.max(3.5) == 3.5
    r.barrier()
    r.close()


def test_weak_scaling_throughput_counts_every_rank():
    import bench
    # 2 ranks, 10 steps of 1000 positions each in 5 ms (the slowest rank)
    assert bench.throughput(1000, 2, 10, 5.0) == pytest.approx(1000 * 2 * 10 / 0.005)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    import bench
    from subquadratic_sequence_b200 import synth

    class Args:
        steps, warmup = 3, 3
    assert bench.run_reference(Args(), synth.WORKLOADS["c0"]) is None
