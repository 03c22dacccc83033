"""The multi-rank host logic of bench.py on CPU: two gloo ranks agree on the
barrier and on the max-over-ranks step time that the whole-job throughput is
computed from (replicas: no collective on the data path)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    import bench
    d = bench.Dist(world, backend="gloo")
    d.barrier()
    local_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
    m = d.max(local_ms)
    q.put((rank, m, bench.tokens_per_s(d.world, 4096, 20, m)))
    d.close()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_max_step_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]
    # 2 ranks x 4096 tokens x 20 steps over the slowest rank's 15 ms
    assert res[0][2] == pytest.approx(2 * 4096 * 20 / 0.015)


def test_single_process_needs_no_process_group():
    import bench
    d = bench.Dist(1, backend="gloo")
    assert d.pg is None and d.max(3.5) == 3.5
