"""Multi-rank host logic on CPU with gloo: bench.py's ranks agree on the
barrier and on the max-over-ranks step time that the whole-job throughput is
computed from (replicas: no collective on the data path); the tensor-parallel
layer's ranks shard the experts' intermediate dimension and sum their shares
with one all-reduce."""
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


def _tp_rank(rank: int, world: int, port: int, q):
    """One rank of the tensor-parallel layer's host logic: shard, compute this
    rank's share (the oracle stands in for the CUDA library on CPU), all-reduce
    over gloo, then round once."""
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    from shared_routed_expert_b200 import synth, tp
    dist.init_process_group("gloo", rank=rank, world_size=world)
    cfg = synth.variant(synth.CONFIGS["prefill_bf16"], T=6, H=256, I=128, n_routed=8, top_k=2)
    inp = synth.make_inputs(cfg)
    shard = tp.shard_weights(inp, cfg.I, rank, world)
    oracle_part = oracle.Layer(tp.local_config(cfg, world), shard)

    def partial_fn(x):
        return torch.from_numpy(oracle_part.forward(n_threads=1)["out"]).float()

    layer = tp.TPMoELayer(cfg, shard, world, partial_fn=partial_fn, cast_fn=lambda t: t.double())
    out = layer.forward(inp["x"])
    if rank == 0:
        full = oracle.Layer(cfg, inp).forward(n_threads=1)["out"]
        q.put(float(np.abs(out.numpy() - full).max() / np.abs(full).max()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world", [2, 4])
def test_tensor_parallel_ranks_sum_their_slices(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_tp_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    err = q.get(timeout=150)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert err < 1e-6          # fp32 shares summed over gloo against the fp64 layer
