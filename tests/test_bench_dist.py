"""bench.py's multi-GPU plumbing on CPU: two gloo ranks (replicas), max-over-ranks
timing and whole-job throughput."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import torch.distributed as dist
    bench.init_dist(world, "gloo")
    assert bench.dist_env() == (rank, rank, world)
    bench.barrier(world)
    # rank r took (r + 1) * 0.1 s per step over 5 steps; 3 requests per step per rank
    steps = [(rank + 1) * 0.1] * 5
    value, t = bench.aggregate(steps, 3, world)
    out[rank] = (value, t, bench.max_over_ranks(float(rank), world))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_replica_aggregation_max_over_ranks(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    slowest = world * 0.1 * 5
    for r in range(world):
        value, t, mx = out[r]
        assert abs(t - slowest) < 1e-9                       # max over ranks, not the local time
        assert abs(value - 3 * 5 * world / slowest) < 1e-9   # all ranks' units / that time
        assert mx == world - 1


def _worker_one_dies(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port), DOMINO_PG_TIMEOUT_S="10")
    bench.init_dist(world, "gloo")
    bench.barrier(world)                      # step boundary both ranks reach
    if rank == world - 1:
        out[rank] = "left"
        os._exit(3)                           # this rank dies between steps
    try:
        bench.max_over_ranks(1.0, world)      # the survivor's next collective
        out[rank] = "returned"
    except Exception as e:                    # noqa: BLE001 - any error ends the wait
        out[rank] = "raised " + type(e).__name__


def test_a_dead_rank_ends_the_others_collective_with_an_error():
    """Failure detection on the host: a replica that dies between steps makes
    the surviving rank's next collective fail within the process-group timeout."""
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker_one_dies, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode is not None for p in procs), "a rank is still waiting"
    assert procs[1].exitcode == 3 and out[1] == "left"
    assert out[0].startswith("raised"), out[0]


def test_single_rank_aggregation():
    value, t = bench.aggregate([0.5, 0.5], 4, 1)
    assert t == 1.0 and value == 8.0


def test_byte_models():
    import synth
    cfg = synth.CONFIGS["qwen3_8b_b1"]
    # 111.87 MB of weights per step plus ~0.62 MB per request per step, 16 steps
    assert abs(bench.loop_bytes(cfg, 1) / 1e9 - 1.800) < 0.005
    assert abs(bench.lm_head_bytes(cfg, 1) / 1e9 - 1.255) < 0.005
    assert bench.lm_head_flops(cfg, 1) == 2 * 16 * 151936 * 4096
