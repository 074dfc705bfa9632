"""The multi-GPU bench path on CPU: two gloo ranks stand in for two GPU replicas.
Each rank is an independent replica (no data exchange); the job's throughput is
the tokens of all ranks over the slowest rank's time, and only rank 0 prints."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local_ms = [120.0, 150.0][rank]           # rank 1 is the slower replica
    local_tokens = [64 * 10, 64 * 10][rank]
    out = bench.aggregate(dist, local_ms, local_tokens)
    ref = bench.run_reference(type("A", (), {"config": "tiny", "steps": 1, "warmup": 3})(),
                              rank, world) if rank == 1 else "skip"
    q.put((rank, out, ref))
    dist.destroy_process_group()


def test_two_rank_aggregation_on_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    for _ in procs:
        r, out, ref = q.get(timeout=120)
        results[r] = (out, ref)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        total_ms, tokens, value = results[r][0]
        assert total_ms == 150.0                      # the slowest rank bounds the job
        assert tokens == 1280.0                       # every replica's tokens count
        assert value == pytest.approx(1280.0 / 0.150)
    assert results[1][1] is None                      # only rank 0 runs the reference arm
