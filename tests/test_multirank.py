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


def _bench(*argv, env=None, timeout=300):
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    e = dict(os.environ)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        e.pop(k, None)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(root, "bench.py"), *argv],
                          capture_output=True, text=True, timeout=timeout, env=e)


def test_gpus_n_launches_n_ranks_and_rank_0_alone_prints():
    """`bench.py --gpus 2` without a launcher relaunches itself as two ranks under
    torch.distributed.run; on the reference arm rank 0 alone runs and prints."""
    import json
    r = _bench("--impl", "reference", "--gpus", "2", "--config", "tiny", "--steps", "1",
               "--warmup", "3", "--cpu-seconds", "0.3")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2
    assert lines[0]["config"]["workload"] == "tiny"


def test_gpu_arm_without_a_gpu_or_with_a_mismatched_world_fails_loudly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("checks the CPU-only failure")
    r = _bench("--gpus", "1", "--config", "tiny", "--steps", "1", "--warmup", "3")
    assert r.returncode != 0 and "CUDA device" in r.stderr
    r = _bench("--gpus", "4", "--config", "tiny", "--steps", "1", "--warmup", "3",
               env={"WORLD_SIZE": "2"})
    assert r.returncode != 0 and "WORLD_SIZE=2" in r.stderr
