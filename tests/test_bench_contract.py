"""bench.py's JSON line on CPU: the reference arm (the oracle on the host cores)
prints the same `config` object as the GPU arm, reports its core counts, and the
decode-only helpers accept the reduced profiling workloads."""
import types

import bench
import workloads


def test_reference_arm_config_equals_the_gpu_arms():
    args = types.SimpleNamespace(config="tiny", steps=1, warmup=3, cpu_seconds=0.3)
    line = bench.run_reference(args, 0, 1)
    wl = workloads.make("tiny")
    assert line["config"] == bench.workload_config(wl, 1)
    assert line["impl"] == "reference" and line["unit"] == "tokens/s"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1
    assert cb["hardware_concurrency"] >= 1 and cb["os_cpu_count"] >= 1
    assert cb["single_thread"]["cores"] == 1 and cb["single_thread"]["value"] > 0
    assert line["e2e"]["value"] == line["value"]


def test_reduced_batch_workloads_for_profiling():
    wl = workloads.make("long_mha", 2)
    assert wl.name == "long_mha_b2" and wl.B == 2
    full = workloads.make("long_mha")
    # bytes scale with the context tokens at a fixed per-sequence length
    assert abs(full.kv_read_bytes() / wl.kv_read_bytes() - 4.0) < 1e-3
    try:
        workloads.make("shared_prefix", 2)
    except ValueError:
        pass
    else:
        raise AssertionError("shared_prefix has a fixed batch")


def test_spread_is_nearest_rank_percentiles_in_microseconds():
    """The per-iteration spread the bench lines carry (median and 10th / 90th
    percentiles of the CUDA-event times): nearest rank over the sorted times,
    reported in microseconds, independent of the input order."""
    import bench
    ms = [0.9, 0.1, 0.5, 0.3, 0.7, 0.2, 0.8, 0.4, 0.6, 1.0, 0.0]
    s = bench._spread(ms)
    assert s == {"p10": 100.0, "p50": 500.0, "p90": 900.0, "n": 11, "unit": "us"}
    assert bench._spread([]) is None
