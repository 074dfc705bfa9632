"""Benchmark of the paged decode hot path on B200.

One step = one decode step of one layer for the whole batch: append each
sequence's new token to the paged cache (pa_reshape_and_cache; block copies
when a shared block must be copied first), then paged decode attention
(pa_decode_attention: one kernel; split contexts are merged in-kernel).

  value  : decode tokens/s (batch / step time), inputs resident in HBM, summed
           over ranks (each rank is an independent replica: weak scaling)
  e2e    : the same metric through the public API from host buffers: the host
           pool allocates each new token's slot (contexts grow by one token per
           step), pinned host q / k / v / slots / tables go to the device, the
           kernels run and the output comes back, all inside the timed region
  roofline: the decode call's algorithmic bytes / its CUDA-event duration
           against the measured HBM copy bandwidth
  cpu_baseline: the fp64 oracle on the host cores, on a bounded sample

``--impl reference`` times the oracle alone as the reference arm.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "paged decode attention tokens/s and KV-read GB/s as % of B200 HBM roofline"
FALLBACK_HBM_GBS = 6650.0
FLUSH_BYTES = 256 << 20  # > 126 MB L2


def _flush_l2(buf):
    """Evict L2 by reading a buffer twice its size.  Reading leaves clean lines, so
    the timed work does not pay for writing back a flush buffer's dirty lines."""
    return buf.sum()


def _peak_hbm():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def _peak_tensor():
    """Dense fp16/bf16 tensor peak (burst): measured bf16 (fp16 has the same nominal rate)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured bf16 (fp16 nominal ratio 1)"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


DECODE_SOURCES = ("decode_tc.cuh", "decode_tc.cu", "decode_common.cuh", "decode_simt.cu")
# the tcgen05 prefill kernels: on pairs of SMs, and on one SM per item (the automatic choice)
PREFILL_SOURCES = ("prefill_pair.cu", "tc5_ptx.cuh", "prefill_launch.h", "decode_tc.cuh",
                   "decode_common.cuh")
PREFILL_1SM_SOURCES = ("prefill_tc5.cu", "tc5_ptx.cuh", "prefill_launch.h", "decode_tc.cuh",
                       "decode_common.cuh")
INT8_SOURCES = ("decode_tc.cuh", "decode_int8.cu", "decode_common.cuh", "int8_launch.h")


def _kernel_sha(names=DECODE_SOURCES):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_486_b200", "csrc")
    for name in names:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(config, names=DECODE_SOURCES):
    """DRAM bytes per launch of the timed kernel from the committed ncu summary, if
    it was taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d.get(config)
        if e and e.get("kernel_sha") == _kernel_sha(names):
            return e["dram_bytes_per_launch"]
    except (OSError, ValueError):
        pass
    return None


def _spread(ms):
    """Median and 10th / 90th percentiles (nearest rank) of per-iteration times in
    ms, reported in microseconds."""
    xs = sorted(ms)
    if not xs:
        return None

    def q(p):
        return xs[min(len(xs) - 1, max(0, int(round(p * (len(xs) - 1)))))] * 1e3

    return {"p10": q(0.1), "p50": q(0.5), "p90": q(0.9), "n": len(xs), "unit": "us"}


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        return dist, dist.get_rank(), ws
    return None, 0, 1


def _reduce(dist, x, op):
    if dist is None:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def _max_over_ranks(dist, x):
    return _reduce(dist, x, None if dist is None else dist.ReduceOp.MAX)


def _sum_over_ranks(dist, x):
    return _reduce(dist, x, None if dist is None else dist.ReduceOp.SUM)


def aggregate(dist, local_ms, local_tokens):
    """Whole-job throughput of independent replicas: tokens summed over ranks divided
    by the slowest rank's device time.  Returns (max_ms, tokens, tokens/s)."""
    total_ms = _max_over_ranks(dist, local_ms)
    tokens = _sum_over_ranks(dist, local_tokens)
    return total_ms, tokens, tokens / (total_ms / 1e3)


def _unique_kv_bytes(wl, table, ctx):
    """K+V bytes of the distinct physical (block, token) rows the batch reads: a block
    shared by several sequences (a common prefix) is counted once, with the most tokens
    any of them reads from it."""
    rows = {}
    for b in range(len(ctx)):
        n = int(ctx[b])
        for j in range((n + wl.bs - 1) // wl.bs):
            blk = int(table[b, j])
            rows[blk] = max(rows.get(blk, 0), min(wl.bs, n - j * wl.bs))
    return sum(rows.values()) * wl.Hkv * wl.D * 2 * wl.elem_bytes


def workload_config(wl, world):
    """The `config` object of the JSON line: the workload and how it is timed.  Both
    arms print this same dict."""
    return {"workload": wl.name, "batch": wl.B, "q_heads": wl.Hq, "kv_heads": wl.Hkv,
            "head_dim": wl.D, "block_size": wl.bs, "layers_per_step": 1,
            "context_tokens": int(wl.context_lens().sum()),
            "kv_read_bytes_per_step": wl.kv_read_bytes(), "parallelism": f"replicas x{world}",
            "timing": "GPU arm: CUDA-graph replay of the step, CUDA events per step; decode "
                      "launched with PA_DECODE_OVERLAP_PROLOGUE after the cache write",
            "l2": "GPU arm: flushed between timed steps (256 MiB read outside the events)"}


# --------------------------------------------------------------- our arm
def _setup(wl, extra_blocks=0):
    """Engine with the workload's pool (plus `extra_blocks` at the bottom of the free
    stack, so the workload's own allocations get the same block ids) after the
    prefill ops and the decode step's allocations."""
    from paged_kv_cache_486_b200.engine import PagedKVCache
    dt = workloads.TORCH_DTYPE[wl.dtype]
    eng = PagedKVCache(wl.num_blocks + extra_blocks, wl.bs, wl.Hkv, wl.D, dt, wl.Hq, wl.B,
                       "cuda")

    def tokens(seq, pos0, n):
        return wl.tokens(seq, pos0, n, 0, "cuda"), wl.tokens(seq, pos0, n, 1, "cuda")

    eng.apply_ops(wl.ops[:wl.n_prefill_ops], tokens)
    # the decode step's slots (and any block copies) for the resident-input loop
    slots, keys, vals, copies = [], [], [], []
    for op in wl.decode_ops():
        _, seq, n, pos0, _w = op
        s, cow = eng.alloc(seq, n)
        slots.append(s)
        copies.extend(cow.tolist())
        k, v = tokens(seq, pos0, n)
        keys.append(k)
        vals.append(v)
    step = dict(slots=torch.from_numpy(np.concatenate(slots)).cuda(),
                key=torch.cat(keys), value=torch.cat(vals),
                pairs=torch.tensor(copies, dtype=torch.int32, device="cuda").reshape(-1, 2))
    bt, ctx = eng.block_tables(wl.batch, wl.max_blocks)
    step.update(bt=bt, ctx=ctx, q=wl.q("cuda"), out=torch.empty_like(wl.q("cuda")))
    torch.cuda.synchronize()
    return eng, step


def run_ours(args, dist, rank, world):
    import paged_kv_cache_486_b200 as pa
    wl = workloads.make(args.config)
    # room for the end-to-end leg, which grows every sequence by one token per step
    eng, st = _setup(wl, extra_blocks=wl.B * ((args.warmup + args.steps) // wl.bs + 2))
    flush = torch.ones(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    n_pairs = st["pairs"].shape[0]
    launches_per_step = 2 + (1 if n_pairs else 0)  # [copy_blocks] + cache write + decode

    def decode(flags=0):
        eng.decode(st["q"], st["bt"], st["ctx"], wl.scale, out=st["out"], flags=flags)

    def step():
        if n_pairs:
            pa.pa_copy_blocks([eng.k_cache], [eng.v_cache], st["pairs"], eng.dev_error)
        eng.write(st["key"], st["value"], st["slots"])
        # the cache write touches only the caches, so decode's prologue may overlap it
        decode(pa.PA_DECODE_OVERLAP_PROLOGUE)

    # One eager pass, then the step and the decode call are captured as CUDA graphs
    # so that host-side launch latency stays out of the device timings.
    step()
    torch.cuda.synchronize()
    g_step, g_dec = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        step()
    with torch.cuda.graph(g_dec):
        decode()
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)

    def timed(graph, n):
        out = []
        for _ in range(n):
            _flush_l2(flush)  # L2 flushed between timed replays, outside the events
            e0.record(stream)
            graph.replay()
            e1.record(stream)
            e1.synchronize()
            out.append(e0.elapsed_time(e1))
        return out

    timed(g_step, args.warmup)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    step_ms = timed(g_step, args.steps)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    timed(g_dec, args.warmup)
    decode_ms = timed(g_dec, args.steps)
    torch.cuda.synchronize()
    assert eng.device_errors() == 0, "device guards fired"

    total_ms, _, value = aggregate(dist, sum(step_ms), wl.B * args.steps)
    alg = wl.kv_read_bytes()
    uniq = _unique_kv_bytes(wl, st["bt"].cpu().numpy(), st["ctx"].cpu().numpy())
    dec_ms = statistics.mean(decode_ms)
    achieved = alg / (dec_ms / 1e3) / 1e9
    peak, peak_kind = _peak_hbm()
    del g_step, g_dec

    e2e = run_e2e(args, wl, eng, dist)
    del eng, st, flush
    torch.cuda.empty_cache()
    bars = {} if args.no_bar_configs else {n: decode_only(n, args) for n in BAR_CONFIGS
                                           if n != wl.name}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded counter-based N(0,1) stand-in values, shuffled block pool)",
        "config": workload_config(wl, world),
        "kv_read_gbs": achieved, "decode_us": dec_ms * 1e3,
        "kv_unique_bytes": uniq, "kv_unique_read_gbs": uniq / (dec_ms / 1e3) / 1e9,
        "decode_us_min": min(decode_ms) * 1e3, "decode_us_spread": _spread(decode_ms),
        "step_us_spread": _spread(step_ms),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": f"{peak_kind} (hbm_gbs copy)",
                     "traffic": _traffic(wl.name),
                     "timed": "pa_decode_attention call (one kernel), graph replay"},
        "e2e": e2e, "gpu_launches": launches_per_step * args.steps, "clocks": clocks,
    }
    if bars:
        line["decode_bar"] = bars
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, target_s=args.cpu_seconds, single_thread=True)
    return line


# The decode configurations on which the >= 70% HBM bar is set (Llama-3-8B- and
# Llama-3-70B-shaped layers); their decode-only roofline rides along the headline.
BAR_CONFIGS = ("llama3_8b", "llama3_70b")


def decode_only(name, args, batch=0):
    """pa_decode_attention alone on a workload: CUDA-graph replays with L2 flushed
    between them, CUDA events on the launching stream."""
    wl = workloads.make(name, batch)
    eng, st = _setup(wl)
    flush = torch.ones(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    eng.decode(st["q"], st["bt"], st["ctx"], wl.scale, out=st["out"])
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        eng.decode(st["q"], st["bt"], st["ctx"], wl.scale, out=st["out"])
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms = []
    for it in range(args.warmup + args.steps):
        _flush_l2(flush)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        e1.synchronize()
        if it >= args.warmup:
            ms.append(e0.elapsed_time(e1))
    assert eng.device_errors() == 0, "device guards fired"
    assert torch.isfinite(st["out"].float()).all()
    del g
    alg = wl.kv_read_bytes()
    t = statistics.mean(ms) / 1e3
    peak, kind = _peak_hbm()
    res = {"workload": wl.name, "batch": wl.B, "q_heads": wl.Hq, "kv_heads": wl.Hkv,
           "dtype": wl.dtype, "kv_read_bytes": alg, "decode_us": t * 1e6,
           "decode_us_min": min(ms) * 1e3, "decode_us_spread": _spread(ms),
           "tokens_per_s": wl.B / t,
           "roofline": {"bound": "hbm", "achieved": alg / t / 1e9, "peak": peak, "unit": "GB/s",
                        "frac": alg / t / 1e9 / peak, "peak_source": f"{kind} (hbm_gbs copy)",
                        "traffic": _traffic(wl.name)},
           "timed": "pa_decode_attention call alone (one kernel), graph replay"}
    del eng, st, flush
    torch.cuda.empty_cache()
    return res


def run_e2e(args, wl, eng, dist):
    """Public-API decode steps from pinned host buffers; contexts grow one token per step.
    Per step: one batched slot allocation and a block-table rebuild on the host, one
    packed host-to-device copy of q / new keys / new values / slots / tables / lengths,
    [block copies], the cache write, decode attention, and the output copied back."""
    import paged_kv_cache_486_b200 as pa
    stream = torch.cuda.current_stream()
    B, Hkv, D, Hq, MB = wl.B, wl.Hkv, wl.D, wl.Hq, wl.max_blocks
    dt = workloads.TORCH_DTYPE[wl.dtype]
    eb = workloads.ELEM_BYTES[wl.dtype]
    parts = [("q", (B, Hq, D), dt, eb), ("k", (B, Hkv, D), dt, eb), ("v", (B, Hkv, D), dt, eb),
             ("slots", (B,), torch.int64, 8), ("table", (B, MB), torch.int32, 4),
             ("ctx", (B,), torch.int32, 4)]
    offs, off = {}, 0
    for name, shape, _, size in parts:
        offs[name] = off
        off += (int(np.prod(shape)) * size + 255) // 256 * 256
    h_buf = torch.empty(off, dtype=torch.uint8).pin_memory()
    d_buf = torch.empty(off, dtype=torch.uint8, device="cuda")

    def view(buf, name):
        _, shape, tdt, size = next(p for p in parts if p[0] == name)
        n = int(np.prod(shape)) * size
        return buf[offs[name]:offs[name] + n].view(tdt).view(shape)

    h = {name: view(h_buf, name) for name, *_ in parts}
    d = {name: view(d_buf, name) for name, *_ in parts}
    h["q"].copy_(wl.q("cpu"))
    h["k"].copy_(wl.tokens(1 << 50, 0, B, 0))
    h["v"].copy_(wl.tokens(1 << 50, 0, B, 1))
    h_out = torch.empty(B, Hq, D, dtype=dt).pin_memory()
    d_out = torch.empty(B, Hq, D, dtype=dt, device="cuda")
    flush = torch.ones(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    seqs = np.asarray(wl.batch, dtype=np.int64)
    np_slots, np_table, np_ctx = h["slots"].numpy(), h["table"].numpy(), h["ctx"].numpy()
    h2d = off
    d2h = h_out.numel() * h_out.element_size()

    def one():
        _, cow = eng.pool.pa_alloc_batch(seqs, 1, slots_out=np_slots)
        eng.pool.pa_block_table(seqs, MB, out_table=np_table, out_ctx=np_ctx)
        d_buf.copy_(h_buf, non_blocking=True)
        if len(cow):
            pa.pa_copy_blocks([eng.k_cache], [eng.v_cache], torch.from_numpy(cow).cuda(),
                              eng.dev_error)
        pa.pa_reshape_and_cache(d["k"], d["v"], eng.k_cache, eng.v_cache, d["slots"],
                                eng.dev_error)
        pa.pa_decode_attention(d_out, d["q"], eng.k_cache, eng.v_cache, d["table"], d["ctx"],
                               wl.scale, eng.workspace, eng.dev_error)
        h_out.copy_(d_out, non_blocking=True)

    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    ms = []
    for _ in range(args.steps):
        _flush_l2(flush)
        torch.cuda.synchronize()
        e0.record(stream)
        one()
        e1.record(stream)
        e1.synchronize()
        ms.append(e0.elapsed_time(e1))
    total, _, e2e_value = aggregate(dist, sum(ms), wl.B * args.steps)
    assert torch.isfinite(h_out.float()).all()
    return {"value": e2e_value, "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": total / args.steps}


def run_swap(args, dist, rank, world):
    """Eviction to host memory and back: swap every sequence of the workload out to a
    pinned host cache and in again (pa_swap on the host pools, pa_swap_blocks on the
    GPU), timed per direction; the reference is a plain pinned copy of the same bytes."""
    import paged_kv_cache_486_b200 as pa
    wl = workloads.make(args.config)
    eng, st = _setup(wl)
    hk = torch.empty(eng.k_cache.shape, dtype=eng.k_cache.dtype).pin_memory()
    hv = torch.empty(eng.v_cache.shape, dtype=eng.v_cache.dtype).pin_memory()
    host = pa.Pool(wl.num_blocks, wl.bs)
    seqs = [int(x) for x in wl.batch]
    out_pairs = np.concatenate([pa.pa_swap(eng.pool, host, s) for s in seqs])
    in_pairs = np.concatenate([pa.pa_swap(host, eng.pool, s) for s in seqs])
    nbytes = len(out_pairs) * 2 * eng.k_cache[0].numel() * eng.k_cache.element_size()
    d_out = torch.from_numpy(out_pairs).cuda()
    d_in = torch.from_numpy(in_pairs).cuda()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ms = []
        for _ in range(args.steps):
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            ms.append(e0.elapsed_time(e1))
        return statistics.mean(ms)

    t_out = timed(lambda: pa.pa_swap_blocks([hk], [hv], [eng.k_cache], [eng.v_cache], d_out,
                                            eng.dev_error))
    t_in = timed(lambda: pa.pa_swap_blocks([eng.k_cache], [eng.v_cache], [hk], [hv], d_in,
                                           eng.dev_error))
    # reference: one contiguous pinned copy of the same number of bytes each way
    hbuf = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dbuf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    r_d2h = timed(lambda: hbuf.copy_(dbuf, non_blocking=True))
    r_h2d = timed(lambda: dbuf.copy_(hbuf, non_blocking=True))
    assert eng.device_errors() == 0
    gbs = lambda ms: nbytes / (ms / 1e3) / 1e9
    return {"metric": "swap_blocks GB/s (device <-> pinned host, whole batch)", "op": "swap",
            "value": 2 * nbytes / ((t_out + t_in) / 1e3) / 1e9, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "dtype": wl.dtype, "data": "synthetic",
            "config": {"workload": wl.name, "blocks": int(len(out_pairs)), "bytes_each_way": nbytes},
            "swap_out_gbs": gbs(t_out), "swap_in_gbs": gbs(t_in),
            "swap_out_ms": t_out, "swap_in_ms": t_in, "gpu_launches": 2 * args.steps,
            "roofline": {"bound": "host link", "unit": "GB/s",
                         "peak": {"d2h": gbs(r_d2h), "h2d": gbs(r_h2d)},
                         "peak_source": "contiguous pinned torch copy of the same bytes, same run",
                         "frac": {"out": r_d2h / t_out, "in": r_h2d / t_in}}}


def run_int8(args, dist, rank, world):
    """The decode step over an INT8 cache (PagedKVCacheInt8): quantising cache write of
    the step's tokens, then decode attention over codes + per-token scales."""
    import paged_kv_cache_486_b200 as pa
    from paged_kv_cache_486_b200.engine import PagedKVCacheInt8
    wl = workloads.make(args.config, args.batch)
    dt = workloads.TORCH_DTYPE[wl.dtype]
    eng = PagedKVCacheInt8(wl.num_blocks, wl.bs, wl.Hkv, wl.D, dt, wl.Hq, wl.B, "cuda")

    def tokens(seq, pos0, n):
        return wl.tokens(seq, pos0, n, 0, "cuda"), wl.tokens(seq, pos0, n, 1, "cuda")

    eng.apply_ops(wl.ops[:wl.n_prefill_ops], tokens)
    slots, keys, vals, copies = [], [], [], []
    for op in wl.decode_ops():
        _, seq, n, pos0, _w = op
        sl, cow = eng.alloc(seq, n)
        slots.append(sl)
        copies.extend(cow.tolist())
        k, v = tokens(seq, pos0, n)
        keys.append(k)
        vals.append(v)
    slots = torch.from_numpy(np.concatenate(slots)).cuda()
    key, value = torch.cat(keys), torch.cat(vals)
    pairs = torch.tensor(copies, dtype=torch.int32, device="cuda").reshape(-1, 2)
    bt, ctx = eng.block_tables(wl.batch, wl.max_blocks)
    q = wl.q("cuda")
    out = torch.empty_like(q)
    flush = torch.ones(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    n_pairs = pairs.shape[0]

    def decode(flags=0):
        eng.decode(q, bt, ctx, wl.scale, out=out, flags=flags)

    def step():
        if n_pairs:
            pa.pa_copy_blocks([eng.k_pool], [eng.v_pool], pairs, eng.dev_error)
        eng.write(key, value, slots)
        decode(pa.PA_DECODE_OVERLAP_PROLOGUE)

    step()
    torch.cuda.synchronize()
    g_step, g_dec = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        step()
    with torch.cuda.graph(g_dec):
        decode()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(graph, n):
        ms = []
        for _ in range(n):
            _flush_l2(flush)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
            e1.synchronize()
            ms.append(e0.elapsed_time(e1))
        return ms

    timed(g_step, args.warmup)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    step_ms = timed(g_step, args.steps)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    timed(g_dec, args.warmup)
    decode_ms = timed(g_dec, args.steps)
    torch.cuda.synchronize()
    assert eng.device_errors() == 0, "device guards fired"
    del g_step, g_dec

    total_ms, _, value = aggregate(dist, sum(step_ms), wl.B * args.steps)
    c = wl.context_lens().astype(np.int64)
    kv = int(c.sum()) * wl.Hkv * (2 * wl.D + 8)        # codes + fp32 scales, keys and values
    qo = 2 * wl.B * wl.Hq * wl.D * wl.elem_bytes
    tables = int(((c + wl.bs - 1) // wl.bs).sum()) * 4 + 4 * wl.B
    alg = kv + qo + tables
    dec_ms = statistics.mean(decode_ms)
    achieved = alg / (dec_ms / 1e3) / 1e9
    peak, peak_kind = _peak_hbm()
    launches = 2 + (1 if n_pairs else 0)
    return {
        "metric": METRIC + " (INT8 KV cache)", "op": "int8", "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": f"{wl.dtype} queries, int8 cache (fp32 scales)",
        "data": "synthetic (seeded counter-based N(0,1) stand-in values, shuffled block pool)",
        "config": {"workload": wl.name, "batch": wl.B, "q_heads": wl.Hq, "kv_heads": wl.Hkv,
                   "head_dim": wl.D, "block_size": wl.bs, "layers_per_step": 1,
                   "context_tokens": int(c.sum()), "kv_read_bytes_per_step": alg,
                   "parallelism": f"replicas x{world}",
                   "timing": "CUDA-graph replay of the step (INT8 cache write + INT8 decode), "
                             "CUDA events per step",
                   "l2": "flushed between timed steps (256 MiB read outside the events)"},
        "kv_read_gbs": achieved, "decode_us": dec_ms * 1e3, "decode_us_min": min(decode_ms) * 1e3,
        "decode_us_spread": _spread(decode_ms), "step_us_spread": _spread(step_ms),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": f"{peak_kind} (hbm_gbs copy)",
                     "traffic": _traffic(wl.name + "_int8", INT8_SOURCES),
                     "timed": "pa_decode_attention_int8 call (one kernel), graph replay"},
        "gpu_launches": launches * args.steps, "clocks": clocks,
    }


def run_decode(args, dist, rank, world):
    """--op decode: the decode call alone on --config (and --batch), one JSON line
    (the form the profiles' ncu captures run)."""
    r = decode_only(args.config, args, args.batch)
    return {"metric": METRIC + " (decode call alone)", "op": "decode",
            "value": r["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": r["dtype"], "data": "synthetic",
            "config": {"workload": r["workload"], "batch": r["batch"],
                       "l2": "flushed between timed calls (256 MiB read outside the events)"},
            "decode_us": r["decode_us"], "roofline": r["roofline"],
            "gpu_launches": args.steps}


def run_prefix(args, dist, rank, world):
    """Prefix caching on the prefix_prompts workload: admission of every request
    through pa_alloc_tokens (host), the K/V write of the tokens the cache does not
    supply, and decode over the shared blocks; each against the same run without
    the cache."""
    import paged_kv_cache_486_b200 as pa
    from paged_kv_cache_486_b200.engine import PagedKVCache
    ps = workloads.prefix_prompts()
    dt = workloads.TORCH_DTYPE[ps.dtype]
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    res = {}
    for on in (True, False):
        eng = PagedKVCache(ps.num_blocks, ps.bs, ps.Hkv, ps.D, dt, ps.Hq, ps.B, "cuda")
        eng.pool.pa_set_prefix_caching(on)
        # host admission: every request, timed on the host clock (pool work only)
        t0 = time.perf_counter()
        adm = [eng.pool.pa_alloc_tokens(i, ids) for i, ids in enumerate(ps.prompts)]
        host_s = time.perf_counter() - t0
        assert all(len(a[1]) == 0 for a in adm)
        slots = np.concatenate([a[0] for a in adm])
        keep = slots >= 0
        # rows of the written tokens only, generated on the device
        ids = np.concatenate(ps.prompts)
        pos = np.concatenate([np.arange(len(p)) for p in ps.prompts])
        k = workloads.token_rows(ps.seed, 0, ids[keep], pos[keep], ps.Hkv, ps.D, ps.dtype, "cuda")
        v = workloads.token_rows(ps.seed, 1, ids[keep], pos[keep], ps.Hkv, ps.D, ps.dtype, "cuda")
        d_slots = torch.from_numpy(slots[keep]).cuda()
        write_ms = []
        for it in range(args.warmup + args.steps):
            e0.record(stream)
            pa.pa_reshape_and_cache(k, v, eng.k_cache, eng.v_cache, d_slots, eng.dev_error)
            e1.record(stream)
            e1.synchronize()
            if it >= args.warmup:
                write_ms.append(e0.elapsed_time(e1))
        bt, ctx = eng.block_tables(list(range(ps.B)), max(len(p) for p in ps.prompts) // ps.bs + 1)
        q = ps.q("cuda")
        out = torch.empty_like(q)
        flush = torch.ones(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        dec_ms = []
        for it in range(args.warmup + args.steps):
            _flush_l2(flush)
            e0.record(stream)
            eng.decode(q, bt, ctx, ps.scale, out=out)
            e1.record(stream)
            e1.synchronize()
            if it >= args.warmup:
                dec_ms.append(e0.elapsed_time(e1))
        assert eng.device_errors() == 0, "device guards fired"
        used = ps.num_blocks - eng.pool.pa_num_free_blocks()  # the free count includes evictable
        res[on] = dict(host_us=1e6 * host_s / ps.B, cached_tokens=int(sum(a[2] for a in adm)),
                       written_tokens=int(keep.sum()), blocks_held=int(used),
                       write_us=1e3 * statistics.mean(write_ms),
                       decode_us=1e3 * statistics.mean(dec_ms), out=out.float().cpu())
        del eng
        torch.cuda.empty_cache()
    on, off = res[True], res[False]
    # decode over shared blocks reads the same logical rows: results agree
    err = float((on["out"] - off["out"]).abs().max())
    ctx_tokens = int(sum(len(p) for p in ps.prompts))
    alg = ctx_tokens * ps.Hkv * ps.D * 2 * 2 + 2 * ps.B * ps.Hq * ps.D * 2
    peak, peak_kind = _peak_hbm()
    achieved = alg / (on["decode_us"] / 1e6) / 1e9
    row_bytes = ps.Hkv * ps.D * 2 * 2
    return {
        "metric": "prefix-cache admission: requests/s through pa_alloc_tokens (host), with "
                  "K/V write and decode over the shared blocks", "op": "prefix",
        "value": 1e6 / on["host_us"], "unit": "requests/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
        "dtype": ps.dtype, "data": "synthetic (16 system prompts x 1024 tokens, U[16,256] own "
                                   "tokens, 32000-id vocabulary; rows a function of (id, position))",
        "config": {"workload": ps.name, "requests": ps.B, "q_heads": ps.Hq, "kv_heads": ps.Hkv,
                   "head_dim": ps.D, "block_size": ps.bs, "context_tokens": ctx_tokens},
        "host_us_per_request": {"cached": on["host_us"], "no_cache": off["host_us"]},
        "cached_token_fraction": on["cached_tokens"] / ctx_tokens,
        "blocks_held": {"cached": on["blocks_held"], "no_cache": off["blocks_held"]},
        "kv_write": {"cached": {"tokens": on["written_tokens"], "us": on["write_us"],
                                "bytes": on["written_tokens"] * row_bytes},
                     "no_cache": {"tokens": off["written_tokens"], "us": off["write_us"],
                                  "bytes": off["written_tokens"] * row_bytes}},
        "decode_us": {"cached": on["decode_us"], "no_cache": off["decode_us"]},
        "decode_max_abs_diff_cached_vs_not": err,
        "decode_kv_unique_read_gbs": {
            k: res[v]["blocks_held"] * ps.bs * row_bytes / (res[v]["decode_us"] / 1e6) / 1e9
            for k, v in (("cached", True), ("no_cache", False))},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": f"{peak_kind} (hbm_gbs copy)",
                     "traffic": None,
                     "timed": "decode over the prefix-cached pool, logical KV bytes (each "
                              "request's rows counted once; shared blocks are read from L2 "
                              "after the first, so this can exceed the HBM copy peak)"},
        "gpu_launches": 2 * 2 * (args.warmup + args.steps),
    }


def run_prefill(args, dist, rank, world):
    """Paged prefill attention over the pool: whole prompts (prefill_8b) or a 512-token
    chunk after earlier context (chunked_8b, --config chunked_8b)."""
    import paged_kv_cache_486_b200 as pa
    from paged_kv_cache_486_b200.engine import PagedKVCache
    name = args.config if args.config in ("prefill_8b", "chunked_8b") else "prefill_8b"
    wl = {"prefill_8b": workloads.prefill_8b, "chunked_8b": workloads.chunked_8b}[name]()
    dt = workloads.TORCH_DTYPE[wl.dtype]
    eng = PagedKVCache(wl.num_blocks, wl.bs, wl.Hkv, wl.D, dt, wl.Hq, wl.B, "cuda")
    eng.apply_ops(wl.ops, lambda s_, p_, n_: (wl.tokens(s_, p_, n_, 0, "cuda"),
                                             wl.tokens(s_, p_, n_, 1, "cuda")))
    bt, ctx = eng.block_tables(wl.batch, wl.max_blocks)
    qsn = workloads.query_start(wl)
    qs = torch.from_numpy(qsn).cuda()
    q = workloads.q_prefill(wl, "cuda")
    out = torch.empty_like(q)
    max_q = int(wl.n_new.max())
    flush = torch.ones(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def run():
        pa.pa_prefill_attention(out, q, eng.k_cache, eng.v_cache, bt, ctx, qs, max_q, wl.scale,
                                eng.dev_error, args.prefill_path, eng.prefill_ws)

    ms = []
    for it in range(args.warmup + args.steps):
        _flush_l2(flush)
        e0.record(stream)
        run()
        e1.record(stream)
        e1.synchronize()
        if it >= args.warmup:
            ms.append(e0.elapsed_time(e1))
    assert eng.device_errors() == 0, "device guards fired"
    c = wl.context_lens().astype(np.int64)
    n = wl.n_new.astype(np.int64)
    # keys attended: new token i of sequence b attends ctx - n + i + 1 keys
    pairs = int(((c - n) * n + n * (n + 1) // 2).sum())
    flops = 4.0 * wl.D * wl.Hq * pairs
    t = statistics.mean(ms) / 1e3
    tflops = flops / t / 1e12
    peak, kind = _peak_tensor()
    tokens = int(n.sum())
    total_ms, _, value = aggregate(dist, sum(ms), tokens * args.steps)
    kv_bytes = int(c.sum()) * wl.Hkv * wl.D * 2 * wl.elem_bytes
    return {
        "metric": "paged prefill attention: new tokens/s", "op": "prefill", "value": value,
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded counter-based N(0,1) stand-in values, shuffled block pool)",
        "config": {"workload": wl.name, "batch": wl.B, "q_heads": wl.Hq, "kv_heads": wl.Hkv,
                   "head_dim": wl.D, "block_size": wl.bs, "new_tokens": tokens,
                   "context_tokens": int(c.sum()), "attended_pairs": pairs,
                   "l2": "flushed between timed calls (256 MiB read outside the events)"},
        "prefill_us": 1e3 * statistics.mean(ms), "prefill_us_spread": _spread(ms),
        "kv_read_bytes": kv_bytes,
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": tflops / peak, "peak_source": kind,
                     "traffic": (None if args.prefill_path == 2 or wl.D != 128
                                 else _traffic(wl.name + "_tc5_pair", PREFILL_SOURCES)
                                 if args.prefill_path == 3
                                 else _traffic(wl.name, PREFILL_1SM_SOURCES)),
                     "timed": "pa_prefill_attention (one kernel, " +
                              ("mma.sync m16n8k16" if args.prefill_path == 2 or wl.D != 128
                               else "tcgen05 UMMA on pairs of SMs (cta_group::2), TMEM "
                                    "accumulators" if args.prefill_path == 3
                               else "tcgen05 UMMA on one SM per item, TMEM accumulators") + ")"},
        "gpu_launches": args.steps,
    }


# ---------------------------------------------------------- oracle timings
# Samples laid out by cpu_baseline, and its one-sequence timings, kept between the
# calls of one run (the reference arm calls it once per warm-up and timed step).
_CPU_SAMPLES = {}
_CPU_T_ONE = {}


def cpu_baseline(wl, target_s=10.0, single_thread=False, max_sample_bytes=2 << 30):
    """The oracle on the host cores (all of them, and with single_thread one more pass
    on one core), on the first S sequences of the workload laid out in a shuffled pool;
    S is chosen for about target_s seconds of work and at most max_sample_bytes of K/V."""
    import oracle
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from oracle_side import raw
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    ctx_all = wl.context_lens()

    def make(S):
        key = (wl.name, S)
        if key not in _CPU_SAMPLES:
            if len(_CPU_SAMPLES) >= 2:  # at most two samples held (the 1-sequence one and S)
                _CPU_SAMPLES.pop(next(k for k in _CPU_SAMPLES if k[1] != 1))
            _CPU_SAMPLES[key] = build(S)
        return _CPU_SAMPLES[key]

    def build(S):
        # lay the first S sequences' logical rows out in a shuffled pool of wl.bs blocks
        rng = np.random.default_rng(wl.seed + S)
        ctx = ctx_all[:S]
        nblk = (ctx + wl.bs - 1) // wl.bs
        nb = int(nblk.sum())
        perm = rng.permutation(nb).astype(np.int32)
        kc = np.zeros((nb, wl.Hkv, wl.bs, wl.D), dtype=np.float32 if wl.dtype == "f32"
                      else np.uint16)
        vc = np.zeros_like(kc)
        table = np.full((S, int(nblk.max())), -1, np.int32)
        off = 0
        for b in range(S):
            blocks = perm[off:off + nblk[b]]
            off += nblk[b]
            table[b, :nblk[b]] = blocks
            seq = int(wl.batch[b])
            for kind, cache in ((0, kc), (1, vc)):
                rows = raw(wl.contiguous_kv(seq, kind, dev))  # [n, Hkv, D]
                pad = np.zeros((nblk[b] * wl.bs,) + rows.shape[1:], rows.dtype)
                pad[:len(rows)] = rows
                cache[blocks] = pad.reshape(nblk[b], wl.bs, wl.Hkv, wl.D).transpose(0, 2, 1, 3)
        q = raw(wl.q(dev)[:S])
        return q, kc, vc, table, ctx.astype(np.int32)

    threads = os.cpu_count() or 1
    q, kc, vc, table, ctx = make(1)
    if wl.name not in _CPU_T_ONE:
        t0 = time.perf_counter()
        oracle.paged_decode_attention(q, kc, vc, table, ctx, wl.scale, wl.dtype,
                                      n_threads=threads)
        _CPU_T_ONE[wl.name] = time.perf_counter() - t0
    t_one = _CPU_T_ONE[wl.name]
    per_seq = kc.nbytes + vc.nbytes
    S = int(min(wl.B, max(1, target_s / max(t_one, 1e-3) / 4),
                max(1, max_sample_bytes // max(per_seq, 1))))
    q, kc, vc, table, ctx = make(S)
    reps, elapsed = 0, 0.0
    while elapsed < target_s and reps < 50:
        t0 = time.perf_counter()
        oracle.paged_decode_attention(q, kc, vc, table, ctx, wl.scale, wl.dtype,
                                      n_threads=threads)
        elapsed += time.perf_counter() - t0
        reps += 1
    res = {"value": S * reps / elapsed, "unit": "tokens/s", "cores": threads, "kind": "oracle",
           "sample": f"first {S} of {wl.B} sequences ({int(ctx.sum())} context tokens) of "
                     f"{wl.name}, fp64 oracle, {reps} passes, {elapsed:.1f} s",
           "nproc": _nproc(), "hardware_concurrency": oracle.hardware_concurrency(),
           "os_cpu_count": os.cpu_count()}
    if single_thread:
        # one sequence on one core, for about a third of the all-core budget
        q1, kc1, vc1, table1, ctx1 = q[:1], kc, vc, table[:1], ctx[:1]
        reps1, el1 = 0, 0.0
        while el1 < target_s / 3 and reps1 < 50:
            t0 = time.perf_counter()
            oracle.paged_decode_attention(q1, kc1, vc1, table1, ctx1, wl.scale, wl.dtype,
                                          n_threads=1)
            el1 += time.perf_counter() - t0
            reps1 += 1
        res["single_thread"] = {"value": reps1 / el1, "unit": "tokens/s", "cores": 1,
                                "sample": f"sequence 0 of {wl.name} ({int(ctx1[0])} context "
                                          f"tokens), {reps1} passes, {el1:.1f} s"}
    return res


def _nproc():
    try:
        return int(subprocess.run(["nproc"], capture_output=True, text=True,
                                  timeout=10).stdout.strip())
    except (OSError, ValueError, subprocess.SubprocessError):
        return None


def run_reference(args, rank, world):
    if rank != 0:
        return None
    wl = workloads.make(args.config)
    per_step = min(args.cpu_seconds, max(2.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(wl, target_s=min(per_step, 2.0))
    vals = [cpu_baseline(wl, target_s=per_step, single_thread=(i == args.steps - 1))
            for i in range(args.steps)]
    v = statistics.mean(x["value"] for x in vals)
    cb = dict(vals[-1])
    cb["value"] = v
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * wl.B / v, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded counter-based N(0,1) stand-in values, shuffled block pool)",
            "config": workload_config(wl, world),
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def _relaunch(n):
    """--gpus N without a launcher: run this same command as N ranks under
    torch.distributed.run on this node (one rank per GPU)."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__), *sys.argv[1:]]
    sys.stdout.flush()
    os.execv(sys.executable, cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="long_mha", choices=sorted(workloads.CONFIGS),
                    help="workload of the step (default long_mha: 8 x 32768 tokens, 64/64 "
                         "heads, the largest single-GPU configuration)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--op", default="step",
                    choices=["step", "decode", "swap", "int8", "prefix", "prefill"],
                    help="step: the decode step (default); decode: the decode call alone; "
                         "swap: eviction to host and back; int8: the decode step over an INT8 "
                         "cache; prefix: prefix caching; prefill: paged prefill attention "
                         "(--config prefill_8b | chunked_8b)")
    ap.add_argument("--batch", type=int, default=0,
                    help="--op decode / int8: override the batch of llama3_8b, llama3_70b or "
                         "long_mha (a reduced case for profiling)")
    ap.add_argument("--prefill-path", type=int, default=0, choices=[0, 1, 2, 3],
                    help="--op prefill kernel: 0 automatic (tcgen05 on one SM per item at "
                         "head_dim 128), 1 tcgen05 on one SM per item, 2 mma.sync, "
                         "3 tcgen05 on pairs of SMs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-bar-configs", action="store_true",
                    help="skip the decode-only lines of llama3_8b and llama3_70b")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1:
        _relaunch(args.gpus)  # does not return
    if env_world is not None and int(env_world) != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={env_world}: launch one rank per GPU")

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        line = run_reference(args, rank, world)
        if line:
            print(json.dumps(line), flush=True)
        return

    if not torch.cuda.is_available():
        sys.exit("bench.py: the GPU arm needs a CUDA device (B200); none is visible")
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist, rank, world = _dist()
    try:
        run = {"swap": run_swap, "int8": run_int8, "prefix": run_prefix,
               "prefill": run_prefill, "decode": run_decode}.get(args.op, run_ours)
        line = run(args, dist, rank, world)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if dist:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
