"""Seeded synthetic workloads for the paged decode hot path.

Shared by the tests, ``bench.py`` and ``__graft_entry__.smoke()``; used by both the
CUDA library's callers and the oracle.  This module holds none of the method's
arithmetic: it draws numbers and writes *op scripts* (alloc / fork / free calls)
that each side executes with its own allocator, and it produces key, value and
query values from a counter-based generator so that either side can regenerate
any slice of them, on the CPU or on the GPU, with identical bits.

Value generator (a statement of its definition, so the two sides agree):
  * 32-bit mixer ``mix32`` (xor-shift / multiply, constants 0x7feb352d and
    0x846ca68b, shifts 16, 15, 16), all arithmetic modulo 2^32;
  * stream key ``key(seed, kind, writer)`` mixes the workload seed, the tensor
    kind (key / value / query) and the sequence that wrote the token;
  * element ``idx`` of a stream draws three words
    ``w_i = mix32((mix32((c >> 32) ^ key) + (c & 0xffffffff)) mod 2^32)`` with
    ``c = 3 * idx + i``, sums their twelve bytes ``S`` (an Irwin-Hall sum, mean
    1530, variance ~ 12 * 256^2 / 12) and returns ``(S - 1530) / 256`` -- a
    N(0, 1) stand-in with exact binary values (multiples of 1/256, |x| < 6),
    exact in fp32 and fp16 and rounded to nearest-even for bf16.
Key/value element (token p, kv head h, dim d) of the stream written by sequence
``writer`` has ``idx = (p * kv_heads + h) * head_dim + d``; query element
(batch row b, q head h, dim d) has ``idx = (b * q_heads + h) * head_dim + d``.

Workload shapes follow the pages' examples: Llama-3-8B-like heads (32 query /
8 KV heads, head_dim 128), Llama-3-70B-like heads (64 / 8), Llama-2-70B-like
full multi-head attention (64 / 64) at 32K context, block size 16, mixed short and
long requests, one shared system prompt with n=4 parallel sampling.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

MASK32 = 0xFFFFFFFF
KIND_K, KIND_V, KIND_Q = 0, 1, 2
DUMMY_BASE = 1 << 40  # sequence ids of churn-only sequences (never read)

TORCH_DTYPE = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2}


# --------------------------------------------------------------- generator
def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    # (x * c) mod 2^32 without leaving int64: split x into 16-bit halves.
    lo = (x & 0xFFFF) * c
    hi = (((x >> 16) * c) & 0xFFFF) << 16
    return (lo + hi) & MASK32


def mix32(x: torch.Tensor) -> torch.Tensor:
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def _mix32_int(x: int) -> int:
    return int(mix32(torch.tensor([x & MASK32], dtype=torch.int64))[0])


def stream_key(seed: int, kind: int, writer: int) -> int:
    k = _mix32_int(seed & MASK32)
    k = _mix32_int(k ^ (kind * 0x9E3779B9 & MASK32))
    k = _mix32_int(k ^ (writer & MASK32))
    k = _mix32_int(k ^ ((writer >> 32) & MASK32))
    return k


def values(key: int, idx: torch.Tensor) -> torch.Tensor:
    """float32 values for int64 element indices ``idx`` of the stream ``key``."""
    acc = torch.zeros_like(idx)
    for i in range(3):
        c = idx * 3 + i
        w = mix32((mix32((c >> 32) ^ key) + (c & MASK32)) & MASK32)
        acc = acc + (w & 255) + ((w >> 8) & 255) + ((w >> 16) & 255) + (w >> 24)
    return (acc - 1530).to(torch.float32) / 256.0


def _gen(key: int, start: int, count: int, device, dtype: str, chunk: int = 1 << 24):
    out = torch.empty(count, dtype=TORCH_DTYPE[dtype], device=device)
    for s in range(0, count, chunk):
        n = min(chunk, count - s)
        idx = torch.arange(start + s, start + s + n, dtype=torch.int64, device=device)
        out[s:s + n] = values(key, idx).to(TORCH_DTYPE[dtype])
    return out


# ---------------------------------------------------------------- workload
@dataclass
class Workload:
    name: str
    dtype: str
    B: int
    Hq: int
    Hkv: int
    D: int
    bs: int
    num_blocks: int
    max_blocks: int
    seed: int
    # ('alloc', seq, n, pos0, write) | ('fork', parent, child) | ('free', seq)
    ops: list = field(default_factory=list)
    n_prefill_ops: int = 0
    batch: np.ndarray = None  # int64 seq ids in batch order
    lengths: dict = field(default_factory=dict)   # seq -> tokens after the script
    segments: dict = field(default_factory=dict)  # seq -> [(p0, p1, writer)] in order
    # Wide-range option (powers of two only, so every value stays exact in every
    # dtype): queries are multiplied by q_mul; the key row at position p by
    # 2^min(p // k_ramp_tokens, k_ramp_max) when k_ramp_tokens > 0, so later keys
    # reach larger scores and a running maximum keeps moving along the context.
    q_mul: float = 1.0
    k_ramp_tokens: int = 0
    k_ramp_max: int = 0

    @property
    def G(self):
        return self.Hq // self.Hkv

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.D)

    @property
    def elem_bytes(self):
        return ELEM_BYTES[self.dtype]

    def context_lens(self):
        return np.array([self.lengths[int(s)] for s in self.batch], dtype=np.int32)

    def decode_ops(self):
        return self.ops[self.n_prefill_ops:]

    # ---- values ----
    def _ramp(self, t, p0, kind):
        """Apply the key ramp to rows t [n, heads, D] at positions p0, p0 + 1, ..."""
        if kind != KIND_K or self.k_ramp_tokens <= 0 or t.shape[0] == 0:
            return t
        p = torch.arange(p0, p0 + t.shape[0], dtype=torch.int64, device=t.device)
        e = torch.clamp(p // self.k_ramp_tokens, max=self.k_ramp_max)
        f = torch.pow(2.0, e.to(torch.float32)).to(t.dtype)
        return t * f[:, None, None]

    def tokens(self, writer, p0, n, kind, device="cpu"):
        """[n, Hkv, D] key (kind 0) or value (kind 1) rows written by ``writer``."""
        per = self.Hkv * self.D
        t = _gen(stream_key(self.seed, kind, writer), p0 * per, n * per, device, self.dtype)
        return self._ramp(t.view(n, self.Hkv, self.D), p0, kind)

    def q(self, device="cpu"):
        n = self.B * self.Hq * self.D
        t = _gen(stream_key(self.seed, KIND_Q, 0), 0, n, device, self.dtype).view(
            self.B, self.Hq, self.D)
        return t if self.q_mul == 1.0 else t * self.q_mul

    def contiguous_kv(self, seq, kind, device="cpu", heads=None):
        """Key/value rows of sequence ``seq`` in logical order: [ctx, Hkv or len(heads), D]."""
        parts = []
        for p0, p1, writer in self.segments[int(seq)]:
            if heads is None:
                parts.append(self.tokens(writer, p0, p1 - p0, kind, device))
            else:
                key = stream_key(self.seed, kind, writer)
                p = torch.arange(p0, p1, dtype=torch.int64, device=device)
                h = torch.as_tensor(heads, dtype=torch.int64, device=device)
                d = torch.arange(self.D, dtype=torch.int64, device=device)
                idx = (p[:, None, None] * self.Hkv + h[None, :, None]) * self.D + d[None, None, :]
                parts.append(self._ramp(values(key, idx.reshape(-1)).to(
                    TORCH_DTYPE[self.dtype]).view(p1 - p0, len(heads), self.D), p0, kind))
        if not parts:
            return torch.empty(0, self.Hkv if heads is None else len(heads), self.D,
                               dtype=TORCH_DTYPE[self.dtype], device=device)
        return torch.cat(parts, 0)

    def kv_read_bytes(self):
        """Algorithmic bytes of one decode call (each context token read once)."""
        ctx = self.context_lens().astype(np.int64)
        kv = int(ctx.sum()) * self.Hkv * self.D * 2 * self.elem_bytes
        qo = 2 * self.B * self.Hq * self.D * self.elem_bytes
        tables = int(((ctx + self.bs - 1) // self.bs).sum()) * 4 + 4 * self.B
        return kv + qo + tables


class _Script:
    """Op-script writer that also keeps per-sequence lengths and content lineage."""

    def __init__(self):
        self.ops = []
        self.lengths = {}
        self.segments = {}

    def alloc(self, seq, n, write=True):
        pos0 = self.lengths.get(seq, 0)
        self.ops.append(("alloc", seq, int(n), pos0, write))
        self.lengths[seq] = pos0 + int(n)
        segs = self.segments.setdefault(seq, [])
        if n > 0:
            segs.append((pos0, pos0 + int(n), seq))

    def fork(self, parent, child):
        self.ops.append(("fork", parent, child))
        self.lengths[child] = self.lengths[parent]
        self.segments[child] = list(self.segments[parent])

    def free(self, seq):
        self.ops.append(("free", seq))
        del self.lengths[seq]
        del self.segments[seq]

    def shuffle_pool(self, rng, num_blocks, bs):
        """Occupy every block with a one-block dummy, then free them in random order,
        so that later allocations come out in a seeded random physical order."""
        ids = [DUMMY_BASE + i for i in range(num_blocks)]
        for s in ids:
            self.alloc(s, bs, write=False)
        for i in rng.permutation(num_blocks):
            self.free(ids[i])


def _finish(wl: Workload, sc: _Script, batch):
    n_prefill = len(sc.ops)
    for s in batch:  # the decode step: one new token per sequence, in batch order
        sc.alloc(int(s), 1)
    wl.ops = sc.ops
    wl.n_prefill_ops = n_prefill
    wl.batch = np.asarray(batch, dtype=np.int64)
    wl.lengths = {int(s): sc.lengths[int(s)] for s in batch}
    wl.segments = {int(s): sc.segments[int(s)] for s in batch}
    return wl


def _simple(name, dtype, B, Hq, Hkv, D, bs, ctx, seed, slack, shuffle=True, extra_mb=16):
    ctx = [int(c) for c in ctx]
    nb = sum((c + bs - 1) // bs for c in ctx) + slack
    mb = (max(ctx) + bs - 1) // bs + extra_mb
    wl = Workload(name, dtype, B, Hq, Hkv, D, bs, nb, mb, seed)
    rng = np.random.default_rng(seed)
    sc = _Script()
    if shuffle:
        sc.shuffle_pool(rng, nb, bs)
    for s, c in enumerate(ctx):
        sc.alloc(s, c - 1)
    return _finish(wl, sc, list(range(B)))


def tiny(seed=486):
    """1 layer, 4 sequences of context {1, 17, 33, 50}, 4 q / 2 kv heads, head_dim 64,
    block 16, fp32, 32-block pool in seeded random physical order."""
    wl = Workload("tiny", "f32", 4, 4, 2, 64, 16, 32, 4, seed)
    rng = np.random.default_rng(seed)
    sc = _Script()
    sc.shuffle_pool(rng, 32, 16)
    for s, c in enumerate([1, 17, 33, 50]):
        sc.alloc(s, c - 1)
    return _finish(wl, sc, [0, 1, 2, 3])


def llama3_8b(seed=4861, B=64):
    """Llama-3-8B-shaped layer: 32 q / 8 kv heads, head_dim 128, fp16, block 16,
    batch 64, context ~ U[128, 4096], shuffled pool (+1024 blocks of slack)."""
    rng = np.random.default_rng(seed)
    ctx = rng.integers(128, 4097, size=B)
    return _simple("llama3_8b", "f16", B, 32, 8, 128, 16, ctx, seed, slack=1024)


def llama3_70b(seed=4862, B=256):
    """Llama-3-70B-shaped layer: 64 q / 8 kv heads, head_dim 128, bf16, block 16,
    batch 256; 70% lengths lognormal (median 300, sigma 1, clipped to [1, 4096]),
    30% ~ U[4096, 8192], order shuffled; pool shuffled then fragmented by churn of
    short-lived dummy sequences interleaved with chunked growth of the real ones."""
    rng = np.random.default_rng(seed)
    n_short = int(round(0.7 * B))
    short = np.clip(np.round(rng.lognormal(math.log(300.0), 1.0, size=n_short)), 1, 4096)
    long_ = rng.integers(4096, 8193, size=B - n_short)
    ctx = rng.permutation(np.concatenate([short, long_]).astype(np.int64))
    bs = 16
    slack = 2048
    nb = int(sum((int(c) + bs - 1) // bs for c in ctx)) + slack
    mb = (int(ctx.max()) + bs - 1) // bs + 16
    wl = Workload("llama3_70b", "bf16", B, 64, 8, 128, bs, nb, mb, seed)
    sc = _Script()
    sc.shuffle_pool(rng, nb, bs)
    remaining = {s: int(c) - 1 for s, c in enumerate(ctx)}
    live_dummies = []
    next_dummy = DUMMY_BASE + nb
    while any(v > 0 for v in remaining.values()):
        for s in rng.permutation(B):
            s = int(s)
            if remaining[s] <= 0:
                continue
            n = min(remaining[s], int(rng.integers(16, 513)))
            sc.alloc(s, n)
            remaining[s] -= n
            if rng.random() < 0.3 and len(live_dummies) < 64:
                sc.alloc(next_dummy, int(rng.integers(1, 65)), write=False)
                live_dummies.append(next_dummy)
                next_dummy += 1
            if rng.random() < 0.3 and live_dummies:
                sc.free(live_dummies.pop(int(rng.integers(0, len(live_dummies)))))
    for s in list(range(B)):
        if remaining[s] == 0 and s not in sc.lengths:
            sc.alloc(s, 0)  # a context of one token: created empty, grown by the decode step
    for d in live_dummies:
        sc.free(d)
    return _finish(wl, sc, list(range(B)))


def shared_prefix(seed=4863, n_groups=128, n_samples=4, prefix_len=1024):
    """8B-shaped heads, fp16, block 16: one 1024-token prefix shared by 128 sequences,
    each with its own suffix ~ U[64, 512], each then forked for n=4 parallel sampling;
    the decode step appends one token to each of the 512 sequences, which copies a
    shared partially filled last block for all but the last holder."""
    rng = np.random.default_rng(seed)
    bs = 16
    suffix = rng.integers(64, 513, size=n_groups)
    prefix_seq = 1 << 30
    child_base = 1 << 31
    nb = (prefix_len // bs + int(sum((int(x) + bs) // bs + 1 for x in suffix))
          + n_groups * n_samples + 256)
    mb = (prefix_len + 512 + 1 + bs - 1) // bs + 16
    wl = Workload("shared_prefix", "f16", n_groups * n_samples, 32, 8, 128, bs, nb, mb, seed)
    sc = _Script()
    sc.shuffle_pool(rng, nb, bs)
    sc.alloc(prefix_seq, prefix_len)
    batch = []
    for i in range(n_groups):
        sc.fork(prefix_seq, i)
        sc.alloc(i, int(suffix[i]))
    for i in range(n_groups):
        batch.append(i)
        for j in range(n_samples - 1):
            c = child_base + i * n_samples + j
            sc.fork(i, c)
            batch.append(c)
    return _finish(wl, sc, batch)


def long_mha(seed=4864, bs=16, B=8, ctx=32768):
    """Full multi-head attention at long context: 64 q / 64 kv heads, head_dim 128,
    fp16, batch 8, context 32768 each, block 16 or 32."""
    name = "long_mha" if bs == 16 else f"long_mha_bs{bs}"
    return _simple(name, "f16", B, 64, 64, 128, bs, [ctx] * B, seed, slack=16)


def custom(name="custom", dtype="f16", B=6, Hq=8, Hkv=2, D=128, bs=16, ctx=None, seed=1,
           slack=8, shuffle=True):
    """Small parity case with explicit context lengths."""
    rng = np.random.default_rng(seed)
    if ctx is None:
        ctx = rng.integers(1, 700, size=B)
    return _simple(name, dtype, len(ctx), Hq, Hkv, D, bs, ctx, seed, slack=slack,
                   shuffle=shuffle)


def spread(wl, q_mul=2.0, ramp_tokens=256, ramp_max=3):
    """The same workload with the wide-range option on (see Workload): scores span
    tens of base-2 units and the largest ones come late in each context."""
    wl.q_mul, wl.k_ramp_tokens, wl.k_ramp_max = float(q_mul), int(ramp_tokens), int(ramp_max)
    wl.name += "_spread"
    return wl


# --------------------------------------------------------------- prefill
def prefill(name, dtype, Hq, Hkv, D, bs, ctx, n_new, seed, slack=8) -> Workload:
    """Sequences of ctx[b] cached tokens whose last n_new[b] are the new chunk being
    prefilled (n_new = ctx: a whole prompt; n_new < ctx: chunked prefill on top of
    earlier context).  The chunk's keys and values are in the cache, written by the
    op script like every other token; `q_prefill` gives the chunk's queries
    [sum n_new, Hq, D] and `query_start` their offsets."""
    wl = _simple(name, dtype, len(ctx), Hq, Hkv, D, bs, ctx, seed, slack=slack, shuffle=True)
    wl.n_new = np.asarray(n_new, dtype=np.int32)
    assert np.all(wl.n_new <= wl.context_lens()) and np.all(wl.n_new >= 0)
    return wl


def query_start(wl) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(wl.n_new)]).astype(np.int32)


def q_prefill(wl, device="cpu") -> torch.Tensor:
    T = int(wl.n_new.sum())
    n = T * wl.Hq * wl.D
    t = _gen(stream_key(wl.seed, KIND_Q, 1), 0, n, device, wl.dtype).view(T, wl.Hq, wl.D)
    return t if wl.q_mul == 1.0 else t * wl.q_mul


def prefill_8b(seed=4866):
    """Llama-3-8B heads (32 / 8, d128, fp16, bs16): 8 whole prompts of 2048 tokens."""
    return prefill("prefill_8b", "f16", 32, 8, 128, 16, [2048] * 8, [2048] * 8, seed)


def chunked_8b(seed=4867):
    """Llama-3-8B heads, fp16, bs16: 16 sequences with U[1024, 8192] tokens whose last
    512 are the chunk being prefilled on top of the earlier context."""
    rng = np.random.default_rng(seed)
    ctx = rng.integers(1024, 8193, size=16)
    return prefill("chunked_8b", "f16", 32, 8, 128, 16, ctx, [512] * 16, seed)


# ------------------------------------------------------------ prompt sets
def token_rows(seed: int, kind: int, ids, positions, Hkv: int, D: int, dtype: str,
               device="cpu") -> torch.Tensor:
    """[n, Hkv, D] key (kind 0) or value (kind 1) rows of tokens with the given ids at
    the given positions.  A function of (id, position) only, so two sequences that
    begin with the same tokens have the same rows there -- what reusing a cached
    prefix block assumes."""
    ids = torch.as_tensor(np.asarray(ids, dtype=np.int64), device=device)
    pos = torch.as_tensor(np.asarray(positions, dtype=np.int64), device=device)
    per = Hkv * D
    key = stream_key(seed, kind, 0x7072656669)
    idx = ((ids << 24) | pos)[:, None] * per + torch.arange(per, dtype=torch.int64, device=device)
    return values(key, idx.reshape(-1)).to(TORCH_DTYPE[dtype]).view(len(ids), Hkv, D)


@dataclass
class PromptSet:
    """Requests that begin with one of a few shared system prompts, each followed by
    its own user tokens (token ids drawn from a vocabulary)."""
    name: str
    dtype: str
    Hq: int
    Hkv: int
    D: int
    bs: int
    num_blocks: int
    seed: int
    prompts: list = field(default_factory=list)   # int32 token-id arrays, one per request
    system_of: list = field(default_factory=list)  # system prompt index of each request

    @property
    def B(self):
        return len(self.prompts)

    @property
    def G(self):
        return self.Hq // self.Hkv

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.D)

    def rows(self, i: int, kind: int, device="cpu") -> torch.Tensor:
        ids = self.prompts[i]
        return token_rows(self.seed, kind, ids, np.arange(len(ids)), self.Hkv, self.D,
                          self.dtype, device)

    def q(self, device="cpu") -> torch.Tensor:
        n = self.B * self.Hq * self.D
        return _gen(stream_key(self.seed, KIND_Q, 0), 0, n, device, self.dtype).view(
            self.B, self.Hq, self.D)


def prompt_set(name="prompts", dtype="f16", n_systems=3, system_lens=(100, 257, 64),
               n_requests=24, user_len=(1, 300), vocab=1000, Hq=32, Hkv=8, D=128, bs=16,
               seed=4865, slack_blocks=0) -> PromptSet:
    rng = np.random.default_rng(seed)
    lens = [system_lens[k % len(system_lens)] for k in range(n_systems)]
    systems = [rng.integers(0, vocab, size=n).astype(np.int32) for n in lens]
    prompts, system_of = [], []
    for _ in range(n_requests):
        k = int(rng.integers(0, n_systems))
        user = rng.integers(0, vocab, size=int(rng.integers(user_len[0], user_len[1] + 1)))
        prompts.append(np.concatenate([systems[k], user.astype(np.int32)]))
        system_of.append(k)
    need = sum((len(p) + bs - 1) // bs for p in prompts)
    return PromptSet(name, dtype, Hq, Hkv, D, bs, need + slack_blocks, seed, prompts, system_of)


def prefix_prompts(seed=4865):
    """Llama-3-8B heads (32 / 8, d128, fp16, bs16): 512 requests over 16 shared
    system prompts of 1024 tokens, each with U[16, 256] own tokens."""
    return prompt_set("prefix_prompts", "f16", n_systems=16, system_lens=(1024,),
                      n_requests=512, user_len=(16, 256), vocab=32000, seed=seed)


CONFIGS = {
    "tiny": tiny,
    "llama3_8b": llama3_8b,
    "llama3_70b": llama3_70b,
    "shared_prefix": shared_prefix,
    "long_mha": long_mha,
    "long_mha_bs32": lambda: long_mha(bs=32),
    "prefill_8b": prefill_8b,
    "chunked_8b": chunked_8b,
}


def make(name: str, batch: int = 0) -> Workload:
    """The named workload; batch > 0 overrides the batch of the configurations
    that take one (llama3_8b, llama3_70b, long_mha, long_mha_bs32)."""
    if batch > 0:
        sized = {"llama3_8b": lambda: llama3_8b(B=batch),
                 "llama3_70b": lambda: llama3_70b(B=batch),
                 "long_mha": lambda: long_mha(B=batch),
                 "long_mha_bs32": lambda: long_mha(bs=32, B=batch)}
        if name not in sized:
            raise ValueError(f"{name} has a fixed batch")
        wl = sized[name]()
        wl.name = f"{wl.name}_b{batch}"
        return wl
    return CONFIGS[name]()
