"""Pins the oracle's prefix cache: hand-worked examples of reuse, the last-token
rule, the eviction order and atomicity, and a content model in which every
memory cell holds an identifier of its token's whole prefix, so a reused block
that held anything else would read back wrong."""
import numpy as np
import pytest

import oracle
from oracle import OK


def _pool(nb, bs):
    p = oracle.Pool(nb, bs)
    p.set_prefix_caching(True)
    return p


def test_reuse_of_a_shared_beginning():
    p = _pool(16, 4)
    a = list(range(1, 11))                       # 10 tokens: blocks [1..4], [5..8] full
    st, slots, cow, n_cached = p.alloc_tokens(1, a)
    assert st == oracle.OK and n_cached == 0 and (slots >= 0).all()
    assert p.num_cached() == 2
    b = list(range(1, 9)) + [99, 100]            # same first 8 tokens
    st, slots_b, _, n_cached = p.alloc_tokens(2, b)
    assert n_cached == 8 and list(slots_b[:8]) == [-1] * 8 and (slots_b[8:] >= 0).all()
    ta, _ = p.block_table([1], 8)[1:]
    tb, _ = p.block_table([2], 8)[1:]
    assert list(tb[0, :2]) == list(ta[0, :2])    # the two full blocks are shared
    assert p.holders(int(ta[0, 0])) == 2 and p.holders(int(ta[0, 1])) == 2
    # a prompt that ends exactly at a block boundary reuses all but the block
    # holding its last token
    st, slots_c, _, n_cached = p.alloc_tokens(3, list(range(1, 9)))
    assert n_cached == 4 and list(slots_c[:4]) == [-1] * 4
    # a different first block: nothing reused, even if later tokens agree
    st, _, _, n_cached = p.alloc_tokens(4, [1, 2, 3, 7, 5, 6, 7, 8, 9])
    assert n_cached == 0
    # growth of an existing sequence never looks up
    st, _, _, n_cached = p.alloc_tokens(4, list(range(1, 9)))
    assert n_cached == 0


def test_partial_blocks_and_unknown_ids_are_never_cached():
    p = _pool(16, 4)
    p.alloc_tokens(1, [1, 2, 3])                  # partial only
    assert p.num_cached() == 0
    p.alloc(2, 8)                                 # no ids: never entered
    assert p.num_cached() == 0
    st, _, _, n_cached = p.alloc_tokens(3, [1, 2, 3, 4, 5])
    assert n_cached == 0 and p.num_cached() == 1  # [1..4] entered now
    p.alloc(3, 4)                                 # ids lost from here on
    p.alloc_tokens(3, [9, 9, 9, 9])
    assert p.num_cached() == 1


def test_eviction_order_and_reuse_after_release():
    p = _pool(4, 2)
    st, slots, _, _ = p.alloc_tokens(1, [1, 2, 3, 4, 5])  # blocks 0, 1 (cached), 2
    assert [int(x) // 2 for x in slots[::2]] == [0, 1, 2]
    assert p.num_cached() == 2
    assert p.free(1) == oracle.OK
    # block 2 (not cached) -> free stack; blocks 1 then 0 -> releasable queue
    assert p.num_free() == 4 and p.num_releasable() == 2 and p.num_cached() == 2
    st, slots, _, n_cached = p.alloc_tokens(2, [7, 8, 9, 10, 11])  # needs 3 blocks
    assert n_cached == 0
    # free stack first (2 on top, then 3), then the queue's front: block 1, whose
    # entry [1, 2, 3, 4] leaves the cache
    assert [int(x) // 2 for x in slots[::2]] == [2, 3, 1]
    assert p.num_cached() == 3                    # [1, 2] stays; [7, 8], [7..10] entered
    assert p.free(2) == OK
    # block 1 (partial) -> free stack; blocks 3 then 2 -> queue, now [0, 3, 2]
    assert p.num_releasable() == 3
    st, slots, _, n_cached = p.alloc_tokens(3, [1, 2, 3, 4, 5, 6])
    assert st == OK and n_cached == 2 and list(slots[:2]) == [-1, -1]  # block 0 found again
    # then block 1 (free stack) and the queue's front, block 3 ([7..10] leaves)
    assert [int(x) // 2 for x in slots[2::2]] == [1, 3]
    assert p.num_releasable() == 1                # block 2 ([7, 8]) still waiting
    assert p.num_cached() == 4                    # [1, 2], [7, 8], [1..4], [1..6]


def test_out_of_memory_changes_nothing():
    p = _pool(3, 2)
    p.alloc_tokens(1, [1, 2, 3, 4, 5])            # 3 blocks, 2 cached
    p.free(1)
    before = (p.num_free(), p.num_cached(), p.num_releasable())
    # [1, 2] would be reused, but 3 more blocks are needed and only 2 remain
    st, _, _, _ = p.alloc_tokens(2, [1, 2, 9, 9, 9, 9, 9, 9])
    assert st == oracle.OOM
    assert (p.num_free(), p.num_cached(), p.num_releasable()) == before
    assert p.seq_len(2) == -1
    # with the cache's own block as a hit, 2 fresh blocks fit
    st, _, _, n_cached = p.alloc_tokens(2, [1, 2, 9, 9, 9, 9])
    assert st == oracle.OK and n_cached == 2


def test_turning_caching_off_frees_the_queue():
    p = _pool(4, 2)
    p.alloc_tokens(1, [1, 2, 3, 4, 5])
    p.free(1)
    p.set_prefix_caching(False)
    assert p.num_cached() == 0 and p.num_releasable() == 0 and p.num_free() == 4
    p.set_prefix_caching(True)
    st, _, _, n_cached = p.alloc_tokens(2, [1, 2, 3, 4, 5])
    assert n_cached == 0


class PrefixContent:
    """Memory simulated cell by cell; a cell written for token i of a sequence
    holds the id of the sequence's tokens 0..i.  Every sequence must read back,
    through its block table, the identifiers of its own prefixes."""

    def __init__(self, nb, bs, seed):
        self.pool = _pool(nb, bs)
        self.nb, self.bs = nb, bs
        self.mem = np.full(nb * bs, -1, dtype=np.int64)
        self.tokens = {}
        self.prefix_id = {}
        self.rng = np.random.default_rng(seed)
        self.cached_tokens = 0

    def pid(self, prefix):
        return self.prefix_id.setdefault(tuple(prefix), len(self.prefix_id))

    def alloc(self, s, ids):
        st, slots, cow, n_cached = self.pool.alloc_tokens(s, ids)
        if st != oracle.OK:
            return st
        for src, dst in cow:
            self.mem[dst * self.bs:(dst + 1) * self.bs] = self.mem[src * self.bs:(src + 1) * self.bs]
        toks = self.tokens.setdefault(s, [])
        assert n_cached == 0 or not toks
        self.cached_tokens += n_cached
        for i, t in enumerate(ids):
            toks.append(int(t))
            if slots[i] >= 0:
                self.mem[slots[i]] = self.pid(toks)
            else:
                assert i < n_cached
        return st

    def check(self):
        seqs = sorted(self.tokens)
        held = {}
        if seqs:
            st, table, ctx = self.pool.block_table(seqs, self.nb + 1)
            assert st == oracle.OK
            for i, s in enumerate(seqs):
                toks = self.tokens[s]
                assert int(ctx[i]) == len(toks)
                pos = np.arange(len(toks))
                got = self.mem[table[i][pos // self.bs] * self.bs + pos % self.bs]
                want = [self.prefix_id[tuple(toks[:k + 1])] for k in range(len(toks))]
                assert list(got) == want
                for b in table[i][table[i] >= 0]:
                    held[int(b)] = held.get(int(b), 0) + 1
        for b in range(self.nb):
            assert self.pool.holders(b) == held.get(b, 0)
        assert self.pool.num_free() + len(held) == self.nb
        assert self.pool.num_releasable() <= self.pool.num_cached()


@pytest.mark.parametrize("seed", range(12))
def test_random_prompt_scripts_read_back_their_prefixes(seed):
    rng = np.random.default_rng(seed)
    bs = int(rng.choice([1, 2, 4]))
    m = PrefixContent(int(rng.integers(6, 40)), bs, seed)
    systems = [list(rng.integers(0, 5, size=int(rng.integers(1, 12)))) for _ in range(3)]
    next_id = 0
    for _ in range(250):
        live = sorted(m.tokens)
        r = rng.random()
        if r < 0.4 or not live:
            sysp = systems[int(rng.integers(0, 3))]
            ids = sysp + list(rng.integers(0, 5, size=int(rng.integers(0, 3 * bs + 2))))
            if ids:
                m.alloc(next_id, ids)
                next_id += 1
        elif r < 0.65:
            s = int(rng.choice(live))
            m.alloc(s, list(rng.integers(0, 5, size=int(rng.integers(1, bs + 2)))))
        elif r < 0.75:
            p_ = int(rng.choice(live))
            if m.pool.fork(p_, next_id) == oracle.OK:
                m.tokens[next_id] = list(m.tokens[p_])
                next_id += 1
        else:
            s = int(rng.choice(live))
            assert m.pool.free(s) == oracle.OK
            del m.tokens[s]
        m.check()
    assert m.cached_tokens > 0  # the scripts do exercise reuse
