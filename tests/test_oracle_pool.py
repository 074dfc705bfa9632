"""Pins the oracle's block-pool model: the pages' printed facts, conservation
invariants, and an exhaustive content check on tiny pools (every sequence must
read back, through its block table, exactly the tokens it was given)."""
import itertools
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _facts():
    with open(os.path.join(GOLD, "allocator.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                yield line.split()


def _used_blocks(pool, seqs, max_blocks=64):
    st, table, ctx = pool.block_table(list(seqs), max_blocks)
    assert st == oracle.OK
    return table, ctx


def test_printed_facts():
    for fact in _facts():
        name, args, expected = fact[0], [int(x) for x in fact[1:-1]], int(fact[-1])
        if name == "blocks_for_tokens":
            bs, n = args
            pool = oracle.Pool(8, bs)
            assert pool.alloc(0, n)[0] == oracle.OK
            table, _ = _used_blocks(pool, [0])
            assert int((table >= 0).sum()) == expected
            assert 8 - pool.num_free() == expected
        elif name == "contiguous_waste":
            max_len, used = args
            assert max_len - used == expected
        elif name == "contiguous_waste_pct":
            max_len, used = args
            assert round(100 * (max_len - used) / max_len) == expected
        elif name == "paged_waste_slots":
            bs, used = args
            pool = oracle.Pool(64, bs)
            pool.alloc(0, used)
            table, ctx = _used_blocks(pool, [0])
            assert int((table >= 0).sum()) * bs - int(ctx[0]) == expected
        else:
            raise AssertionError(name)


def test_growth_one_token_at_a_time_takes_a_block_every_16():
    pool = oracle.Pool(16, 16)
    for n in range(1, 80):
        st, slots, cow = pool.alloc(7, 1)
        assert st == oracle.OK and len(cow) == 0
        table, ctx = _used_blocks(pool, [7])
        assert ctx[0] == n
        assert int((table >= 0).sum()) == (n + 15) // 16   # waste only in the last block


def test_fresh_pool_order_and_immediate_reuse():
    pool = oracle.Pool(10, 4)
    pool.alloc(1, 12)
    t1, _ = _used_blocks(pool, [1])
    assert list(t1[0, :3]) == [0, 1, 2]
    pool.free(1)
    assert pool.num_free() == 10
    pool.alloc(2, 12)
    t2, _ = _used_blocks(pool, [2])
    assert set(t2[0, :3]) == {0, 1, 2}  # the freed blocks are taken at once
    assert list(t2[0, :3]) == [2, 1, 0]  # last freed, first reused


@pytest.mark.parametrize("suffix_len, expect_new, expect_copies",
                         [(1030, 3, 3), (1024, 4, 0)])
def test_parallel_sampling_n4_costs_about_n1(suffix_len, expect_new, expect_copies):
    pool = oracle.Pool(200, 16)
    pool.alloc(0, suffix_len)
    used0 = 200 - pool.num_free()
    for c in (1, 2, 3):
        assert pool.fork(0, c) == oracle.OK
    assert 200 - pool.num_free() == used0  # forks share every block
    copies = 0
    for s in (0, 1, 2, 3):
        st, slots, cow = pool.alloc(s, 1)
        assert st == oracle.OK
        copies += len(cow)
    assert copies == expect_copies
    assert 200 - pool.num_free() == used0 + expect_new


def test_oom_changes_nothing():
    pool = oracle.Pool(4, 4)
    pool.alloc(0, 10)  # 3 blocks
    pool.fork(0, 1)
    before = (pool.num_free(), [pool.holders(b) for b in range(4)], pool.seq_len(0),
              pool.seq_len(1))
    assert pool.alloc(1, 7)[0] == oracle.OOM  # needs a copy of the last block + 1 more
    assert pool.alloc(5, 17)[0] == oracle.OOM  # new sequence, 5 blocks
    after = (pool.num_free(), [pool.holders(b) for b in range(4)], pool.seq_len(0),
             pool.seq_len(1))
    assert before == after
    assert pool.seq_len(5) == -1


def test_error_codes():
    pool = oracle.Pool(4, 4)
    assert pool.free(3) == oracle.NOT_FOUND
    assert pool.fork(3, 4) == oracle.NOT_FOUND
    pool.alloc(3, 1)
    assert pool.fork(3, 3) == oracle.INVALID
    pool.alloc(4, 9)
    st, _, _ = pool.block_table([4], 2)
    assert st == oracle.INVALID
    st, _, _ = pool.block_table([99], 8)
    assert st == oracle.NOT_FOUND
    assert pool.alloc(3, -1)[0] == oracle.INVALID


class ContentModel:
    """What each sequence holds, by definition: alloc appends fresh tokens, fork
    copies the parent's tokens, free forgets the sequence.  Physical memory is
    simulated cell by cell from the pool's slots and copy pairs only."""

    def __init__(self, nb, bs):
        self.pool = oracle.Pool(nb, bs)
        self.nb, self.bs = nb, bs
        self.mem = np.full(nb * bs, -1, dtype=np.int64)
        self.expected = {}
        self.next_token = 0

    def apply(self, op):
        kind = op[0]
        if kind == "alloc":
            _, s, n = op
            st, slots, cow = self.pool.alloc(s, n)
            if st != oracle.OK:
                return st
            for src, dst in cow:
                self.mem[dst * self.bs:(dst + 1) * self.bs] = \
                    self.mem[src * self.bs:(src + 1) * self.bs]
            toks = list(range(self.next_token, self.next_token + n))
            self.next_token += n
            for b in {int(x) // self.bs for x in slots}:
                assert self.pool.holders(b) == 1  # never write into a block others hold
            self.mem[slots] = toks
            self.expected.setdefault(s, []).extend(toks)
            return st
        if kind == "fork":
            _, p, c = op
            st = self.pool.fork(p, c)
            if st == oracle.OK:
                self.expected[c] = list(self.expected[p])
            return st
        _, s = op
        st = self.pool.free(s)
        if st == oracle.OK:
            del self.expected[s]
        return st

    def check(self):
        seqs = sorted(self.expected)
        held = {}
        if seqs:
            st, table, ctx = self.pool.block_table(seqs, self.nb + 1)
            assert st == oracle.OK
            for i, s in enumerate(seqs):
                n = int(ctx[i])
                assert n == len(self.expected[s])
                nblk = int((table[i] >= 0).sum())
                assert nblk == (n + self.bs - 1) // self.bs
                pos = np.arange(n)
                got = self.mem[table[i][pos // self.bs] * self.bs + pos % self.bs]
                assert list(got) == self.expected[s]
                for b in table[i][:nblk]:
                    held[int(b)] = held.get(int(b), 0) + 1
        for b in range(self.nb):
            assert self.pool.holders(b) == held.get(b, 0)
        assert self.pool.num_free() + len(held) == self.nb


def test_exhaustive_short_scripts_on_a_tiny_pool():
    # every script of 4 ops over sequences {0, 1} on a 3-block pool of 2-token blocks
    alphabet = ([("alloc", s, n) for s in (0, 1) for n in (0, 1, 2, 3)]
                + [("fork", 0, 1), ("fork", 1, 0), ("free", 0), ("free", 1)])
    count = 0
    for script in itertools.product(alphabet, repeat=4):
        m = ContentModel(3, 2)
        for op in script:
            m.apply(op)
            m.check()
        count += 1
    assert count == len(alphabet) ** 4


def test_random_long_scripts():
    rng = np.random.default_rng(7)
    for trial in range(20):
        nb, bs = int(rng.integers(4, 40)), int(rng.choice([1, 2, 4, 16]))
        m = ContentModel(nb, bs)
        for _ in range(300):
            live = sorted(m.expected)
            r = rng.random()
            if r < 0.55 or not live:
                s = int(rng.integers(0, 12))
                m.apply(("alloc", s, int(rng.integers(0, 2 * bs + 2))))
            elif r < 0.75:
                p = int(rng.choice(live))
                c = int(rng.integers(0, 12))
                m.apply(("fork", p, c))
            else:
                m.apply(("free", int(rng.choice(live))))
            m.check()


def test_swap_moves_a_sequence_and_its_content():
    """Swapping out and back in keeps every sequence's content (checked cell by cell)."""
    dev, host = oracle.Pool(6, 2), oracle.Pool(4, 2)
    mem = {"d": np.full(12, -1), "h": np.full(8, -1)}
    dev.alloc(1, 5)            # 3 blocks
    dev.fork(1, 2)             # shares them
    _, s3, _ = dev.alloc(3, 2)
    t, _ = _used_blocks(dev, [1, 3])
    pos = np.arange(5)
    mem["d"][t[0][pos // 2] * 2 + pos % 2] = [10, 11, 12, 13, 14]
    mem["d"][s3] = [30, 31]
    st, pairs = oracle.swap(dev, host, 1)
    assert st == oracle.OK and len(pairs) == 3
    for a, b in pairs:
        mem["h"][b * 2:(b + 1) * 2] = mem["d"][a * 2:(a + 1) * 2]
    assert dev.seq_len(1) == -1 and host.seq_len(1) == 5
    assert dev.num_free() == 6 - 3 - 1     # seq 2 still holds the shared blocks
    th, _ = _used_blocks(host, [1])
    assert list(mem["h"][th[0][pos // 2] * 2 + pos % 2]) == [10, 11, 12, 13, 14]
    assert oracle.swap(dev, host, 3)[0] == oracle.OK      # 1 more host block
    assert oracle.swap(dev, host, 2)[0] == oracle.OOM     # 3 blocks, 0 free: nothing moves
    assert dev.seq_len(2) == 5 and host.num_free() == 0
    st, back = oracle.swap(host, dev, 1)
    assert st == oracle.OK
    for a, b in back:
        mem["d"][b * 2:(b + 1) * 2] = mem["h"][a * 2:(a + 1) * 2]
    td, _ = _used_blocks(dev, [1])
    assert list(mem["d"][td[0][pos // 2] * 2 + pos % 2]) == [10, 11, 12, 13, 14]
    assert host.num_free() == 3            # the swapped-in sequence's host blocks came back
    assert oracle.swap(dev, host, 9)[0] == oracle.NOT_FOUND
    assert oracle.swap(host, dev, 3)[0] == oracle.OOM      # seqs 1 and 2 fill the device pool
    assert dev.free(2) == oracle.OK
    assert oracle.swap(host, dev, 3)[0] == oracle.OK
    assert oracle.swap(dev, dev, 3)[0] == oracle.INVALID   # already in the destination
