"""The product's host block pool against the oracle's pool model: identical
slots, copy pairs, block tables, free counts and holder counts, bit for bit,
on every workload script and on random op scripts; plus the validators."""
import numpy as np
import pytest

import oracle
import paged_kv_cache_486_b200 as pa
import workloads


def _same_state(p, o, nb, seqs, max_blocks):
    assert p.pa_num_free_blocks() == o.num_free()
    for b in range(nb):
        assert p.pa_refcount(b) == o.holders(b)
    if seqs:
        t1, c1 = p.pa_block_table(seqs, max_blocks)
        st, t2, c2 = o.block_table(seqs, max_blocks)
        assert st == oracle.OK
        assert np.array_equal(t1, t2) and np.array_equal(c1, c2)


def _run_both(wl):
    p = pa.Pool(wl.num_blocks, wl.bs)
    o = oracle.Pool(wl.num_blocks, wl.bs)
    for op in wl.ops:
        if op[0] == "alloc":
            slots, cow = p.pa_alloc(op[1], op[2])
            st, slots2, cow2 = o.alloc(op[1], op[2])
            assert st == oracle.OK
            assert np.array_equal(slots, slots2) and np.array_equal(cow, cow2)
        elif op[0] == "fork":
            p.pa_fork(op[1], op[2])
            assert o.fork(op[1], op[2]) == oracle.OK
        else:
            p.pa_free(op[1])
            assert o.free(op[1]) == oracle.OK
    _same_state(p, o, wl.num_blocks, list(wl.batch), wl.max_blocks)


@pytest.mark.parametrize("name", ["tiny", "llama3_8b", "shared_prefix", "llama3_70b"])
def test_workload_scripts_match_the_oracle(name):
    _run_both(workloads.make(name))


def test_random_scripts_match_the_oracle():
    rng = np.random.default_rng(99)
    for trial in range(30):
        nb, bs = int(rng.integers(1, 50)), int(rng.choice([1, 3, 8, 16]))
        p, o = pa.Pool(nb, bs), oracle.Pool(nb, bs)
        live = set()
        for _ in range(250):
            r = rng.random()
            if r < 0.5 or not live:
                s, n = int(rng.integers(0, 10)), int(rng.integers(0, 3 * bs + 1))
                st, slots2, cow2 = o.alloc(s, n)
                try:
                    slots, cow = p.pa_alloc(s, n)
                    assert st == oracle.OK
                    assert np.array_equal(slots, slots2) and np.array_equal(cow, cow2)
                    live.add(s)
                except pa.PagedAttnError as e:
                    assert e.status == st == pa.PA_ERR_OOM
            elif r < 0.7:
                parent, child = int(rng.choice(sorted(live))), int(rng.integers(0, 10))
                st = o.fork(parent, child)
                try:
                    p.pa_fork(parent, child)
                    assert st == oracle.OK
                    live.add(child)
                except pa.PagedAttnError as e:
                    assert e.status == st
            else:
                s = int(rng.choice(sorted(live)))
                p.pa_free(s)
                assert o.free(s) == oracle.OK
                live.discard(s)
            _same_state(p, o, nb, sorted(live), nb + 1)


def test_errors_and_atomicity():
    p = pa.Pool(4, 4)
    with pytest.raises(pa.PagedAttnError) as e:
        p.pa_free(1)
    assert e.value.status == pa.PA_ERR_NOT_FOUND
    p.pa_alloc(1, 10)
    p.pa_fork(1, 2)
    before = (p.pa_num_free_blocks(), [p.pa_refcount(b) for b in range(4)])
    with pytest.raises(pa.PagedAttnError) as e:
        p.pa_alloc(2, 7)
    assert e.value.status == pa.PA_ERR_OOM
    assert (p.pa_num_free_blocks(), [p.pa_refcount(b) for b in range(4)]) == before
    with pytest.raises(pa.PagedAttnError) as e:
        p.pa_fork(1, 2)
    assert e.value.status == pa.PA_ERR_INVALID
    with pytest.raises(pa.PagedAttnError):
        p.pa_block_table([1], 2)
    assert p.pa_refcount(-1) == -1 and p.pa_refcount(4) == -1
    assert p.pa_seq_len(1) == 10 and p.pa_seq_len(9) == -1


def test_validators():
    assert pa.pa_validate_slot_mapping([0, 5, -1, 63], 16, 4) == pa.PA_OK
    assert pa.pa_validate_slot_mapping([0, 64], 16, 4) == pa.PA_ERR_INVALID
    assert pa.pa_validate_slot_mapping([3, 3], 16, 4) == pa.PA_ERR_INVALID
    assert pa.pa_validate_slot_mapping([-2], 16, 4) == pa.PA_ERR_INVALID
    t = np.array([[0, 1, -1], [2, -1, -1]], np.int32)
    assert pa.pa_validate_block_table(t, np.array([20, 16], np.int32), 16, 3) == pa.PA_OK
    assert pa.pa_validate_block_table(t, np.array([33, 16], np.int32), 16, 3) == pa.PA_ERR_INVALID
    assert pa.pa_validate_block_table(t, np.array([20, 17], np.int32), 16, 3) == pa.PA_ERR_INVALID
    assert pa.pa_validate_block_table(t, np.array([20, 16], np.int32), 16, 2) == pa.PA_ERR_INVALID
    assert pa.pa_validate_copy_pairs([[1, 2], [3, 4]], 5) == pa.PA_OK
    assert pa.pa_validate_copy_pairs([[1, 2], [3, 2]], 5) == pa.PA_ERR_INVALID
    assert pa.pa_validate_copy_pairs([[1, 2], [2, 4]], 5) == pa.PA_ERR_INVALID
    assert pa.pa_validate_copy_pairs([[1, 5]], 5) == pa.PA_ERR_INVALID


def test_pool_slots_are_valid_for_the_kernels():
    wl = workloads.make("shared_prefix")
    p = pa.Pool(wl.num_blocks, wl.bs)
    for op in wl.ops:
        if op[0] == "alloc":
            slots, cow = p.pa_alloc(op[1], op[2])
            assert pa.pa_validate_slot_mapping(slots, wl.bs, wl.num_blocks) == pa.PA_OK
            if len(cow):
                assert pa.pa_validate_copy_pairs(cow, wl.num_blocks) == pa.PA_OK
        elif op[0] == "fork":
            p.pa_fork(op[1], op[2])
        else:
            p.pa_free(op[1])
    t, c = p.pa_block_table(wl.batch, wl.max_blocks)
    assert pa.pa_validate_block_table(t, c, wl.bs, wl.num_blocks) == pa.PA_OK


def test_batched_alloc_equals_sequential_and_rolls_back():
    rng = np.random.default_rng(5)
    for trial in range(40):
        nb, bs = int(rng.integers(4, 60)), int(rng.choice([1, 4, 16]))
        a, b = pa.Pool(nb, bs), pa.Pool(nb, bs)
        live = []
        for _ in range(30):
            r = rng.random()
            if r < 0.2 and live:
                p, c = int(rng.choice(live)), int(rng.integers(100, 200))
                if c not in live:
                    a.pa_fork(p, c)
                    b.pa_fork(p, c)
                    live.append(c)
                continue
            ids = [int(x) for x in rng.integers(0, 8, size=int(rng.integers(1, 6)))]
            n = int(rng.integers(0, 2 * bs + 1))
            before = ([a.pa_refcount(i) for i in range(nb)], a.pa_num_free_blocks(),
                      {s: a.pa_seq_len(s) for s in range(8)})
            try:
                slots, cow = a.pa_alloc_batch(ids, n)
            except pa.PagedAttnError as e:
                assert e.status == pa.PA_ERR_OOM
                after = ([a.pa_refcount(i) for i in range(nb)], a.pa_num_free_blocks(),
                         {s: a.pa_seq_len(s) for s in range(8)})
                assert before == after  # all or nothing
                # and the free stack order is intact: the next allocations agree
                continue
            exp_slots, exp_cow = [], []
            for s in ids:
                sl, cw = b.pa_alloc(s, n)
                exp_slots.append(sl)
                exp_cow.extend(cw.tolist())
            assert np.array_equal(slots, np.concatenate(exp_slots) if exp_slots else slots)
            assert cow.tolist() == exp_cow
            live = sorted(set(live) | set(ids))
            assert a.pa_num_free_blocks() == b.pa_num_free_blocks()
            assert [a.pa_refcount(i) for i in range(nb)] == [b.pa_refcount(i) for i in range(nb)]
            t1, c1 = a.pa_block_table(live, nb + 1)
            t2, c2 = b.pa_block_table(live, nb + 1)
            assert np.array_equal(t1, t2) and np.array_equal(c1, c2)


def test_swap_matches_the_oracle():
    rng = np.random.default_rng(13)
    for trial in range(25):
        bs = int(rng.choice([1, 4, 16]))
        nd, nh = int(rng.integers(4, 40)), int(rng.integers(2, 30))
        pd, ph = pa.Pool(nd, bs), pa.Pool(nh, bs)
        od, oh = oracle.Pool(nd, bs), oracle.Pool(nh, bs)
        where = {}  # seq -> "d" / "h"
        for _ in range(120):
            r = rng.random()
            dev_seqs = [s for s, w in where.items() if w == "d"]
            host_seqs = [s for s, w in where.items() if w == "h"]
            if r < 0.45 or not where:
                s = int(rng.integers(0, 10))
                if where.get(s) == "h":
                    continue
                n = int(rng.integers(0, 2 * bs + 1))
                st, sl2, cw2 = od.alloc(s, n)
                try:
                    sl, cw = pd.pa_alloc(s, n)
                    assert st == oracle.OK and np.array_equal(sl, sl2) and np.array_equal(cw, cw2)
                    where[s] = "d"
                except pa.PagedAttnError as e:
                    assert e.status == st
            elif r < 0.55 and dev_seqs:
                p, c = int(rng.choice(dev_seqs)), int(rng.integers(0, 10))
                if c in where:
                    continue
                assert od.fork(p, c) == oracle.OK
                pd.pa_fork(p, c)
                where[c] = "d"
            elif r < 0.75 and dev_seqs:
                s = int(rng.choice(dev_seqs))
                st, pr2 = oracle.swap(od, oh, s)
                try:
                    pr = pa.pa_swap(pd, ph, s)
                    assert st == oracle.OK and np.array_equal(pr, pr2)
                    where[s] = "h"
                except pa.PagedAttnError as e:
                    assert e.status == st == pa.PA_ERR_OOM
            elif r < 0.95 and host_seqs:
                s = int(rng.choice(host_seqs))
                st, pr2 = oracle.swap(oh, od, s)
                try:
                    pr = pa.pa_swap(ph, pd, s)
                    assert st == oracle.OK and np.array_equal(pr, pr2)
                    where[s] = "d"
                except pa.PagedAttnError as e:
                    assert e.status == st == pa.PA_ERR_OOM
            elif where:
                s = int(rng.choice(sorted(where)))
                if where[s] == "d":
                    pd.pa_free(s)
                    assert od.free(s) == oracle.OK
                else:
                    ph.pa_free(s)
                    assert oh.free(s) == oracle.OK
                del where[s]
            _same_state(pd, od, nd, sorted(s for s, w in where.items() if w == "d"), nd + 1)
            _same_state(ph, oh, nh, sorted(s for s, w in where.items() if w == "h"), nh + 1)


def _prefix_state(p, o, nb, seqs):
    _same_state(p, o, nb, seqs, nb + 1)
    assert p.pa_num_cached_blocks() == o.num_cached()
    assert p.pa_num_evictable_blocks() == o.num_releasable()


@pytest.mark.parametrize("seed", range(8))
def test_prefix_cache_scripts_match_the_oracle(seed):
    """Prompts sharing system prompts (pa_alloc_tokens), growth with and without
    ids, batches, forks, frees, swaps and toggles: every status, slot, copy pair,
    cached-token count, table and counter equals the oracle's."""
    rng = np.random.default_rng(100 + seed)
    bs = int(rng.choice([1, 2, 4, 16]))
    nb = int(rng.integers(8, 60))
    p, o = pa.Pool(nb, bs), oracle.Pool(nb, bs)
    hp, ho = pa.Pool(nb, bs), oracle.Pool(nb, bs)  # a second pool to swap into
    p.pa_set_prefix_caching(True)
    o.set_prefix_caching(True)
    systems = [list(rng.integers(0, 4, size=int(rng.integers(1, 3 * bs + 3)))) for _ in range(3)]
    live, away, nxt, hits = set(), set(), 0, 0
    for step in range(300):
        r = rng.random()
        if r < 0.35 or not live:
            ids = systems[int(rng.integers(0, 3))] + list(
                rng.integers(0, 4, size=int(rng.integers(0, 2 * bs + 2))))
            ids = np.array(ids or [1], dtype=np.int32)
            st_o, slots_o, cow_o, cached_o = o.alloc_tokens(nxt, ids)
            try:
                slots_p, cow_p, cached_p = p.pa_alloc_tokens(nxt, ids)
                assert st_o == oracle.OK
                assert np.array_equal(slots_p, slots_o) and np.array_equal(cow_p, cow_o)
                assert cached_p == cached_o
                hits += cached_p
                live.add(nxt)
            except pa.PagedAttnError as e:
                assert st_o == oracle.OOM and e.status == pa.PA_ERR_OOM
            nxt += 1
        elif r < 0.55:
            s = int(rng.choice(sorted(live)))
            if rng.random() < 0.8:
                ids = np.array(rng.integers(0, 4, size=int(rng.integers(1, bs + 2))), np.int32)
                st_o, slots_o, cow_o, cached_o = o.alloc_tokens(s, ids)
                try:
                    slots_p, cow_p, cached_p = p.pa_alloc_tokens(s, ids)
                    assert st_o == oracle.OK and cached_p == cached_o == 0
                    assert np.array_equal(slots_p, slots_o) and np.array_equal(cow_p, cow_o)
                except pa.PagedAttnError as e:
                    assert st_o == oracle.OOM and e.status == pa.PA_ERR_OOM
            elif o.num_free() >= 2 * 3:  # growth without ids: a batch that fits
                ids_b = sorted(live)[: int(rng.integers(1, 4))]
                exp = []
                for sid in ids_b:
                    exp.append(o.alloc(sid, 1))
                try:
                    slots_p, cow_p = p.pa_alloc_batch(ids_b, 1)
                    assert all(e[0] == oracle.OK for e in exp)
                    assert np.array_equal(slots_p, np.concatenate([e[1] for e in exp]))
                except pa.PagedAttnError as e:  # cannot happen: at most 2 blocks each
                    raise AssertionError(f"batch failed: {e}")
        elif r < 0.65:
            par = int(rng.choice(sorted(live)))
            assert o.fork(par, nxt) == oracle.OK
            p.pa_fork(par, nxt)
            live.add(nxt)
            nxt += 1
        elif r < 0.72 and live:
            s = int(rng.choice(sorted(live)))
            st_o, pairs_o = oracle.swap(o, ho, s)
            try:
                pairs_p = pa.pa_swap(p, hp, s)
                assert st_o == oracle.OK and np.array_equal(pairs_p, pairs_o)
                live.discard(s)
                away.add(s)
            except pa.PagedAttnError as e:
                assert st_o == oracle.OOM and e.status == pa.PA_ERR_OOM
        elif r < 0.75 and away:
            s = int(rng.choice(sorted(away)))
            st_o, pairs_o = oracle.swap(ho, o, s)
            try:
                pairs_p = pa.pa_swap(hp, p, s)
                assert st_o == oracle.OK and np.array_equal(pairs_p, pairs_o)
                away.discard(s)
                live.add(s)
            except pa.PagedAttnError as e:
                assert st_o == oracle.OOM and e.status == pa.PA_ERR_OOM
        elif r < 0.76:
            on = bool(rng.random() < 0.7)
            p.pa_set_prefix_caching(on)
            o.set_prefix_caching(on)
        else:
            s = int(rng.choice(sorted(live)))
            assert o.free(s) == oracle.OK
            p.pa_free(s)
            live.discard(s)
        _prefix_state(p, o, nb, sorted(live))
        _prefix_state(hp, ho, nb, sorted(away))
    assert hits > 0
