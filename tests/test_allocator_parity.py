"""The C++ block manager of libpagedkv.so agrees bit for bit with the oracle's
(block tables, context lengths, slots, copy-on-write pairs, reference counts,
free stack, OOM behaviour) on the worked example, the workloads and long
random operation sequences.  CPU only."""
import numpy as np
import pytest

import paged_kv_cache_443_b200 as pk
import workloads as W
from oracle.allocator import OOM, BlockManager, Invalid
from pa_testlib import read_golden


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_443_b200 import build
    build.build()


def same_state(a: pk.BlockAllocator, o: BlockManager, live):
    assert a.num_free() == o.num_free()
    assert a.free_stack() == o.free_stack()
    for b in range(o.num_blocks):
        assert a.refcount(b) == o.refcount[b]
    if live:
        mb = max(1, max(len(o.blocks_of(s)) for s in live))
        ta, la = a.build_tables(live, mb)
        to, lo = o.build_tables(live, mb)
        assert np.array_equal(ta, to) and np.array_equal(la, lo)


def test_worked_example():
    g = read_golden("block_table_example.txt")
    bs, L, table = g["block_size"][0], g["seq_len"][0], g["table"]
    order = [b for b in range(12) if b not in table] + list(reversed(table))
    a = pk.BlockAllocator(12, bs, order)
    a.add(5)
    slots, pairs = a.append(5, L)
    t, lens = a.build_tables([5], 3)
    assert t.tolist() == [table] and lens.tolist() == [L] and pairs == []
    assert slots[36] == 148


def test_errors_map_to_statuses():
    a = pk.BlockAllocator(4, 4)
    a.add(0)
    with pytest.raises(pk.PagedKVError):
        a.add(0)
    with pytest.raises(pk.PagedKVError):
        a.fork(3, 4)
    with pytest.raises(pk.PagedKVError):
        a.append(9, 1)
    with pytest.raises(pk.PagedKVError):
        a.release(9)
    a.append(0, 6)
    a.fork(0, 1)
    before = (a.free_stack(), a.num_tokens(1))
    with pytest.raises(pk.OutOfBlocks):
        a.append(1, 11)
    assert before == (a.free_stack(), a.num_tokens(1))
    with pytest.raises(pk.PagedKVError):
        pk.BlockAllocator(3, 4, [0, 1, 1])
    with pytest.raises(pk.PagedKVError):
        a.build_tables([0], 1)
    assert a.refcount(-1) == -1 and a.refcount(4) == -1


@pytest.mark.parametrize("seed", range(6))
def test_random_operation_sequences_match_oracle(seed):
    rng = np.random.default_rng(1000 + seed)
    for trial in range(8):
        NB, bs = int(rng.integers(3, 48)), int(rng.choice([1, 2, 8, 16, 32]))
        order = rng.permutation(NB).tolist() if rng.random() < 0.7 else None
        a = pk.BlockAllocator(NB, bs, order)
        o = BlockManager(NB, bs, order)
        next_id = 0
        for _ in range(150):
            live = sorted(o.seqs)
            r = rng.random()
            if r < 0.18 or not live:
                a.add(next_id)
                o.add(next_id)
                next_id += 1
            elif r < 0.33:
                p = int(rng.choice(live))
                a.fork(p, next_id)
                o.fork(p, next_id)
                next_id += 1
            elif r < 0.85:
                sid = int(rng.choice(live))
                n = int(rng.integers(0, 3 * bs + 3))
                try:
                    want = o.append(sid, n)
                except OOM:
                    with pytest.raises(pk.OutOfBlocks):
                        a.append(sid, n)
                else:
                    got = a.append(sid, n)
                    assert got[0] == want[0] and [tuple(x) for x in got[1]] == want[1]
            else:
                sid = int(rng.choice(live))
                a.release(sid)
                o.release(sid)
            same_state(a, o, sorted(o.seqs))


@pytest.mark.parametrize("name", ["tiny", "opt13b", "llama13b_ps", "gqa70b", "long_prefix"])
def test_workload_scripts_match_oracle(name):
    sc = W.scenario(W.small(name) if name != "tiny" else W.TINY)
    a = pk.BlockAllocator(sc.num_blocks, sc.spec.block_size, sc.free_order.tolist())
    o = BlockManager(sc.num_blocks, sc.spec.block_size, sc.free_order.tolist())
    for op in sc.setup_ops + sc.step_ops:
        if op.kind == "add":
            a.add(op.seq); o.add(op.seq)
        elif op.kind == "fork":
            a.fork(op.seq, op.arg); o.fork(op.seq, op.arg)
        elif op.kind == "release":
            a.release(op.seq); o.release(op.seq)
        else:
            ga, wo = a.append(op.seq, op.arg), o.append(op.seq, op.arg)
            assert ga[0] == wo[0] and [tuple(x) for x in ga[1]] == wo[1]
    ta, la = a.build_tables(sc.batch, sc.max_blocks)
    to, lo = o.build_tables(sc.batch, sc.max_blocks)
    assert np.array_equal(ta, to) and np.array_equal(la, lo)


@pytest.mark.parametrize("seed", range(4))
def test_random_moves_between_two_managers_match_oracle(seed):
    """A device pool and a host pool on each side; sequences grow, fork, free
    and move back and forth in random groups.  Copy pairs, tables, refcounts,
    free stacks and OOM outcomes equal on both sides after every operation."""
    rng = np.random.default_rng(2000 + seed)
    for trial in range(6):
        bs = int(rng.choice([1, 2, 4, 16]))
        sizes = [int(rng.integers(6, 40)), int(rng.integers(3, 30))]
        orders = [rng.permutation(n).tolist() for n in sizes]
        A = [pk.BlockAllocator(n, bs, o) for n, o in zip(sizes, orders)]
        O = [BlockManager(n, bs, o) for n, o in zip(sizes, orders)]
        next_id = 0
        for _ in range(120):
            side = int(rng.integers(0, 2))
            a, o = A[side], O[side]
            live = sorted(o.seqs)
            r = rng.random()
            if r < 0.15 or not live:
                a.add(next_id); o.add(next_id)
                next_id += 1
            elif r < 0.3:
                p = int(rng.choice(live))
                a.fork(p, next_id); o.fork(p, next_id)
                next_id += 1
            elif r < 0.6:
                sid = int(rng.choice(live))
                n = int(rng.integers(0, 2 * bs + 2))
                try:
                    want = o.append(sid, n)
                except OOM:
                    with pytest.raises(pk.OutOfBlocks):
                        a.append(sid, n)
                else:
                    got = a.append(sid, n)
                    assert got[0] == want[0] and [tuple(x) for x in got[1]] == want[1]
            elif r < 0.9:
                k = int(rng.integers(1, len(live) + 1))
                group = [int(x) for x in rng.choice(live, size=k, replace=False)]
                try:
                    want = o.move_to(O[1 - side], group)
                except OOM:
                    with pytest.raises(pk.OutOfBlocks):
                        a.move_to(A[1 - side], group)
                else:
                    got = a.move_to(A[1 - side], group)
                    assert [tuple(x) for x in got] == [tuple(x) for x in want]
            else:
                sid = int(rng.choice(live))
                a.release(sid); o.release(sid)
            for s_ in (0, 1):
                same_state(A[s_], O[s_], sorted(O[s_].seqs))


def test_move_errors_map_to_statuses():
    a, b = pk.BlockAllocator(8, 4), pk.BlockAllocator(2, 4)
    a.add(0)
    a.append(0, 9)
    snap = (a.free_stack(), b.free_stack())
    with pytest.raises(pk.OutOfBlocks):
        a.move_to(b, [0])
    for bad in ([0, 0], [7]):
        with pytest.raises(pk.PagedKVError):
            a.move_to(b, bad)
    with pytest.raises(pk.PagedKVError):
        a.move_to(a, [0])
    with pytest.raises(pk.PagedKVError):
        a.move_to(pk.BlockAllocator(8, 2), [0])
    c = pk.BlockAllocator(8, 4)
    with pytest.raises(pk.PagedKVError):   # capacity below the distinct blocks
        pk.pa_seq_move(a.h, c.h, [0], 2)
    assert snap == (a.free_stack(), b.free_stack()) and a.num_tokens(0) == 9
    assert a.move_to(b, []) == []


def same_prefix_state(a: pk.BlockAllocator, o: BlockManager, live):
    same_state(a, o, live)
    assert a.evictable() == o.evictable


@pytest.mark.parametrize("seed", range(5))
def test_random_prefix_cache_scripts_match_oracle(seed):
    """Requests drawn from a few prompts (so prefixes repeat), forks, appends,
    commits, releases and pool pressure (evictions): cached token counts,
    slots, copy pairs, tables, refcounts, free stack and evictable list equal
    on both sides after every operation."""
    rng = np.random.default_rng(3000 + seed)
    for trial in range(8):
        NB, bs = int(rng.integers(4, 40)), int(rng.choice([1, 2, 4, 16]))
        order = rng.permutation(NB).tolist()
        a, o = pk.BlockAllocator(NB, bs, order), BlockManager(NB, bs, order)
        if rng.random() < 0.9:
            a.enable_prefix_cache()
            o.enable_prefix_cache()
        prompts = [rng.integers(0, 3, size=int(rng.integers(1, 5 * bs + 2))).tolist()
                   for _ in range(4)]
        toks = {}
        next_id = 0
        for _ in range(150):
            live = sorted(o.seqs)
            r = rng.random()
            if r < 0.3 or not live:
                p = prompts[int(rng.integers(0, 4))] + \
                    rng.integers(0, 3, size=int(rng.integers(0, 3))).tolist()
                got_o = o.add_cached(next_id, p)
                assert a.add_cached(next_id, p) == got_o
                toks[next_id] = p[:got_o]
                try:
                    want = o.append(next_id, len(p) - got_o)
                except OOM:
                    with pytest.raises(pk.OutOfBlocks):
                        a.append(next_id, len(p) - got_o)
                else:
                    got = a.append(next_id, len(p) - got_o)
                    assert got[0] == want[0] and [tuple(x) for x in got[1]] == want[1]
                    toks[next_id] = p
                    a.commit(next_id, p)
                    o.commit(next_id, p)
                next_id += 1
            elif r < 0.4:
                q = int(rng.choice(live))
                a.fork(q, next_id)
                o.fork(q, next_id)
                toks[next_id] = list(toks[q])
                next_id += 1
            elif r < 0.7:
                sid = int(rng.choice(live))
                n = int(rng.integers(1, 2 * bs + 1))
                try:
                    want = o.append(sid, n)
                except OOM:
                    with pytest.raises(pk.OutOfBlocks):
                        a.append(sid, n)
                else:
                    got = a.append(sid, n)
                    assert got[0] == want[0] and [tuple(x) for x in got[1]] == want[1]
                    toks[sid] = toks[sid] + rng.integers(0, 3, size=n).tolist()
                    k = int(rng.integers(0, len(toks[sid]) + 1))     # commit a prefix of it
                    a.commit(sid, toks[sid][:k])
                    o.commit(sid, toks[sid][:k])
            else:
                sid = int(rng.choice(live))
                a.release(sid)
                o.release(sid)
            same_prefix_state(a, o, sorted(o.seqs))


def test_prefix_cache_errors_map_to_statuses():
    a = pk.BlockAllocator(8, 2)
    a.enable_prefix_cache()
    assert a.add_cached(0, [1, 2, 3]) == 0
    with pytest.raises(pk.PagedKVError):
        a.add_cached(0, [1])                      # exists
    with pytest.raises(pk.PagedKVError):
        a.commit(5, [1])                          # unknown
    with pytest.raises(pk.PagedKVError):
        a.commit(0, [1, 2, 3])                    # more tokens than it holds (0)
    a.append(0, 3)
    a.commit(0, [1, 2, 3])
    assert a.add_cached(1, [1, 2, 3, 4]) == 2 and a.evictable() == []
    a.release(0)
    a.release(1)
    assert len(a.evictable()) == 1 and a.num_free() == 8
