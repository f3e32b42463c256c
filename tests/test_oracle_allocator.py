"""Pins of the oracle block manager (CPU only).

The worked example of "4.2 PagedAttention의 접근" (hjr-study-book Day 3), the
rules of "3. vLLM: KV cache를 블록 단위로 관리하기" (blog.aqudi.me: a new block
only when the current one is full; shared prompt blocks copied only on
modification) and bookkeeping invariants that any correct block manager keeps,
checked on long random operation sequences.
"""
import os

import numpy as np
import pytest

from oracle.allocator import OOM, BlockManager, Invalid
from pa_testlib import read_golden


def test_worked_example_table():
    g = read_golden("block_table_example.txt")
    bs, L, table = g["block_size"][0], g["seq_len"][0], g["table"]
    NB = 12
    # free stack whose top three entries are 7, 2, 9 (popped in that order)
    rest = [b for b in range(NB) if b not in table]
    bm = BlockManager(NB, bs, rest + list(reversed(table)))
    bm.add(0)
    slots, pairs = bm.append(0, L)
    assert pairs == []
    assert bm.blocks_of(0) == table
    tables, lens = bm.build_tables([0], 4)
    assert tables.tolist() == [table + [-1]] and lens.tolist() == [L]
    assert slots[36] == 148 and slots[0] == 7 * 16 and slots[16] == 2 * 16
    # internal fragmentation confined to the last block: 16*3 - 37 = 11 free slots
    assert len(table) * bs - L == 11 and L - 2 * bs == g["last_block_tokens"][0]


def test_new_block_only_when_current_block_is_full():
    bm = BlockManager(8, 4)
    bm.add(1)
    counts = []
    for _ in range(9):
        bm.append(1, 1)
        counts.append(len(bm.blocks_of(1)))
    assert counts == [1, 1, 1, 1, 2, 2, 2, 2, 3]
    assert bm.num_free() == 5


def test_default_free_order_hands_out_block_zero_first():
    bm = BlockManager(5, 2)
    bm.add(0)
    bm.append(0, 5)
    assert bm.blocks_of(0) == [0, 1, 2]


def test_parallel_samples_share_then_copy_on_write():
    """Six samples of one prompt share its blocks; the first five to write into
    the shared partial block copy it, the last writes in place."""
    bs = 16
    bm = BlockManager(64, bs)
    bm.add(0)
    bm.append(0, 40)                          # blocks: 2 full + 1 partial (8 tokens)
    for c in range(1, 6):
        bm.fork(0, c)
    shared = bm.blocks_of(0)
    assert all(bm.refcount[b] == 6 for b in shared)
    n_pairs = []
    for s in range(6):
        slots, pairs = bm.append(s, 3)
        n_pairs.append(len(pairs))
        if pairs:
            assert pairs[0][0] == shared[2]
            assert bm.blocks_of(s)[:2] == shared[:2] and bm.blocks_of(s)[2] == pairs[0][1]
        assert slots == [bm.blocks_of(s)[2] * bs + 8 + i for i in range(3)]
    assert n_pairs == [1, 1, 1, 1, 1, 0]
    assert bm.refcount[shared[2]] == 1 and bm.refcount[shared[0]] == 6
    assert bm.blocks_of(5)[2] == shared[2]


def test_no_copy_when_prompt_fills_its_last_block():
    bm = BlockManager(16, 8)
    bm.add(0)
    bm.append(0, 16)
    bm.fork(0, 1)
    _, p0 = bm.append(0, 1)
    _, p1 = bm.append(1, 1)
    assert p0 == [] and p1 == []
    assert bm.blocks_of(0)[:2] == bm.blocks_of(1)[:2]
    assert bm.blocks_of(0)[2] != bm.blocks_of(1)[2]


def test_oom_is_all_or_nothing():
    bm = BlockManager(4, 4)
    bm.add(0)
    bm.append(0, 6)
    bm.fork(0, 1)
    state = (bm.free_stack(), list(bm.refcount), bm.blocks_of(1), bm.num_tokens(1))
    with pytest.raises(OOM):
        bm.append(1, 11)                      # needs a CoW copy + 3 new blocks, 2 free
    assert state == (bm.free_stack(), list(bm.refcount), bm.blocks_of(1), bm.num_tokens(1))
    bm.append(1, 6)                           # CoW + 1 new block fits exactly
    assert bm.num_free() == 0


def test_release_returns_unshared_blocks_in_logical_order():
    bm = BlockManager(10, 2)
    bm.add(0)
    bm.append(0, 3)                           # blocks 0, 1
    bm.fork(0, 1)
    bm.append(1, 3)                           # CoW of block 1 -> 2, new block 3
    bm.release(1)
    assert bm.free_stack()[-2:] == [2, 3]
    bm.release(0)
    assert bm.free_stack()[-2:] == [0, 1] and bm.num_free() == 10


def test_invalid_operations():
    bm = BlockManager(4, 4)
    bm.add(0)
    with pytest.raises(Invalid):
        bm.add(0)
    with pytest.raises(Invalid):
        bm.fork(7, 8)
    with pytest.raises(Invalid):
        bm.fork(0, 0)
    with pytest.raises(Invalid):
        bm.append(3, 1)
    with pytest.raises(Invalid):
        bm.append(0, -1)
    with pytest.raises(Invalid):
        bm.release(9)
    with pytest.raises(Invalid):
        BlockManager(3, 4, [0, 1, 1])
    bm.append(0, 9)
    with pytest.raises(Invalid):
        bm.build_tables([0], 2)


def _check_invariants(bm):
    NB = bm.num_blocks
    free = bm.free_stack()
    assert len(set(free)) == len(free)
    refs = np.zeros(NB, dtype=int)
    for sid, s in bm.seqs.items():
        assert len(s.blocks) == -(-s.num_tokens // bm.block_size)
        for b in s.blocks:
            refs[b] += 1
    assert refs.tolist() == bm.refcount
    used = {b for b in range(NB) if refs[b] > 0}
    assert used.isdisjoint(free) and len(used) + len(free) == NB


def test_random_operation_sequences_keep_invariants():
    rng = np.random.default_rng(int(os.environ.get("PA_TEST_SEED", "3")))
    for trial in range(30):
        NB, bs = int(rng.integers(4, 40)), int(rng.choice([1, 2, 4, 8, 16]))
        bm = BlockManager(NB, bs, rng.permutation(NB).tolist())
        next_id = 0
        for _ in range(200):
            live = list(bm.seqs)
            r = rng.random()
            try:
                if r < 0.2 or not live:
                    bm.add(next_id)
                    next_id += 1
                elif r < 0.35:
                    bm.fork(int(rng.choice(live)), next_id)
                    next_id += 1
                elif r < 0.85:
                    sid = int(rng.choice(live))
                    before = bm.blocks_of(sid)
                    T = bm.num_tokens(sid)
                    n = int(rng.integers(0, 3 * bs + 2))
                    slots, pairs = bm.append(sid, n)
                    after = bm.blocks_of(sid)
                    assert len(slots) == n and len(pairs) <= 1
                    # full blocks never change; the written tail block is private
                    assert after[: T // bs] == before[: T // bs]
                    for s_ in slots:
                        assert bm.refcount[s_ // bs] == 1
                    assert slots == [after[t // bs] * bs + t % bs for t in range(T, T + n)]
                else:
                    bm.release(int(rng.choice(live)))
            except OOM:
                pass
            _check_invariants(bm)
        for sid in list(bm.seqs):
            bm.release(sid)
        assert bm.num_free() == NB
