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
    ev = list(bm.evictable)
    assert len(set(ev)) == len(ev) and set(ev).isdisjoint(free) and used.isdisjoint(ev)
    assert used.isdisjoint(free) and len(used) + len(free) + len(ev) == NB
    # every evictable block is cached; cached blocks and keys pair up one to one
    assert all(b in bm.key_of_block for b in ev)
    assert all(bm.block_of_key[k] == b for b, k in bm.key_of_block.items())
    assert len(bm.block_of_key) == len(bm.key_of_block)


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


# ---------------------------------------------------------------------------
# moving sequences to a second manager (swap to host memory and back)


def _sharing(bm, seqs):
    """Which (sequence, logical block) positions hold the same physical block:
    the equivalence classes, independent of the ids themselves."""
    first = {}
    out = []
    for sid in seqs:
        row = []
        for blk in bm.blocks_of(sid):
            row.append(first.setdefault(blk, len(first)))
        out.append(row)
    return out


def test_move_keeps_sharing_among_moved_sequences():
    bs = 4
    dev = BlockManager(32, bs)
    host = BlockManager(16, bs)
    dev.add(0)
    dev.append(0, 10)                      # 2 full + 1 partial block
    for c in (1, 2, 3):
        dev.fork(0, c)
    dev.append(1, 1)                       # copy-on-write of the partial block
    free_before = dev.num_free()
    pattern = _sharing(dev, [1, 2, 3])
    pairs = dev.move_to(host, [1, 2, 3])
    # distinct blocks of 1, 2, 3: the two full prompt blocks, the shared partial
    # block (held by 0, 2, 3) and 1's private copy
    assert len(pairs) == 4 and host.num_free() == 12
    assert _sharing(host, [1, 2, 3]) == pattern
    assert [host.num_tokens(s) for s in (1, 2, 3)] == [11, 10, 10]
    for blk in host.blocks_of(2):
        assert host.refcount[blk] == (3 if blk in host.blocks_of(1) else 2)
    # device: 1's private block freed; the prompt blocks now held by 0 alone
    assert dev.num_free() == free_before + 1
    assert all(dev.refcount[b] == 1 for b in dev.blocks_of(0))
    assert sorted(dev.seqs) == [0]
    # every pair copies a block one of the moved sequences held, into the block
    # that takes its place in the same logical position
    src_of = dict((d, s) for s, d in pairs)
    assert len(src_of) == len(pairs)


def test_move_there_and_back_restores_contents_and_sharing():
    """Track block contents as labels: after a round trip every sequence reads
    the same labels in logical order, and the sharing pattern is unchanged."""
    rng = np.random.default_rng(11)
    bs = 2
    dev = BlockManager(40, bs, rng.permutation(40).tolist())
    host = BlockManager(40, bs, rng.permutation(40).tolist())
    dev.add(0)
    dev.append(0, 7)
    dev.fork(0, 1)
    dev.fork(0, 2)
    dev.append(2, 3)
    dev.add(5)
    dev.append(5, 4)
    label_dev = {b: ("d", b) for b in range(40)}
    before = {s: [label_dev[b] for b in dev.blocks_of(s)] for s in (0, 1, 2, 5)}
    pattern = _sharing(dev, [1, 2, 5])
    out_pairs = dev.move_to(host, [1, 2, 5])
    label_host = {}
    for s_blk, d_blk in out_pairs:
        label_host[d_blk] = label_dev[s_blk]
    for s in (1, 2, 5):
        assert [label_host[b] for b in host.blocks_of(s)] == before[s]
    in_pairs = host.move_to(dev, [5, 2, 1])
    for s_blk, d_blk in in_pairs:
        label_dev[d_blk] = label_host[s_blk]
    for s in (0, 1, 2, 5):
        assert [label_dev[b] for b in dev.blocks_of(s)] == before[s]
    assert _sharing(dev, [1, 2, 5]) == pattern
    assert host.num_free() == 40 and not host.seqs
    _check_invariants(dev)
    _check_invariants(host)


def test_move_single_sample_takes_private_copies():
    dev = BlockManager(16, 4)
    host = BlockManager(16, 4)
    dev.add(0)
    dev.append(0, 8)
    dev.fork(0, 1)
    pairs = dev.move_to(host, [1])
    assert [s for s, _ in pairs] == dev.blocks_of(0)
    assert all(host.refcount[b] == 1 for b in host.blocks_of(1))
    assert all(dev.refcount[b] == 1 for b in dev.blocks_of(0))


def test_move_errors_change_nothing():
    dev = BlockManager(8, 4)
    host = BlockManager(2, 4)
    dev.add(0)
    dev.append(0, 9)                       # 3 blocks > 2 free in host
    snap = (dev.free_stack(), list(dev.refcount), host.free_stack())
    with pytest.raises(OOM):
        dev.move_to(host, [0])
    with pytest.raises(Invalid):
        dev.move_to(host, [0, 0])
    with pytest.raises(Invalid):
        dev.move_to(host, [7])
    with pytest.raises(Invalid):
        dev.move_to(dev, [0])
    with pytest.raises(Invalid):
        dev.move_to(BlockManager(8, 2), [0])
    host.add(0)
    with pytest.raises(Invalid):
        dev.move_to(host, [0])
    assert snap == (dev.free_stack(), list(dev.refcount), host.free_stack())
    assert dev.num_tokens(0) == 9



# ---------------------------------------------------------------------------
# prefix caching: reuse of a repeated prompt prefix's blocks


def _prompt(*parts):
    return [t for p in parts for t in p]


SYS = list(range(100, 110))        # a 10-token system prompt


def test_repeated_prompt_prefix_reuses_full_blocks():
    bm = BlockManager(32, 4)
    bm.enable_prefix_cache()
    a = _prompt(SYS, [1, 2, 3, 4, 5])
    assert bm.add_cached(0, a) == 0
    bm.append(0, len(a))
    bm.commit(0, a)
    b = _prompt(SYS, [7, 8, 9, 9, 9, 9, 9])
    assert bm.add_cached(1, b) == 8            # blocks 0, 1 hit; block 2 mixes in user tokens
    assert bm.blocks_of(1) == bm.blocks_of(0)[:2]
    assert [bm.refcount[x] for x in bm.blocks_of(0)] == [2, 2, 1, 1]
    slots, pairs = bm.append(1, len(b) - 8)
    assert pairs == [] and bm.num_tokens(1) == len(b)
    assert bm.blocks_of(1)[2] not in bm.blocks_of(0)
    _check_invariants(bm)


def test_lookup_follows_the_content_chain_and_leaves_one_token():
    bm = BlockManager(32, 4)
    bm.enable_prefix_cache()
    a = list(range(12))                         # exactly three full blocks
    bm.add_cached(0, a)
    bm.append(0, 12)
    bm.commit(0, a)
    # same second block after a different first block: no hit (keys chain)
    assert bm.add_cached(1, [99, 1, 2, 3] + a[4:]) == 0
    # the very same prompt: two blocks, the last one is computed again
    assert bm.add_cached(2, a) == 8
    # a longer prompt with the same 12 tokens: all three
    assert bm.add_cached(3, a + [50]) == 12
    assert bm.add_cached(4, []) == 0 and bm.add_cached(5, a[:4]) == 0
    _check_invariants(bm)


def test_released_cached_blocks_wait_evictable_and_come_back():
    bm = BlockManager(8, 4, list(range(7, -1, -1)))   # block 0 handed out first
    bm.enable_prefix_cache()
    a = _prompt(SYS, [1, 2])                    # 12 tokens: 3 full blocks
    bm.add_cached(0, a)
    bm.append(0, 12)
    bm.commit(0, a)
    bm.append(0, 1)                             # a 4th, partial block (uncommitted)
    blocks = bm.blocks_of(0)
    bm.release(0)
    assert bm.evictable == blocks[:3]           # logical order, oldest first
    assert bm.free_stack()[-1] == blocks[3]
    assert bm.num_free() == 8
    assert bm.add_cached(1, a + [5]) == 12      # taken back from the evictable list
    assert bm.blocks_of(1) == blocks[:3] and bm.evictable == []
    _check_invariants(bm)


def test_eviction_takes_free_blocks_first_then_least_recently_released():
    bm = BlockManager(6, 2)
    bm.enable_prefix_cache()
    p1, p2 = [1, 1, 2, 2, 3], [4, 4, 5, 5, 6]
    for sid, p in ((0, p1), (1, p2)):
        bm.add_cached(sid, p)
        bm.append(sid, len(p))
        bm.commit(sid, p)
    bm.release(0)
    bm.release(1)
    b1, b2 = bm.evictable[:2], bm.evictable[2:]
    assert len(b1) == 2 and len(b2) == 2 and len(bm.free) == 2
    bm.add(7)
    bm.append(7, 4)                             # the two free blocks, no eviction
    assert bm.evictable == b1 + b2
    bm.append(7, 2)                             # evicts p1's first block
    assert bm.evictable == b1[1:] + b2 and bm.blocks_of(7)[-1] == b1[0]
    assert bm.add_cached(8, p1 + [9]) == 0       # p1's chain starts with a miss now
    assert bm.add_cached(9, p2 + [9]) == 4
    _check_invariants(bm)


def test_first_committed_block_wins_a_key():
    bm = BlockManager(16, 2)
    bm.enable_prefix_cache()
    p = [3, 3, 4, 4, 5]
    for sid in (0, 1):                          # both miss: computed twice
        assert bm.add_cached(sid, p) == 0
        bm.append(sid, len(p))
    bm.commit(0, p)
    bm.commit(1, p)
    assert bm.add_cached(2, p) == 4 and bm.blocks_of(2) == bm.blocks_of(0)[:2]
    bm.release(1)                               # 1's full blocks were never cached
    assert bm.evictable == [] and len(bm.free) == 16 - 3 - 3 + 3
    _check_invariants(bm)


def test_prefix_cache_off_is_plain_allocation():
    bm = BlockManager(8, 2)
    assert bm.add_cached(0, [1, 2, 3]) == 0
    bm.append(0, 3)
    bm.commit(0, [1, 2, 3])
    assert bm.add_cached(1, [1, 2, 3]) == 0 and not bm.block_of_key
    with pytest.raises(Invalid):
        bm.commit(0, [1, 2, 3, 4])
    with pytest.raises(Invalid):
        bm.add_cached(0, [1])


def test_random_prefix_cache_sequences_keep_invariants():
    rng = np.random.default_rng(17)
    for trial in range(20):
        NB, bs = int(rng.integers(4, 30)), int(rng.choice([1, 2, 4]))
        bm = BlockManager(NB, bs, rng.permutation(NB).tolist())
        bm.enable_prefix_cache()
        prompts = [rng.integers(0, 3, size=int(rng.integers(1, 4 * bs + 2))).tolist() for _ in range(4)]
        toks = {}
        next_id = 0
        for _ in range(150):
            live = sorted(bm.seqs)
            r = rng.random()
            try:
                if r < 0.3 or not live:
                    p = prompts[int(rng.integers(0, 4))] + rng.integers(0, 3, size=int(rng.integers(0, 3))).tolist()
                    got = bm.add_cached(next_id, p)
                    assert got % bs == 0 and got < max(1, len(p))
                    toks[next_id] = p[:got]
                    try:
                        bm.append(next_id, len(p) - got)
                        toks[next_id] = p
                        bm.commit(next_id, p)
                    except OOM:
                        pass
                    next_id += 1
                elif r < 0.4:
                    q = int(rng.choice(live))
                    bm.fork(q, next_id)
                    toks[next_id] = list(toks[q])
                    next_id += 1
                elif r < 0.7:
                    sid = int(rng.choice(live))
                    n = int(rng.integers(1, 2 * bs + 1))
                    bm.append(sid, n)
                    toks[sid] = toks[sid] + rng.integers(0, 3, size=n).tolist()
                    bm.commit(sid, toks[sid])
                else:
                    bm.release(int(rng.choice(live)))
            except OOM:
                pass
            _check_invariants(bm)
            # a cached block's key is the content chain of the tokens it holds for
            # every live sequence that uses it in that logical position
            for sid, s in bm.seqs.items():
                key = None
                for k, blk in enumerate(s.blocks[: len(toks[sid]) // bs]):
                    key = (key, tuple(toks[sid][k * bs:(k + 1) * bs]))
                    if blk in bm.key_of_block:
                        assert bm.key_of_block[blk] == key
