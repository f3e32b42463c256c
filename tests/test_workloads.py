"""The seeded workloads replay cleanly on the oracle block manager (CPU only)."""
import numpy as np
import pytest

import workloads as W
from oracle.allocator import BlockManager


def replay(sc):
    bm = BlockManager(sc.num_blocks, sc.spec.block_size, sc.free_order.tolist())
    pairs_setup, pairs_step = [], []
    for ops, pairs in ((sc.setup_ops, pairs_setup), (sc.step_ops, pairs_step)):
        for op in ops:
            if op.kind == "add":
                bm.add(op.seq)
            elif op.kind == "fork":
                bm.fork(op.seq, op.arg)
            elif op.kind == "release":
                bm.release(op.seq)
            else:
                _, p = bm.append(op.seq, op.arg)
                pairs += p
    return bm, pairs_setup, pairs_step


@pytest.mark.parametrize("name", ["tiny", "opt13b", "llama13b_ps", "gqa70b", "long_prefix"])
def test_small_workloads_replay(name):
    sc = W.scenario(W.small(name))
    bm, _, pairs = replay(sc)
    tables, lens = bm.build_tables(sc.batch, sc.max_blocks)
    assert np.array_equal(lens, sc.context_lens)
    assert lens.max() == sc.max_context_len
    if name == "llama13b_ps":
        assert len(pairs) > 0            # the divergent appends copy shared prompt tails


@pytest.mark.parametrize("name", ["tiny", "opt13b", "llama13b_ps", "gqa70b", "long_prefix"])
def test_full_workloads_replay(name):
    spec = W.FULL[name]
    sc = W.scenario(spec)
    bm, _, pairs = replay(sc)
    tables, lens = bm.build_tables(sc.batch, sc.max_blocks)
    assert np.array_equal(lens, sc.context_lens)
    assert len(sc.batch) == spec.num_seqs
    if name == "opt13b":
        assert lens.min() >= 16 and lens.max() <= 2048 and 500 < np.median(lens) < 700
    if name == "gqa70b":
        assert lens.min() >= 256 and lens.max() <= 4096
    if name == "long_prefix":
        # every request reads the same physical prefix blocks
        npre = spec.prefix_len // spec.block_size
        assert (tables[:, :npre] == tables[0, :npre]).all()
        assert lens.min() >= spec.prefix_len + 1 and lens.max() <= spec.prefix_len + spec.suffix_hi
    if name == "llama13b_ps":
        assert len(pairs) > 0


def test_long_prefix_block_sizes():
    for bs in (8, 16, 32):
        sc = W.scenario(W.long_prefix(bs))
        bm, _, _ = replay(sc)
        t, l = bm.build_tables(sc.batch, sc.max_blocks)
        assert np.array_equal(l, sc.context_lens)
