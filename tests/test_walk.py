"""The aligned walk order (paged_block_quantized_b200.walk): a permutation of the batch in which the
members of every sharing group (sequences on the same first block: forks of one parent) sit a
whole number of worker ranges apart, within the stated tolerance, so that two warps reach each
shared block at about the same time. Host logic only."""
import numpy as np

from paged_block_quantized_b200 import workloads as W
from paged_block_quantized_b200.walk import aligned_walk_order, sharing_groups


def _positions(order, nblk):
    pos, x = {}, 0
    for s in order:
        pos[int(s)] = x
        x += int(nblk[s])
    return pos


def test_mixed_forks_are_aligned():
    w = W.make("mixed", seed=0)
    workers = 148 * 16
    order, mis = aligned_walk_order(w.block_tables, w.context_lens, w.block_size, workers)
    assert np.array_equal(np.sort(order), np.arange(w.num_seqs))
    nblk = (w.context_lens + w.block_size - 1) // w.block_size
    rng = nblk.sum() / workers
    pos = _positions(order, nblk)
    groups = sharing_groups(w.block_tables, w.context_lens, w.block_size)
    assert len(groups) == 16 and all(len(g) == 2 for g in groups)
    assert all(m is not None and abs(m) <= 0.08 for m in mis)
    for g in groups:
        # the distance from the first member to the other, in warp ranges, is a whole number (±8%)
        d = (pos[g[1]] - pos[g[0]]) / rng
        assert d >= 1 - 0.08 and abs(d - round(d)) <= 0.08
        # every shared block has the same offset in the two ranges (the members have equal lengths)
        assert nblk[g[0]] == nblk[g[1]]


def test_no_sharing_keeps_everything_and_small_cases():
    w = W.make("llama7b", seed=1)
    order, mis = aligned_walk_order(w.block_tables, w.context_lens, w.block_size, 2368)
    assert np.array_equal(np.sort(order), np.arange(w.num_seqs)) and mis == []
    # empty batch, no workers
    assert aligned_walk_order(np.zeros((0, 4), np.int32), np.zeros(0, np.int32), 16, 10)[0].size == 0
    o, _ = aligned_walk_order(w.block_tables, w.context_lens, w.block_size, 0)
    assert np.array_equal(o, np.arange(w.num_seqs))


def test_group_of_three_and_no_fillers():
    # three sequences on one first block and nothing to fill the gaps with: still a permutation,
    # the members that cannot be aligned follow directly (reported as None)
    bt = np.array([[5, 6, 7], [5, 8, 9], [5, 10, 11]], np.int32)
    lens = np.array([40, 40, 40], np.int32)
    order, mis = aligned_walk_order(bt, lens, 16, 4)
    assert sorted(order.tolist()) == [0, 1, 2]
    assert len(mis) == 2
    # deterministic
    assert np.array_equal(order, aligned_walk_order(bt, lens, 16, 4)[0])
