"""Walk orders for the decode (`pkv_decode_options.seq_order`).

The decode's persistent grid cuts the stream of (sequence, head group, block) positions into equal
contiguous ranges, one per worker warp, and every warp walks its range at about the same pace. A
position at offset x inside its warp's range is therefore reached at about the same time as every
other position at offset x of any other range. Sequences that share blocks (a forked beam and its
parent: deepinsea.top "PagedAttention 内存管理深度解析", Copy-on-Write 机制) read those blocks twice;
in the natural order the two reads are tens to hundreds of microseconds apart and the second one
comes from HBM again.

`aligned_walk_order` places the members of each sharing group a whole number of warp ranges apart
in the walk, so that the same block of the same head group lands at the same offset of two ranges
and is read by two warps at about the same moment: the second read finds it in L2. The gap between
two members is filled with sequences that share nothing, chosen so that their block counts add up
exactly to the gap (a subset sum over the remaining ones). Measured in blocks of one sequence, a
warp range is sum(blocks) / workers long; the number of head groups scales every sequence's
positions alike and drops out.
"""
from __future__ import annotations

import math

import numpy as np


def _subset_exact(items, sizes, target: int):
    """Items (in the given order) whose sizes add up to exactly `target`, or None."""
    if target < 0:
        return None
    reach = {0: []}
    for it in items:
        sz = int(sizes[it])
        if sz > target:
            continue
        for s, chosen in list(reach.items()):
            t = s + sz
            if t <= target and t not in reach:
                reach[t] = chosen + [it]
        if target in reach:
            return reach[target]
    return reach.get(target)


def sharing_groups(block_tables: np.ndarray, context_lens: np.ndarray, block_size: int):
    """Sequences that start on the same physical block (forks of one parent), as lists of
    sequence indices with more than one member, in order of first appearance."""
    groups = {}
    for s in range(len(context_lens)):
        if int(context_lens[s]) > 0:
            groups.setdefault(int(block_tables[s, 0]), []).append(s)
    return [g for g in groups.values() if len(g) > 1]


def aligned_walk_order(block_tables: np.ndarray, context_lens: np.ndarray, block_size: int, num_workers: int,
                       max_ranges: int = 64, tolerance: float = 0.08):
    """int32 [S]: a permutation of the sequences for the decode's walk.

    Each group of `sharing_groups` keeps its first member where the walk reaches it; every other
    member is placed k warp ranges after it, with k the first count (from the smallest that fits)
    for which the gap is within `tolerance` of a range of a whole number of blocks and a subset of
    the not-yet-placed non-sharing sequences fills it exactly. A member for which no such k exists
    (up to `max_ranges` ranges later) follows directly. Returns (order, misalignment): the second
    is, per placed member, its distance from exact alignment in warp ranges (None where none was
    found).
    """
    context_lens = np.asarray(context_lens)
    S = len(context_lens)
    nblk = (context_lens.astype(np.int64) + block_size - 1) // block_size
    total = int(nblk.sum())
    if S == 0 or total == 0 or num_workers <= 0:
        return np.arange(S, dtype=np.int32), []
    rng_blocks = total / num_workers  # one warp range, in blocks of one sequence
    groups = sharing_groups(block_tables, context_lens, block_size)
    grouped = {s for g in groups for s in g}
    free = sorted((s for s in range(S) if s not in grouped), key=lambda s: (int(nblk[s]), s))
    order, misalign = [], []
    x = 0  # blocks placed so far
    for g in sorted(groups, key=lambda g: (-int(nblk[g[0]]), g[0])):
        p = x
        order.append(g[0])
        x += int(nblk[g[0]])
        for m in g[1:]:
            k0 = max(1, math.ceil((x - p) / rng_blocks))
            placed = False
            for k in range(k0, k0 + max_ranges):
                target = p + k * rng_blocks - x
                n = round(target)
                if abs(n - target) > tolerance * rng_blocks:
                    continue
                fill = _subset_exact(free, nblk, n)
                if fill is None:
                    continue
                for s in fill:
                    free.remove(s)
                order.extend(fill)
                x += sum(int(nblk[s]) for s in fill)
                misalign.append(((x - p) - k * rng_blocks) / rng_blocks)
                placed = True
                break
            if not placed:
                misalign.append(None)
            order.append(m)
            x += int(nblk[m])
    order.extend(free)
    out = np.asarray(order, dtype=np.int32)
    assert np.array_equal(np.sort(out), np.arange(S))
    return out, misalign
