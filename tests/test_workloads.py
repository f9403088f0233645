"""Structure of the seeded synthetic workloads (shapes, block assignment, sharing, slots)."""
import numpy as np
import pytest

from paged_block_quantized_b200 import workloads as W


@pytest.mark.parametrize("name", W.CONFIGS + ("llama7b_fp16",))
def test_layout_is_consistent(name):
    w = W.make(name)
    bs = w.block_size
    assert w.context_lens.min() >= 1
    used = []
    for s in range(w.num_seqs):
        nblk = (int(w.context_lens[s]) + bs - 1) // bs
        row = w.block_tables[s, :nblk]
        assert (row >= 0).all() and (row < w.num_blocks).all()
        assert (w.block_tables[s, nblk:] == -1).all()
        used.extend(row.tolist())
    # a physical block is shared only where the workload says so (prefix or fork)
    counts = np.bincount(used, minlength=w.num_blocks)
    if name == "gqa_prefix":
        assert (counts == w.num_seqs).sum() == 64 and counts.max() == 64
    elif name == "mixed":
        assert w.cow_pairs.shape == (16, 2)
        assert len(set(w.cow_pairs[:, 1])) == 16
        assert counts.max() == 2
    else:
        assert counts.max() == 1
    # the step's slots land in each sequence's last block at offset (L-1) % bs
    slots = w.step_slots()
    for s in range(w.num_seqs):
        p = int(w.context_lens[s]) - 1
        assert slots[s] == w.block_tables[s, p // bs] * bs + p % bs


def test_named_sizes():
    assert list(W.make("tiny").context_lens) == [17, 33, 50, 64]
    w = W.make("llama7b")
    assert w.num_seqs == 32 and w.num_blocks == 8192 and 500 <= w.context_lens.min() and w.context_lens.max() <= 2000
    w = W.make("long")
    assert w.num_seqs == 8 and 8192 <= w.context_lens.min() and w.context_lens.max() <= 32768 and w.block_size == 32
    w = W.make("gqa_prefix")
    assert (w.num_q_heads, w.num_kv_heads, int(w.context_lens[0])) == (64, 8, 2048)
    w = W.make("mixed")
    assert w.num_seqs == 128 and 16 <= w.context_lens.min() and w.context_lens.max() <= 16384
    for src, dst in w.cow_pairs:
        parent = np.nonzero((w.block_tables == src).any(axis=1))[0]
        assert len(parent) == 1
        assert (w.context_lens[parent[0]] - 1) % 16 != 0  # the shared last block is partial


def test_values_are_deterministic_and_fp16():
    w = W.make("llama7b", seed=3, num_seqs=2)
    a = w.block_values(1, 5)
    b = W.make("llama7b", seed=3, num_seqs=2).block_values(1, 5)
    assert a[0].dtype == np.float16
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    # outlier channels: about 1% of channels scaled by 8
    k = np.concatenate([w.block_values(0, j)[0] for j in range(40)]).astype(np.float32)
    ch_std = k.reshape(-1, w.num_kv_heads * w.head_dim).std(axis=0)
    assert (ch_std > 4).sum() == round(0.01 * w.num_kv_heads * w.head_dim)


def test_prefill_covers_positions_once():
    w = W.make("mixed", num_seqs=20, children=3)
    seen = set()
    for k, v, slots in w.prefill_batches(max_tokens=100):
        assert k.shape == v.shape and k.shape[0] == slots.shape[0]
        for sl in slots.tolist():
            assert sl not in seen
            seen.add(sl)
    expected = set()
    for s in range(w.num_seqs):
        for p in range(int(w.context_lens[s]) - 1):
            expected.add(int(w.prefill_tables[s, p // w.block_size]) * w.block_size + p % w.block_size)
    assert seen == expected


def test_beam_order_and_prefix_groups():
    from paged_block_quantized_b200 import workloads as W
    w = W.make("mixed", seed=0, num_seqs=24, children=4)
    order = w.beam_walk_order()
    assert sorted(order) == list(range(24))
    for src, dst in w.cow_pairs:  # each child right after its parent
        child = int(np.nonzero((w.block_tables == dst).any(axis=1))[0][0])
        parent = int(np.nonzero((w.block_tables == src).any(axis=1))[0][0])
        assert list(order).index(child) == list(order).index(parent) + 1
    starts, members, shared = w.prefix_groups()
    assert len(starts) == 5 and (np.diff(starts) == 2).all()
    for g in range(4):
        a, b = members[starts[g]:starts[g + 1]]
        k = shared[a]
        assert k == shared[b] > 0
        assert (w.block_tables[a, :k] == w.block_tables[b, :k]).all()
        assert w.block_tables[a, k] != w.block_tables[b, k]
    g = W.make("gqa_prefix", seed=0, num_seqs=5, prefix_blocks=3, private_blocks=2)
    starts, members, shared = g.prefix_groups()
    assert list(starts) == [0, 5] and (shared == 3).all()
    assert W.make("llama7b", seed=0, num_seqs=4).prefix_groups() is None


def test_k_ramp_scales_keys_by_block():
    # the option that makes scores grow along the context: K of logical block j times 1 + r * j
    # (before the fp16 rounding), V untouched
    a = W.make("prefill", seed=3, num_seqs=1, chunk=8, prefix_lens=[100], num_q_heads=4, num_kv_heads=4)
    b = W.make("prefill", seed=3, num_seqs=1, chunk=8, prefix_lens=[100], num_q_heads=4, num_kv_heads=4, k_ramp=0.25)
    for j in (0, 3, 6):
        ka, va = a.block_values(a.block_streams[0, j], j)
        kb, vb = b.block_values(b.block_streams[0, j], j)
        np.testing.assert_array_equal(va, vb)
        if j == 0:
            np.testing.assert_array_equal(kb, ka)
        ratio = kb.astype(np.float64) / np.where(ka == 0, 1, ka).astype(np.float64)
        assert np.allclose(ratio[ka != 0], 1 + 0.25 * j, rtol=2e-3)
