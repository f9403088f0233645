"""Automatic prefix caching (host index from token blocks to physical blocks): hits, misses,
eviction of blocks only the cache holds, forked beams, and the shared-prefix layout of the GQA
workload built by the index itself. No GPU needed.

Source: yunthe.com "LLM推理显存优化KV Cache量化与PagedAttention实现详解", section "Prefix Caching与多轮
对话场景优化实践" (a new request looks up blocks holding its prefix and maps onto them on a hit) and
section "PagedAttention分页注意力机制与vLLM实现" (requests with the same prefix share physical blocks).
"""
import numpy as np
import pytest

BS = 16


@pytest.fixture(scope="module")
def pkv():
    from paged_block_quantized_b200 import build
    build.build()
    from paged_block_quantized_b200 import pkv as mod
    return mod


def _prefill(pc, tokens):
    """What a serving loop does for a new request: reuse the cached prefix, take fresh blocks for the
    rest, store, then register the request's whole blocks. Returns the request's block table."""
    hit = pc.match(tokens)
    need = -(-len(tokens) // BS) - len(hit)
    fresh = pc.alloc(need)
    table = hit + fresh
    pc.insert(tokens, table)
    return table, len(hit)


def test_hit_miss_and_chain(pkv):
    a = pkv.Allocator(32)
    pc = pkv.PrefixCache(a, BS)
    req1 = list(range(40))                     # 2 whole blocks + 8 tokens
    t1, hits = _prefill(pc, req1)
    assert hits == 0 and len(t1) == 3 and pc.size == 2
    assert [a.refcount(b) for b in t1] == [2, 2, 1]          # caller + cache on the whole blocks
    req2 = list(range(32)) + [900, 901]        # same two whole blocks, other tail
    t2, hits = _prefill(pc, req2)
    assert hits == 2 and t2[:2] == t1[:2] and t2[2] != t1[2]
    assert [a.refcount(b) for b in t1[:2]] == [3, 3]
    # the second block's content alone is not enough: its prefix differs
    req3 = [7] * 16 + list(range(16, 32))
    assert pc.match(req3) == []
    # one token different inside the first block: no hit at all
    req4 = list(range(15)) + [999] + list(range(16, 32))
    assert pc.match(req4) == []
    # partial blocks are never matched
    assert pc.match(list(range(15))) == []
    # a longer request than anything cached matches only what is cached
    got = pc.match(list(range(64)))
    assert got == t1[:2]
    a.release(got)
    pc.close()
    assert all(a.refcount(b) == 2 for b in t1[:2])           # the cache's references are gone


def test_eviction_least_recently_used_and_all_or_nothing(pkv):
    a = pkv.Allocator(8)
    pc = pkv.PrefixCache(a, BS)
    ta, _ = _prefill(pc, list(range(32)))      # blocks A0 A1
    tb, _ = _prefill(pc, list(range(100, 132)))  # blocks B0 B1
    assert a.num_free == 4 and pc.size == 4
    a.release(ta)                              # request A ends: its blocks stay cached
    assert pc.evictable == 2 and a.num_free == 4
    assert pc.match(list(range(32))) == ta     # a later request reuses them...
    a.release(ta)
    _ = pc.match(list(range(100, 132)))        # ...B is used more recently than A
    a.release(tb)
    a.release(tb)
    assert pc.evictable == 4
    # too many for free + evictable: refused without evicting anything
    assert pc.alloc(9, raise_on_error=False) is None and pc.size == 4 and a.num_free == 4
    # 5 blocks: one eviction, the least recently used whole-block chain head first (A0, whose
    # descendant A1 is dropped with it since it can no longer be reached)
    got = pc.alloc(5)
    assert len(got) == 5 and pc.size == 2
    assert pc.match(list(range(32))) == []
    assert pc.match(list(range(100, 132))) == tb


def test_forked_beam_shares_then_copies(pkv):
    """A beam fork shares the parent's blocks; the first write into the shared partial last block
    takes a private copy (copy-on-write); the cached whole blocks stay shared."""
    a = pkv.Allocator(16)
    pc = pkv.PrefixCache(a, BS)
    parent, _ = _prefill(pc, list(range(40)))  # 2 whole + 1 partial
    a.fork(parent)                             # the child shares all three
    assert [a.refcount(b) for b in parent] == [3, 3, 2]
    new_last = a.cow(parent[2])                # the child writes its next token
    child = parent[:2] + [new_last]
    assert new_last != parent[2] and a.refcount(parent[2]) == 1 and a.refcount(new_last) == 1
    # both continue; when the child's last block fills up it is registered under its own tokens
    child_tokens = list(range(40)) + [500 + i for i in range(8)]
    pc.insert(child_tokens, child)
    assert pc.size == 3 and pc.match(child_tokens) == child
    a.release(child)


def test_builds_the_shared_prefix_layout(pkv):
    """64 requests with one 1024-token system prompt and private continuations: the index alone
    gives every request the same 64 physical prefix blocks (one copy, referenced by all) and
    private blocks for the rest, the sharing structure of the GQA prefix workload."""
    from paged_block_quantized_b200 import workloads as W
    w = W.make("gqa_prefix", seed=0)
    n_pre = 64 * BS
    a = pkv.Allocator(w.num_blocks)
    pc = pkv.PrefixCache(a, BS)
    rng = np.random.default_rng(0)
    prompt = list(rng.integers(0, 32000, n_pre))
    tables = []
    for s in range(w.num_seqs):
        tokens = prompt + list(rng.integers(0, 32000, int(w.context_lens[s]) - n_pre))
        t, hits = _prefill(pc, tokens)
        assert hits == (0 if s == 0 else 64)
        tables.append(t)
    tables = np.array(tables)
    assert tables.shape == w.block_tables.shape
    assert (tables[:, :64] == tables[0, :64]).all()                       # one shared prefix
    assert np.unique(tables[:, 64:]).size == tables[:, 64:].size           # private blocks distinct
    assert set(tables[0, :64]).isdisjoint(set(tables[:, 64:].ravel()))
    # same structure as the workload's own tables (shared prefix columns, private rest)
    wt = w.block_tables
    assert (wt[:, :64] == wt[0, :64]).all() and np.unique(wt[:, 64:]).size == wt[:, 64:].size
    assert all(a.refcount(int(b)) == w.num_seqs + 1 for b in tables[0, :64])
