"""Host block allocator (C ABI): the page's worked example, ceil-division sizing, all-or-nothing
out-of-blocks failure, reference counts, fork and copy-on-write. No GPU needed."""
import pytest

from _golden import read


@pytest.fixture(scope="module")
def pkv():
    from paged_block_quantized_b200 import build
    build.build()
    from paged_block_quantized_b200 import pkv as mod
    return mod


def test_worked_example(pkv):
    g = read("allocator_example.txt")
    n = pkv.pkv_blocks_for_tokens(int(g["num_tokens"]), int(g["block_size"]))
    assert n == g["blocks_needed"]
    a = pkv.Allocator(int(g["num_blocks"]))
    ids = a.alloc(n)
    assert len(set(ids)) == n
    assert a.num_free == g["free_after"]


def test_ceil_division(pkv):
    assert [pkv.pkv_blocks_for_tokens(t, 16) for t in (0, 1, 15, 16, 17, 32, 33)] == [0, 1, 1, 1, 2, 2, 3]
    assert pkv.pkv_blocks_for_tokens(-1, 16) == -1
    assert pkv.pkv_blocks_for_tokens(5, 0) == -1


def test_out_of_blocks_is_all_or_nothing(pkv):
    a = pkv.Allocator(5)
    assert a.alloc(3) is not None
    assert a.alloc(3, raise_on_error=False) is None
    assert a.num_free == 2
    with pytest.raises(pkv.PkvError) as e:
        a.alloc(3)
    assert e.value.status == pkv.PKV_ERR_OUT_OF_BLOCKS


def test_refcounts_fork_release(pkv):
    a = pkv.Allocator(4)
    ids = a.alloc(2)
    a.fork(ids)
    assert [a.refcount(i) for i in ids] == [2, 2]
    a.release(ids)
    assert a.num_free == 2 and [a.refcount(i) for i in ids] == [1, 1]
    a.release(ids)
    assert a.num_free == 4 and [a.refcount(i) for i in ids] == [0, 0]
    # double free and unknown ids are rejected without changing anything
    assert a.release(ids, raise_on_error=False) == pkv.PKV_ERR_INVALID_ARG
    assert a.release([9], raise_on_error=False) == pkv.PKV_ERR_INVALID_ARG
    x = a.alloc(1)
    assert a.release(x + x, raise_on_error=False) == pkv.PKV_ERR_INVALID_ARG
    assert a.refcount(x[0]) == 1
    assert a.fork([3 if x[0] != 3 else 2], raise_on_error=False) == pkv.PKV_ERR_INVALID_ARG
    assert a.refcount(99) == -1


def test_lifo_reuse(pkv):
    a = pkv.Allocator(8)
    first = a.alloc(3)
    assert first == [0, 1, 2]
    a.release([1])
    assert a.alloc(1) == [1]


def test_copy_on_write(pkv):
    a = pkv.Allocator(4)
    (b,) = a.alloc(1)
    assert a.cow(b) == b              # sole owner: write in place
    a.fork([b])
    nb = a.cow(b)                     # shared: a private copy for the writer
    assert nb != b and a.refcount(b) == 1 and a.refcount(nb) == 1
    a.alloc(2)
    a.fork([b])
    assert a.cow(b, raise_on_error=False) is None  # no free block for the copy
    assert a.refcount(b) == 2


def test_swap_bookkeeping(pkv):
    """A sequence swapped out and back in ([deepinsea] "Swap 机制") with one allocator per pool:
    host blocks are taken before the swap-out and the device blocks released after it; device
    blocks are taken before the swap-in and the host blocks released after it. A block shared with
    another sequence stays on the device until its last reference goes."""
    dev, host = pkv.Allocator(16), pkv.Allocator(8)
    seq_a = dev.alloc(5)
    seq_b = dev.alloc(3)
    dev.fork(seq_a[:2])                       # seq_b's beam shares seq_a's first two blocks
    # swap seq_a out: one host block per device block
    h = host.alloc(len(seq_a))
    mapping_out = list(zip(seq_a, h))
    assert len(mapping_out) == 5 and host.num_free == 3
    dev.release(seq_a)
    assert [dev.refcount(b) for b in seq_a] == [1, 1, 0, 0, 0]  # the shared two stay for the beam
    assert dev.num_free == 16 - 3 - 2
    # not enough host room for a second sequence of 5: all or nothing
    assert host.alloc(5, raise_on_error=False) is None and host.num_free == 3
    # swap seq_a back in under fresh device ids
    d = dev.alloc(len(h))
    mapping_in = list(zip(h, d))
    assert len(set(d) & set(seq_b)) == 0 and all(dev.refcount(b) == 1 for b in d)
    host.release(h)
    assert host.num_free == 8
    assert [src for src, _ in mapping_in] == [dst for _, dst in mapping_out]
