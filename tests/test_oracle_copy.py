"""Pins for the oracle's block copy (copy-on-write): deepinsea.top "PagedAttention 内存管理深度解析",
section "Copy-on-Write 机制" (share blocks, copy only the block that diverges)."""
import numpy as np

import oracle


def test_copy_is_byte_identity_and_leaves_others():
    rng = np.random.default_rng(20)
    nb, bs, H, D = 6, 16, 2, 32
    c = oracle.OracleCache.empty(nb, bs, H, D, oracle.INT8_SYM, oracle.INT4_ASYM)
    x = rng.standard_normal((nb * bs, H, D)).astype(np.float16)
    oracle.store(c, x, x, np.arange(nb * bs))
    before = c.copy()
    assert oracle.copy_blocks(c, np.array([[1, 4], [2, 0]])) == 0
    for src, dst in ((1, 4), (2, 0)):
        for a in ("k_codes", "v_codes", "k_scale", "v_scale", "v_zp"):
            np.testing.assert_array_equal(getattr(c, a)[dst], getattr(before, a)[src])
    for b in (1, 2, 3, 5):
        for a in ("k_codes", "v_codes", "k_scale", "v_scale", "v_zp"):
            np.testing.assert_array_equal(getattr(c, a)[b], getattr(before, a)[b])


def test_copy_then_append_leaves_parent_unchanged():
    """After copy-on-write and an append into the child's copy, the parent's block is intact."""
    rng = np.random.default_rng(21)
    bs, H, D = 16, 1, 16
    c = oracle.OracleCache.empty(4, bs, H, D, oracle.INT8_SYM, oracle.INT4_ASYM)
    x = rng.standard_normal((5, H, D)).astype(np.float16)
    oracle.store(c, x, x, np.arange(5))
    parent = c.copy()
    oracle.copy_blocks(c, np.array([[0, 3]]))
    y = (rng.standard_normal((1, H, D)) * 10).astype(np.float16)  # forces a rebuild in the copy
    oracle.store(c, y, y, np.array([3 * bs + 5]))
    for a in ("k_codes", "v_codes", "k_scale", "v_scale", "v_zp"):
        np.testing.assert_array_equal(getattr(c, a)[0], getattr(parent, a)[0])
    assert c.k_scale[3, 0] != parent.k_scale[0, 0]


def test_bad_ids_are_skipped_and_reported():
    c = oracle.OracleCache.empty(2, 16, 1, 16, oracle.INT8_SYM, oracle.INT8_SYM, poison=0)
    before = c.copy()
    assert oracle.copy_blocks(c, np.array([[0, 2]])) == oracle.DEVERR_BLOCK_ID
    np.testing.assert_array_equal(c.k_codes, before.k_codes)
