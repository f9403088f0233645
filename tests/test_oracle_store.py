"""Pins for the oracle's quantize + scatter (store): worked examples, the rounding error bound,
extremes and special cases of the formulas, scatter positions, and the append rule's invariants.

Formulas: tbr8.org "如何通过 PagedAttention 与分块量化结合..." §4 store_kv (scale = absmax/127) and
yunthe.com "LLM推理显存优化KV Cache量化与PagedAttention实现详解", section "KV Cache量化技术原理"
(Q(x) = clamp(round(x/scale + zp), 0, 2^bits-1), x_hat = (Q - zp) * scale).
"""
import numpy as np
import pytest

import oracle
from _golden import read

EPS = 2.0 ** -16  # allowance for the binary32 rounding of x/scale (and + zp) before rint


def unpack(packed):
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), np.int64)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


def dequant_rows(cache, which, block, head, rows):
    """x_hat of token rows of a tile, by the page's formula (float64)."""
    if which == "k":
        return cache.k_codes[block, head, rows].astype(np.float64) * float(cache.k_scale[block, head])
    if cache.v_dtype == oracle.INT8_SYM:
        return cache.v_codes[block, head, rows].astype(np.float64) * float(cache.v_scale[block, head])
    codes = unpack(cache.v_codes[block, head, rows])
    return (codes - float(cache.v_zp[block, head])) * float(cache.v_scale[block, head])


def one_tile_cache(d, v_dtype=oracle.INT8_SYM, bs=16, nb=2, heads=1):
    return oracle.OracleCache.empty(nb, bs, heads, d, oracle.INT8_SYM, v_dtype)


def test_int8_worked_example():
    g = read("int8_sym_example.txt")
    d = int(g["head_dim"])
    x = np.zeros((1, 1, d), np.float16)
    x[0, 0, :len(g["values"])] = g["values"]
    c = one_tile_cache(d)
    assert oracle.store(c, x, x, np.array([0])) == 0
    assert c.k_scale[0, 0] == np.float32(g["scale"])
    np.testing.assert_array_equal(c.k_codes[0, 0, 0, :len(g["codes"])], g["codes"])
    np.testing.assert_array_equal(c.k_codes[0, 0, 0, len(g["codes"]):], 0)


def test_int4_worked_example_and_packing():
    g = read("int4_asym_example.txt")
    d = int(g["head_dim"])
    x = np.zeros((1, 1, d), np.float16)
    x[0, 0, :len(g["values"])] = g["values"]
    c = one_tile_cache(d, oracle.INT4_ASYM)
    assert oracle.store(c, x, x, np.array([0])) == 0
    assert c.v_scale[0, 0] == np.float32(g["scale"])
    assert c.v_zp[0, 0] == g["zero_point"]
    codes = unpack(c.v_codes[0, 0, 0])
    np.testing.assert_array_equal(codes[:len(g["codes"])], g["codes"])
    np.testing.assert_array_equal(c.v_codes[0, 0, 0], np.array(g["packed_bytes"], np.uint8))


@pytest.mark.parametrize("v_dtype", [oracle.INT8_SYM, oracle.INT4_ASYM])
@pytest.mark.parametrize("bs,n", [(16, 16), (16, 5), (32, 32), (32, 1)])
def test_single_shot_error_bound_and_extremes(v_dtype, bs, n):
    """|x - x_hat| <= scale * (1/2 + eps) for every element quantized in one shot; the absmax
    element maps to +-127; INT4 codes span [0, 15] with the extremes at lo / hi."""
    rng = np.random.default_rng(5)
    H, D = 3, 64
    c = oracle.OracleCache.empty(4, bs, H, D, oracle.INT8_SYM, v_dtype)
    k = (rng.standard_normal((n, H, D)) * rng.uniform(0.1, 10, size=(1, H, 1))).astype(np.float16)
    v = (rng.standard_normal((n, H, D)) * 3 + 0.5).astype(np.float16)
    slots = 2 * bs + np.arange(n)
    assert oracle.store(c, k, v, slots) == 0
    for h in range(H):
        xk = k[:, h].astype(np.float64)
        s = float(c.k_scale[2, h])
        assert np.float32(s) == np.float32(np.float32(np.abs(xk).max()) / np.float32(127))
        err = np.abs(dequant_rows(c, "k", 2, h, slice(0, n)) - xk)
        assert err.max() <= s * (0.5 + EPS)
        codes = c.k_codes[2, h, :n].astype(np.int64)
        assert np.abs(codes).max() == 127
        assert codes.min() >= -127
        xv = v[:, h].astype(np.float64)
        sv = float(c.v_scale[2, h])
        err = np.abs(dequant_rows(c, "v", 2, h, slice(0, n)) - xv)
        assert err.max() <= sv * (0.5 + EPS)
        if v_dtype == oracle.INT4_ASYM:
            vc = unpack(c.v_codes[2, h, :n])
            lo, hi = min(0.0, xv.min()), max(0.0, xv.max())
            assert np.float32(sv) == np.float32(np.float32(hi) - np.float32(lo)) / np.float32(15)
            assert vc.min() >= 0 and vc.max() <= 15
            assert vc[xv == xv.max()].max() == 15 or hi == 0
            assert vc[xv == xv.min()].min() <= 1  # lo maps to 0 up to the zp rounding


def test_zero_tile_and_constant_tile():
    D = 32
    c = one_tile_cache(D, oracle.INT4_ASYM)
    z = np.zeros((3, 1, D), np.float16)
    assert oracle.store(c, z, z, np.arange(3)) == 0
    assert c.k_scale[0, 0] == 0 and c.v_scale[0, 0] == 0 and c.v_zp[0, 0] == 0
    np.testing.assert_array_equal(c.k_codes[0, 0, :3], 0)
    np.testing.assert_array_equal(c.v_codes[0, 0, :3], 0)
    # a constant positive tile c: lo = 0, hi = c, scale = c/15, zp = 0, every code 15
    const = np.full((2, 1, D), 0.75, np.float16)
    assert oracle.store(c, const, const, 16 + np.arange(2)) == 0
    assert c.v_scale[1, 0] == np.float32(0.75) / np.float32(15) and c.v_zp[1, 0] == 0
    np.testing.assert_array_equal(unpack(c.v_codes[1, 0, :2]), 15)
    # K: constant tile -> every code 127
    np.testing.assert_array_equal(c.k_codes[1, 0, :2], 127)


def test_negative_constant_tile_int4():
    """All values equal to -c < 0: lo = -c, hi = 0 -> scale c/15, zp = 15, codes 0."""
    D = 16
    c = one_tile_cache(D, oracle.INT4_ASYM)
    x = np.full((1, 1, D), -3.0, np.float16)
    assert oracle.store(c, x, x, np.array([0])) == 0
    assert c.v_zp[0, 0] == 15
    np.testing.assert_array_equal(unpack(c.v_codes[0, 0, :1]), 0)


def test_scatter_positions_and_untouched_bytes():
    """Every token lands in the row its slot names; every other byte keeps the poison value."""
    rng = np.random.default_rng(1)
    nb, bs, H, D = 8, 16, 2, 32
    c = oracle.OracleCache.empty(nb, bs, H, D, oracle.INT8_SYM, oracle.INT4_ASYM)
    before = c.copy()
    # three groups: block 5 offsets 0..3, block 1 offsets 0..15 (full), block 6 offset 0; plus skips
    slots = np.concatenate([5 * bs + np.arange(4), [-1], 1 * bs + np.arange(16), [-7], [6 * bs]])
    T = slots.size
    k = rng.standard_normal((T, H, D)).astype(np.float16)
    v = rng.standard_normal((T, H, D)).astype(np.float16)
    assert oracle.store(c, k, v, slots) == 0
    written = np.zeros((nb, bs), bool)
    for t, sl in enumerate(slots):
        if sl < 0:
            continue
        b, o = divmod(int(sl), bs)
        written[b, o] = True
        for h in range(H):
            xk = k[t, h].astype(np.float64)
            assert np.abs(dequant_rows(c, "k", b, h, o) - xk).max() <= c.k_scale[b, h] * (0.5 + EPS)
            xv = v[t, h].astype(np.float64)
            assert np.abs(dequant_rows(c, "v", b, h, o) - xv).max() <= c.v_scale[b, h] * (0.5 + EPS)
    for b in range(nb):
        for o in range(bs):
            if not written[b, o]:
                np.testing.assert_array_equal(c.k_codes[b, :, o], before.k_codes[b, :, o])
                np.testing.assert_array_equal(c.v_codes[b, :, o], before.v_codes[b, :, o])
        if not written[b].any():
            np.testing.assert_array_equal(c.k_scale[b], before.k_scale[b])
            np.testing.assert_array_equal(c.v_zp[b], before.v_zp[b])


def test_fp16_side_is_stored_verbatim():
    rng = np.random.default_rng(2)
    c = oracle.OracleCache.empty(4, 16, 2, 16, oracle.FP16, oracle.FP16)
    k = rng.standard_normal((5, 2, 16)).astype(np.float16)
    v = rng.standard_normal((5, 2, 16)).astype(np.float16)
    assert oracle.store(c, k, v, 3 * 16 + 4 + np.arange(5)) == 0
    np.testing.assert_array_equal(c.k_codes[3, :, 4:9].transpose(1, 0, 2), k.view(np.uint16))
    np.testing.assert_array_equal(c.v_codes[3, :, 4:9].transpose(1, 0, 2), v.view(np.uint16))


def test_malformed_slots_report_errors():
    c = one_tile_cache(16)
    x = np.ones((2, 1, 16), np.float16)
    assert oracle.store(c, x[:1], x[:1], np.array([2 * 16])) == oracle.DEVERR_SLOT  # pool has 2 blocks
    assert oracle.store(c, x, x, np.array([3, 5])) == oracle.DEVERR_SLOT_GROUP      # gap in a group
    assert oracle.store(c, x, x, np.array([-1, -1])) == 0


# ---- append into a partly filled tile (fit-or-rebuild reading; the pages only store whole blocks)


@pytest.mark.parametrize("v_dtype", [oracle.INT8_SYM, oracle.INT4_ASYM])
def test_append_that_fits_equals_single_shot(v_dtype):
    """When the first tokens already hold the tile's extremes, storing them first and appending
    the rest gives exactly the single-shot result."""
    rng = np.random.default_rng(3)
    bs, H, D = 16, 2, 32
    n0, n = 6, 16
    k = rng.uniform(-1, 1, (n, H, D)).astype(np.float16)
    v = rng.uniform(-1, 1, (n, H, D)).astype(np.float16)
    k[0, :, 0], k[1, :, 1] = 4.0, -4.0     # absmax in the first part
    v[0, :, 0], v[1, :, 1] = 4.0, -2.0     # min and max in the first part
    one = oracle.OracleCache.empty(2, bs, H, D, oracle.INT8_SYM, v_dtype)
    assert oracle.store(one, k, v, np.arange(n)) == 0
    two = oracle.OracleCache.empty(2, bs, H, D, oracle.INT8_SYM, v_dtype)
    assert oracle.store(two, k[:n0], v[:n0], np.arange(n0)) == 0
    for t in range(n0, n):  # token-by-token appends, as decode does
        assert oracle.store(two, k[t:t + 1], v[t:t + 1], np.array([t])) == 0
    np.testing.assert_array_equal(one.k_codes[0], two.k_codes[0])
    np.testing.assert_array_equal(one.v_codes[0], two.v_codes[0])
    np.testing.assert_array_equal(one.k_scale[0], two.k_scale[0])
    np.testing.assert_array_equal(one.v_scale[0], two.v_scale[0])
    if v_dtype == oracle.INT4_ASYM:
        np.testing.assert_array_equal(one.v_zp[0], two.v_zp[0])


@pytest.mark.parametrize("v_dtype", [oracle.INT8_SYM, oracle.INT4_ASYM])
def test_append_rebuild_invariants(v_dtype):
    """A new value outside the stored range rebuilds the tile: the new scale covers old and new
    values, every code stays in range, new tokens meet the single-shot bound and old tokens
    drift by at most half an old step plus half a new step."""
    rng = np.random.default_rng(4)
    bs, H, D = 16, 2, 32
    n0 = 7
    k = rng.uniform(-1, 1, (n0 + 1, H, D)).astype(np.float16)
    v = rng.uniform(-1, 1, (n0 + 1, H, D)).astype(np.float16)
    k[n0, :, 3] = 9.0
    v[n0, :, 3] = -9.0
    c = oracle.OracleCache.empty(2, bs, H, D, oracle.INT8_SYM, v_dtype)
    assert oracle.store(c, k[:n0], v[:n0], np.arange(n0)) == 0
    s_old_k, s_old_v = c.k_scale[0].copy(), c.v_scale[0].copy()
    old_k = [dequant_rows(c, "k", 0, h, slice(0, n0)) for h in range(H)]
    old_v = [dequant_rows(c, "v", 0, h, slice(0, n0)) for h in range(H)]
    assert oracle.store(c, k[n0:], v[n0:], np.array([n0])) == 0
    for h in range(H):
        s = float(c.k_scale[0, h])
        assert s > s_old_k[h]
        assert np.float32(s) == np.float32(max(np.float32(np.abs(old_k[h]).max()), np.float32(9.0))) / np.float32(127)
        codes = c.k_codes[0, h, :n0 + 1].astype(np.int64)
        assert np.abs(codes).max() <= 127
        new = dequant_rows(c, "k", 0, h, slice(0, n0 + 1))
        assert np.abs(new[n0] - k[n0, h]).max() <= s * (0.5 + EPS)
        assert np.abs(new[:n0] - old_k[h]).max() <= s * (0.5 + EPS)
        assert np.abs(new[:n0] - k[:n0, h]).max() <= (s + s_old_k[h]) * (0.5 + EPS)
        sv = float(c.v_scale[0, h])
        assert sv > s_old_v[h]
        newv = dequant_rows(c, "v", 0, h, slice(0, n0 + 1))
        assert np.abs(newv[n0] - v[n0, h]).max() <= sv * (0.5 + EPS)
        assert np.abs(newv[:n0] - v[:n0, h]).max() <= (sv + s_old_v[h]) * (0.5 + EPS)
        if v_dtype == oracle.INT4_ASYM:
            vc = unpack(c.v_codes[0, h, :n0 + 1])
            assert vc.min() >= 0 and vc.max() <= 15


def test_append_sequence_never_leaves_range():
    rng = np.random.default_rng(6)
    bs, H, D = 16, 1, 16
    c = oracle.OracleCache.empty(1, bs, H, D, oracle.INT8_SYM, oracle.INT4_ASYM)
    for t in range(bs):
        scale = 10.0 ** rng.uniform(-2, 2)
        k = (rng.standard_normal((1, H, D)) * scale).astype(np.float16)
        v = (rng.standard_normal((1, H, D)) * scale + rng.uniform(-5, 5)).astype(np.float16)
        assert oracle.store(c, k, v, np.array([t])) == 0
        kc = c.k_codes[0, 0, :t + 1].astype(np.int64)
        assert np.abs(kc).max() <= 127
        vc = unpack(c.v_codes[0, 0, :t + 1])
        assert vc.min() >= 0 and vc.max() <= 15
        # the newest token always meets the single-shot bound under the tile's current scale
        assert np.abs(dequant_rows(c, "k", 0, 0, t) - k[0, 0]).max() <= c.k_scale[0, 0] * (0.5 + EPS)
        assert np.abs(dequant_rows(c, "v", 0, 0, t) - v[0, 0]).max() <= c.v_scale[0, 0] * (0.5 + EPS)
