"""Pins for the oracle's FP8 E4M3 cache mode: the format's values and rounding (hand-worked codes,
and every code and a large random sample against torch's independent float8_e4m3fn type), one
hand-worked tile, the single-shot error bound, and the append rule's invariants.

Source: yunthe.com "LLM推理显存优化KV Cache量化与PagedAttention实现详解", section
"vLLM推理引擎部署与KV Cache量化配置实战" (the fp8 KV-cache mode stores E4M3 values). Reading taken for
what the page leaves open: one binary32 scale per (block, KV head) = absmax / 448, codes rounded to
nearest (ties to even) and saturated at +-448, x_hat = value(code) * scale; appended values fit
when |x / scale| <= 448, otherwise the tile is rebuilt as for INT8.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from _golden import read

E4M3 = oracle.FP8_E4M3


def torch_value(codes):
    """E4M3 values of code bytes through torch's own float8_e4m3fn type (float64)."""
    t = torch.from_numpy(np.asarray(codes, np.uint8).copy()).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def half_step(y):
    """Half the spacing of E4M3 values around |y| (the bound of nearest rounding in range)."""
    a = abs(y)
    if a < 2.0 ** -6:
        return 2.0 ** -10                       # subnormals: spacing 2^-9
    return 2.0 ** (math.floor(math.log2(a)) - 4)  # 3 mantissa bits: spacing 2^(e-3)


def test_hand_worked_codes_and_values():
    g = read("fp8_e4m3_example.txt")
    got = [oracle.fp8_e4m3_encode(x) for x in g["inputs"]]
    assert got == [int(c) for c in g["codes"]]
    assert [oracle.fp8_e4m3_decode(int(c)) for c in g["decode_codes"]] == list(g["decode_values"])
    assert math.isnan(oracle.fp8_e4m3_decode(0x7F)) and math.isnan(oracle.fp8_e4m3_decode(0xFF))
    assert oracle.fp8_e4m3_decode(0x80) == 0.0 and math.copysign(1, oracle.fp8_e4m3_decode(0x80)) < 0


def test_every_code_matches_torch_and_round_trips():
    codes = np.arange(256)
    ours = np.array([oracle.fp8_e4m3_decode(int(c)) for c in codes])
    ref = torch_value(codes)
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[ok], ref[ok])
    for c in codes[ok]:
        assert oracle.fp8_e4m3_encode(float(ours[c])) == c  # every finite code encodes back to itself
    assert (np.diff(ours[:127]) > 0).all()                    # codes 0..126 ascend


def test_rounding_matches_torch_in_range():
    rng = np.random.default_rng(0)
    n = 20000
    mag = np.exp2(rng.uniform(-12, 8.8, n)).astype(np.float32)
    x = np.where(rng.random(n) < 0.5, -mag, mag).astype(np.float32)
    x = x[np.abs(x) <= 448]
    # exact midpoints between neighbouring values (ties) and the values themselves
    vals = torch_value(np.arange(127))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, vals.astype(np.float32)])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.fp8_e4m3_encode(float(v)) for v in x], np.uint8)
    np.testing.assert_array_equal(ours, ref)


def test_saturation_beyond_448():
    for x in (448.0, 449.0, 463.9, 464.0, 480.0, 1e5, 3.0e38):
        assert oracle.fp8_e4m3_encode(x) == 0x7E
        assert oracle.fp8_e4m3_encode(-x) == 0xFE


def test_tile_worked_example():
    g = read("fp8_e4m3_example.txt")
    d = int(g["head_dim"])
    x = np.zeros((1, 1, d), np.float16)
    x[0, 0, :len(g["values"])] = g["values"]
    c = oracle.OracleCache.empty(2, 16, 1, d, E4M3, E4M3)
    assert oracle.store(c, x, x, np.array([0])) == 0
    assert c.k_scale[0, 0] == np.float32(g["scale"]) and c.v_scale[0, 0] == np.float32(g["scale"])
    n = len(g["tile_codes"])
    np.testing.assert_array_equal(c.k_codes[0, 0, 0, :n], g["tile_codes"])
    np.testing.assert_array_equal(c.v_codes[0, 0, 0, :n], g["tile_codes"])
    np.testing.assert_array_equal(c.k_codes[0, 0, 0, n:], 0)


def _check_bound(x, codes, s):
    xh = torch_value(codes.reshape(-1)).reshape(codes.shape) * float(s)
    y = x.astype(np.float64) / float(s)
    bound = np.vectorize(half_step)(y) * float(s) * (1 + 2.0 ** -20)  # + binary32 rounding of x / s
    assert (np.abs(xh - x) <= bound).all()


@pytest.mark.parametrize("bs,n", [(16, 16), (16, 3), (32, 32)])
def test_single_shot_error_bound_and_extremes(bs, n):
    rng = np.random.default_rng(bs + n)
    H, D = 3, 64
    k = (rng.standard_normal((n, H, D)) * np.exp2(rng.uniform(-6, 6, (1, H, 1)))).astype(np.float16)
    v = (rng.standard_normal((n, H, D)) * 3).astype(np.float16)
    c = oracle.OracleCache.empty(2, bs, H, D, E4M3, E4M3)
    assert oracle.store(c, k, v, np.arange(n)) == 0
    for h in range(H):
        for which, x, codes, s in (("k", k, c.k_codes, c.k_scale), ("v", v, c.v_codes, c.v_scale)):
            xs = x[:, h].astype(np.float32)
            m = np.abs(xs).max()
            assert s[0, h] == np.float32(m) / np.float32(448)
            _check_bound(xs, codes[0, h, :n], s[0, h])
            top = codes[0, h, :n][np.abs(xs) == m]
            assert set(int(t) & 0x7F for t in top) == {0x7E}     # the absmax element lands on 448


def test_zero_tile():
    c = oracle.OracleCache.empty(1, 16, 1, 16, E4M3, E4M3)
    x = np.zeros((2, 1, 16), np.float16)
    assert oracle.store(c, x, x, np.arange(2)) == 0
    assert c.k_scale[0, 0] == 0 and (c.k_codes[0, 0, :2] == 0).all()
    # appending non-zero values into a zero tile rebuilds it
    y = np.full((1, 1, 16), 2.0, np.float16)
    assert oracle.store(c, y, y, np.array([2])) == 0
    assert c.k_scale[0, 0] == np.float32(2.0) / np.float32(448)
    assert (c.k_codes[0, 0, 2] == 0x7E).all() and (c.k_codes[0, 0, :2] == 0).all()


def test_append_that_fits_equals_single_shot():
    rng = np.random.default_rng(5)
    bs, H, D, n0, n = 16, 2, 32, 5, 16
    k = rng.uniform(-1, 1, (n, H, D)).astype(np.float16)
    k[0, :, 0] = 4.0
    v = k[::-1].copy()
    v[0, :, 1] = -4.0
    one = oracle.OracleCache.empty(1, bs, H, D, E4M3, E4M3)
    assert oracle.store(one, k, v, np.arange(n)) == 0
    two = oracle.OracleCache.empty(1, bs, H, D, E4M3, E4M3)
    assert oracle.store(two, k[:n0], v[:n0], np.arange(n0)) == 0
    for t in range(n0, n):
        assert oracle.store(two, k[t:t + 1], v[t:t + 1], np.array([t])) == 0
    for a, b in ((one.k_codes, two.k_codes), (one.v_codes, two.v_codes), (one.k_scale, two.k_scale),
                 (one.v_scale, two.v_scale)):
        np.testing.assert_array_equal(a, b)


def test_append_rebuild_invariants():
    """Appended values beyond the stored range rebuild the tile: the new scale covers old and new
    values, new tokens meet the single-shot bound, old tokens move by at most an old plus a new
    half step; values just past 448 steps (that would merely saturate) rebuild too."""
    rng = np.random.default_rng(6)
    bs, H, D, n0 = 16, 1, 32, 6
    for grow in (1.04, 3.0, 100.0):
        k = rng.uniform(-1, 1, (n0 + 1, H, D)).astype(np.float16)
        k[0, 0, 0] = 2.0
        c = oracle.OracleCache.empty(1, bs, H, D, E4M3, E4M3)
        assert oracle.store(c, k[:n0], k[:n0], np.arange(n0)) == 0
        s_old = float(c.k_scale[0, 0])
        old = torch_value(c.k_codes[0, 0, :n0].reshape(-1)).reshape(n0, D) * s_old
        k[n0, 0, 5] = np.float16(2.0 * grow)
        assert oracle.store(c, k[n0:], k[n0:], np.array([n0])) == 0
        s = float(c.k_scale[0, 0])
        x_new = float(k[n0, 0, 5])
        assert np.float32(s) == np.float32(max(np.float32(np.abs(old).max()), np.float32(x_new))) / np.float32(448)
        _check_bound(k[n0, 0].astype(np.float32), c.k_codes[0, 0, n0], s)
        new_old = torch_value(c.k_codes[0, 0, :n0].reshape(-1)).reshape(n0, D) * s
        bound = np.vectorize(half_step)(old / s) * s * (1 + 2.0 ** -20)
        assert (np.abs(new_old - old) <= bound).all()
