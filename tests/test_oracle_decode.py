"""Pins for the oracle's decode attention: a library attention routine on the contiguous layout,
invariance under physical block permutation and prefix sharing, closed-form special cases,
agreement with the independent NumPy brute force, and error reporting.

Paged layout: tbr8.org "如何通过 PagedAttention 与分块量化结合..." §2 (blocks mapped by a block table,
non-contiguous in memory) and yunthe.com "LLM推理显存优化KV Cache量化与PagedAttention实现详解",
section "PagedAttention分页注意力机制与vLLM实现" (block_table[seq_id] = [physical ids]); contiguous
reference layout [batch, heads, seq_len, head_dim] from the same page's section "KV Cache量化技术原理".
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import brute

DTYPES = [(oracle.INT8_SYM, oracle.INT8_SYM), (oracle.INT8_SYM, oracle.INT4_ASYM), (oracle.FP16, oracle.FP16),
          (oracle.FP8_E4M3, oracle.FP8_E4M3)]


def unpack(packed):
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), np.int64)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


def filled_cache(rng, nb, bs, H, D, kd, vd, tables, lens):
    """Store random fp16 tokens for every sequence through the oracle (whole blocks, one shot)."""
    c = oracle.OracleCache.empty(nb, bs, H, D, kd, vd)
    S = len(lens)
    for s in range(S):
        L = int(lens[s])
        if L == 0:
            continue
        k = (rng.standard_normal((L, H, D)) * 1.5).astype(np.float16)
        v = (rng.standard_normal((L, H, D)) + 0.3).astype(np.float16)
        slots = tables[s, np.arange(L) // bs].astype(np.int64) * bs + np.arange(L) % bs
        assert oracle.store(c, k, v, slots) == 0
    return c


def page_dequant(c, which, b, h):
    """x_hat = (Q - zp) * scale of one tile (yunthe.com, KV Cache量化技术原理), float64 [bs][D]."""
    dt = c.k_dtype if which == "k" else c.v_dtype
    codes = c.k_codes[b, h] if which == "k" else c.v_codes[b, h]
    if dt == oracle.FP16:
        return codes.view(np.float16).astype(np.float64)
    if dt == oracle.INT8_SYM:
        s = c.k_scale[b, h] if which == "k" else c.v_scale[b, h]
        return codes.astype(np.float64) * float(s)
    if dt == oracle.FP8_E4M3:  # E4M3 values through torch's own float8 type, times the scale
        s = c.k_scale[b, h] if which == "k" else c.v_scale[b, h]
        vals = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
        return vals * float(s)
    return (unpack(codes) - float(c.v_zp[b, h])) * float(c.v_scale[b, h])


def sdpa_reference(c, q, tables, lens, scale):
    """torch's scaled_dot_product_attention in float64 on the contiguous [S, H, L, D] layout."""
    S, Hq, D = q.shape
    H = c.num_kv_heads
    out = np.zeros((S, Hq, D))
    for s in range(S):
        L = int(lens[s])
        if L == 0:
            continue
        K = np.zeros((H, L, D))
        V = np.zeros((H, L, D))
        for t in range(L):
            b = tables[s, t // c.block_size]
            for h in range(H):
                K[h, t] = page_dequant(c, "k", b, h)[t % c.block_size]
                V[h, t] = page_dequant(c, "v", b, h)[t % c.block_size]
        G = Hq // H
        Kt = torch.from_numpy(K).repeat_interleave(G, dim=0)[None]
        Vt = torch.from_numpy(V).repeat_interleave(G, dim=0)[None]
        qt = torch.from_numpy(q[s].astype(np.float64))[None, :, None, :]
        o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=float(np.float32(scale)))
        out[s] = o[0, :, 0].numpy()
    return out


@pytest.mark.parametrize("kd,vd", DTYPES)
@pytest.mark.parametrize("G", [1, 4])
def test_matches_library_attention(kd, vd, G):
    rng = np.random.default_rng(10)
    nb, bs, H, D = 24, 16, 2, 32
    lens = np.array([1, 16, 17, 70])
    perm = rng.permutation(nb).astype(np.int32)
    tables = perm[:20].reshape(4, 5)
    c = filled_cache(rng, nb, bs, H, D, kd, vd, tables, lens)
    q = rng.standard_normal((4, H * G, D)).astype(np.float16)
    scale = 1 / np.sqrt(D)
    out, err = oracle.decode(c, q, tables, lens, scale)
    assert err == 0
    ref = sdpa_reference(c, q, tables, lens, scale)
    np.testing.assert_allclose(out, ref, atol=1e-12, rtol=0)


@pytest.mark.parametrize("kd,vd", DTYPES)
def test_physical_permutation_invariance(kd, vd):
    """Moving blocks to other physical ids (and rewriting the table) changes nothing."""
    rng = np.random.default_rng(11)
    nb, bs, H, D = 16, 16, 2, 16
    lens = np.array([40, 7, 64])
    tables = np.arange(12, dtype=np.int32).reshape(3, 4)
    c = filled_cache(rng, nb, bs, H, D, kd, vd, tables, lens)
    q = rng.standard_normal((3, H, D)).astype(np.float16)
    out, _ = oracle.decode(c, q, tables, lens, 0.25)
    perm = rng.permutation(nb)
    moved = c.copy()
    for arr_name in ("k_codes", "v_codes", "k_scale", "v_scale", "v_zp"):
        getattr(moved, arr_name)[perm] = getattr(c, arr_name)
    out2, _ = oracle.decode(moved, q, perm[tables].astype(np.int32), lens, 0.25)
    np.testing.assert_array_equal(out, out2)


def test_shared_prefix_equals_private_copies():
    rng = np.random.default_rng(12)
    nb, bs, H, D = 16, 16, 2, 16
    lens = np.array([48, 40])
    shared = np.array([[0, 1, 2], [0, 1, 3]], np.int32)   # blocks 0, 1 shared
    c = filled_cache(rng, nb, bs, H, D, oracle.INT8_SYM, oracle.INT4_ASYM, shared[:1], lens[:1])
    k = rng.standard_normal((8, H, D)).astype(np.float16)
    assert oracle.store(c, k, k, 3 * bs + np.arange(8)) == 0
    private = c.copy()
    assert oracle.copy_blocks(private, np.array([[0, 4], [1, 5]])) == 0
    priv_tables = np.array([[0, 1, 2], [4, 5, 3]], np.int32)
    q = rng.standard_normal((2, H, D)).astype(np.float16)
    a, _ = oracle.decode(c, q, shared, lens, 0.25)
    b, _ = oracle.decode(private, q, priv_tables, lens, 0.25)
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("kd,vd", DTYPES)
def test_closed_forms(kd, vd):
    rng = np.random.default_rng(13)
    nb, bs, H, D = 8, 16, 1, 16
    tables = np.array([[3, 5]], np.int32)
    c = filled_cache(rng, nb, bs, H, D, kd, vd, tables, [32])
    vhat = np.concatenate([page_dequant(c, "v", 3, 0), page_dequant(c, "v", 5, 0)])
    khat = np.concatenate([page_dequant(c, "k", 3, 0), page_dequant(c, "k", 5, 0)])
    q = rng.standard_normal((1, 1, D)).astype(np.float16)
    # one token: the output is that token's v_hat
    out, _ = oracle.decode(c, q, tables, [1], 0.5)
    np.testing.assert_array_equal(out[0, 0], vhat[0])
    # q = 0: uniform weights, the output is the mean of v_hat
    out, _ = oracle.decode(c, np.zeros_like(q), tables, [23], 0.5)
    np.testing.assert_allclose(out[0, 0], vhat[:23].mean(axis=0), atol=1e-13)
    # a logit that dominates by >= 40: the output is that token's v_hat (to e^-40)
    t_star = 20
    q_dom = (khat[t_star] / np.linalg.norm(khat[t_star]) * 4).astype(np.float16)[None, None]
    z = (khat[:32] @ q_dom[0, 0].astype(np.float64))
    sm = 60.0 / (z[t_star] - np.max(np.delete(z, t_star)))
    assert sm > 0
    out, _ = oracle.decode(c, q_dom, tables, [32], float(sm))
    np.testing.assert_allclose(out[0, 0], vhat[t_star], atol=1e-12 * np.abs(vhat).max() + 1e-15)


def test_empty_and_error_reporting():
    rng = np.random.default_rng(14)
    nb, bs, H, D = 4, 16, 1, 16
    tables = np.array([[0, 1], [2, 3]], np.int32)
    c = filled_cache(rng, nb, bs, H, D, oracle.INT8_SYM, oracle.INT8_SYM, tables, [20, 32])
    q = rng.standard_normal((2, 1, D)).astype(np.float16)
    out, err = oracle.decode(c, q, tables, [0, 32], 0.25)
    assert err == 0 and not out[0].any()
    _, err = oracle.decode(c, q, tables, [33, 1], 0.25, max_context_len=40)
    assert err == oracle.DEVERR_CONTEXT_LEN
    bad = tables.copy()
    bad[1, 1] = 9
    out_bad, err = oracle.decode(c, q, bad, [20, 32], 0.25)
    assert err == oracle.DEVERR_BLOCK_ID
    # the bad block's tokens are left out: the same as attending over the first block only
    out_16, _ = oracle.decode(c, q, tables, [20, 16], 0.25)
    np.testing.assert_array_equal(out_bad[1], out_16[1])


@pytest.mark.parametrize("seed", range(8))
def test_brute_force_agreement(seed):
    rng = np.random.default_rng(100 + seed)
    kd, vd = DTYPES[seed % len(DTYPES)]
    bs = [16, 32][seed % 2]
    H = int(rng.integers(1, 3))
    G = int(rng.choice([1, 2, 4]))
    D = 16
    S = int(rng.integers(1, 5))
    lens = rng.integers(0, 41, size=S)
    mb = 3
    nb = S * mb + 2
    tables = rng.permutation(nb)[:S * mb].astype(np.int32).reshape(S, mb)
    c = filled_cache(rng, nb, bs, H, D, kd, vd, tables, lens)
    q = rng.standard_normal((S, H * G, D)).astype(np.float16)
    out, err = oracle.decode(c, q, tables, lens, 0.3)
    assert err == 0
    ref = brute.decode(c, q, tables, lens, 0.3)
    np.testing.assert_allclose(out, ref, atol=1e-12, rtol=0)


def test_quantized_attention_tracks_fp16_attention():
    """Attention over the INT8/INT4 cache stays close to attention over the fp16 originals:
    per-element dequant error is at most half a step, so outputs move by a few steps."""
    rng = np.random.default_rng(15)
    nb, bs, H, D = 8, 16, 2, 64
    tables = np.arange(8, dtype=np.int32).reshape(2, 4)
    lens = np.array([64, 50])
    k = rng.standard_normal((2, 64, H, D)).astype(np.float16)
    v = rng.standard_normal((2, 64, H, D)).astype(np.float16)
    q = rng.standard_normal((2, H, D)).astype(np.float16)
    outs = {}
    for kd, vd in DTYPES:
        c = oracle.OracleCache.empty(nb, bs, H, D, kd, vd)
        for s in range(2):
            L = lens[s]
            slots = tables[s, np.arange(L) // bs].astype(np.int64) * bs + np.arange(L) % bs
            oracle.store(c, k[s, :L], v[s, :L], slots)
        outs[(kd, vd)], _ = oracle.decode(c, q, tables, lens, 1 / 8)
    ref = outs[(oracle.FP16, oracle.FP16)]
    assert np.abs(outs[(oracle.INT8_SYM, oracle.INT8_SYM)] - ref).max() < 0.03
    assert np.abs(outs[(oracle.INT8_SYM, oracle.INT4_ASYM)] - ref).max() < 0.2
    assert np.abs(outs[(oracle.FP8_E4M3, oracle.FP8_E4M3)] - ref).max() < 0.1
