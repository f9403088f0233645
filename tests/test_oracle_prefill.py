"""Pins for the oracle's chunked prefill: torch's scaled_dot_product_attention in binary64 with an
explicit causal mask on the contiguous layout, equality with decode for one-token chunks and with
two half chunks, the NumPy brute force per query, and error reporting.

Source: yunthe.com "LLM推理显存优化KV Cache量化与PagedAttention实现详解", section "Prefix Caching与多轮对话
场景优化实践" (only the new tokens are computed, over the cached prefix) and tbr8.org "如何通过
PagedAttention 与分块量化结合..." §5 item 2 (dequantization inside the attention operator). Reading
taken: a chunk holds the last q_len tokens of a sequence's context (already stored), and the query
at position p attends causally to tokens 0..p.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from test_oracle_decode import DTYPES, filled_cache, page_dequant


def contiguous(c, tables, s, L, h):
    rows_k, rows_v = [], []
    for t in range(L):
        b = tables[s, t // c.block_size]
        rows_k.append(page_dequant(c, "k", b, h)[t % c.block_size])
        rows_v.append(page_dequant(c, "v", b, h)[t % c.block_size])
    return np.array(rows_k), np.array(rows_v)


def sdpa_causal(c, q, cu, tables, lens, scale):
    T, Hq, D = q.shape
    H = c.num_kv_heads
    G = Hq // H
    out = np.zeros((T, Hq, D))
    for s in range(len(lens)):
        n = cu[s + 1] - cu[s]
        L = int(lens[s])
        if n == 0:
            continue
        pos = L - n + np.arange(n)
        mask = torch.from_numpy(np.arange(L)[None, :] <= pos[:, None])          # [n, L]
        for h in range(H):
            K, V = contiguous(c, tables, s, L, h)
            qs = torch.from_numpy(q[cu[s]:cu[s + 1], h * G:(h + 1) * G].astype(np.float64)).permute(1, 0, 2)
            o = torch.nn.functional.scaled_dot_product_attention(
                qs[None], torch.from_numpy(K)[None, None].expand(1, G, L, D),
                torch.from_numpy(V)[None, None].expand(1, G, L, D), attn_mask=mask, scale=float(np.float32(scale)))
            out[cu[s]:cu[s + 1], h * G:(h + 1) * G] = o[0].permute(1, 0, 2).numpy()
    return out


def setup(rng, kd, vd, lens, qlens, H=2, G=2, D=32, bs=16):
    S = len(lens)
    mb = max(-(-int(L) // bs) for L in lens)
    nb = S * mb + 3
    tables = rng.permutation(nb)[:S * mb].astype(np.int32).reshape(S, mb)
    c = filled_cache(rng, nb, bs, H, D, kd, vd, tables, lens)
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = rng.standard_normal((int(cu[-1]), H * G, D)).astype(np.float16)
    return c, tables, cu, q


@pytest.mark.parametrize("kd,vd", DTYPES)
def test_matches_library_attention_with_causal_mask(kd, vd):
    rng = np.random.default_rng(20)
    lens, qlens = [40, 17, 64], [40, 5, 23]
    c, tables, cu, q = setup(rng, kd, vd, lens, qlens)
    out, err = oracle.prefill(c, q, cu, tables, np.array(lens), 0.2)
    assert err == 0
    np.testing.assert_allclose(out, sdpa_causal(c, q, cu, tables, lens, 0.2), atol=1e-12, rtol=0)


def test_one_token_chunks_equal_decode_and_halves_equal_whole():
    rng = np.random.default_rng(21)
    lens, qlens = [33, 50], [1, 1]
    c, tables, cu, q = setup(rng, oracle.INT8_SYM, oracle.INT4_ASYM, lens, qlens, G=4)
    pre, _ = oracle.prefill(c, q, cu, tables, np.array(lens), 0.3)
    dec, _ = oracle.decode(c, q, tables, np.array(lens), 0.3)
    np.testing.assert_array_equal(pre, dec)
    # a chunk of 20 equals two chunks of 10 (the first one over a context 10 tokens shorter)
    c, tables, cu, q = setup(rng, oracle.INT8_SYM, oracle.INT8_SYM, [60], [20])
    whole, _ = oracle.prefill(c, q, cu, tables, np.array([60]), 0.3)
    a, _ = oracle.prefill(c, q[:10], np.array([0, 10]), tables, np.array([50]), 0.3)
    b, _ = oracle.prefill(c, q[10:], np.array([0, 10]), tables, np.array([60]), 0.3)
    np.testing.assert_array_equal(whole, np.concatenate([a, b]))


@pytest.mark.parametrize("seed", range(4))
def test_brute_force_per_query(seed):
    rng = np.random.default_rng(30 + seed)
    kd, vd = DTYPES[seed % len(DTYPES)]
    lens = list(rng.integers(1, 45, 3))
    qlens = [int(rng.integers(0, L + 1)) for L in lens]
    c, tables, cu, q = setup(rng, kd, vd, lens, qlens, H=1, G=3, bs=[16, 32][seed % 2])
    out, err = oracle.prefill(c, q, cu, tables, np.array(lens), 0.25)
    assert err == 0
    for s in range(3):
        for i in range(qlens[s]):
            L = lens[s] - qlens[s] + i + 1
            ref = brute.decode(c, q[cu[s] + i][None], tables[s:s + 1], np.array([L]), 0.25)
            np.testing.assert_allclose(out[cu[s] + i], ref[0], atol=1e-12, rtol=0)


def test_errors():
    rng = np.random.default_rng(22)
    c, tables, cu, q = setup(rng, oracle.INT8_SYM, oracle.INT8_SYM, [20, 20], [4, 4])
    _, err = oracle.prefill(c, q, cu, tables, np.array([20, 3]), 0.3)  # a chunk longer than its context
    assert err == oracle.DEVERR_CONTEXT_LEN
    bad = tables.copy()
    bad[0, 0] = 999
    _, err = oracle.prefill(c, q, cu, bad, np.array([20, 20]), 0.3)
    assert err == oracle.DEVERR_BLOCK_ID
