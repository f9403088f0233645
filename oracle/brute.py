"""NumPy binary64 brute force of paged decode attention -- TEST INFRASTRUCTURE ONLY.

A second, independent route to the decode result for tiny inputs, written separately from
``oracle.c``: it first rebuilds each sequence's contiguous K_hat / V_hat ([seq_len, head_dim],
the per-layer [batch, heads, seq_len, head_dim] view of yunthe.com "LLM推理显存优化KV Cache量化与
PagedAttention实现详解", section "KV Cache量化技术原理") by walking the block table, dequantizes
with x_hat = (Q - zp) * scale (same section), and then evaluates softmax attention with array
operations. It only supports well-formed inputs.
"""
from __future__ import annotations

import numpy as np

FP16, INT8_SYM, INT4_ASYM, FP8_E4M3 = 0, 1, 2, 3


def _e4m3_values(codes: np.ndarray) -> np.ndarray:
    """E4M3 code bytes -> float64 values: sign, 4 exponent bits (bias 7), 3 mantissa bits;
    exponent field 0 = subnormal m * 2^-9 (the all-ones NaN codes never occur in a tile)."""
    c = codes.astype(np.int64)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    return np.where(c & 0x80, -mag, mag)


def _unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    """[..., D/2] bytes -> [..., D] codes, low nibble = even dimension."""
    lo = packed & 0x0F
    hi = packed >> 4
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.int64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def dequant_tile(codes: np.ndarray, dtype: int, scale=None, zp=None) -> np.ndarray:
    """One (block, head) tile [bs][row] -> float64 [bs][D]."""
    if dtype == FP16:
        return codes.view(np.float16).astype(np.float64)
    if dtype == INT8_SYM:
        return codes.astype(np.float64) * np.float64(scale)
    if dtype == FP8_E4M3:
        return _e4m3_values(codes) * np.float64(scale)
    return (_unpack_nibbles(codes).astype(np.float64) - np.float64(zp)) * np.float64(scale)


def contiguous_kv(cache, block_table_row: np.ndarray, length: int, kv_head: int):
    """Walk one sequence's block table and stack its dequantized K and V rows in token order."""
    bs = cache.block_size
    ks, vs = [], []
    for i in range((length + bs - 1) // bs):
        b = int(block_table_row[i])
        k = dequant_tile(cache.k_codes[b, kv_head], cache.k_dtype, cache.k_scale[b, kv_head])
        v = dequant_tile(cache.v_codes[b, kv_head], cache.v_dtype, cache.v_scale[b, kv_head],
                         cache.v_zp[b, kv_head])
        ks.append(k)
        vs.append(v)
    if not ks:
        d = cache.head_dim
        return np.zeros((0, d)), np.zeros((0, d))
    return np.concatenate(ks)[:length], np.concatenate(vs)[:length]


def decode(cache, q: np.ndarray, block_tables: np.ndarray, context_lens: np.ndarray,
           softmax_scale: float) -> np.ndarray:
    """out[s, h] = softmax(scale * K_hat q) . V_hat over the first context_lens[s] tokens."""
    S, Hq, D = q.shape
    G = Hq // cache.num_kv_heads
    out = np.zeros((S, Hq, D), dtype=np.float64)
    scale = np.float64(np.float32(softmax_scale))
    for s in range(S):
        L = int(context_lens[s])
        if L == 0:
            continue
        for g in range(cache.num_kv_heads):
            K, V = contiguous_kv(cache, block_tables[s], L, g)
            qs = q[s, g * G:(g + 1) * G].astype(np.float64)          # [G, D]
            z = scale * (qs @ K.T)                                  # [G, L]
            w = np.exp(z - z.max(axis=1, keepdims=True))
            out[s, g * G:(g + 1) * G] = (w @ V) / w.sum(axis=1, keepdims=True)
    return out
