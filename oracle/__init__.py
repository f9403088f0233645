"""CPU oracle for the paged, block-quantized KV-cache path -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously correct implementation (``oracle.c``, binary32 for quantization and
binary64 for attention) plus a NumPy binary64 brute force for tiny inputs (``brute.py``).
It shares no code with the GPU library and never imports it. Only the tests, the smoke check
and the benchmark's CPU-baseline / reference leg may use it.

This module is argument marshalling around ``liboracle.so`` (built by ``oracle/build.py``).

Parity status of each function (what pins it; see ``tests/test_oracle_*.py``):
  store  INT8 / INT4 single-shot quantization: pinned (worked examples, error bound, extremes,
         special cases). Append into a partly filled block (fit-or-rebuild rule): the pages only
         quantize whole blocks, so the rule itself is **parity unpinned**; only invariants
         (range, error bound, fit == single shot) are checked.
  FP8 E4M3 store (scale = absmax / 448, nearest-even saturating codes): pinned (the format's
         hand-decoded values, ties and saturation, every code round-trips, error bound); its
         append rule is parity unpinned like the INT8 one.
  copy   pinned (byte identity, untouched blocks).
  decode pinned (library attention on contiguous data, permutation / prefix-sharing
         invariance, closed-form special cases, brute-force agreement).
  prefill (chunked, causal) pinned (library attention with an explicit causal mask on contiguous
         data, equality with decode for one-token chunks, chunk splitting, brute force).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

from . import build as _build

FP16, INT8_SYM, INT4_ASYM, FP8_E4M3 = 0, 1, 2, 3

DEVERR_BLOCK_ID, DEVERR_SLOT, DEVERR_SLOT_GROUP, DEVERR_CONTEXT_LEN = 1, 2, 3, 4


class _COracleCache(ctypes.Structure):
    _fields_ = [
        ("num_blocks", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("k_dtype", ctypes.c_int32),
        ("v_dtype", ctypes.c_int32),
        ("k_codes", ctypes.c_void_p),
        ("v_codes", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p),
        ("v_scale", ctypes.c_void_p),
        ("v_zp", ctypes.c_void_p),
    ]


_lib = None


def _load():
    global _lib
    if _lib is None:
        # PKV_ORACLE_LIB: another build of oracle.c (the mutation test loads seeded-mistake builds)
        path = os.environ.get("PKV_ORACLE_LIB") or _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        lib.oracle_store.argtypes = [P, P, P, P, ctypes.c_int32]
        lib.oracle_store.restype = ctypes.c_int32
        lib.oracle_copy_blocks.argtypes = [P, P, ctypes.c_int32]
        lib.oracle_copy_blocks.restype = ctypes.c_int32
        lib.oracle_decode.argtypes = [P, P, ctypes.c_int32, ctypes.c_int32, P, ctypes.c_int32, P,
                                      ctypes.c_int32, ctypes.c_float, P, ctypes.c_int32]
        lib.oracle_decode.restype = ctypes.c_int32
        lib.oracle_prefill.argtypes = [P, P, ctypes.c_int32, ctypes.c_int32, P, P, ctypes.c_int32, P,
                                       ctypes.c_float, P, ctypes.c_int32]
        lib.oracle_prefill.restype = ctypes.c_int32
        lib.oracle_fp8_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_fp8_e4m3_decode.restype = ctypes.c_double
        lib.oracle_fp8_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_fp8_e4m3_encode.restype = ctypes.c_uint8
        _lib = lib
    return _lib


def _row_shape(dtype: int, head_dim: int):
    if dtype == FP16:
        return head_dim, np.uint16  # fp16 bit patterns
    if dtype == INT8_SYM:
        return head_dim, np.int8
    if dtype == FP8_E4M3:
        return head_dim, np.uint8  # E4M3 bytes
    if dtype == INT4_ASYM:
        return head_dim // 2, np.uint8
    raise ValueError(f"unknown dtype {dtype}")


@dataclass
class OracleCache:
    """Host pool with the device layout: codes [nb][H][bs][row], scales/zps [nb][H]."""

    num_blocks: int
    block_size: int
    num_kv_heads: int
    head_dim: int
    k_dtype: int
    v_dtype: int
    k_codes: np.ndarray
    v_codes: np.ndarray
    k_scale: np.ndarray
    v_scale: np.ndarray
    v_zp: np.ndarray

    @classmethod
    def empty(cls, num_blocks, block_size, num_kv_heads, head_dim, k_dtype, v_dtype, poison=0xA5):
        """A pool whose every byte is `poison` (so unwritten bytes are recognisable)."""
        def codes(dtype):
            row, np_dtype = _row_shape(dtype, head_dim)
            nbytes = num_blocks * num_kv_heads * block_size * row * np.dtype(np_dtype).itemsize
            raw = np.full(nbytes, poison, dtype=np.uint8)
            return raw.view(np_dtype).reshape(num_blocks, num_kv_heads, block_size, row)

        def meta(np_dtype):
            nbytes = num_blocks * num_kv_heads * np.dtype(np_dtype).itemsize
            return np.full(nbytes, poison, dtype=np.uint8).view(np_dtype).reshape(num_blocks, num_kv_heads)

        return cls(num_blocks, block_size, num_kv_heads, head_dim, k_dtype, v_dtype,
                   codes(k_dtype), codes(v_dtype), meta(np.float32), meta(np.float32), meta(np.uint8))

    def copy(self) -> "OracleCache":
        return OracleCache(self.num_blocks, self.block_size, self.num_kv_heads, self.head_dim,
                           self.k_dtype, self.v_dtype, self.k_codes.copy(), self.v_codes.copy(),
                           self.k_scale.copy(), self.v_scale.copy(), self.v_zp.copy())

    def _c(self) -> _COracleCache:
        for a in (self.k_codes, self.v_codes, self.k_scale, self.v_scale, self.v_zp):
            assert a.flags["C_CONTIGUOUS"]
        return _COracleCache(self.num_blocks, self.block_size, self.num_kv_heads, self.head_dim,
                             self.k_dtype, self.v_dtype, self.k_codes.ctypes.data, self.v_codes.ctypes.data,
                             self.k_scale.ctypes.data, self.v_scale.ctypes.data, self.v_zp.ctypes.data)


def _fp16_bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    if x.dtype == np.float16:
        return x.view(np.uint16)
    if x.dtype == np.uint16:
        return x
    raise TypeError("expected float16 data")


def fp8_e4m3_decode(code: int) -> float:
    """The E4M3 value of a code byte (binary64, exact)."""
    return float(_load().oracle_fp8_e4m3_decode(int(code) & 0xFF))


def fp8_e4m3_encode(x: float) -> int:
    """The E4M3 code of a binary32 value: nearest, ties to even, saturating at +-448."""
    return int(_load().oracle_fp8_e4m3_encode(float(np.float32(x))))


def store(cache: OracleCache, k_new: np.ndarray, v_new: np.ndarray, slot_mapping: np.ndarray) -> int:
    """Quantize + scatter T tokens (fp16 [T][H][D]) in place. Returns the error code (0 = none)."""
    k_bits, v_bits = _fp16_bits(k_new), _fp16_bits(v_new)
    slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    T = slots.shape[0]
    assert k_bits.shape == v_bits.shape == (T, cache.num_kv_heads, cache.head_dim)
    c = cache._c()
    rc = _load().oracle_store(ctypes.byref(c), k_bits.ctypes.data, v_bits.ctypes.data, slots.ctypes.data, T)
    if rc < 0:
        raise ValueError("unsupported cache descriptor")
    return int(rc)


def copy_blocks(cache: OracleCache, block_mapping: np.ndarray) -> int:
    """Copy blocks in place for pairs {src, dst}. Returns the error code (0 = none)."""
    m = np.ascontiguousarray(block_mapping, dtype=np.int32).reshape(-1, 2)
    c = cache._c()
    rc = _load().oracle_copy_blocks(ctypes.byref(c), m.ctypes.data, m.shape[0])
    if rc < 0:
        raise ValueError("unsupported cache descriptor")
    return int(rc)


def decode(cache: OracleCache, q: np.ndarray, block_tables: np.ndarray, context_lens: np.ndarray,
           softmax_scale: float, max_context_len: int | None = None, num_threads: int | None = None):
    """Binary64 decode attention. Returns (out float64 [S][Hq][D], error code)."""
    q_bits = _fp16_bits(q)
    S, Hq, D = q_bits.shape
    assert D == cache.head_dim
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    assert bt.shape[0] == S and cl.shape == (S,)
    if max_context_len is None:
        max_context_len = int(cl.max()) if S else 0
    if num_threads is None:
        num_threads = os.cpu_count() or 1
    out = np.zeros((S, Hq, D), dtype=np.float64)
    c = cache._c()
    rc = _load().oracle_decode(ctypes.byref(c), q_bits.ctypes.data, S, Hq, bt.ctypes.data, bt.shape[1],
                               cl.ctypes.data, int(max_context_len), ctypes.c_float(softmax_scale),
                               out.ctypes.data, int(num_threads))
    if rc < 0:
        raise ValueError("unsupported cache descriptor or head split")
    return out, int(rc)


def prefill(cache: OracleCache, q: np.ndarray, cu_q_lens: np.ndarray, block_tables: np.ndarray,
            context_lens: np.ndarray, softmax_scale: float, num_threads: int | None = None):
    """Binary64 chunked-prefill attention: the rows of sequence s (q[cu_q_lens[s]:cu_q_lens[s+1]])
    are its last q_len context tokens, each attending causally. Returns (out [T][Hq][D], error)."""
    q_bits = _fp16_bits(q)
    T, Hq, D = q_bits.shape
    assert D == cache.head_dim
    cu = np.ascontiguousarray(cu_q_lens, dtype=np.int32)
    S = cu.shape[0] - 1
    assert cu[-1] == T if S > 0 else T == 0
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    assert bt.shape[0] == S and cl.shape == (S,)
    if num_threads is None:
        num_threads = os.cpu_count() or 1
    out = np.zeros((T, Hq, D), dtype=np.float64)
    c = cache._c()
    rc = _load().oracle_prefill(ctypes.byref(c), q_bits.ctypes.data, S, Hq, cu.ctypes.data, bt.ctypes.data,
                                bt.shape[1], cl.ctypes.data, ctypes.c_float(softmax_scale), out.ctypes.data,
                                int(num_threads))
    if rc < 0:
        raise ValueError("unsupported cache descriptor or head split")
    return out, int(rc)
