"""ctypes binding of libpkv.so -- the C ABI declared in include/pkv.h, under the same names.

Argument marshalling only: every step of the store, decode and copy runs in the library's CUDA
kernels. Device buffers may be passed as torch tensors (their data_ptr is used) or as raw
integer addresses. Streams default to torch's current stream on the current device.

Importing this module loads libpkv.so and raises ImportError if it has not been built
(``python -m paged_block_quantized_b200.build``); there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpkv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libpkv.so not built at {LIB_PATH}: run `python -m paged_block_quantized_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

# ---- enums (values fixed by include/pkv.h) ----
PKV_OK, PKV_ERR_INVALID_ARG, PKV_ERR_UNSUPPORTED, PKV_ERR_OUT_OF_BLOCKS, PKV_ERR_CUDA, PKV_ERR_DEVICE_TIMEOUT = range(6)
PKV_FP16, PKV_INT8_SYM, PKV_INT4_ASYM, PKV_FP8_E4M3 = 0, 1, 2, 3
(PKV_DEVERR_NONE, PKV_DEVERR_BLOCK_ID, PKV_DEVERR_SLOT, PKV_DEVERR_SLOT_GROUP, PKV_DEVERR_CONTEXT_LEN,
 PKV_DEVERR_TIMEOUT, PKV_DEVERR_SEQ_ORDER, PKV_DEVERR_SHARED) = range(8)

EXPORTED = (
    "pkv_status_string", "pkv_tile_bytes", "pkv_store_quantized", "pkv_decode_workspace_size",
    "pkv_decode_partitioning", "pkv_paged_attention_decode_static", "pkv_static_scratch_address",
    "pkv_paged_attention_decode", "pkv_paged_attention_decode_ex", "pkv_decode_ex_workspace_size",
    "pkv_paged_attention_prefill",
    "pkv_copy_blocks", "pkv_swap_blocks", "pkv_decode_step", "pkv_blocks_for_tokens", "pkv_alloc_create",
    "pkv_alloc_destroy", "pkv_alloc_num_free", "pkv_alloc_refcount", "pkv_alloc_blocks", "pkv_alloc_fork",
    "pkv_alloc_release", "pkv_alloc_cow", "pkv_prefix_cache_create", "pkv_prefix_cache_destroy",
    "pkv_prefix_cache_size", "pkv_prefix_cache_evictable", "pkv_prefix_match", "pkv_prefix_insert",
    "pkv_prefix_alloc",
)


class pkv_cache_desc(ctypes.Structure):
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


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_DESC = ctypes.POINTER(pkv_cache_desc)


def _sig(name, restype, *argtypes):
    f = getattr(_lib, name)
    f.restype = restype
    f.argtypes = list(argtypes)
    return f


_status_string = _sig("pkv_status_string", ctypes.c_char_p, ctypes.c_int)
_tile_bytes = _sig("pkv_tile_bytes", ctypes.c_size_t, _DESC, _I32)
_store = _sig("pkv_store_quantized", ctypes.c_int, _DESC, _P, _P, _P, _I32, _P, _P)
_ws_size = _sig("pkv_decode_workspace_size", ctypes.c_int, _DESC, _I32, _I32, _I32, _I32,
                ctypes.POINTER(ctypes.c_size_t))
_partitioning = _sig("pkv_decode_partitioning", ctypes.c_int, _DESC, _I32, _I32, _I32, _I32,
                     ctypes.POINTER(_I32), ctypes.POINTER(_I32))
_decode = _sig("pkv_paged_attention_decode", ctypes.c_int, _DESC, _P, _P, _I32, _I32, _P, _I32, _P, _I32,
               ctypes.c_float, _I32, _P, ctypes.c_size_t, _P, _P)


class pkv_decode_options(ctypes.Structure):
    _fields_ = [("struct_bytes", ctypes.c_size_t), ("seq_order", ctypes.c_void_p),
                ("num_prefix_groups", ctypes.c_int32), ("num_prefix_members", ctypes.c_int32),
                ("max_group_size", ctypes.c_int32), ("max_shared_blocks", ctypes.c_int32),
                ("prefix_group_start", ctypes.c_void_p), ("prefix_members", ctypes.c_void_p),
                ("shared_blocks", ctypes.c_void_p)]


def decode_options(seq_order=None, prefix=None):
    """pkv_decode_options: seq_order (device int32 [S]) and/or prefix = dict(group_start, members,
    shared_blocks: device int32 tensors; num_groups, num_members, max_group_size, max_shared_blocks: ints)."""
    o = pkv_decode_options()
    o.struct_bytes = ctypes.sizeof(pkv_decode_options)
    o.seq_order = _ptr(seq_order)
    if prefix is not None:
        o.num_prefix_groups = int(prefix["num_groups"])
        o.num_prefix_members = int(prefix["num_members"])
        o.max_group_size = int(prefix["max_group_size"])
        o.max_shared_blocks = int(prefix["max_shared_blocks"])
        o.prefix_group_start = _ptr(prefix["group_start"])
        o.prefix_members = _ptr(prefix["members"])
        o.shared_blocks = _ptr(prefix["shared_blocks"])
    return o


_decode_ex = _sig("pkv_paged_attention_decode_ex", ctypes.c_int, _DESC, _P, _P, _I32, _I32, _P, _I32, _P, _I32,
                  ctypes.c_float, _I32, ctypes.POINTER(pkv_decode_options), _P, ctypes.c_size_t, _P, _P)
_ws_ex = _sig("pkv_decode_ex_workspace_size", ctypes.c_int, _DESC, _I32, _I32, _I32, _I32,
              ctypes.POINTER(pkv_decode_options), ctypes.POINTER(ctypes.c_size_t))
_prefill = _sig("pkv_paged_attention_prefill", ctypes.c_int, _DESC, _P, _P, _I32, _I32, _P, _I32, _I32, _P, _I32, _P,
                _I32, ctypes.c_float, _P, _P)
_decode_static = _sig("pkv_paged_attention_decode_static", ctypes.c_int, _DESC, _P, _P, _I32, _I32, _P, _I32, _P,
                      _I32, ctypes.c_float, _I32, _P, _P)
PKV_STATIC_SCRATCH_BYTES = 8 << 20
_static_addr = _sig("pkv_static_scratch_address", ctypes.c_int, ctypes.POINTER(_P), ctypes.POINTER(ctypes.c_size_t))
_copy = _sig("pkv_copy_blocks", ctypes.c_int, _DESC, _P, _I32, _P, _P)
_swap = _sig("pkv_swap_blocks", ctypes.c_int, _DESC, _DESC, _P, _I32, _I32, _P, _P)
PKV_SWAP_OUT, PKV_SWAP_IN = 0, 1
_step = _sig("pkv_decode_step", ctypes.c_int, _DESC, _P, _I32, _P, _P, _P, _I32, _P, _P, _I32, _I32, _P, _I32, _P,
             _I32, ctypes.c_float, _I32, _P, ctypes.c_size_t, _P, _P)
_blocks_for_tokens = _sig("pkv_blocks_for_tokens", _I32, ctypes.c_int64, _I32)
_alloc_create = _sig("pkv_alloc_create", ctypes.c_int, _I32, ctypes.POINTER(_P))
_alloc_destroy = _sig("pkv_alloc_destroy", None, _P)
_alloc_num_free = _sig("pkv_alloc_num_free", _I32, _P)
_alloc_refcount = _sig("pkv_alloc_refcount", _I32, _P, _I32)
_alloc_blocks = _sig("pkv_alloc_blocks", ctypes.c_int, _P, _I32, _P)
_alloc_fork = _sig("pkv_alloc_fork", ctypes.c_int, _P, _P, _I32)
_alloc_release = _sig("pkv_alloc_release", ctypes.c_int, _P, _P, _I32)
_alloc_cow = _sig("pkv_alloc_cow", ctypes.c_int, _P, _I32, ctypes.POINTER(_I32))
_pc_create = _sig("pkv_prefix_cache_create", ctypes.c_int, _P, _I32, ctypes.POINTER(_P))
_pc_destroy = _sig("pkv_prefix_cache_destroy", None, _P)
_pc_size = _sig("pkv_prefix_cache_size", _I32, _P)
_pc_evictable = _sig("pkv_prefix_cache_evictable", _I32, _P)
_pc_match = _sig("pkv_prefix_match", ctypes.c_int, _P, _P, ctypes.c_int64, _P, _I32, ctypes.POINTER(_I32))
_pc_insert = _sig("pkv_prefix_insert", ctypes.c_int, _P, _P, ctypes.c_int64, _P, _I32)
_pc_alloc = _sig("pkv_prefix_alloc", ctypes.c_int, _P, _I32, _P)


class PkvError(RuntimeError):
    def __init__(self, status: int, call: str):
        super().__init__(f"{call}: {pkv_status_string(status)}")
        self.status = status


def _ptr(x) -> int | None:
    """Device/host address of a tensor (data_ptr), an integer address, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):  # numpy array (host buffers for the allocator)
        return x.ctypes.data
    raise TypeError(f"cannot take the address of {type(x)}")


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, call: str, raise_on_error: bool) -> int:
    if raise_on_error and status != PKV_OK:
        raise PkvError(status, call)
    return status


def pkv_status_string(status: int) -> str:
    return _status_string(int(status)).decode()


def pkv_tile_bytes(desc: pkv_cache_desc, which_v: int) -> int:
    return int(_tile_bytes(ctypes.byref(desc), int(which_v)))


def pkv_store_quantized(desc, k_new, v_new, slot_mapping, T, dev_error=None, stream=None, raise_on_error=True):
    st = _store(ctypes.byref(desc), _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), int(T), _ptr(dev_error),
                _stream(stream))
    return _check(st, "pkv_store_quantized", raise_on_error)


def pkv_decode_workspace_size(desc, num_seqs, num_q_heads, max_context_len, partition_tokens=0) -> int:
    out = ctypes.c_size_t(0)
    st = _ws_size(ctypes.byref(desc), int(num_seqs), int(num_q_heads), int(max_context_len),
                  int(partition_tokens), ctypes.byref(out))
    _check(st, "pkv_decode_workspace_size", True)
    return int(out.value)


def pkv_decode_partitioning(desc, num_seqs, num_q_heads, max_context_len, partition_tokens=0):
    """(worker warps, persistent CTAs) the decode will use on the current device."""
    nw, nc = _I32(0), _I32(0)
    st = _partitioning(ctypes.byref(desc), int(num_seqs), int(num_q_heads), int(max_context_len),
                       int(partition_tokens), ctypes.byref(nw), ctypes.byref(nc))
    _check(st, "pkv_decode_partitioning", True)
    return int(nw.value), int(nc.value)


def pkv_paged_attention_decode(desc, out, q, num_seqs, num_q_heads, block_tables, max_blocks_per_seq,
                               context_lens, max_context_len, softmax_scale, partition_tokens=0,
                               workspace=None, workspace_bytes=0, dev_error=None, stream=None,
                               raise_on_error=True):
    st = _decode(ctypes.byref(desc), _ptr(out), _ptr(q), int(num_seqs), int(num_q_heads), _ptr(block_tables),
                 int(max_blocks_per_seq), _ptr(context_lens), int(max_context_len), float(softmax_scale),
                 int(partition_tokens), _ptr(workspace), int(workspace_bytes), _ptr(dev_error), _stream(stream))
    return _check(st, "pkv_paged_attention_decode", raise_on_error)


def pkv_decode_ex_workspace_size(desc, num_seqs, num_q_heads, max_context_len, partition_tokens=0, seq_order=None,
                                 prefix=None) -> int:
    opts = decode_options(seq_order, prefix)
    out = ctypes.c_size_t(0)
    st = _ws_ex(ctypes.byref(desc), int(num_seqs), int(num_q_heads), int(max_context_len), int(partition_tokens),
                ctypes.byref(opts), ctypes.byref(out))
    _check(st, "pkv_decode_ex_workspace_size", True)
    return int(out.value)


def pkv_paged_attention_decode_ex(desc, out, q, num_seqs, num_q_heads, block_tables, max_blocks_per_seq,
                                  context_lens, max_context_len, softmax_scale, partition_tokens=0, seq_order=None,
                                  workspace=None, workspace_bytes=0, dev_error=None, stream=None,
                                  raise_on_error=True, prefix=None):
    """Decode with options: seq_order (device int32 [num_seqs]) = the walk order of the sequences;
    prefix = the shared-prefix groups (see decode_options)."""
    opts = decode_options(seq_order, prefix)
    st = _decode_ex(ctypes.byref(desc), _ptr(out), _ptr(q), int(num_seqs), int(num_q_heads), _ptr(block_tables),
                    int(max_blocks_per_seq), _ptr(context_lens), int(max_context_len), float(softmax_scale),
                    int(partition_tokens), ctypes.byref(opts), _ptr(workspace), int(workspace_bytes),
                    _ptr(dev_error), _stream(stream))
    return _check(st, "pkv_paged_attention_decode_ex", raise_on_error)


def pkv_paged_attention_prefill(desc, out, q, num_seqs, num_q_heads, cu_q_lens, total_q, max_q_len, block_tables,
                                max_blocks_per_seq, context_lens, max_context_len, softmax_scale, dev_error=None,
                                stream=None, raise_on_error=True):
    """Chunked prefill: causal attention of each sequence's last q_len tokens (rows of q given by
    cu_q_lens) over the paged cache."""
    st = _prefill(ctypes.byref(desc), _ptr(out), _ptr(q), int(num_seqs), int(num_q_heads), _ptr(cu_q_lens),
                  int(total_q), int(max_q_len), _ptr(block_tables), int(max_blocks_per_seq), _ptr(context_lens),
                  int(max_context_len), float(softmax_scale), _ptr(dev_error), _stream(stream))
    return _check(st, "pkv_paged_attention_prefill", raise_on_error)


def pkv_paged_attention_decode_static(desc, out, q, num_seqs, num_q_heads, block_tables, max_blocks_per_seq,
                                      context_lens, max_context_len, softmax_scale, partition_tokens=0,
                                      dev_error=None, stream=None, raise_on_error=True):
    """Decode without a workspace, for callers that cannot provide scratch memory; uses the
    library's own fixed device array (see include/pkv.h: calls must not overlap on the GPU)."""
    st = _decode_static(ctypes.byref(desc), _ptr(out), _ptr(q), int(num_seqs), int(num_q_heads), _ptr(block_tables),
                        int(max_blocks_per_seq), _ptr(context_lens), int(max_context_len), float(softmax_scale),
                        int(partition_tokens), _ptr(dev_error), _stream(stream))
    return _check(st, "pkv_paged_attention_decode_static", raise_on_error)


def pkv_static_scratch_address():
    """(device address, bytes) of the static decode's array on the current device (diagnostics)."""
    ptr, n = _P(), ctypes.c_size_t(0)
    _check(_static_addr(ctypes.byref(ptr), ctypes.byref(n)), "pkv_static_scratch_address", True)
    return int(ptr.value or 0), int(n.value)


def pkv_copy_blocks(desc, block_mapping, n_pairs, dev_error=None, stream=None, raise_on_error=True):
    st = _copy(ctypes.byref(desc), _ptr(block_mapping), int(n_pairs), _ptr(dev_error), _stream(stream))
    return _check(st, "pkv_copy_blocks", raise_on_error)


def pkv_swap_blocks(device_desc, host_desc, block_mapping, n_pairs, direction, dev_error=None, stream=None,
                    raise_on_error=True):
    """Whole blocks device pool -> host pool (PKV_SWAP_OUT) or back (PKV_SWAP_IN); the host pool's
    arrays must be pinned host memory (e.g. torch tensors from pin_memory())."""
    st = _swap(ctypes.byref(device_desc), ctypes.byref(host_desc), _ptr(block_mapping), int(n_pairs), int(direction),
               _ptr(dev_error), _stream(stream))
    return _check(st, "pkv_swap_blocks", raise_on_error)


def pkv_decode_step(desc, block_mapping, n_pairs, k_new, v_new, slot_mapping, T, out, q, num_seqs, num_q_heads,
                    block_tables, max_blocks_per_seq, context_lens, max_context_len, softmax_scale,
                    partition_tokens=0, workspace=None, workspace_bytes=0, dev_error=None, stream=None,
                    raise_on_error=True):
    """Copies, store and decode of one step in one launch (the three calls above, in that order)."""
    st = _step(ctypes.byref(desc), _ptr(block_mapping), int(n_pairs), _ptr(k_new), _ptr(v_new), _ptr(slot_mapping),
               int(T), _ptr(out), _ptr(q), int(num_seqs), int(num_q_heads), _ptr(block_tables),
               int(max_blocks_per_seq), _ptr(context_lens), int(max_context_len), float(softmax_scale),
               int(partition_tokens), _ptr(workspace), int(workspace_bytes), _ptr(dev_error), _stream(stream))
    return _check(st, "pkv_decode_step", raise_on_error)


# ---- host allocator ----

def pkv_blocks_for_tokens(num_tokens: int, block_size: int) -> int:
    return int(_blocks_for_tokens(int(num_tokens), int(block_size)))


class Allocator:
    """Owning wrapper of a pkv_allocator handle (host memory)."""

    def __init__(self, num_blocks: int):
        h = _P()
        _check(_alloc_create(int(num_blocks), ctypes.byref(h)), "pkv_alloc_create", True)
        self._h = h

    def close(self):
        if self._h:
            _alloc_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    @property
    def num_free(self) -> int:
        return int(_alloc_num_free(self._h))

    def refcount(self, block_id: int) -> int:
        return int(_alloc_refcount(self._h, int(block_id)))

    def alloc(self, n: int, raise_on_error=True):
        ids = (ctypes.c_int32 * max(n, 1))()
        st = _alloc_blocks(self._h, int(n), ids)
        if st != PKV_OK:
            _check(st, "pkv_alloc_blocks", raise_on_error)
            return None
        return [int(ids[i]) for i in range(n)]

    def fork(self, ids, raise_on_error=True):
        arr = (ctypes.c_int32 * max(len(ids), 1))(*ids)
        return _check(_alloc_fork(self._h, arr, len(ids)), "pkv_alloc_fork", raise_on_error)

    def release(self, ids, raise_on_error=True):
        arr = (ctypes.c_int32 * max(len(ids), 1))(*ids)
        return _check(_alloc_release(self._h, arr, len(ids)), "pkv_alloc_release", raise_on_error)

    def cow(self, block_id: int, raise_on_error=True):
        new = _I32(-1)
        st = _alloc_cow(self._h, int(block_id), ctypes.byref(new))
        if st != PKV_OK:
            _check(st, "pkv_alloc_cow", raise_on_error)
            return None
        return int(new.value)


class PrefixCache:
    """Owning wrapper of a pkv_prefix_cache handle over an Allocator (which must outlive it)."""

    def __init__(self, allocator: Allocator, block_size: int):
        h = _P()
        _check(_pc_create(allocator._h, int(block_size), ctypes.byref(h)), "pkv_prefix_cache_create", True)
        self._h = h
        self.allocator = allocator
        self.block_size = int(block_size)

    def close(self):
        if self._h:
            _pc_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    @property
    def size(self) -> int:
        return int(_pc_size(self._h))

    @property
    def evictable(self) -> int:
        return int(_pc_evictable(self._h))

    @staticmethod
    def _tokens(tokens):
        arr = (ctypes.c_int32 * max(len(tokens), 1))(*[int(t) for t in tokens])
        return arr, len(tokens)

    def match(self, tokens, max_blocks=None):
        """Physical ids of the longest cached whole-block prefix (each gains a caller reference)."""
        arr, n = self._tokens(tokens)
        mb = n // self.block_size if max_blocks is None else int(max_blocks)
        out = (ctypes.c_int32 * max(mb, 1))()
        got = _I32(0)
        _check(_pc_match(self._h, arr, n, out, mb, ctypes.byref(got)), "pkv_prefix_match", True)
        return [int(out[i]) for i in range(got.value)]

    def insert(self, tokens, block_ids, raise_on_error=True):
        arr, n = self._tokens(tokens)
        ids = (ctypes.c_int32 * max(len(block_ids), 1))(*[int(b) for b in block_ids])
        return _check(_pc_insert(self._h, arr, n, ids, len(block_ids)), "pkv_prefix_insert", raise_on_error)

    def alloc(self, n: int, raise_on_error=True):
        ids = (ctypes.c_int32 * max(n, 1))()
        st = _pc_alloc(self._h, int(n), ids)
        if st != PKV_OK:
            _check(st, "pkv_prefix_alloc", raise_on_error)
            return None
        return [int(ids[i]) for i in range(n)]


# ---- device pool (torch tensors used as plain device memory) ----

@dataclass
class DevicePool:
    """One layer's pool in device memory plus its pkv_cache_desc. Byte layout as in pkv.h."""

    desc: pkv_cache_desc
    k_codes: object
    v_codes: object
    k_scale: object
    v_scale: object
    v_zp: object

    @classmethod
    def allocate(cls, num_blocks, block_size, num_kv_heads, head_dim, k_dtype, v_dtype, device="cuda",
                 fill: int | None = None, pinned_host: bool = False):
        """Device pool, or with pinned_host=True a pool in page-locked host memory (a swap target)."""
        import torch

        def empty(shape, dtype):
            if pinned_host:
                return torch.empty(shape, dtype=dtype, device="cpu", pin_memory=True)
            return torch.empty(shape, dtype=dtype, device=device)

        def codes(dt):
            row = {PKV_FP16: 2 * head_dim, PKV_INT8_SYM: head_dim, PKV_INT4_ASYM: head_dim // 2,
                   PKV_FP8_E4M3: head_dim}[dt]
            return empty((num_blocks, num_kv_heads, block_size, row), torch.uint8)

        k = codes(k_dtype)
        v = codes(v_dtype)
        ks = empty((num_blocks, num_kv_heads), torch.float32)
        vs = empty((num_blocks, num_kv_heads), torch.float32)
        zp = empty((num_blocks, num_kv_heads), torch.uint8)
        if fill is not None:
            for t in (k, v, zp):
                t.fill_(fill)
            for t in (ks, vs):
                t.view(torch.uint8).fill_(fill)
        desc = pkv_cache_desc(num_blocks, block_size, num_kv_heads, head_dim, k_dtype, v_dtype,
                              k.data_ptr(), v.data_ptr(), ks.data_ptr(), vs.data_ptr(), zp.data_ptr())
        return cls(desc, k, v, ks, vs, zp)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.k_codes, self.v_codes, self.k_scale, self.v_scale,
                                                           self.v_zp))
