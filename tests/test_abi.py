"""The C-ABI library loads without a GPU, exports every function include/pkv.h declares, and
rejects bad arguments on the host before any launch (no CUDA device needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pkv():
    from paged_block_quantized_b200 import build
    build.build()
    from paged_block_quantized_b200 import pkv as mod
    return mod


def declared_functions():
    text = open(os.path.join(ROOT, "include", "pkv.h")).read()
    return sorted(set(re.findall(r"PKV_API\s+[\w\s\*]+?\b(pkv_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(pkv):
    names = declared_functions()
    assert len(names) >= 16
    lib = ctypes.CDLL(pkv.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(pkv.EXPORTED) == names


def desc(pkv, **kw):
    d = dict(num_blocks=8, block_size=16, num_kv_heads=2, head_dim=64, k_dtype=pkv.PKV_INT8_SYM,
             v_dtype=pkv.PKV_INT4_ASYM, k_codes=0x1000, v_codes=0x2000, k_scale=0x3000, v_scale=0x4000,
             v_zp=0x5000)
    d.update(kw)
    return pkv.pkv_cache_desc(**d)


def test_status_strings(pkv):
    assert pkv.pkv_status_string(pkv.PKV_OK) == "PKV_OK"
    assert pkv.pkv_status_string(pkv.PKV_ERR_UNSUPPORTED) == "PKV_ERR_UNSUPPORTED"
    assert pkv.pkv_status_string(99) == "PKV_ERR_UNKNOWN"


def test_tile_bytes(pkv):
    d = desc(pkv)
    assert pkv.pkv_tile_bytes(d, 0) == 16 * 64
    assert pkv.pkv_tile_bytes(d, 1) == 16 * 32
    assert pkv.pkv_tile_bytes(desc(pkv, k_dtype=pkv.PKV_FP16), 0) == 16 * 128


@pytest.mark.parametrize("bad,code", [
    (dict(block_size=8), "PKV_ERR_UNSUPPORTED"),
    (dict(head_dim=96), "PKV_ERR_UNSUPPORTED"),
    (dict(head_dim=72), "PKV_ERR_INVALID_ARG"),
    (dict(num_blocks=0), "PKV_ERR_INVALID_ARG"),
    (dict(k_dtype=2), "PKV_ERR_INVALID_ARG"),      # INT4 is V-only
    (dict(v_dtype=7), "PKV_ERR_INVALID_ARG"),
    (dict(k_codes=0x1001), "PKV_ERR_INVALID_ARG"),  # misaligned
    (dict(v_zp=0), "PKV_ERR_INVALID_ARG"),          # INT4 needs zero points
    (dict(k_scale=0), "PKV_ERR_INVALID_ARG"),
])
def test_descriptor_validation(pkv, bad, code):
    d = desc(pkv, **bad)
    st = pkv.pkv_store_quantized(d, 0x6000, 0x7000, 0x8000, 4, stream=0, raise_on_error=False)
    assert pkv.pkv_status_string(st) == code
    st = pkv.pkv_copy_blocks(d, 0x6000, 1, stream=0, raise_on_error=False)
    assert pkv.pkv_status_string(st) == code


def test_call_validation(pkv):
    """Every call here is rejected on the host before any launch (the pointers are fake)."""
    d = desc(pkv)
    E = pkv.PKV_ERR_INVALID_ARG
    assert pkv.pkv_store_quantized(d, 0x6000, 0x7000, 0x8000, -1, stream=0, raise_on_error=False) == E
    assert pkv.pkv_store_quantized(d, 0x6008, 0x7000, 0x8000, 1, stream=0, raise_on_error=False) == E
    assert pkv.pkv_store_quantized(d, None, 0x7000, 0x8000, 1, stream=0, raise_on_error=False) == E
    assert pkv.pkv_store_quantized(d, 0x6000, 0x7000, 0x8000, 0, stream=0, raise_on_error=False) == pkv.PKV_OK
    assert pkv.pkv_copy_blocks(d, 0x6000, -2, stream=0, raise_on_error=False) == E
    assert pkv.pkv_copy_blocks(d, 0x6000, 0, stream=0, raise_on_error=False) == pkv.PKV_OK
    big = 1 << 40  # a (fake) workspace large enough for any size, so that the intended check fires
    dec = lambda **kw: pkv.pkv_paged_attention_decode(
        d, kw.get("out", 0x9000), kw.get("q", 0xA000), kw.get("S", 2), kw.get("Hq", 4), 0xB000,
        kw.get("mbps", 4), 0xC000, kw.get("max_len", 64), kw.get("scale", 0.125), kw.get("pt", 0),
        kw.get("ws", 0xD000), kw.get("ws_bytes", big), stream=0, raise_on_error=False)
    assert dec(Hq=3) == E                        # not a multiple of the KV heads
    assert dec(q=0xA004) == E                    # misaligned
    assert dec(out=None) == E
    assert dec(mbps=0) == E
    assert dec(pt=24) == E                       # not a multiple of the block size
    assert dec(pt=-16) == E
    assert dec(scale=float("nan")) == E
    assert dec(max_len=-1) == E
    assert dec(S=-1) == E
    assert dec(S=0) == pkv.PKV_OK                # nothing to do
    assert dec(ws=None) == E                     # a workspace is required
    assert dec(ws_bytes=16) == E                 # too small
    assert dec(ws=0xD004) == E                   # misaligned
    assert pkv.pkv_paged_attention_decode(desc(pkv, k_dtype=pkv.PKV_FP16), 0x9000, 0xA000, 2, 4, 0xB000, 4,
                                          0xC000, 64, 0.1, 0, 0xD000, big, stream=0,
                                          raise_on_error=False) == pkv.PKV_ERR_UNSUPPORTED
    # a pool beyond 2^31 - 1 token rows per cache side: the tile copies' row coordinate is 32-bit
    huge = desc(pkv, num_blocks=(1 << 26), num_kv_heads=2, block_size=16)  # 2^31 rows
    assert pkv.pkv_paged_attention_decode(huge, 0x9000, 0xA000, 2, 4, 0xB000, 4, 0xC000, 64, 0.1, 0, 0xD000,
                                          big, stream=0, raise_on_error=False) == pkv.PKV_ERR_UNSUPPORTED
    with pytest.raises(pkv.PkvError):
        pkv.pkv_decode_workspace_size(huge, 2, 4, 64, 0)
    just = desc(pkv, num_blocks=(1 << 26) - 1, num_kv_heads=2, block_size=16)  # 2^31 - 32 rows
    assert pkv.pkv_decode_workspace_size(just, 2, 4, 64, 0) > 0


def test_step_validation(pkv):
    """pkv_decode_step checks the arguments of its three parts on the host, before any launch (fake
    pointers), with the same answers as the separate calls."""
    d = desc(pkv)
    E = pkv.PKV_ERR_INVALID_ARG
    big = 1 << 40

    def step(**kw):
        return pkv.pkv_decode_step(
            kw.get("desc", d), kw.get("mapping", 0x6000), kw.get("n_pairs", 1), kw.get("k_new", 0x7000),
            kw.get("v_new", 0x7800), kw.get("slots", 0x8000), kw.get("T", 2), kw.get("out", 0x9000), 0xA000,
            kw.get("S", 2), 4, 0xB000, 4, 0xC000, 64, 0.125, 0, kw.get("ws", 0xD000), kw.get("ws_bytes", big),
            stream=0, raise_on_error=False)

    assert step(n_pairs=-1) == E
    assert step(T=-1) == E
    assert step(mapping=None) == E                  # copies requested without a mapping
    assert step(mapping=0x6002) == E                # misaligned mapping
    assert step(k_new=0x7008) == E                  # misaligned new values
    assert step(slots=None) == E
    assert step(out=None) == E
    assert step(ws=None) == E
    assert step(ws_bytes=16) == E
    assert step(desc=desc(pkv, block_size=8)) == pkv.PKV_ERR_UNSUPPORTED
    assert step(desc=desc(pkv, k_dtype=pkv.PKV_FP16, v_dtype=pkv.PKV_INT8_SYM)) == pkv.PKV_ERR_UNSUPPORTED
    # nothing at all to do: no copies, no tokens, no sequences
    assert step(n_pairs=0, T=0, S=0, mapping=None, k_new=None, v_new=None, slots=None) == pkv.PKV_OK


def test_partitioning(pkv):
    d = desc(pkv)
    workers, ctas = pkv.pkv_decode_partitioning(d, 200, 4, 1000, 0)  # a batch that fills the device
    wpc = workers // ctas                      # one CTA per SM, 8 to 16 warps by engine
    assert ctas > 0 and workers % ctas == 0 and wpc in (8, 12, 16)
    up = lambda n: -(-n // wpc) * wpc          # worker counts are whole CTAs
    # a small batch: about one worker per 4 blocks of the largest possible work (2 x 2 x 63)
    assert pkv.pkv_decode_partitioning(d, 2, 4, 1000, 0)[0] == up(63)
    # with partition_tokens: about one worker per partition_tokens tokens of the largest work
    # (2 seqs x 2 head groups x 63 blocks = 252 blocks, 8 blocks each -> 32 workers)
    w2, c2 = pkv.pkv_decode_partitioning(d, 2, 4, 1000, 128)
    assert w2 == up(32) and c2 == w2 // wpc
    w3, _ = pkv.pkv_decode_partitioning(d, 2, 4, 1000, 1 << 20)   # never fewer than one CTA of warps
    assert w3 == wpc
    w4, _ = pkv.pkv_decode_partitioning(d, 2, 4, 1000, 16)        # one block each: 252 workers
    assert w4 == up(252)
    w5, _ = pkv.pkv_decode_partitioning(d, 200, 4, 1000, 16)      # never more than fit on the device
    assert w5 == workers


def test_workspace_size(pkv):
    """Tickets per (sequence, head group), then one partial slot per (sequence, head group) and per
    worker: sizes follow the batch shape and the worker count, never the cache size."""
    d = desc(pkv)  # D 64, 2 KV heads; 4 query heads -> groups of 2 handled together
    def expect(S, Hq, workers, gt=2, D=64):
        units = S * (Hq // gt)
        slots = units + workers
        pad = lambda x: (x + 255) // 256 * 256
        return pad(units * 4) + pad(slots * gt * 2 * 4) + slots * gt * D * 4
    for S, L, pt in ((2, 64, 0), (3, 1000, 128), (8, 32768, 0), (1, 16, 0)):
        workers, _ = pkv.pkv_decode_partitioning(d, S, 4, L, pt)
        assert pkv.pkv_decode_workspace_size(d, S, 4, L, pt) == expect(S, 4, workers)
    assert pkv.pkv_decode_workspace_size(d, 0, 4, 64, 0) == 0
    # independent of the context length once the device is full (no copy of the cache)
    assert pkv.pkv_decode_workspace_size(d, 64, 4, 8192, 0) == pkv.pkv_decode_workspace_size(d, 64, 4, 32768, 0)


def test_swap_validation(pkv):
    """pkv_swap_blocks refuses mismatched pools, a bad direction and bad counts on the host before
    it looks at where the memory lives (fake pointers, no device needed)."""
    d = desc(pkv)
    E = pkv.PKV_ERR_INVALID_ARG
    swap = lambda h, n=1, direction=pkv.PKV_SWAP_OUT, mapping=0x6000: pkv.pkv_swap_blocks(
        d, h, mapping, n, direction, stream=0, raise_on_error=False)
    # a smaller host pool is fine; the fake pointers are then refused by the memory-kind check (or,
    # without a device, the device query fails): never a launch
    assert swap(desc(pkv, num_blocks=4)) in (E, pkv.PKV_ERR_CUDA)
    assert swap(desc(pkv, head_dim=128)) == E            # geometry must match
    assert swap(desc(pkv, num_kv_heads=4)) == E
    assert swap(desc(pkv, block_size=32)) == E
    assert swap(desc(pkv, v_dtype=pkv.PKV_INT8_SYM, v_zp=0)) == E
    assert swap(desc(pkv), direction=2) == E
    assert swap(desc(pkv), n=-1) == E
    assert swap(desc(pkv), mapping=None) == E
    assert swap(desc(pkv), mapping=0x6002) == E
    assert swap(desc(pkv), n=0) == pkv.PKV_OK
    assert swap(desc(pkv, k_codes=0x1008)) == E          # a misaligned host array


def test_decode_ex_options_validation(pkv):
    """pkv_paged_attention_decode_ex / pkv_decode_ex_workspace_size check their options on the host
    (fake pointers, no device): the struct size, the shared-prefix bounds and the cache types the
    shared-prefix pass is built for; the shared-prefix pass adds its partials to the workspace."""
    import ctypes
    d = desc(pkv, head_dim=128, v_dtype=pkv.PKV_INT8_SYM, v_zp=0)
    prefix = dict(group_start=0x6000, members=0x6100, shared_blocks=0x6200, num_groups=1, num_members=2,
                  max_group_size=2, max_shared_blocks=4)
    base = pkv.pkv_decode_workspace_size(d, 2, 4, 256, 0)
    assert pkv.pkv_decode_ex_workspace_size(d, 2, 4, 256, 0) == base
    with_prefix = pkv.pkv_decode_ex_workspace_size(d, 2, 4, 256, 0, None, prefix)
    assert with_prefix > base
    dec = lambda **kw: pkv.pkv_paged_attention_decode_ex(
        kw.get("desc", d), 0x9000, 0xA000, 2, 4, 0xB000, 16, 0xC000, 256, 0.1, 0, None, 0xD000,
        kw.get("ws_bytes", 1 << 40), stream=0, raise_on_error=False, prefix=kw.get("prefix", prefix))
    E = pkv.PKV_ERR_INVALID_ARG
    assert dec(ws_bytes=base) == E                                    # too small for the partials
    assert dec(prefix=dict(prefix, max_group_size=0)) == E
    assert dec(prefix=dict(prefix, members=None)) == E
    assert dec(prefix=dict(prefix, shared_blocks=0x6202)) == E         # misaligned
    fp16 = desc(pkv, head_dim=128, k_dtype=pkv.PKV_FP16, v_dtype=pkv.PKV_FP16, k_scale=0, v_scale=0, v_zp=0)
    assert dec(desc=fp16) == pkv.PKV_ERR_UNSUPPORTED                   # the pass is built for INT8 K
    # a struct of another size is refused
    opts = pkv.decode_options()
    opts.struct_bytes = ctypes.sizeof(pkv.pkv_decode_options) + 8
    st = pkv._decode_ex(ctypes.byref(d), 0x9000, 0xA000, 2, 4, 0xB000, 16, 0xC000, 256, 0.1, 0, ctypes.byref(opts),
                        0xD000, 1 << 40, None, 0)
    assert st == pkv.PKV_ERR_UNSUPPORTED


def test_prefill_validation(pkv):
    d = desc(pkv, head_dim=128, v_dtype=pkv.PKV_INT8_SYM, v_zp=0)
    E = pkv.PKV_ERR_INVALID_ARG
    pf = lambda **kw: pkv.pkv_paged_attention_prefill(
        kw.get("desc", d), kw.get("out", 0x9000), 0xA000, kw.get("S", 2), kw.get("Hq", 4), 0xB000,
        kw.get("T", 10), kw.get("maxq", 8), 0xC000, 16, 0xD000, 256, kw.get("scale", 0.1), stream=0,
        raise_on_error=False)
    assert pf(Hq=3) == E
    assert pf(out=None) == E
    assert pf(T=-1) == E
    assert pf(scale=float("nan")) == E
    assert pf(T=0) == pkv.PKV_OK and pf(S=0) == pkv.PKV_OK
    assert pf(desc=desc(pkv, head_dim=64, v_dtype=pkv.PKV_INT8_SYM, v_zp=0)) == pkv.PKV_ERR_UNSUPPORTED
    assert pf(desc=desc(pkv, head_dim=128, k_dtype=pkv.PKV_FP8_E4M3, v_dtype=pkv.PKV_FP8_E4M3,
                        v_zp=0)) == pkv.PKV_ERR_UNSUPPORTED
