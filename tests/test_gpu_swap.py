"""GPU: block swap between the device pool and a pinned host pool (pkv_swap_blocks).

Swap-out then swap-in of scattered blocks is a byte-exact round trip (codes, scales, zero points,
every head), a sequence whose blocks went out and came back under new ids decodes to the same
output bit for bit, bad ids are skipped and flagged, and host memory the device cannot address
(pageable) is refused on the host before anything is launched.
"""
import numpy as np
import pytest
import torch

from paged_block_quantized_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _pools(w, host_blocks):
    from paged_block_quantized_b200 import pkv
    from paged_block_quantized_b200.step import DeviceStep
    g = DeviceStep(w)
    g.prefill()
    g.step()
    torch.cuda.synchronize()
    host = pkv.DevicePool.allocate(host_blocks, w.block_size, w.num_kv_heads, w.head_dim, w.k_dtype, w.v_dtype,
                                   fill=0x3C, pinned_host=True)
    return g, host


def _arrays(pool):
    """The arrays a swap moves for this pool's dtypes: codes always, scales of quantized sides, zero
    points of INT4 V (the others are not part of the cache and keep whatever they held)."""
    from paged_block_quantized_b200 import pkv
    d = pool.desc
    arrs = [pool.k_codes, pool.v_codes]
    if d.k_dtype != pkv.PKV_FP16:
        arrs.append(pool.k_scale)
    if d.v_dtype != pkv.PKV_FP16:
        arrs.append(pool.v_scale)
    if d.v_dtype == pkv.PKV_INT4_ASYM:
        arrs.append(pool.v_zp)
    return [t.cpu().numpy().view(np.uint8) for t in arrs]


@pytest.mark.parametrize("name,over", [("mixed", dict(num_seqs=10, children=2)), ("llama7b_fp16", dict(num_seqs=3))])
def test_swap_round_trip_is_byte_exact(name, over):
    from paged_block_quantized_b200 import pkv
    w = W.make(name, seed=3, **over)
    g, host = _pools(w, host_blocks=64)
    # every block of sequence 1, out to scattered host ids, back in to free device ids
    nblk = (int(w.context_lens[1]) + w.block_size - 1) // w.block_size
    dev_ids = [int(b) for b in w.block_tables[1, :nblk]]
    host_ids = list(np.random.default_rng(0).permutation(64)[:nblk])
    used = set(int(b) for b in w.block_tables[w.block_tables >= 0]) | set(int(b) for b in w.cow_pairs.reshape(-1))
    free = [b for b in range(w.num_blocks) if b not in used][:nblk]
    assert len(free) == nblk
    before = _arrays(g.pool)
    out_map = torch.tensor(list(zip(dev_ids, host_ids)), dtype=torch.int32, device="cuda")
    pkv.pkv_swap_blocks(g.pool.desc, host.desc, out_map, nblk, pkv.PKV_SWAP_OUT, g.dev_error)
    torch.cuda.synchronize()
    assert g.error() == 0
    got_host = _arrays(host)
    for a, b in zip(before, got_host):
        np.testing.assert_array_equal(b[host_ids], a[dev_ids])
    in_map = torch.tensor(list(zip(host_ids, free)), dtype=torch.int32, device="cuda")
    pkv.pkv_swap_blocks(g.pool.desc, host.desc, in_map, nblk, pkv.PKV_SWAP_IN, g.dev_error)
    torch.cuda.synchronize()
    assert g.error() == 0
    after = _arrays(g.pool)
    for a, b in zip(before, after):
        np.testing.assert_array_equal(b[free], a[dev_ids])
        keep = np.ones(w.num_blocks, bool)
        keep[free] = False
        np.testing.assert_array_equal(b[keep], a[keep])  # nothing else touched
    # the sequence decodes identically from its new blocks
    ref = g.out.clone()
    tables = g.block_tables.clone()
    tables[1, :nblk] = torch.tensor(free, dtype=torch.int32, device="cuda")
    pkv.pkv_paged_attention_decode(g.pool.desc, g.out, g.q, w.num_seqs, w.num_q_heads, tables, w.max_blocks_per_seq,
                                   g.context_lens, w.max_context_len, w.softmax_scale, g.partition_tokens,
                                   g.workspace, g.ws_bytes, g.dev_error)
    torch.cuda.synchronize()
    assert torch.equal(g.out, ref)


def test_swap_bad_ids_and_unmapped_host_memory():
    from paged_block_quantized_b200 import pkv
    w = W.make("tiny", seed=4)
    g, host = _pools(w, host_blocks=8)
    before = _arrays(host)
    bad = torch.tensor([[0, 8], [w.num_blocks, 1], [2, 3]], dtype=torch.int32, device="cuda")
    pkv.pkv_swap_blocks(g.pool.desc, host.desc, bad, 3, pkv.PKV_SWAP_OUT, g.dev_error)
    torch.cuda.synchronize()
    assert g.error() == pkv.PKV_DEVERR_BLOCK_ID
    after = _arrays(host)
    dev = _arrays(g.pool)
    for a, b, d in zip(before, after, dev):
        np.testing.assert_array_equal(b[3], d[2])      # the good pair went through
        mask = np.ones(8, bool)
        mask[3] = False
        np.testing.assert_array_equal(b[mask], a[mask])  # nothing else written
    # pageable host memory cannot be reached by the device: refused on the host
    pageable = pkv.DevicePool.allocate(8, w.block_size, w.num_kv_heads, w.head_dim, w.k_dtype, w.v_dtype,
                                       device="cpu")
    ok = torch.tensor([[0, 0]], dtype=torch.int32, device="cuda")
    st = pkv.pkv_swap_blocks(g.pool.desc, pageable.desc, ok, 1, pkv.PKV_SWAP_OUT, g.dev_error, raise_on_error=False)
    assert st == pkv.PKV_ERR_INVALID_ARG
    # a device pool given where the host pool belongs is refused too
    st = pkv.pkv_swap_blocks(g.pool.desc, g.pool.desc, ok, 1, pkv.PKV_SWAP_OUT, g.dev_error, raise_on_error=False)
    assert st == pkv.PKV_ERR_INVALID_ARG
