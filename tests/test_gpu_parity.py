"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the same seeded inputs.

Bar: quantized codes, scales, zero points, slot scatter and copy-on-write bytes bit-exact (whole
blocks, including never-written rows, starting from identically poisoned pools); attention output
(fp16) within max-abs 2e-3 of the oracle's binary64 result computed on the oracle's own codes.
Reduced sizes run the oracle over everything; full sizes (the benchmark's launch configuration)
compare sampled sequences.
"""
import numpy as np
import pytest
import torch

from paged_block_quantized_b200 import workloads as W
from _oracle_run import oracle_step

pytestmark = pytest.mark.gpu
TOL = 2e-3


def run_gpu(w, partition_tokens=None, fused=False):
    """Prefill, then one step: the three launches the benchmark times by default (copy kernel,
    store kernel, decode with a programmatic dependent launch), or the one-launch pkv_decode_step."""
    from paged_block_quantized_b200.step import DeviceStep
    g = DeviceStep(w, partition_tokens=partition_tokens)
    g.prefill()
    pre = g.pool_numpy()
    g.step(fused=fused)
    torch.cuda.synchronize()
    return g, pre


def assert_pool_equal(gpu_arrays, cache, phys, what):
    k, v, ks, vs, zp = gpu_arrays
    phys = np.asarray(phys)
    np.testing.assert_array_equal(k[phys], cache.k_codes, err_msg=f"{what}: K codes")
    np.testing.assert_array_equal(v[phys], cache.v_codes, err_msg=f"{what}: V codes")
    np.testing.assert_array_equal(ks[phys].view(np.uint32), cache.k_scale.view(np.uint32), err_msg=f"{what}: K scales")
    np.testing.assert_array_equal(vs[phys].view(np.uint32), cache.v_scale.view(np.uint32), err_msg=f"{what}: V scales")
    np.testing.assert_array_equal(zp[phys], cache.v_zp, err_msg=f"{what}: zero points")


def check(w, seqs=None, partition_tokens=None, fused=False):
    g, pre = run_gpu(w, partition_tokens, fused)
    o = oracle_step(w, seqs)
    assert all(e == 0 for e in o["errors"]), o["errors"]
    assert g.error() == 0
    assert_pool_equal(pre, o["prefill_cache"], o["phys"], "prefill store")
    assert_pool_equal(g.pool_numpy(), o["cache"], o["phys"], "after copy + append")
    out = g.out.float().cpu().numpy()[o["seqs"]]
    err = np.abs(out - o["out"]).max()
    assert err <= TOL, f"max abs error {err}"
    return g, o


REDUCED = {
    "tiny": {},
    "llama7b": dict(num_seqs=4),
    "llama7b_fp16": dict(num_seqs=4),
    "llama7b_fp8": dict(num_seqs=4),
    "long": dict(num_seqs=2, context_lens=[8192 + 37, 9001]),
    "gqa_prefix": dict(num_seqs=4, prefix_blocks=8, private_blocks=9),
    "mixed": dict(num_seqs=24, children=4),
}


@pytest.mark.parametrize("path", ["separate", "fused"])
@pytest.mark.parametrize("name", list(REDUCED))
def test_config_reduced_sizes(name, path):
    check(W.make(name, seed=0, **REDUCED[name]), fused=path == "fused")


FULL_SAMPLES = {
    "llama7b": [0, 7, 31],
    "llama7b_fp16": [3, 30],
    "llama7b_fp8": [0, 31],
    "long": [int(np.argmin(W.make("long").context_lens))],
    "gqa_prefix": [0, 33, 63],
    "mixed": None,  # a parent, its child and two others, chosen below
}


@pytest.mark.parametrize("path", ["separate", "fused"])
@pytest.mark.parametrize("name", list(FULL_SAMPLES))
def test_config_full_size_sampled(name, path):
    w = W.make(name, seed=0)
    seqs = FULL_SAMPLES[name]
    if seqs is None:
        src, dst = (int(x) for x in w.cow_pairs[0])
        child = int(np.nonzero((w.block_tables == dst).any(axis=1))[0][0])
        parent = int(np.nonzero((w.block_tables == src).any(axis=1))[0][0])
        seqs = [parent, child, 1, int(np.argmax(w.context_lens))]
    check(w, seqs, fused=path == "fused")


def test_split_matches_unsplit():
    w = W.make("llama7b", seed=1, num_seqs=3)
    g_small, o = check(w, partition_tokens=64)
    g_big, _ = check(w, partition_tokens=2048)
    a = g_small.out.float().cpu().numpy()
    b = g_big.out.float().cpu().numpy()
    assert np.abs(a - b).max() <= 1e-3


@pytest.mark.parametrize("case", [
    dict(head_dim=64, block_size=32, num_q_heads=4, num_kv_heads=4),
    dict(head_dim=256, block_size=16, num_q_heads=2, num_kv_heads=2),
    dict(head_dim=128, block_size=32, num_q_heads=8, num_kv_heads=4),
    dict(head_dim=128, block_size=16, num_q_heads=16, num_kv_heads=2),
    dict(head_dim=64, block_size=16, num_q_heads=12, num_kv_heads=4, v_dtype=W.INT4_ASYM),
    dict(head_dim=256, block_size=32, num_q_heads=4, num_kv_heads=1, v_dtype=W.INT4_ASYM),
    dict(head_dim=64, block_size=16, num_q_heads=4, num_kv_heads=2, k_dtype=W.FP16, v_dtype=W.FP16),
    # tensor-core engine: FP16 with 256-byte rows, INT8 with head_dim 256, block size 32, 4 heads
    dict(head_dim=128, block_size=16, num_q_heads=32, num_kv_heads=4, k_dtype=W.FP16, v_dtype=W.FP16),
    dict(head_dim=256, block_size=32, num_q_heads=16, num_kv_heads=2),
    dict(head_dim=64, block_size=32, num_q_heads=16, num_kv_heads=4, k_dtype=W.FP16, v_dtype=W.FP16),
    dict(head_dim=128, block_size=32, num_q_heads=16, num_kv_heads=4),
    # E4M3 cache: the tensor-core engine for every group size (1, 2, 4 and 8 heads per warp)
    dict(head_dim=128, block_size=16, num_q_heads=4, num_kv_heads=4, k_dtype=W.FP8_E4M3, v_dtype=W.FP8_E4M3),
    dict(head_dim=256, block_size=32, num_q_heads=8, num_kv_heads=4, k_dtype=W.FP8_E4M3, v_dtype=W.FP8_E4M3),
    dict(head_dim=128, block_size=32, num_q_heads=16, num_kv_heads=4, k_dtype=W.FP8_E4M3, v_dtype=W.FP8_E4M3),
    dict(head_dim=128, block_size=16, num_q_heads=16, num_kv_heads=2, k_dtype=W.FP8_E4M3, v_dtype=W.FP8_E4M3),
    # the tcgen05 grouped-query kernel: 8 or 16 query heads per KV head (one or two units), INT8 or
    # INT4 V, block size 16 or 32
    dict(head_dim=128, block_size=32, num_q_heads=16, num_kv_heads=2, v_dtype=W.INT4_ASYM),
    dict(head_dim=128, block_size=16, num_q_heads=32, num_kv_heads=2),
    dict(head_dim=128, block_size=32, num_q_heads=8, num_kv_heads=1),
    # one query head per KV head: INT8 K on the integer tensor cores with 32-token blocks (head_dim
    # 128 and 256), and the paired walk of 16-token blocks (two blocks per tile; the odd block
    # counts above leave the last tile of a unit half full)
    dict(head_dim=128, block_size=32, num_q_heads=4, num_kv_heads=4),
    dict(head_dim=128, block_size=32, num_q_heads=4, num_kv_heads=4, v_dtype=W.INT4_ASYM),
    dict(head_dim=256, block_size=32, num_q_heads=2, num_kv_heads=2),
    dict(head_dim=128, block_size=16, num_q_heads=4, num_kv_heads=4, v_dtype=W.INT4_ASYM),
    dict(head_dim=64, block_size=16, num_q_heads=4, num_kv_heads=4, v_dtype=W.INT4_ASYM),
    # INT4 V on the CUDA-core engine with 2 and 4 query heads per warp (per-head zero-point sums),
    # paired 16-token blocks and 32-token blocks
    dict(head_dim=128, block_size=16, num_q_heads=8, num_kv_heads=4, v_dtype=W.INT4_ASYM),
    dict(head_dim=64, block_size=16, num_q_heads=16, num_kv_heads=4, v_dtype=W.INT4_ASYM),
    dict(head_dim=64, block_size=32, num_q_heads=8, num_kv_heads=4, v_dtype=W.INT4_ASYM),
])
def test_shapes_and_groups(case):
    lens = [1, 2, 16, 17, 31, 32, 33, 100, 700]
    w = W.make("tiny", seed=2, num_seqs=len(lens), context_lens=lens, num_blocks=128, **case)
    check(w)


@pytest.mark.parametrize("pt", [64, 128, 512])
def test_partition_boundaries(pt):
    lens = [pt - 1, pt, pt + 1, 2 * pt, 2 * pt + 1, 5 * pt - 3]
    w = W.make("llama7b", seed=3, num_seqs=len(lens), context_lens=lens)
    check(w, partition_tokens=pt)


@pytest.mark.parametrize("pt", [0, 32768])
def test_long_sequence_split_and_whole(pt):
    # pt 0: every resident warp, each of the 32 heads cut across many warps (merge of many
    # partials); pt 32768: 32 workers, one whole head each (no merge)
    w = W.make("long", seed=4, num_seqs=1, context_lens=[32768])
    g, _ = check(w, partition_tokens=pt)
    if pt:
        assert g.num_workers == 32


@pytest.mark.parametrize("vt", [W.INT8_SYM, W.INT4_ASYM])
def test_gqa_long_context_many_splits(vt):
    # the tcgen05 grouped-query kernel with one long sequence: its blocks cut into many splits whose
    # partials the last split merges, next to a one-token sequence (one split, written directly)
    w = W.make("tiny", seed=6, num_seqs=2, context_lens=[20011, 5], num_blocks=1400, head_dim=128, block_size=16,
               num_q_heads=16, num_kv_heads=2, v_dtype=vt)
    assert _gqa_tc_shape(w)
    check(w)


def test_zero_length_and_empty_batch():
    from paged_block_quantized_b200 import pkv
    import oracle
    w = W.make("tiny", seed=5)
    g, o = check(w)
    lens = w.context_lens.copy()
    lens[1] = 0
    lens[3] = 1
    g.context_lens.copy_(torch.from_numpy(lens))
    g.decode()
    torch.cuda.synchronize()
    ref, err = oracle.decode(o["cache"], o["q"], o["tables"], lens, w.softmax_scale, max_context_len=w.max_context_len)
    assert err == 0 and g.error() == 0
    out = g.out.float().cpu().numpy()
    assert not out[1].any()
    assert np.abs(out - ref).max() <= TOL
    # no sequences / no tokens: accepted, nothing launched
    assert pkv.pkv_paged_attention_decode(g.pool.desc, g.out, g.q, 0, w.num_q_heads, g.block_tables,
                                          w.max_blocks_per_seq, g.context_lens, 0, 0.1) == pkv.PKV_OK
    assert pkv.pkv_store_quantized(g.pool.desc, g.k_new, g.v_new, g.step_slots, 0) == pkv.PKV_OK


@pytest.mark.parametrize("j", [0, 1, 2])
def test_bad_block_id_is_skipped_and_flagged(j):
    # a bad id in either block of a paired tile (the tiny cache walks two 16-token blocks per tile)
    import oracle
    w = W.make("tiny", seed=6)
    g, o = check(w)
    tables = o["tables"].copy()
    bad_gpu = g.block_tables.clone()
    bad_gpu[2, j] = w.num_blocks + 5
    tables[2, j] = len(o["phys"]) + 5
    from paged_block_quantized_b200 import pkv
    pkv.pkv_paged_attention_decode(g.pool.desc, g.out, g.q, w.num_seqs, w.num_q_heads, bad_gpu,
                                   w.max_blocks_per_seq, g.context_lens, w.max_context_len, w.softmax_scale,
                                   g.partition_tokens, g.workspace, g.ws_bytes, g.dev_error)
    torch.cuda.synchronize()
    assert g.error() == pkv.PKV_DEVERR_BLOCK_ID
    ref, err = oracle.decode(o["cache"], o["q"], tables, w.context_lens, w.softmax_scale)
    assert err == oracle.DEVERR_BLOCK_ID
    assert np.abs(g.out.float().cpu().numpy() - ref).max() <= TOL


def test_context_longer_than_table_is_flagged():
    from paged_block_quantized_b200 import pkv
    w = W.make("tiny", seed=7)
    g, _ = check(w)
    lens = g.context_lens.clone()
    lens[0] = w.max_blocks_per_seq * w.block_size + 1
    g.dev_error.zero_()
    # longer than both the table and max_context_len (which sizes the grid and workspace)
    pkv.pkv_paged_attention_decode(g.pool.desc, g.out, g.q, w.num_seqs, w.num_q_heads, g.block_tables,
                                   w.max_blocks_per_seq, lens, w.max_context_len, w.softmax_scale,
                                   g.partition_tokens, g.workspace, g.ws_bytes, g.dev_error)
    torch.cuda.synchronize()
    assert g.error() == pkv.PKV_DEVERR_CONTEXT_LEN
    # negative lengths are flagged too and treated as empty
    lens[0] = -3
    g.dev_error.zero_()
    pkv.pkv_paged_attention_decode(g.pool.desc, g.out, g.q, w.num_seqs, w.num_q_heads, g.block_tables,
                                   w.max_blocks_per_seq, lens, w.max_context_len, w.softmax_scale,
                                   g.partition_tokens, g.workspace, g.ws_bytes, g.dev_error)
    torch.cuda.synchronize()
    assert g.error() == pkv.PKV_DEVERR_CONTEXT_LEN
    assert not g.out[0].float().abs().sum().item()


def test_store_slot_errors_are_flagged():
    from paged_block_quantized_b200 import pkv
    w = W.make("tiny", seed=8)
    g, _ = check(w)
    for slots, code in (([w.num_blocks * w.block_size, -1, -1, -1], pkv.PKV_DEVERR_SLOT),
                        ([5, 7, -1, -1], pkv.PKV_DEVERR_SLOT_GROUP)):
        g.dev_error.zero_()
        st = torch.tensor(slots, dtype=torch.int64, device="cuda")
        pkv.pkv_store_quantized(g.pool.desc, g.k_new, g.v_new, st, 4, g.dev_error)
        torch.cuda.synchronize()
        assert g.error() == code


def test_append_rebuild_bit_exact():
    """Tokens far outside a tile's stored range force the rebuild path; bytes match the oracle."""
    import oracle
    from paged_block_quantized_b200 import pkv
    rng = np.random.default_rng(9)
    nb, bs, H, D = 8, 16, 4, 128
    for v_dtype in (W.INT8_SYM, W.INT4_ASYM):
        pool = pkv.DevicePool.allocate(nb, bs, H, D, W.INT8_SYM, v_dtype, fill=0xA5)
        c = oracle.OracleCache.empty(nb, bs, H, D, oracle.INT8_SYM, {1: oracle.INT8_SYM, 2: oracle.INT4_ASYM}[v_dtype])
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        # 5 tokens; appends of 1 that does not fit, 3 that fit, 2 that do not, 4 that do not
        plan = [(0, 5, 1.0), (5, 1, 50.0), (6, 3, 0.01), (9, 2, 30.0), (11, 4, 400.0)]
        for start, n, scale in plan:
            k = (rng.standard_normal((n, H, D)) * scale).astype(np.float16)
            v = (rng.standard_normal((n, H, D)) * scale - scale / 3).astype(np.float16)
            slots = 3 * bs + start + np.arange(n, dtype=np.int64)
            oracle.store(c, k, v, slots)
            pkv.pkv_store_quantized(pool.desc, torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(),
                                    torch.from_numpy(slots).cuda(), n, err)
        torch.cuda.synchronize()
        assert err.item() == 0
        np.testing.assert_array_equal(pool.k_codes.cpu().numpy().view(np.int8), c.k_codes)
        np.testing.assert_array_equal(pool.v_codes.cpu().numpy().view(c.v_codes.dtype), c.v_codes)
        np.testing.assert_array_equal(pool.k_scale.cpu().numpy().view(np.uint32), c.k_scale.view(np.uint32))
        np.testing.assert_array_equal(pool.v_scale.cpu().numpy().view(np.uint32), c.v_scale.view(np.uint32))
        np.testing.assert_array_equal(pool.v_zp.cpu().numpy(), c.v_zp)


@pytest.mark.parametrize("bs,D,kt,vt", [(32, 256, W.INT8_SYM, W.INT4_ASYM), (32, 128, W.INT8_SYM, W.INT8_SYM),
                                         (16, 64, W.FP16, W.INT4_ASYM), (16, 256, W.INT8_SYM, W.INT8_SYM),
                                         (32, 64, W.INT8_SYM, W.FP16), (16, 128, W.FP8_E4M3, W.FP8_E4M3),
                                         (32, 256, W.FP8_E4M3, W.FP8_E4M3), (16, 64, W.FP8_E4M3, W.FP8_E4M3)])
def test_token_by_token_appends_bit_exact(bs, D, kt, vt):
    """Decode-step appends one token at a time into every offset of a tile, with tokens that force a
    rebuild at early and late offsets (tiles larger than one batch of a rebuild's loads included),
    an all-zero first token (stored scale 0), and multi-token groups that rebuild late in the tile."""
    import oracle
    from paged_block_quantized_b200 import pkv
    rng = np.random.default_rng(21 + bs + D)
    nb, H = 6, 3
    ot = {W.FP16: oracle.FP16, W.INT8_SYM: oracle.INT8_SYM, W.INT4_ASYM: oracle.INT4_ASYM, W.FP8_E4M3: oracle.FP8_E4M3}
    pool = pkv.DevicePool.allocate(nb, bs, H, D, kt, vt, fill=0x5A)
    c = oracle.OracleCache.empty(nb, bs, H, D, ot[kt], ot[vt], poison=0x5A)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    grow = {3: 3.0, 9: 9.0, 17: 27.0, 25: 81.0, bs - 1: 300.0}

    def put(block, start, n, scale, zero=False):
        k = (rng.standard_normal((n, H, D)) * scale).astype(np.float16)
        v = (rng.standard_normal((n, H, D)) * scale + scale / 4).astype(np.float16)
        if zero:
            k[:] = 0
            v[:] = 0
        slots = block * bs + start + np.arange(n, dtype=np.int64)
        oracle.store(c, k, v, slots)
        pkv.pkv_store_quantized(pool.desc, torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(),
                                torch.from_numpy(slots).cuda(), n, err)

    for o in range(bs):                       # block 1: one token at a time, rebuilds at `grow`
        put(1, o, 1, grow.get(o, 0.5))
    put(2, 0, 1, 1.0, zero=True)              # block 2: zero tile, then non-zero tokens
    for o in range(1, bs):
        put(2, o, 1, 1.0 + o)
    put(4, 0, bs - 6, 1.0)                    # block 4: late group that rebuilds, then one that fits
    put(4, bs - 6, 4, 50.0)
    put(4, bs - 2, 2, 0.1)
    torch.cuda.synchronize()
    assert err.item() == 0
    got = (pool.k_codes.cpu().numpy(), pool.v_codes.cpu().numpy(), pool.k_scale.cpu().numpy().view(np.uint32),
           pool.v_scale.cpu().numpy().view(np.uint32), pool.v_zp.cpu().numpy())
    for b in (1, 2, 4):
        np.testing.assert_array_equal(got[0][b].reshape(-1), c.k_codes[b].view(np.uint8).reshape(-1))
        np.testing.assert_array_equal(got[1][b].reshape(-1), c.v_codes[b].view(np.uint8).reshape(-1))
        if kt != W.FP16:
            np.testing.assert_array_equal(got[2][b], c.k_scale[b].view(np.uint32))
        if vt != W.FP16:
            np.testing.assert_array_equal(got[3][b], c.v_scale[b].view(np.uint32))
        if vt == W.INT4_ASYM:
            np.testing.assert_array_equal(got[4][b], c.v_zp[b])


def _gqa_tc_shape(w):
    """True for the shapes the tcgen05 grouped-query kernel covers (INT8 K, INT8 or INT4 V, head_dim
    128, query heads in groups of 8): a library built with PKV_DECODE_GQA_TC=1 decodes them there,
    the default build on the stream-K kernel's tensor-core engine."""
    group = w.num_q_heads // w.num_kv_heads
    return (w.k_dtype == W.INT8_SYM and w.v_dtype in (W.INT8_SYM, W.INT4_ASYM) and w.head_dim == 128
            and group % 8 == 0)



@pytest.mark.parametrize("name,over", [("mixed", dict(num_seqs=24, children=4)), ("llama7b", dict(num_seqs=6)),
                                       ("gqa_prefix", dict(num_seqs=4, prefix_blocks=8, private_blocks=9)),
                                       ("llama7b_fp16", dict(num_seqs=3)), ("llama7b_fp8", dict(num_seqs=3))])
def test_fused_step_matches_separate_launches(name, over):
    """pkv_decode_step (copies, store and decode in one cooperative launch) gives the same pool
    bytes and the same outputs as the three separate calls, on several steps in a row (its grid
    barrier counters come back to zero every call)."""
    from paged_block_quantized_b200.step import DeviceStep
    w = W.make(name, seed=5, **over)
    gf, gs = DeviceStep(w), DeviceStep(w)
    for g in (gf, gs):
        g.prefill()
    for it in range(3):
        gf.step(fused=True)
        gs.step(fused=False)
        torch.cuda.synchronize()
        assert gf.error() == 0 and gs.error() == 0
        for a, b in zip(gf.pool_numpy(), gs.pool_numpy()):
            np.testing.assert_array_equal(a, b)
        # (both on the stream-K kernel; a library built with PKV_DECODE_GQA_TC=1 would decode the
        # separate GQA step on the tcgen05 kernel, the same attention rounded differently)
        np.testing.assert_array_equal(gf.out.cpu().numpy(), gs.out.cpu().numpy())
        # tickets (one per sequence and head group) and the two barrier counters lead the workspace
        group = w.num_q_heads // w.num_kv_heads
        mma = (w.k_dtype, w.v_dtype) in ((W.FP16, W.FP16), (W.FP8_E4M3, W.FP8_E4M3)) or (
            (w.k_dtype, w.v_dtype) == (W.INT8_SYM, W.INT8_SYM) and w.head_dim >= 128)
        gt = 8 if mma and group % 8 == 0 else 4 if group % 4 == 0 else 2 if group % 2 == 0 else 1
        units = w.num_seqs * (w.num_q_heads // gt)
        ws = gf.workspace.view(torch.int32)[: units + 2].cpu().numpy()
        assert (ws == 0).all(), "tickets and barrier counters must be back at zero"


def test_copy_blocks_bit_exact_and_bad_ids():
    import oracle
    from paged_block_quantized_b200 import pkv
    w = W.make("mixed", seed=10, num_seqs=12, children=2)
    g, o = check(w)
    before = g.pool_numpy()
    pairs = np.array([[1, 40], [7, 41], [w.num_blocks - 1, 0]], np.int32)
    gp = torch.from_numpy(pairs).cuda()
    pkv.pkv_copy_blocks(g.pool.desc, gp, 3, g.dev_error)
    torch.cuda.synchronize()
    after = g.pool_numpy()
    for a, b in zip(before, after):
        exp = a.copy()
        exp[pairs[:, 1]] = a[pairs[:, 0]]
        np.testing.assert_array_equal(b.view(np.uint8), exp.view(np.uint8))
    g.dev_error.zero_()
    pkv.pkv_copy_blocks(g.pool.desc, torch.tensor([[0, w.num_blocks]], dtype=torch.int32, device="cuda"), 1,
                        g.dev_error)
    torch.cuda.synchronize()
    assert g.error() == pkv.PKV_DEVERR_BLOCK_ID
    np.testing.assert_array_equal(g.pool_numpy()[0], after[0])


@pytest.mark.parametrize("name,over,walk", [("mixed", dict(num_seqs=24, children=4), "beam"), ("mixed", {}, "beam"),
                                           ("mixed", dict(num_seqs=24, children=4), "aligned"),
                                           ("mixed", {}, "aligned")])
def test_walk_order(name, over, walk):
    """pkv_paged_attention_decode_ex with a walk order (every forked child right after its parent, or
    sharing sequences a whole number of worker ranges apart) gives the oracle's outputs (reduced and
    full size), and an order entry outside the batch is skipped and flagged, never a fault or a
    hang."""
    from paged_block_quantized_b200 import pkv
    from paged_block_quantized_b200.step import DeviceStep
    w = W.make(name, seed=0, **over)
    g = DeviceStep(w, walk=walk)
    assert g.seq_order is not None
    g.prefill()
    g.step()
    torch.cuda.synchronize()
    assert g.error() == 0
    seqs = None if over else [int(s) for s in g.seq_order[:6].cpu()] + [int(np.argmax(w.context_lens))]
    o = oracle_step(w, seqs)
    out = g.out.float().cpu().numpy()[o["seqs"]]
    assert np.abs(out - o["out"]).max() <= TOL
    bad = g.seq_order.clone()
    bad[1] = w.num_seqs + 3
    g.dev_error.zero_()
    pkv.pkv_paged_attention_decode_ex(g.pool.desc, g.out, g.q, w.num_seqs, w.num_q_heads, g.block_tables,
                                      w.max_blocks_per_seq, g.context_lens, w.max_context_len, w.softmax_scale, 0,
                                      bad, g.workspace, g.ws_bytes, g.dev_error)
    torch.cuda.synchronize()
    assert g.error() == pkv.PKV_DEVERR_SEQ_ORDER


@pytest.mark.parametrize("name,over,seqs,beam", [
    ("gqa_prefix", dict(num_seqs=4, prefix_blocks=8, private_blocks=9), None, False),
    ("gqa_prefix", dict(num_seqs=5, prefix_blocks=3, private_blocks=2, block_size=32), None, False),
    ("gqa_prefix", dict(num_seqs=40, prefix_blocks=2, private_blocks=1), None, False),  # a group > 128 columns
    ("mixed", dict(num_seqs=24, children=4), None, False),
    ("mixed", dict(num_seqs=24, children=4), None, True),
    ("gqa_prefix", {}, [0, 33, 63], False),
    ("mixed", {}, "pairs", True),
])
def test_shared_prefix_decode(name, over, seqs, beam):
    """pkv_paged_attention_decode_ex with shared-prefix groups (each shared block attended once per
    group by the prefix pass, merged into the decode) gives the oracle's outputs."""
    from paged_block_quantized_b200.step import DeviceStep
    w = W.make(name, seed=0, **over)
    g = DeviceStep(w, shared_prefix=True, beam_order=beam)
    assert g.prefix is not None
    g.prefill()
    g.step()
    torch.cuda.synchronize()
    assert g.error() == 0
    if seqs == "pairs":  # two parent/child pairs and the longest sequence
        members = g.members.cpu().numpy()
        seqs = [int(x) for x in members[:4]] + [int(np.argmax(w.context_lens))]
    o = oracle_step(w, seqs)
    out = g.out.float().cpu().numpy()[o["seqs"]]
    err = np.abs(out - o["out"]).max()
    assert err <= TOL, f"max abs error {err}"


def test_shared_prefix_count_beyond_the_sequence_is_flagged():
    from paged_block_quantized_b200 import pkv
    from paged_block_quantized_b200.step import DeviceStep
    w = W.make("gqa_prefix", seed=1, num_seqs=3, prefix_blocks=2, private_blocks=1)
    g = DeviceStep(w, shared_prefix=True)
    g.prefill()
    g.step()
    torch.cuda.synchronize()
    ref = g.out.clone()
    # a count covering every block of the sequences: clamped to leave the last block, reported
    g.shared_blocks.fill_(3)
    g.prefix["max_shared_blocks"] = 3
    g.ws_bytes = pkv.pkv_decode_ex_workspace_size(g.pool.desc, w.num_seqs, w.num_q_heads, w.max_context_len,
                                                  g.partition_tokens, None, g.prefix)
    g.workspace = torch.zeros(g.ws_bytes, dtype=torch.uint8, device="cuda")
    g.dev_error.zero_()
    g.decode()
    torch.cuda.synchronize()
    assert g.error() == pkv.PKV_DEVERR_SHARED
    assert (g.out.float() - ref.float()).abs().max().item() <= 1e-3
