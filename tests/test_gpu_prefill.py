"""GPU parity of chunked prefill (pkv_paged_attention_prefill) against the CPU oracle, through the
C ABI: the chunk's stored codes bit-exact, every output row within 2e-3 of the binary64 oracle,
across block sizes, V types, group sizes, chunk and prefix lengths (chunks shorter and longer than a
CTA's 128 columns, prefixes ending mid-block, empty prefixes), plus error reporting.
"""
import numpy as np
import pytest
import torch

from paged_block_quantized_b200 import workloads as W
from _oracle_run import oracle_prefill_step

pytestmark = pytest.mark.gpu
TOL = 2e-3


def run(w, seqs=None):
    from paged_block_quantized_b200.step import PrefillStep
    g = PrefillStep(w)
    g.prefill()
    g.step()
    torch.cuda.synchronize()
    assert g.error() == 0
    o = oracle_prefill_step(w, seqs)
    assert all(e == 0 for e in o["errors"]), o["errors"]
    # the chunk's codes and scales, byte for byte, on the blocks the sample uses
    k, v = g.pool.k_codes.cpu().numpy(), g.pool.v_codes.cpu().numpy()
    phys = np.asarray(o["phys"])
    np.testing.assert_array_equal(k[phys].reshape(-1), o["cache"].k_codes.view(np.uint8).reshape(-1))
    np.testing.assert_array_equal(v[phys].reshape(-1), o["cache"].v_codes.view(np.uint8).reshape(-1))
    got = g.out.float().cpu().numpy()[o["rows"]]
    err = np.abs(got - o["out"]).max()
    assert err <= TOL, f"max abs error {err}"
    return g, o


@pytest.mark.parametrize("case", [
    dict(num_seqs=3, chunk=40, prefix_lens=[0, 23, 100]),
    dict(num_seqs=2, chunk=200, prefix_lens=[7, 300]),                       # more than one CTA of columns
    dict(num_seqs=2, chunk=33, prefix_lens=[16, 45], block_size=32),
    dict(num_seqs=2, chunk=64, prefix_lens=[1, 70], v_dtype=W.INT4_ASYM),
    dict(num_seqs=2, chunk=70, prefix_lens=[31, 0], v_dtype=W.INT4_ASYM, block_size=32),
    dict(num_seqs=2, chunk=48, prefix_lens=[5, 90], num_q_heads=8, num_kv_heads=2),    # 4 heads per KV head
    dict(num_seqs=2, chunk=20, prefix_lens=[17, 0], num_q_heads=32, num_kv_heads=4),   # 8 heads per KV head
    dict(num_seqs=1, chunk=1, prefix_lens=[500]),                              # a one-token chunk: a decode
])
def test_prefill_matches_oracle(case):
    case = dict(case)
    case.setdefault("num_q_heads", 4)
    case.setdefault("num_kv_heads", 4)
    run(W.make("prefill", seed=1, **case))


def test_prefill_growing_scores_rescale_in_place():
    # K grows along the context, so a column's running maximum rises by more than 2^8 many times:
    # the accumulator in tensor memory is rescaled in place again and again
    w = W.make("prefill", seed=5, num_seqs=2, chunk=96, prefix_lens=[700, 333], num_q_heads=4, num_kv_heads=4,
               k_ramp=0.5)
    run(w)


def test_prefill_bad_block_id_is_flagged():
    from paged_block_quantized_b200 import pkv
    from paged_block_quantized_b200.step import PrefillStep
    w = W.make("prefill", seed=6, num_seqs=2, chunk=40, prefix_lens=[100, 60], num_q_heads=4, num_kv_heads=4)
    g = PrefillStep(w)
    g.prefill()
    g.step()
    torch.cuda.synchronize()
    ref = g.out.clone()
    tables = g.block_tables.clone()
    tables[0, 2] = w.num_blocks + 5  # one block of sequence 0 out of the pool
    g.dev_error.zero_()
    pkv.pkv_paged_attention_prefill(g.pool.desc, g.out, g.q, 2, 4, g.cu, g.total_q, g.max_q_len, tables,
                                    w.max_blocks_per_seq, g.context_lens, w.max_context_len, w.softmax_scale,
                                    g.dev_error)
    torch.cuda.synchronize()
    assert g.error() == pkv.PKV_DEVERR_BLOCK_ID
    assert torch.equal(g.out[40:], ref[40:])  # the other sequence is untouched
    assert torch.isfinite(g.out[:40].float()).all()


def test_prefill_full_size_sampled():
    w = W.make("prefill", seed=0)
    run(w, seqs=[0, int(np.argmax(w.context_lens))])


def test_prefill_errors_and_empty():
    from paged_block_quantized_b200 import pkv
    from paged_block_quantized_b200.step import PrefillStep
    w = W.make("prefill", seed=2, num_seqs=2, chunk=16, prefix_lens=[10, 20], num_q_heads=4, num_kv_heads=4)
    g = PrefillStep(w)
    g.prefill()
    g.step()
    torch.cuda.synchronize()
    # a chunk longer than its context: flagged, its rows zeroed, the other sequence untouched
    ref = g.out.clone()
    lens = g.context_lens.clone()
    lens[0] = 8
    g.dev_error.zero_()
    g.out.fill_(1.0)
    pkv.pkv_paged_attention_prefill(g.pool.desc, g.out, g.q, 2, 4, g.cu, g.total_q, g.max_q_len, g.block_tables,
                                    w.max_blocks_per_seq, lens, w.max_context_len, w.softmax_scale, g.dev_error)
    torch.cuda.synchronize()
    assert g.error() == pkv.PKV_DEVERR_CONTEXT_LEN
    assert not g.out[:16].float().abs().sum().item()
    assert torch.equal(g.out[16:], ref[16:])
    # nothing to do: accepted, nothing launched
    assert pkv.pkv_paged_attention_prefill(g.pool.desc, g.out, g.q, 0, 4, g.cu, 0, 0, g.block_tables,
                                           w.max_blocks_per_seq, lens, w.max_context_len, 0.1) == pkv.PKV_OK
    # unsupported cache types are refused on the host
    fp16 = pkv.DevicePool.allocate(4, 16, 4, 128, pkv.PKV_FP16, pkv.PKV_FP16)
    st = pkv.pkv_paged_attention_prefill(fp16.desc, g.out, g.q, 2, 4, g.cu, g.total_q, g.max_q_len, g.block_tables,
                                         w.max_blocks_per_seq, lens, w.max_context_len, 0.1, raise_on_error=False)
    assert st == pkv.PKV_ERR_UNSUPPORTED
