"""The decode entry point that needs no scratch memory from its caller.

Some callers cannot give the library a workspace: a plugin that its host engine hands only the
input and output buffers, or a serving loop that fixed its device-memory budget up front and may
not allocate per request. pkv_paged_attention_decode_static serves them from a fixed device array
inside the library. These tests call it through the C ABI and check it against the regular
pkv_paged_attention_decode (which takes a caller-provided workspace) on the same pool, for calls
made back to back, including a call whose sizes differ from the previous one's. Both run the same
kernel with the same work split on the same inputs, so their outputs must be identical bit for bit.

Before each call the whole array is filled with 0xFF, which is what a previous call that never
completed (or a stray write) could leave behind: the call must clear the part that has to start at
zero (the split-unit tickets) on its own, or some outputs are never written.

This file is collected last on purpose: a run that stops at the first failure has already run
every other test by the time it gets here. It builds all of its own state, so it also passes on
its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from paged_block_quantized_b200 import workloads as W

pytestmark = pytest.mark.gpu


class _Raw:
    """A device byte range seen by torch through the CUDA array interface (no copy, no ownership)."""

    def __init__(self, ptr, nbytes):
        self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1", "data": (ptr, False), "version": 3}


def _static_array():
    from paged_block_quantized_b200 import pkv
    ptr, nbytes = pkv.pkv_static_scratch_address()
    assert ptr != 0 and nbytes == pkv.PKV_STATIC_SCRATCH_BYTES
    return torch.as_tensor(_Raw(ptr, nbytes), device="cuda")


def _prepared(name, **over):
    from paged_block_quantized_b200.step import DeviceStep
    w = W.make(name, seed=11, **over)
    g = DeviceStep(w)
    g.prefill()
    g.copy()
    g.store()
    torch.cuda.synchronize()
    return w, g


def _regular(w, g):
    g.decode()
    torch.cuda.synchronize()
    assert g.error() == 0
    return g.out.clone()


def _static(w, g):
    from paged_block_quantized_b200 import pkv
    out = torch.full_like(g.out, float("nan"))
    pkv.pkv_paged_attention_decode_static(
        g.pool.desc, out, g.q, w.num_seqs, w.num_q_heads, g.block_tables, w.max_blocks_per_seq, g.context_lens,
        w.max_context_len, w.softmax_scale, g.partition_tokens, g.dev_error)
    torch.cuda.synchronize()
    assert g.error() == 0
    return out


def test_static_scratch_decode_matches_workspace_decode():
    from paged_block_quantized_b200 import pkv
    cases = [_prepared("mixed", num_seqs=12, children=2),   # INT8 K / INT4 V, forked sequences
             _prepared("llama7b", num_seqs=3),               # INT8 / INT8, other sizes
             _prepared("long", num_seqs=1, context_lens=[20000])]  # every head cut across many warps
    array = _static_array()
    for w, g in (cases[0], cases[0], cases[1], cases[2], cases[0]):  # back-to-back calls, sizes changing
        assert pkv.pkv_decode_workspace_size(g.pool.desc, w.num_seqs, w.num_q_heads, w.max_context_len,
                                             g.partition_tokens) <= pkv.PKV_STATIC_SCRATCH_BYTES
        ref = _regular(w, g).cpu().numpy()
        array.fill_(0xFF)  # what an interrupted call could leave: the call must clear its tickets itself
        torch.cuda.synchronize()
        got = _static(w, g).cpu().numpy()
        assert np.isfinite(got.astype(np.float32)).all()
        np.testing.assert_array_equal(got.view(np.uint16), ref.view(np.uint16))


def test_static_scratch_rejects_sizes_beyond_its_array():
    from paged_block_quantized_b200 import pkv
    w, g = _prepared("tiny")
    # a batch whose partials would not fit in the fixed array: rejected before anything runs
    S, Hq = 65535, 64
    assert pkv.pkv_decode_workspace_size(g.pool.desc, S, Hq, 64, 0) > pkv.PKV_STATIC_SCRATCH_BYTES
    st = pkv.pkv_paged_attention_decode_static(g.pool.desc, g.out, g.q, S, Hq, g.block_tables, w.max_blocks_per_seq,
                                               g.context_lens, 64, w.softmax_scale, 0, g.dev_error,
                                               raise_on_error=False)
    assert st == pkv.PKV_ERR_UNSUPPORTED


def test_static_scratch_rejected_call_writes_nothing():
    """Arguments are checked before anything is enqueued: a call rejected for a missing output
    leaves the array (and the output) exactly as they were."""
    from paged_block_quantized_b200 import pkv
    w, g = _prepared("tiny")
    array = _static_array()
    array.fill_(0xFF)
    before_out = g.out.clone()
    torch.cuda.synchronize()
    st = pkv.pkv_paged_attention_decode_static(g.pool.desc, None, g.q, w.num_seqs, w.num_q_heads, g.block_tables,
                                               w.max_blocks_per_seq, g.context_lens, w.max_context_len,
                                               w.softmax_scale, 0, g.dev_error, raise_on_error=False)
    assert st == pkv.PKV_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert bool((array == 0xFF).all().item()), "a rejected call wrote to the array"
    assert torch.equal(g.out, before_out)
