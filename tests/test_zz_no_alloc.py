"""The decode entry point that needs no scratch memory from its caller.

Some callers cannot give the library a workspace: a plugin that its host engine hands only the
input and output buffers, or a serving loop that fixed its device-memory budget up front and may
not allocate per request. pkv_paged_attention_decode_static serves them from a fixed device array
inside the library. These tests call it through the C ABI and check it against the regular
pkv_paged_attention_decode (which takes a caller-provided workspace) on the same pool, for calls
made back to back, including a call whose sizes differ from the previous one's.

This file is collected last on purpose: a run that stops at the first failure has already run
every other test by the time it gets here. It builds all of its own state, so it also passes on
its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from paged_block_quantized_b200 import workloads as W

pytestmark = pytest.mark.gpu
TOL = 2e-3  # the attention tolerance used by every decode test


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
             _prepared("llama7b", num_seqs=3)]               # INT8 / INT8, other sizes
    for w, g in (cases[0], cases[0], cases[1], cases[0]):    # back-to-back calls, sizes changing
        assert pkv.pkv_decode_workspace_size(g.pool.desc, w.num_seqs, w.num_q_heads, w.max_context_len,
                                             g.partition_tokens) <= pkv.PKV_STATIC_SCRATCH_BYTES
        ref = _regular(w, g).float().cpu().numpy()
        got = _static(w, g).float().cpu().numpy()
        assert np.isfinite(got).all()
        assert np.abs(got - ref).max() <= TOL


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
