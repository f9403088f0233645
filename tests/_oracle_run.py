"""Run a workload's prefill + step + decode on the CPU oracle, for all sequences or a sample.

The oracle pool is compact: it holds only the physical blocks the chosen sequences reference,
renumbered 0..n-1 in increasing physical order. Per-block quantization only depends on a
block's own values and grouping, so the compact pool's bytes must equal the GPU pool's bytes for
the same physical blocks.
"""
from __future__ import annotations

import numpy as np

import oracle


def _odt(dt):
    return {0: oracle.FP16, 1: oracle.INT8_SYM, 2: oracle.INT4_ASYM, 3: oracle.FP8_E4M3}[dt]


def oracle_step(w, seqs=None, num_threads=None):
    S, bs = w.num_seqs, w.block_size
    seqs = list(range(S)) if seqs is None else sorted(set(int(s) for s in seqs))
    # blocks referenced before and after copy-on-write, and what fills each one in prefill
    fill = {}  # physical block -> (stream, logical index, tokens stored in prefill)
    used = set()
    for s in seqs:
        L = int(w.context_lens[s])
        nblk = (L + bs - 1) // bs
        n_pre = L - 1
        for j in range(nblk):
            used.add(int(w.block_tables[s, j]))
            b = int(w.prefill_tables[s, j])
            used.add(b)
            ntok = min(n_pre - j * bs, bs)
            if ntok > 0:
                fill[b] = (int(w.block_streams[s, j]), j, ntok)
    phys = sorted(used)
    remap = {b: i for i, b in enumerate(phys)}
    c = oracle.OracleCache.empty(len(phys), bs, w.num_kv_heads, w.head_dim, _odt(w.k_dtype), _odt(w.v_dtype))
    err_prefill = 0
    for b in phys:
        if b not in fill:
            continue
        stream, j, ntok = fill[b]
        k, v = w.block_values(stream, j)
        slots = remap[b] * bs + np.arange(ntok, dtype=np.int64)
        err_prefill |= oracle.store(c, k[:ntok], v[:ntok], slots)
    pre = c.copy()
    # copy-on-write pairs whose target belongs to the sample
    pairs = [(remap[int(a)], remap[int(b)]) for a, b in w.cow_pairs if int(b) in remap]
    err_copy = oracle.copy_blocks(c, np.array(pairs, np.int32).reshape(-1, 2)) if pairs else 0
    # the step's store: one token per sampled sequence at position L-1
    k_new, v_new = w.new_token_values()
    slots = []
    for s in seqs:
        p = int(w.context_lens[s]) - 1
        slots.append(remap[int(w.block_tables[s, p // bs])] * bs + p % bs)
    err_store = oracle.store(c, k_new[seqs], v_new[seqs], np.array(slots, np.int64))
    # decode
    tables = np.full((len(seqs), w.max_blocks_per_seq), -1, np.int32)
    for i, s in enumerate(seqs):
        nblk = (int(w.context_lens[s]) + bs - 1) // bs
        tables[i, :nblk] = [remap[int(b)] for b in w.block_tables[s, :nblk]]
    q = w.queries()[seqs]
    out, err_decode = oracle.decode(c, q, tables, w.context_lens[seqs], w.softmax_scale,
                                    max_context_len=w.max_context_len, num_threads=num_threads)
    return dict(seqs=seqs, out=out, cache=c, prefill_cache=pre, phys=phys, remap=remap, tables=tables, q=q,
                errors=(err_prefill, err_copy, err_store, err_decode))


def oracle_prefill_step(w, seqs=None, num_threads=None):
    """The chunked-prefill step of a workload with q_lens on the oracle: the prefix positions
    stored block by block, each chunk stored as one group per block, then oracle.prefill over the
    chosen sequences' chunks. Returns the outputs of those sequences' rows."""
    S, bs = w.num_seqs, w.block_size
    seqs = list(range(S)) if seqs is None else sorted(set(int(s) for s in seqs))
    used = sorted(set(int(b) for s in seqs for b in w.block_tables[s, :(int(w.context_lens[s]) + bs - 1) // bs]))
    remap = {b: i for i, b in enumerate(used)}
    c = oracle.OracleCache.empty(len(used), bs, w.num_kv_heads, w.head_dim, _odt(w.k_dtype), _odt(w.v_dtype))
    errors = []
    for s in seqs:
        L, q = int(w.context_lens[s]), int(w.q_lens[s])
        n_pre = L - q
        for j in range((n_pre + bs - 1) // bs):
            ntok = min(n_pre - j * bs, bs)
            k, v = w.block_values(w.block_streams[s, j], j)
            slots = remap[int(w.block_tables[s, j])] * bs + np.arange(ntok, dtype=np.int64)
            errors.append(oracle.store(c, k[:ntok], v[:ntok], slots))
    k_all, v_all, _ = w.chunk_tokens()
    cu = w.cu_q_lens
    q_all = w.chunk_queries()
    rows, cu_sel = [], [0]
    for s in seqs:
        L, q = int(w.context_lens[s]), int(w.q_lens[s])
        pos = np.arange(L - q, L)
        slots = np.array([remap[int(w.block_tables[s, t // bs])] * bs + t % bs for t in pos], np.int64)
        errors.append(oracle.store(c, k_all[cu[s]:cu[s + 1]], v_all[cu[s]:cu[s + 1]], slots))
        rows.extend(range(cu[s], cu[s + 1]))
        cu_sel.append(cu_sel[-1] + q)
    tables = np.full((len(seqs), w.max_blocks_per_seq), -1, np.int32)
    for i, s in enumerate(seqs):
        nblk = (int(w.context_lens[s]) + bs - 1) // bs
        tables[i, :nblk] = [remap[int(b)] for b in w.block_tables[s, :nblk]]
    out, err = oracle.prefill(c, q_all[rows], np.array(cu_sel, np.int32), tables, w.context_lens[seqs],
                              w.softmax_scale, num_threads=num_threads)
    errors.append(err)
    return dict(seqs=seqs, rows=np.array(rows), out=out, cache=c, phys=used, errors=errors)
