"""Seeded synthetic workloads for the decode step over a paged, block-quantized KV cache.

This module only produces inputs -- shapes, context lengths, physical block assignment, slot
mappings, copy-on-write pairs and fp16 token values. It contains none of the method's
arithmetic (no quantization, no attention), so both the GPU path and the CPU oracle can take
their inputs from it.

Every value is a deterministic function of (seed, what it is): token values of logical block j
of a value stream come from ``numpy.random.default_rng([seed, 11, stream, j])``, so any block
can be regenerated on its own (the oracle recomputes sampled sequences this way at full size).

A "step" is what one decode iteration does to the cache: copy-on-write copies for forked
sequences (if any), store of one new token per sequence at position L-1, then attention over
L tokens. Before the step the pool holds positions [0, L-1) of every sequence, stored
block by block ("prefill").

Named workloads (sizes from the pages' scenarios):
  tiny       4 seqs, L = {17, 33, 50, 64}, 4 heads MHA, D 64, bs 16, 64-block pool, INT8/INT8
  llama7b    32 seqs, L ~ U{500..2000}, 32 heads MHA, D 128, bs 16, 8192-block pool, INT8/INT8,
             K/V with 1% outlier channels x8 (``llama7b_fp16``: same with an FP16 cache;
             ``llama7b_fp8``: same with an FP8 E4M3 cache)
  long       8 seqs, L ~ U{8192..32768}, 32 heads, D 128, bs 32, K INT8 / V INT4 (the decode
             splits the long contexts across worker warps itself)
  gqa_prefix 64 seqs, 64 q heads / 8 KV heads, D 128, bs 16, 64 shared prefix blocks then 64
             private blocks each (L = 2048), INT8/INT8
  mixed      128 seqs, L = clamp(round(exp(N(ln 1000, 1))), 16, 16384), 32 heads, D 128, bs 16,
             K INT8 / V INT4, 16 beam children forked from 16 parents with a partial last block
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

FP16, INT8_SYM, INT4_ASYM, FP8_E4M3 = 0, 1, 2, 3

_VALUES, _NEWTOK, _OUTLIER, _LAYOUT, _QUERY = 11, 12, 13, 14, 15


@dataclass
class Workload:
    name: str
    seed: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    k_dtype: int
    v_dtype: int
    softmax_scale: float
    context_lens: np.ndarray          # int32 [S]: tokens attended in the step (after the append)
    block_tables: np.ndarray          # int32 [S][max_blocks]: final tables (after copy-on-write)
    block_streams: np.ndarray         # int64 [S][max_blocks]: value stream of each logical block
    prefill_tables: np.ndarray        # int32 [S][max_blocks]: tables before copy-on-write
    prefill_owner: np.ndarray         # bool  [S][max_blocks]: this seq stores this block in prefill
    cow_pairs: np.ndarray             # int32 [n][2]: (src, dst) copies the step makes
    partition_tokens: int = 0         # 0 = let the library choose
    q_lens: np.ndarray | None = None  # int32 [S]: chunked prefill, new tokens per sequence (None: decode)
    outliers: bool = False
    k_ramp: float = 0.0               # K of logical block j scaled by 1 + k_ramp * j (scores grow along the context)
    description: str = ""
    _mult: dict = field(default_factory=dict, repr=False)

    # ---- sizes ----
    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def total_tokens(self) -> int:
        return int(self.context_lens.sum())

    def unique_blocks(self) -> int:
        return int(np.unique(self.block_tables[self.block_tables >= 0]).size)

    # ---- values ----
    def _multipliers(self, which: str) -> np.ndarray:
        """Per-channel multipliers [H][D]: 1, or 8 for a seeded 1% of the channels."""
        if which not in self._mult:
            m = np.ones((self.num_kv_heads, self.head_dim), dtype=np.float32)
            if self.outliers:
                rng = np.random.default_rng([self.seed, _OUTLIER, 0 if which == "k" else 1])
                n_ch = self.num_kv_heads * self.head_dim
                idx = rng.choice(n_ch, size=max(1, round(0.01 * n_ch)), replace=False)
                m.reshape(-1)[idx] = 8.0
            self._mult[which] = m
        return self._mult[which]

    def _scaled(self, x: np.ndarray, which: str) -> np.ndarray:
        return (x * self._multipliers(which)).astype(np.float16)

    def block_values(self, stream: int, j: int):
        """fp16 K, V [bs][H][D] of logical block j of a value stream: N(0,1) draws in fp32 (K times
        1 + k_ramp * j), outlier channels scaled, rounded to fp16 (round to nearest)."""
        rng = np.random.default_rng([self.seed, _VALUES, int(stream), int(j)])
        shape = (self.block_size, self.num_kv_heads, self.head_dim)
        k = rng.standard_normal(shape, dtype=np.float32)
        v = rng.standard_normal(shape, dtype=np.float32)
        if self.k_ramp:
            k *= np.float32(1.0 + self.k_ramp * int(j))
        return self._scaled(k, "k"), self._scaled(v, "v")

    def seq_values(self, s: int, start: int, stop: int):
        """fp16 K, V [stop-start][H][D] of sequence s at positions [start, stop) as they are
        before the step's append (the prefill content)."""
        bs = self.block_size
        ks, vs = [], []
        for j in range(start // bs, (stop + bs - 1) // bs):
            k, v = self.block_values(self.block_streams[s, j], j)
            lo = max(start - j * bs, 0)
            hi = min(stop - j * bs, bs)
            ks.append(k[lo:hi])
            vs.append(v[lo:hi])
        H, D = self.num_kv_heads, self.head_dim
        if not ks:
            return np.zeros((0, H, D), np.float16), np.zeros((0, H, D), np.float16)
        return np.concatenate(ks), np.concatenate(vs)

    def new_token_values(self):
        """fp16 K, V [S][H][D]: the token each sequence appends in the step (position L-1)."""
        shape = (self.num_seqs, self.num_kv_heads, self.head_dim)
        k = np.empty(shape, np.float16)
        v = np.empty(shape, np.float16)
        for s in range(self.num_seqs):
            rng = np.random.default_rng([self.seed, _NEWTOK, s])
            ramp = np.float32(1.0 + self.k_ramp * ((int(self.context_lens[s]) - 1) // self.block_size))
            k[s] = self._scaled(rng.standard_normal(shape[1:], dtype=np.float32) * ramp, "k")
            v[s] = self._scaled(rng.standard_normal(shape[1:], dtype=np.float32), "v")
        return k, v

    def queries(self) -> np.ndarray:
        """fp16 q [S][Hq][D], N(0,1)."""
        rng = np.random.default_rng([self.seed, _QUERY])
        q = rng.standard_normal((self.num_seqs, self.num_q_heads, self.head_dim), dtype=np.float32)
        return q.astype(np.float16)

    # ---- slots ----
    def slots(self, tables: np.ndarray, s: int, positions: np.ndarray) -> np.ndarray:
        """slot = physical_block * block_size + offset for positions of sequence s."""
        bs = self.block_size
        positions = np.asarray(positions, dtype=np.int64)
        return tables[s, positions // bs].astype(np.int64) * bs + positions % bs

    def prefill_batches(self, max_tokens: int = 1 << 16):
        """Yield (k [T][H][D], v, slot_mapping [T]) that fill positions [0, L-1) of every
        sequence, one whole-or-leading-partial block per group, each shared block once."""
        bs = self.block_size
        ks, vs, sl = [], [], []
        count = 0
        for s in range(self.num_seqs):
            n_pre = int(self.context_lens[s]) - (1 if self.q_lens is None else int(self.q_lens[s]))
            for j in range((n_pre + bs - 1) // bs):
                if not self.prefill_owner[s, j]:
                    continue
                hi = min(n_pre - j * bs, bs)
                k, v = self.block_values(self.block_streams[s, j], j)
                ks.append(k[:hi])
                vs.append(v[:hi])
                sl.append(self.slots(self.prefill_tables, s, np.arange(j * bs, j * bs + hi)))
                count += hi
                if count >= max_tokens:
                    yield np.concatenate(ks), np.concatenate(vs), np.concatenate(sl)
                    ks, vs, sl, count = [], [], [], 0
        if ks:
            yield np.concatenate(ks), np.concatenate(vs), np.concatenate(sl)

    # ---- chunked prefill: the new tokens of every sequence ----
    @property
    def cu_q_lens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.q_lens)]).astype(np.int32)

    def chunk_tokens(self):
        """fp16 K, V [T][H][D] and slots [T] of every sequence's chunk (its last q_len positions),
        sequences one after another: the values of those positions' blocks."""
        ks, vs, sl = [], [], []
        for s in range(self.num_seqs):
            L, q = int(self.context_lens[s]), int(self.q_lens[s])
            k, v = self.seq_values(s, L - q, L)
            ks.append(k)
            vs.append(v)
            sl.append(self.slots(self.block_tables, s, np.arange(L - q, L)))
        return np.concatenate(ks), np.concatenate(vs), np.concatenate(sl).astype(np.int64)

    def chunk_queries(self) -> np.ndarray:
        """fp16 q [T][Hq][D] of the chunks' tokens, N(0,1)."""
        rng = np.random.default_rng([self.seed, _QUERY, 1])
        T = int(self.q_lens.sum())
        return rng.standard_normal((T, self.num_q_heads, self.head_dim), dtype=np.float32).astype(np.float16)

    def prefill_flops(self) -> int:
        """Multiply-adds x 2 of one chunked-prefill attention: q.k and p.v over every visible
        (query, token) pair of every query head."""
        pairs = 0
        for s in range(self.num_seqs):
            L, q = int(self.context_lens[s]), int(self.q_lens[s])
            pairs += sum(L - q + i + 1 for i in range(q))
        return int(4 * pairs * self.num_q_heads * self.head_dim)

    def step_slots(self) -> np.ndarray:
        """int64 [S]: slot of position L-1 of every sequence in its final (post-copy) table."""
        return np.array([self.slots(self.block_tables, s, [int(self.context_lens[s]) - 1])[0]
                         for s in range(self.num_seqs)], dtype=np.int64)

    def beam_walk_order(self) -> np.ndarray:
        """int32 [S]: the sequence indices in order, except that every beam child forked from a
        parent (a copy-on-write pair) comes right after that parent, so that the blocks they share
        are walked back to back."""
        S = self.num_seqs
        kids = {}
        child_set = set()
        for src, dst in self.cow_pairs:
            c = int(np.nonzero((self.block_tables == dst).any(axis=1))[0][0])
            par = int(np.nonzero((self.block_tables == src).any(axis=1))[0][0])
            kids.setdefault(par, []).append(c)
            child_set.add(c)
        order = []
        for s in range(S):
            if s in child_set:
                continue
            order.append(s)
            order.extend(kids.get(s, []))
        assert sorted(order) == list(range(S))
        return np.array(order, np.int32)

    def prefix_groups(self):
        """Sequences that share their first blocks, as the shared-prefix decode takes them: a group
        per first block id used by more than one sequence, its shared count the longest common run
        of leading block ids of all its members, kept below every member's own block count (the
        decode keeps each sequence's last block). Returns (group_start int32 [G+1], members int32,
        shared_blocks int32 [S]), or None when nothing is shared."""
        bs = self.block_size
        by_first = {}
        for s in range(self.num_seqs):
            if int(self.context_lens[s]) > 0:
                by_first.setdefault(int(self.block_tables[s, 0]), []).append(s)
        starts, members = [0], []
        shared = np.zeros(self.num_seqs, np.int32)
        for seqs in by_first.values():
            if len(seqs) < 2:
                continue
            nb = [(int(self.context_lens[s]) + bs - 1) // bs for s in seqs]
            k = 0
            while k < min(nb) - 1 and all(self.block_tables[s, k] == self.block_tables[seqs[0], k] for s in seqs):
                k += 1
            if k == 0:
                continue
            members.extend(seqs)
            starts.append(len(members))
            shared[seqs] = k
        if not members:
            return None
        return np.array(starts, np.int32), np.array(members, np.int32), shared

    # ---- bytes read by one decode (the algorithmic minimum) ----
    def decode_bytes(self, unique: bool = True) -> int:
        """Algorithmic bytes one decode reads: K/V codes of valid tokens, per-block scales and
        zero points, block-table entries, q, context lens. With unique=True a physical block
        shared by several sequences is counted once."""
        H, D, bs = self.num_kv_heads, self.head_dim, self.block_size
        code_b = {FP16: 2.0, INT8_SYM: 1.0, INT4_ASYM: 0.5, FP8_E4M3: 1.0}
        per_tok = H * D * (code_b[self.k_dtype] + code_b[self.v_dtype])
        meta = H * ((4 if self.k_dtype != FP16 else 0) + (4 if self.v_dtype != FP16 else 0)
                    + (1 if self.v_dtype == INT4_ASYM else 0))
        total = 0.0
        seen = set()
        for s in range(self.num_seqs):
            L = int(self.context_lens[s])
            nblk = (L + bs - 1) // bs
            total += nblk * 4  # table entries
            for j in range(nblk):
                b = int(self.block_tables[s, j])
                ntok = min(L - j * bs, bs)
                if unique:
                    # a block shared by several sequences is read from DRAM once
                    if b in seen:
                        continue
                    seen.add(b)
                total += ntok * per_tok + meta
        total += self.num_seqs * self.num_q_heads * D * 2 + self.num_seqs * 4
        return int(total)

    def store_bytes(self) -> int:
        """Algorithmic bytes of the step's store: each new token's fp16 K and V rows read, its codes
        written, the slot read, and the per-(block, head) scale (and zero point) written."""
        H, D = self.num_kv_heads, self.head_dim
        code_b = {FP16: 2.0, INT8_SYM: 1.0, INT4_ASYM: 0.5, FP8_E4M3: 1.0}
        row = D * (code_b[self.k_dtype] + code_b[self.v_dtype])
        meta = (4 if self.k_dtype != FP16 else 0) + (4 if self.v_dtype != FP16 else 0) + (1 if self.v_dtype == INT4_ASYM else 0)
        return int(self.num_seqs * (8 + H * (4 * D + row + meta)))

    def copy_bytes(self) -> int:
        """Algorithmic bytes of the step's copy-on-write copies: each whole block (all heads, codes,
        scales, zero points) read once and written once, plus the mapping entries."""
        H, D, bs = self.num_kv_heads, self.head_dim, self.block_size
        code_b = {FP16: 2.0, INT8_SYM: 1.0, INT4_ASYM: 0.5, FP8_E4M3: 1.0}
        meta = (4 if self.k_dtype != FP16 else 0) + (4 if self.v_dtype != FP16 else 0) + (1 if self.v_dtype == INT4_ASYM else 0)
        block = H * (bs * D * (code_b[self.k_dtype] + code_b[self.v_dtype]) + meta)
        return int(self.cow_pairs.shape[0] * (2 * block + 8))

    def decode_write_bytes(self) -> int:
        return self.num_seqs * self.num_q_heads * self.head_dim * 2


def _layout(seed, name, S, bs, context_lens, nb=None, prefix_blocks=0, children=None):
    """Assign physical blocks by a seeded permutation of the pool.

    prefix_blocks: number of leading logical blocks every sequence shares (one copy).
    children: dict child -> parent; a child shares all of its parent's blocks and gets a
    private copy of the last one in the step (copy-on-write).
    Returns tables (final), prefill tables, value streams, prefill owners, cow pairs, nb.
    """
    children = children or {}
    nblk = [(int(L) + bs - 1) // bs for L in context_lens]
    max_blocks = max(nblk) if nblk else 1
    needed = prefix_blocks
    for s in range(S):
        if s in children:
            needed += 1  # the copy-on-write target
        else:
            needed += nblk[s] - prefix_blocks
    if nb is None:
        nb = math.ceil(1.25 * needed)
    assert nb >= needed, f"{name}: pool of {nb} blocks < {needed} needed"
    rng = np.random.default_rng([seed, _LAYOUT])
    perm = rng.permutation(nb).astype(np.int32)
    nxt = 0
    tables = np.full((S, max_blocks), -1, np.int32)
    streams = np.full((S, max_blocks), -1, np.int64)
    owner = np.zeros((S, max_blocks), bool)
    prefix_ids = perm[nxt:nxt + prefix_blocks]
    nxt += prefix_blocks
    for s in range(S):
        if s in children:
            continue
        tables[s, :prefix_blocks] = prefix_ids
        streams[s, :prefix_blocks] = S  # one stream for the shared prefix
        owner[s, :prefix_blocks] = (s == 0)
        k = nblk[s] - prefix_blocks
        tables[s, prefix_blocks:nblk[s]] = perm[nxt:nxt + k]
        nxt += k
        streams[s, prefix_blocks:nblk[s]] = s
        owner[s, prefix_blocks:nblk[s]] = True
    prefill_tables = tables.copy()
    cow = []
    for c, p in sorted(children.items()):
        assert nblk[c] == nblk[p]
        tables[c] = tables[p]
        prefill_tables[c] = tables[p]
        streams[c] = streams[p]
        new_id = perm[nxt]
        nxt += 1
        cow.append((int(tables[p, nblk[p] - 1]), int(new_id)))
        tables[c, nblk[c] - 1] = new_id
    cow = np.array(cow, np.int32).reshape(-1, 2)
    return tables, prefill_tables, streams, owner, cow, nb


def make(name: str, seed: int = 0, **over) -> Workload:
    """Build a named workload. Keyword overrides (for reduced test sizes): num_seqs,
    context_lens, num_blocks, k_dtype, v_dtype, partition_tokens, block_size, head_dim,
    num_q_heads, num_kv_heads, outliers."""
    rng = np.random.default_rng([seed, 1, sum(map(ord, name))])
    children = None
    prefix_blocks = 0
    if name == "tiny":
        p = dict(num_seqs=4, num_q_heads=4, num_kv_heads=4, head_dim=64, block_size=16,
                 num_blocks=64, k_dtype=INT8_SYM, v_dtype=INT8_SYM, outliers=False,
                 partition_tokens=0, context_lens=np.array([17, 33, 50, 64]))
        desc = "4 seqs, L={17,33,50,64}, 4 heads MHA, D 64, bs 16, 64-block pool, INT8/INT8"
    elif name in ("llama7b", "llama7b_fp16", "llama7b_fp8"):
        S = over.get("num_seqs", 32)
        dt = {"llama7b": INT8_SYM, "llama7b_fp16": FP16, "llama7b_fp8": FP8_E4M3}[name]
        rng = np.random.default_rng([seed, 1, sum(map(ord, "llama7b"))])  # the same lengths for all three
        p = dict(num_seqs=S, num_q_heads=32, num_kv_heads=32, head_dim=128, block_size=16,
                 num_blocks=8192, k_dtype=dt, v_dtype=dt, outliers=True, partition_tokens=0,
                 context_lens=rng.integers(500, 2001, size=S))
        desc = ("Llama-2-7B-shaped decode layer: 32 seqs, L~U{500..2000}, 32 heads MHA, D 128, "
                "bs 16, 8192-block pool, 1% outlier channels x8, "
                + {INT8_SYM: "INT8/INT8", FP16: "FP16 cache", FP8_E4M3: "FP8 E4M3 cache"}[dt])
    elif name == "long":
        S = over.get("num_seqs", 8)
        p = dict(num_seqs=S, num_q_heads=32, num_kv_heads=32, head_dim=128, block_size=32,
                 num_blocks=None, k_dtype=INT8_SYM, v_dtype=INT4_ASYM, outliers=False,
                 partition_tokens=0, context_lens=rng.integers(8192, 32769, size=S))
        desc = "long context: 8 seqs, L~U{8192..32768}, 32 heads, D 128, bs 32, K INT8 / V INT4, contexts split across worker warps"
    elif name == "gqa_prefix":
        S = over.get("num_seqs", 64)
        prefix_blocks = over.pop("prefix_blocks", 64)
        private = over.pop("private_blocks", 64)
        bs = over.get("block_size", 16)
        p = dict(num_seqs=S, num_q_heads=64, num_kv_heads=8, head_dim=128, block_size=bs,
                 num_blocks=None, k_dtype=INT8_SYM, v_dtype=INT8_SYM, outliers=False,
                 partition_tokens=0, context_lens=np.full(S, (prefix_blocks + private) * bs))
        desc = "LLaMA-70B-shaped GQA: 64 seqs, 64 q / 8 KV heads, D 128, bs 16, 64 shared prefix blocks + 64 private, INT8/INT8"
    elif name == "prefill":
        S = over.get("num_seqs", 8)
        bs = over.get("block_size", 16)
        chunk = over.pop("chunk", 512)
        prefix = np.asarray(over.pop("prefix_lens", rng.integers(0, 2049, size=S)))
        p = dict(num_seqs=S, num_q_heads=32, num_kv_heads=32, head_dim=128, block_size=bs,
                 num_blocks=None, k_dtype=INT8_SYM, v_dtype=INT8_SYM, outliers=False,
                 partition_tokens=0, context_lens=prefix + chunk)
        q_lens = np.full(S, chunk, np.int32)
        desc = ("chunked prefill: 8 seqs, a 512-token chunk each over a cached prefix of U{0..2048} tokens, "
                "32 heads MHA, D 128, bs 16, INT8/INT8")
    elif name == "mixed":
        S = over.get("num_seqs", 128)
        n_children = over.pop("children", 16)
        L = np.clip(np.rint(np.exp(rng.normal(math.log(1000.0), 1.0, size=S))), 16, 16384).astype(np.int64)
        bs = over.get("block_size", 16)
        # parents: distinct sequences whose last prefill block is partial ((L-1) % bs != 0);
        # children: the last n_children sequences, which take their parent's length and blocks
        cand = [s for s in range(S - n_children) if (L[s] - 1) % bs != 0]
        parents = rng.choice(cand, size=n_children, replace=False)
        children = {S - n_children + i: int(par) for i, par in enumerate(parents)}
        for c, par in children.items():
            L[c] = L[par]
        p = dict(num_seqs=S, num_q_heads=32, num_kv_heads=32, head_dim=128, block_size=bs,
                 num_blocks=None, k_dtype=INT8_SYM, v_dtype=INT4_ASYM, outliers=False,
                 partition_tokens=0, context_lens=L)
        desc = "mixed step: 128 seqs, lognormal L (median 1000, sigma 1) in [16,16384], 32 heads, D 128, bs 16, K INT8 / V INT4, 16 forked"
    else:
        raise KeyError(name)
    q_lens = q_lens if name == "prefill" else None
    p.update(over)
    S = p["num_seqs"]
    cl = np.asarray(p["context_lens"], dtype=np.int32)
    assert cl.shape == (S,) and (cl >= 1).all()
    tables, pre_tables, streams, owner, cow, nb = _layout(
        seed, name, S, p["block_size"], cl, p["num_blocks"], prefix_blocks, children)
    return Workload(
        name=name, seed=seed, num_seqs=S, num_q_heads=p["num_q_heads"], num_kv_heads=p["num_kv_heads"],
        head_dim=p["head_dim"], block_size=p["block_size"], num_blocks=nb, k_dtype=p["k_dtype"],
        v_dtype=p["v_dtype"], softmax_scale=float(np.float32(1.0 / math.sqrt(p["head_dim"]))),
        context_lens=cl, block_tables=tables, block_streams=streams, prefill_tables=pre_tables,
        prefill_owner=owner, cow_pairs=cow, partition_tokens=p["partition_tokens"],
        outliers=p["outliers"], k_ramp=float(p.get("k_ramp", 0.0)), description=desc,
        q_lens=None if q_lens is None else np.asarray(q_lens, np.int32)[:S])


CONFIGS = ("tiny", "llama7b", "long", "gqa_prefix", "mixed")
