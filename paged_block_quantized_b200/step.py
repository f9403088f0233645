"""Drive one decode step of a workload through the C ABI on one GPU.

A `DeviceStep` owns the device pool and the step's inputs for a `workloads.Workload`:
  prefill()  store positions [0, L-1) of every sequence (whole blocks, untimed set-up)
  step()     copy-on-write copies, store of the token at L-1 for every sequence, decode over L:
             the three separate calls, or one pkv_decode_step launch (fused=True)
Each call is a thin sequence of pkv_* calls on one stream; torch provides the device memory.
"""
from __future__ import annotations

import numpy as np
import torch

from . import pkv
from .walk import aligned_walk_order
from .workloads import Workload


class _nullctx:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


_TORCH_DTYPE = {np.dtype(np.float16): torch.float16, np.dtype(np.int32): torch.int32, np.dtype(np.int64): torch.int64}


class DeviceStep:
    def __init__(self, w: Workload, device="cuda", poison: int | None = 0xA5, partition_tokens: int | None = None,
                 beam_order: bool = False, shared_prefix: bool = False, walk: str | None = None):
        self.w = w
        self.device = torch.device(device)
        self.pool = pkv.DevicePool.allocate(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, w.k_dtype,
                                            w.v_dtype, device=self.device, fill=poison)
        self.dev_error = torch.zeros(1, dtype=torch.int32, device=self.device)
        dev = self.device
        self.partition_tokens = w.partition_tokens if partition_tokens is None else partition_tokens
        self.num_workers, self.num_ctas = pkv.pkv_decode_partitioning(
            self.pool.desc, w.num_seqs, w.num_q_heads, w.max_context_len, self.partition_tokens)
        # the step's inputs live in one device buffer (views below), so that a caller feeding the
        # step from host memory moves them with one copy
        k_new, v_new = w.new_token_values()
        inputs = [("q", w.queries()), ("k_new", k_new), ("v_new", v_new), ("step_slots", w.step_slots()),
                  ("block_tables", w.block_tables), ("context_lens", w.context_lens), ("cow", w.cow_pairs)]
        # the decode's walk: the sequences in index order; forked children right after their
        # parents ("beam"); or sharing sequences a whole number of worker ranges apart ("aligned")
        walk = walk if walk is not None else ("beam" if beam_order else "index")
        if walk not in ("index", "beam", "aligned"):
            raise ValueError(f"walk {walk!r}")
        self.walk = walk
        self.walk_misalignment = None
        use_order = walk != "index" and w.cow_pairs.shape[0] > 0
        if use_order and walk == "beam":
            inputs.append(("seq_order", w.beam_walk_order()))
        elif use_order:
            order, self.walk_misalignment = aligned_walk_order(w.block_tables, w.context_lens, w.block_size,
                                                               self.num_workers)
            inputs.append(("seq_order", order))
        # with shared_prefix, blocks shared by several sequences are attended once per group
        groups = w.prefix_groups() if shared_prefix else None
        if groups is not None:
            inputs += [("group_start", groups[0]), ("members", groups[1]), ("shared_blocks", groups[2])]
        offs, total = [], 0
        for _, a in inputs:
            offs.append(total)
            total += (np.ascontiguousarray(a).nbytes + 255) // 256 * 256
        host = np.zeros(max(total, 256), dtype=np.uint8)
        for (_, a), o in zip(inputs, offs):
            a = np.ascontiguousarray(a)
            host[o:o + a.nbytes] = a.view(np.uint8).reshape(-1)
        self.inbuf = torch.from_numpy(host).to(dev)
        for (name, a), o in zip(inputs, offs):
            t = self.inbuf[o:o + a.nbytes].view(_TORCH_DTYPE[np.dtype(a.dtype)]).view(a.shape)
            setattr(self, name, t)
        self.out = torch.zeros_like(self.q)
        if not use_order:
            self.seq_order = None
        self.prefix = None
        if groups is not None:
            sizes = np.diff(groups[0])
            self.prefix = dict(group_start=self.group_start, members=self.members, shared_blocks=self.shared_blocks,
                               num_groups=len(sizes), num_members=int(groups[0][-1]),
                               max_group_size=int(sizes.max()), max_shared_blocks=int(groups[2].max()))
        self.ws_bytes = pkv.pkv_decode_ex_workspace_size(self.pool.desc, w.num_seqs, w.num_q_heads,
                                                         w.max_context_len, self.partition_tokens, self.seq_order,
                                                         self.prefix)
        # zero-filled once: the decode leaves its arrival counters at zero after every call
        self.workspace = torch.zeros(max(self.ws_bytes, 16), dtype=torch.uint8, device=dev)

    # ---- set-up ----
    def prefill(self, max_tokens: int = 1 << 16):
        w = self.w
        for k, v, slots in w.prefill_batches(max_tokens):
            kt = torch.from_numpy(k).to(self.device)
            vt = torch.from_numpy(v).to(self.device)
            st = torch.from_numpy(slots).to(self.device)
            pkv.pkv_store_quantized(self.pool.desc, kt, vt, st, st.numel(), self.dev_error)
        torch.cuda.synchronize(self.device)

    # ---- first-time appends when a step is repeated ----
    def snapshot_step_tiles(self):
        """Remember the pool state of every block the step writes (copy-on-write targets and the
        blocks receiving the new tokens), so that restore_step_tiles() can put it back: a repeated
        step then appends tokens its tiles have not seen yet, and the store's rebuilds happen at
        their natural rate instead of every repeat taking the "fits" path."""
        bs = self.w.block_size
        blocks = set(int(b) for b in (self.w.step_slots() // bs))
        blocks |= set(int(b) for b in self.w.cow_pairs[:, 1]) if self.w.cow_pairs.size else set()
        self._touched = torch.tensor(sorted(blocks), dtype=torch.int64, device=self.device)
        p = self.pool
        self._snap = [t.index_select(0, self._touched) for t in (p.k_codes, p.v_codes, p.k_scale, p.v_scale, p.v_zp)]

    def restore_step_tiles(self, stream=None):
        """Put the snapshot back (plain device copies on `stream`, outside any timed region)."""
        p = self.pool
        with torch.cuda.stream(stream) if stream is not None else _nullctx():
            for t, s in zip((p.k_codes, p.v_codes, p.k_scale, p.v_scale, p.v_zp), self._snap):
                t.index_copy_(0, self._touched, s)

    def rebuilt_tiles(self):
        """After one step from the snapshot: (tiles rebuilt, tiles appended into). A tile is a
        (block, KV head) pair whose block receives a token at an offset > 0; it was rebuilt when its
        K or V scale differs from the snapshot (a token at offset 0 starts a fresh tile instead)."""
        slots = self.w.step_slots()
        bs = self.w.block_size
        appended = sorted(set(int(s // bs) for s in slots if s % bs != 0))
        if not appended:
            return 0, 0
        # a copy-on-write target starts the step as a copy of its source: compare it with that
        ref = {int(d): int(s) for s, d in self.w.cow_pairs}
        touched = self._touched.cpu().tolist()
        rows = torch.tensor([touched.index(ref.get(b, b)) for b in appended], device=self.device)
        blocks = torch.tensor(appended, dtype=torch.int64, device=self.device)
        p = self.pool
        ks = p.k_scale.index_select(0, blocks).view(torch.int32)
        vs = p.v_scale.index_select(0, blocks).view(torch.int32)
        changed = (ks != self._snap[2].index_select(0, rows).view(torch.int32)) | (
            vs != self._snap[3].index_select(0, rows).view(torch.int32))
        return int(changed.sum().item()), int(changed.numel())

    # ---- the step ----
    def copy(self, stream=None):
        n = self.cow.shape[0]
        if n:
            pkv.pkv_copy_blocks(self.pool.desc, self.cow, n, self.dev_error, stream=stream)

    def store(self, stream=None):
        pkv.pkv_store_quantized(self.pool.desc, self.k_new, self.v_new, self.step_slots, self.w.num_seqs,
                                self.dev_error, stream=stream)

    def decode(self, stream=None, out=None, q=None):
        w = self.w
        if self.seq_order is not None or self.prefix is not None:
            pkv.pkv_paged_attention_decode_ex(
                self.pool.desc, self.out if out is None else out, self.q if q is None else q, w.num_seqs,
                w.num_q_heads, self.block_tables, w.max_blocks_per_seq, self.context_lens, w.max_context_len,
                w.softmax_scale, self.partition_tokens, self.seq_order, self.workspace, self.ws_bytes,
                self.dev_error, stream=stream, prefix=self.prefix)
            return
        pkv.pkv_paged_attention_decode(
            self.pool.desc, self.out if out is None else out, self.q if q is None else q, w.num_seqs,
            w.num_q_heads, self.block_tables, w.max_blocks_per_seq, self.context_lens, w.max_context_len,
            w.softmax_scale, self.partition_tokens, self.workspace, self.ws_bytes, self.dev_error, stream=stream)

    def step(self, stream=None, fused: bool = False):
        if not fused:
            self.copy(stream)
            self.store(stream)
            self.decode(stream)
            return self.out
        w = self.w
        pkv.pkv_decode_step(
            self.pool.desc, self.cow, self.cow.shape[0], self.k_new, self.v_new, self.step_slots, w.num_seqs,
            self.out, self.q, w.num_seqs, w.num_q_heads, self.block_tables, w.max_blocks_per_seq, self.context_lens,
            w.max_context_len, w.softmax_scale, self.partition_tokens, self.workspace, self.ws_bytes,
            self.dev_error, stream=stream)
        return self.out

    # ---- read-back ----
    def error(self) -> int:
        return int(self.dev_error.item())

    def pool_numpy(self):
        """Host copies of the pool arrays with the oracle's element types."""
        from . import workloads as W
        p = self.pool
        def codes(t, dt):
            a = t.cpu().numpy()
            if dt == W.FP16:
                return a.view(np.uint16)
            if dt == W.INT8_SYM:
                return a.view(np.int8)
            return a
        return (codes(p.k_codes, self.w.k_dtype), codes(p.v_codes, self.w.v_dtype), p.k_scale.cpu().numpy(),
                p.v_scale.cpu().numpy(), p.v_zp.cpu().numpy())


class PrefillStep:
    """One chunked-prefill step of a workload with q_lens: store every sequence's chunk (its last
    q_len positions) into the pool, then causal attention of the chunk's queries over the cache
    (pkv_paged_attention_prefill). Before the step the pool holds positions [0, L - q_len)."""

    def __init__(self, w: Workload, device="cuda", poison: int | None = 0xA5):
        assert w.q_lens is not None
        self.w = w
        self.device = torch.device(device)
        dev = self.device
        self.pool = pkv.DevicePool.allocate(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, w.k_dtype,
                                            w.v_dtype, device=dev, fill=poison)
        self.dev_error = torch.zeros(1, dtype=torch.int32, device=dev)
        k, v, slots = w.chunk_tokens()
        self.k_new = torch.from_numpy(k).to(dev)
        self.v_new = torch.from_numpy(v).to(dev)
        self.slots = torch.from_numpy(slots).to(dev)
        self.q = torch.from_numpy(w.chunk_queries()).to(dev)
        self.out = torch.zeros_like(self.q)
        self.cu = torch.from_numpy(w.cu_q_lens).to(dev)
        self.context_lens = torch.from_numpy(w.context_lens).to(dev)
        self.block_tables = torch.from_numpy(w.block_tables).to(dev)
        self.total_q = int(w.q_lens.sum())
        self.max_q_len = int(w.q_lens.max())

    def prefill(self, max_tokens: int = 1 << 16):
        for k, v, slots in self.w.prefill_batches(max_tokens):
            pkv.pkv_store_quantized(self.pool.desc, torch.from_numpy(k).to(self.device),
                                    torch.from_numpy(v).to(self.device), torch.from_numpy(slots).to(self.device),
                                    slots.shape[0], self.dev_error)
        torch.cuda.synchronize(self.device)

    def store(self, stream=None):
        pkv.pkv_store_quantized(self.pool.desc, self.k_new, self.v_new, self.slots, self.total_q, self.dev_error,
                                stream=stream)

    def attend(self, stream=None):
        w = self.w
        pkv.pkv_paged_attention_prefill(self.pool.desc, self.out, self.q, w.num_seqs, w.num_q_heads, self.cu,
                                        self.total_q, self.max_q_len, self.block_tables, w.max_blocks_per_seq,
                                        self.context_lens, w.max_context_len, w.softmax_scale, self.dev_error,
                                        stream=stream)

    def step(self, stream=None):
        self.store(stream)
        self.attend(stream)
        return self.out

    def error(self) -> int:
        return int(self.dev_error.item())
