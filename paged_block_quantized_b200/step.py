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
from .workloads import Workload


_TORCH_DTYPE = {np.dtype(np.float16): torch.float16, np.dtype(np.int32): torch.int32, np.dtype(np.int64): torch.int64}


class DeviceStep:
    def __init__(self, w: Workload, device="cuda", poison: int | None = 0xA5, partition_tokens: int | None = None):
        self.w = w
        self.device = torch.device(device)
        self.pool = pkv.DevicePool.allocate(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, w.k_dtype,
                                            w.v_dtype, device=self.device, fill=poison)
        self.dev_error = torch.zeros(1, dtype=torch.int32, device=self.device)
        dev = self.device
        # the step's inputs live in one device buffer (views below), so that a caller feeding the
        # step from host memory moves them with one copy
        k_new, v_new = w.new_token_values()
        inputs = [("q", w.queries()), ("k_new", k_new), ("v_new", v_new), ("step_slots", w.step_slots()),
                  ("block_tables", w.block_tables), ("context_lens", w.context_lens), ("cow", w.cow_pairs)]
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
        self.partition_tokens = w.partition_tokens if partition_tokens is None else partition_tokens
        self.num_workers, self.num_ctas = pkv.pkv_decode_partitioning(
            self.pool.desc, w.num_seqs, w.num_q_heads, w.max_context_len, self.partition_tokens)
        self.ws_bytes = pkv.pkv_decode_workspace_size(self.pool.desc, w.num_seqs, w.num_q_heads,
                                                      w.max_context_len, self.partition_tokens)
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
