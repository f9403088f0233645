#!/usr/bin/env python
"""Benchmark: one decode step over a paged, block-quantized KV cache on B200, through the C ABI.

A step is the whole hot path once: copy-on-write block copies (when the workload forks), store of
one new token per sequence (quantize + scatter, pkv_store_quantized), then decode attention over
every sequence (pkv_paged_attention_decode). The default workload is the mixed serving step, the
largest one-GPU configuration and the only one that runs all three kernels: 128 sequences with
lognormal context lengths (median 1000, sigma 1, clamped to [16, 16384]), 32 heads MHA, head_dim
128, block size 16, INT8 K / INT4 V, 16 beam children forked from 16 parents (16 copy-on-write
copies per step). Other workloads: --config llama7b | llama7b_fp16 | long | gqa_prefix | tiny.

Every timed step appends tokens that its tiles have not seen yet: before each step (outside the
timed region) the blocks the step writes are restored from a snapshot taken after the prefill, so
the store rebuilds tiles at their natural rate (reported as store_rebuilt_tiles).

Prints ONE JSON line (rank 0). `value` is whole-job decode KV tokens/s: tokens attended by all
ranks / the slowest rank's device time (CUDA events, per step, L2 flushed between steps, inputs
resident in HBM). `e2e` is the same metric with each step's inputs copied from pinned host memory
and the output copied back inside the timed region. `roofline` rates the decode kernel's own
event-timed duration against the measured HBM copy bandwidth. `cpu_baseline` times the CPU
oracle (binary64) on a bounded sample of the workload (rank 0, one GPU only).

The step runs as three launches by default; --fused runs it as one (pkv_decode_step), and the
roofline then rates that launch with the step's algorithmic bytes.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl pkv|reference] [--fused]
Multi-GPU: launched under torch.distributed.run, one process per GPU; each rank runs its own
independently seeded copy of the workload (data-parallel over sequences, no exchange): weak scaling.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode KV tokens/s and effective HBM GB/s (fraction of ~8 TB/s) on 1 B200"
UNIT = "KV tokens/s"
FALLBACK_HBM_GBS = 6650.0
KV_NAMES = {0: "fp16", 1: "int8", 2: "int4", 3: "fp8e4m3"}


def dtype_label(w) -> str:
    """The types the path computes in: cache codes, activations, accumulation."""
    return f"k={KV_NAMES[w.k_dtype]},v={KV_NAMES[w.v_dtype]},q/out=fp16,acc=f32"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("pkv", "reference"), default="pkv")
    ap.add_argument("--op", choices=("step", "swap"), default="step",
                    help="step: the decode step (or the prefill step for --config prefill); swap: block swap")
    ap.add_argument("--config", default="mixed")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--partition-tokens", type=int, default=None)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--walk", choices=("index", "beam", "aligned"), default=None,
                    help="the decode's walk over the sequences: index order; each forked child right after "
                         "its parent; or sequences that share blocks a whole number of worker ranges apart "
                         "(reads of a shared block coincide and the second hits L2)")
    ap.add_argument("--beam-order", action="store_true", help="same as --walk beam")
    ap.add_argument("--shared-prefix", choices=("auto", "on", "off"), default="off",
                    help="attend blocks shared by a group of sequences once per group (auto: when a group has "
                         "more than two members)")
    ap.add_argument("--fused", action="store_true",
                    help="time the step as one fused launch (pkv_decode_step) instead of copy, store, decode")
    return ap.parse_args()


# ----------------------------------------------------------------------------- distributed
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "pkv":  # the reference arm runs on rank 0 alone, no group
        import torch.distributed as dist
        import torch
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def dist_max(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_sum(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def dist_barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str, enabled: bool = True):
        self.gpu_index = gpu_index
        self.enabled = enabled
        self.proc = None
        self.lines = []

    def __enter__(self):
        if self.enabled:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                     "-i", str(self.gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.reader = threading.Thread(target=self._read, daemon=True)
                self.reader.start()
                time.sleep(0.3)
            except OSError:
                self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.reader.join(timeout=2)

    def summary(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons = [], 0.0, set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- helpers
class L2Flush:
    """Leave L2 cold and clean: write a buffer of twice the L2 size (evicting everything), then
    read a second one of the same size, so that the dirty lines of the write are written back here
    and not during the next timed kernel."""

    def __init__(self, dev):
        import torch
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        n = max(2 * l2, 256 << 20)
        self.wbuf = torch.empty(n, dtype=torch.uint8, device=dev)
        self.rbuf = torch.ones(n // 4, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.wbuf.zero_()
        self.sink.copy_(self.rbuf.sum())



def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs: STREAM-style copy)"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (earlier copy measurement on this pool)"


def _source_hash(names) -> str:
    """Hash of kernel device sources with comments and blank lines removed (a profile stays valid
    across comment edits and host-side changes, not across kernel code changes)."""
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "paged_block_quantized_b200", "csrc", name), encoding="utf-8") as f:
            for line in f:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def decode_source_hash() -> str:
    return _source_hash(("decode_kernel.cuh", "decode_i8i8.cu", "decode_i8i4.cu", "decode_f16.cu", "decode_fp8.cu",
                         "common.cuh", "store_impl.cuh", "copy_impl.cuh"))


def prefill_source_hash() -> str:
    return _source_hash(("prefill_tc.cuh", "tc_common.cuh", "common.cuh", "prefill.cu"))


def ncu_traffic(profile: str, key: str = "decode_source_sha256_16", source_hash=decode_source_hash):
    """DRAM bytes per launch from the committed ncu summary `profiles/<profile>.md`, if the summary
    was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"{profile}.md")
    try:
        text = open(path, encoding="utf-8").read()
    except OSError:
        return None, None
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    hsh = re.search(key + r":\s*([0-9a-f]+)", text)
    if not m or not hsh or hsh.group(1) != source_hash():
        return None, path
    return float(m.group(1)), path


def traffic_note(profile: str, key: str = "decode_source_sha256_16", source_hash=decode_source_hash):
    """Why `traffic` is null although the summary exists: it was taken on other kernel sources."""
    path = os.path.join(ROOT, "profiles", f"{profile}.md")
    try:
        text = open(path, encoding="utf-8").read()
    except OSError:
        return None
    hsh = re.search(key + r":\s*([0-9a-f]+)", text)
    cur = source_hash()
    if hsh and hsh.group(1) != cur:
        return f"profiles/{profile}.md was taken on kernel sources {hsh.group(1)}; these are {cur}"
    return None


def config_block(w, g, step_desc):
    return {
        "workload": f"{w.name}: {w.description}",
        "num_seqs": w.num_seqs, "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
        "head_dim": w.head_dim, "block_size": w.block_size, "num_blocks": w.num_blocks,
        "kv_dtype": f"{KV_NAMES[w.k_dtype]}/{KV_NAMES[w.v_dtype]}",
        "tokens_per_step": w.total_tokens, "max_context_len": w.max_context_len,
        "partition_tokens": g.partition_tokens if g is not None else w.partition_tokens,
        "decode_worker_warps": g.num_workers if g is not None else None,
        "step": step_desc, "seed": w.seed,
    }


# ----------------------------------------------------------------------------- CPU oracle
def oracle_pool_for(w, seqs):
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from _oracle_run import oracle_step  # noqa: E402
    return oracle_step(w, seqs)


def time_oracle_decode(w, budget_s: float, threads: int):
    """Time the binary64 oracle decode on a bounded sample of the workload's sequences."""
    import numpy as np
    import oracle
    order = list(range(w.num_seqs))
    # calibrate on one sequence, then take as many sequences as fit about half the budget per run
    o1 = oracle_pool_for(w, order[:1])
    t0 = time.perf_counter()
    oracle.decode(o1["cache"], o1["q"], o1["tables"], w.context_lens[o1["seqs"]], w.softmax_scale,
                  max_context_len=w.max_context_len, num_threads=threads)
    per_tok = max((time.perf_counter() - t0) / max(int(w.context_lens[0]), 1), 1e-9)
    n = 1
    while n < w.num_seqs and per_tok * w.context_lens[:n + 1].sum() < budget_s / 2:
        n += 1
    o = oracle_pool_for(w, order[:n])
    lens = w.context_lens[o["seqs"]]
    reps, elapsed = 0, 0.0
    while elapsed < budget_s / 2 or reps == 0:
        t0 = time.perf_counter()
        oracle.decode(o["cache"], o["q"], o["tables"], lens, w.softmax_scale, max_context_len=w.max_context_len,
                      num_threads=threads)
        elapsed += time.perf_counter() - t0
        reps += 1
    tokens = int(lens.sum()) * reps
    return {"value": tokens / elapsed, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n} of {w.num_seqs} sequences ({int(lens.sum())} KV tokens) x {reps} runs of the binary64 "
                      f"oracle decode ({elapsed:.1f} s, OpenMP over (sequence, head), {threads} threads)"}


# ----------------------------------------------------------------------------- pkv arm
def run_pkv(args, rank, world, local):
    import numpy as np
    import torch
    from paged_block_quantized_b200 import workloads as W
    from paged_block_quantized_b200.step import DeviceStep

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = W.make(args.config, seed=args.seed + rank)
    groups = w.prefix_groups()
    shared = args.shared_prefix == "on" or (
        args.shared_prefix == "auto" and groups is not None and int(np.diff(groups[0]).max()) > 2)
    walk = args.walk or ("beam" if args.beam_order else "index")
    g = DeviceStep(w, device=dev, poison=None, partition_tokens=args.partition_tokens, walk=walk,
                   shared_prefix=shared and not args.fused)
    g.prefill()
    g.snapshot_step_tiles()
    has_cow = w.cow_pairs.shape[0] > 0
    fused = args.fused
    launches_per_step = 1 if fused else (1 if has_cow else 0) + 2
    stream = torch.cuda.current_stream(dev)
    flush = L2Flush(dev)

    for _ in range(args.warmup):
        g.restore_step_tiles()
        flush()
        g.step(fused=fused)
    torch.cuda.synchronize(dev)
    assert g.error() == 0, f"device error {g.error()} in warm-up"
    rebuilt, appended = g.rebuilt_tiles()  # of the last warm-up step, which started from the snapshot

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    props = torch.cuda.get_device_properties(dev)
    smi_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) is not None else str(dev.index)
    with ClockSampler(smi_id, enabled=not args.no_clocks) as clk:
        # the timed steps: the three kernels back to back (the decode overlapping its set-up with
        # the store through a programmatic dependent launch), or with --fused one launch per step
        dist_barrier(world, dev)
        torch.cuda.synchronize(dev)
        wall0 = time.perf_counter()
        for i in range(K):
            g.restore_step_tiles()        # outside the events: first-time appends every step
            flush()                       # and a cold, clean L2
            ev[i][0].record(stream)
            g.step(fused=fused)
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        dist_barrier(world, dev)
        wall_ms = (time.perf_counter() - wall0) * 1e3
        # each kernel on its own (for reference): the same steps as separate launches with events
        # around the store and the decode
        dev_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
        for i in range(K):
            g.restore_step_tiles()
            flush()
            g.copy()
            dev_ev[i][0].record(stream)
            g.store()
            dev_ev[i][1].record(stream)
            g.decode()
            dev_ev[i][2].record(stream)
        torch.cuda.synchronize(dev)
    step_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    store_ms = [dev_ev[i][0].elapsed_time(dev_ev[i][1]) for i in range(K)]
    dec_ms = [dev_ev[i][1].elapsed_time(dev_ev[i][2]) for i in range(K)]
    total_s = dist_max(sum(step_ms) / 1e3, world, dev)
    tokens_all = dist_sum(float(w.total_tokens * K), world, dev)  # every rank runs its own workload
    value = tokens_all / total_s

    # ---- e2e: same step through the public runner with host buffers copied in and out ----
    e2e = None
    if not args.no_e2e:
        # the step's inputs (q, new K/V, slots, block tables, lengths, copy pairs) are one packed
        # buffer on the device; the host side holds the same bytes in pinned memory
        host_in = g.inbuf.cpu().pin_memory()
        host_out = torch.empty_like(g.out, device="cpu").pin_memory()
        h2d = host_in.numel() * host_in.element_size()
        d2h = host_out.numel() * host_out.element_size()

        def e2e_step():
            g.inbuf.copy_(host_in, non_blocking=True)
            g.step(fused=fused)
            host_out.copy_(g.out, non_blocking=True)

        for _ in range(args.warmup):
            g.restore_step_tiles()
            e2e_step()
        torch.cuda.synchronize(dev)
        e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        dist_barrier(world, dev)
        for i in range(K):
            g.restore_step_tiles()
            flush()
            e_ev[i][0].record(stream)
            e2e_step()
            e_ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        e_total = dist_max(sum(e_ev[i][0].elapsed_time(e_ev[i][1]) for i in range(K)) / 1e3, world, dev)
        e2e = {"value": tokens_all / e_total, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": e_total * 1e3 / K}
        assert np.array_equal(host_out.numpy(), g.out.cpu().numpy())

    assert g.error() == 0, f"device error {g.error()}"
    dec_s = dist_max(statistics.mean(dec_ms) / 1e3, world, dev)
    dec_bytes = w.decode_bytes(unique=True)
    if fused:
        # the dominant (only) kernel of the step is the fused launch: its algorithmic bytes are the
        # step's (decode + store + copies) and its duration is the step's
        alg_bytes = dec_bytes + w.store_bytes() + w.copy_bytes()
        launch_s = total_s / K
        kernel = "paged_decode_kernel (fused step: copies + store + decode)"
    elif g.prefix is not None:
        alg_bytes, launch_s = dec_bytes, dec_s
        kernel = "paged_prefill_tc_kernel (prefix mode) + paged_decode_kernel"
    else:
        alg_bytes, launch_s, kernel = dec_bytes, dec_s, "paged_decode_kernel"
    achieved = alg_bytes / launch_s / 1e9
    peak, peak_src = measured_hbm_peak()
    # the committed summaries are of the plain decode launch, in the walk order they name
    traffic = None
    if not fused and g.prefix is None:
        traffic, prof = ncu_traffic(f"paged_decode_{args.config}")
        if prof is not None:
            m = re.search(r"^walk:\s*(\w+)", open(prof, encoding="utf-8").read(), re.M)
            if (m.group(1) if m else "index") != (g.walk if g.seq_order is not None else "index"):
                traffic = None
    step_desc = (("copy-on-write copies + " if has_cow else "") + "store 1 token/seq (quantize+scatter) + decode"
                 + (", one fused launch (pkv_decode_step)" if fused else ", separate launches")
                 + (", decode walks each forked child right after its parent (pkv_paged_attention_decode_ex)"
                    if g.seq_order is not None and not fused and g.walk == "beam" else "")
                 + (", decode walks sharing sequences a whole number of worker ranges apart "
                    "(pkv_paged_attention_decode_ex)" if g.seq_order is not None and not fused and g.walk == "aligned"
                    else "")
                 + (", shared-prefix decode: each shared block attended once per group (prefix pass + decode)"
                    if g.prefix is not None else ""))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": total_s * 1e3 / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": dtype_label(w), "data": "synthetic (seeded N(0,1) fp16 K/V/q, permuted block pool)",
        "config": {**config_block(w, g, step_desc), "parallelism": f"dp{world} (independent sequences per rank)",
                   "l2": "flushed before every timed step (2x L2 written, then 2x L2 read: cold and clean)", "timing": "CUDA events per step"},
        "effective_hbm_gbs": achieved, "frac_of_8tbs": achieved / 8000.0,
        "decode_us": dec_s * 1e6, "store_us": statistics.mean(store_ms) * 1e3,
        "store_rebuilt_tiles": f"{rebuilt} of {appended} (block, head) tiles appended into (first-time appends)",
        **({"decode_logical_gbs": w.decode_bytes(unique=False) / dec_s / 1e9,
            "logical_bytes_per_launch": w.decode_bytes(unique=False)}
           if w.decode_bytes(unique=False) != dec_bytes else {}),
        "decode_only_gbs": dec_bytes / dec_s / 1e9,
        # medians over the timed steps (the value above is their total)
        "ms_per_step_median": statistics.median(step_ms), "decode_us_median": statistics.median(dec_ms) * 1e3,
        "roofline": {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                     "algorithmic_bytes_per_launch": alg_bytes, "peak_source": peak_src,
                     **({"traffic_note": note} if traffic is None and not fused and g.prefix is None
                        and (note := traffic_note(f"paged_decode_{args.config}")) else {})},
        "e2e": e2e,
        "gpu_launches": launches_per_step * K,  # in the timed steps (the roofline pass runs as many again)
        "wall_ms_timed_region": wall_ms,
    }
    clocks = clk.summary()
    if clocks is not None:
        line["clocks"] = clocks
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        line["cpu_baseline"] = time_oracle_decode(w, args.cpu_seconds, threads)
        if threads > 1:  # the same oracle on one host thread, a smaller bounded sample
            one = time_oracle_decode(w, min(args.cpu_seconds, 6.0), 1)
            line["cpu_baseline"]["single_thread"] = {"value": one["value"], "sample": one["sample"]}
    return line


# ----------------------------------------------------------------------------- chunked prefill
def run_prefill(args, rank, world, local):
    """--config prefill: one step = store every sequence's chunk (quantize + scatter) and the causal
    attention of the chunk's queries over the cache (pkv_paged_attention_prefill). Tensor-bound:
    the roofline is the attention's multiply-add FLOPs over the prefill kernel's duration."""
    import torch
    from paged_block_quantized_b200 import workloads as W
    from paged_block_quantized_b200.step import PrefillStep

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = W.make(args.config, seed=args.seed + rank)
    g = PrefillStep(w, device=dev, poison=None)
    g.prefill()
    stream = torch.cuda.current_stream(dev)
    flush = L2Flush(dev)
    for _ in range(args.warmup):
        flush()
        g.step()
    torch.cuda.synchronize(dev)
    assert g.error() == 0, f"device error {g.error()} in warm-up"
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    props = torch.cuda.get_device_properties(dev)
    smi_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) is not None else str(dev.index)
    with ClockSampler(smi_id, enabled=not args.no_clocks) as clk:
        dist_barrier(world, dev)
        torch.cuda.synchronize(dev)
        for i in range(K):
            flush()
            ev[i][0].record(stream)
            g.store()
            ev[i][1].record(stream)
            g.attend()
            ev[i][2].record(stream)
        torch.cuda.synchronize(dev)
        dist_barrier(world, dev)
    step_ms = [ev[i][0].elapsed_time(ev[i][2]) for i in range(K)]
    att_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(K)]
    total_s = dist_max(sum(step_ms) / 1e3, world, dev)
    q_tokens = float(w.q_lens.sum())
    tokens_all = dist_sum(q_tokens * K, world, dev)
    att_s = dist_max(statistics.mean(att_ms) / 1e3, world, dev)
    flops = w.prefill_flops()
    peak = 1590.0  # TFLOP/s, dense bf16/fp16 (recipe fallback: MEASURED_PEAKS.json has no entry here)
    peak_src = "fallback 1.59 PFLOP/s dense fp16/bf16 (earlier cuBLAS measurement on this pool)"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            mp = json.load(f)
        if "bf16_tflops" in mp:
            peak, peak_src = float(mp["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, cuBLAS burst)"
    except (OSError, ValueError):
        pass
    achieved = flops / att_s / 1e12
    assert g.error() == 0, f"device error {g.error()}"
    line = {
        "metric": "chunked-prefill query tokens/s over the paged INT8 cache", "value": tokens_all / total_s,
        "unit": "query tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": total_s * 1e3 / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": dtype_label(w), "data": "synthetic (seeded N(0,1) fp16 K/V/q, permuted block pool)",
        "config": {"workload": f"{w.name}: {w.description}", "num_seqs": w.num_seqs, "num_q_heads": w.num_q_heads,
                   "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size,
                   "query_tokens_per_step": int(q_tokens), "context_tokens": w.total_tokens,
                   "step": "store the chunks (quantize+scatter) + chunked-prefill attention",
                   "parallelism": f"dp{world}", "l2": "flushed before every timed step"},
        "prefill_attention_us": att_s * 1e6,
        "roofline": {"bound": "tensor", "kernel": "paged_prefill_tc_kernel", "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": ncu_traffic("paged_prefill_tc_prefill", "prefill_source_sha256_16",
                                            prefill_source_hash)[0],
                     "algorithmic_flops_per_launch": flops, "peak_source": peak_src},
        "gpu_launches": 2 * K,
    }
    clocks = clk.summary()
    if clocks is not None:
        line["clocks"] = clocks
    return line


# ----------------------------------------------------------------------------- block swap
def run_swap(args, rank, world, local):
    """--op swap: every block of a quarter of the workload's sequences (scattered physical ids) out to a
    pinned host pool and back in (pkv_swap_blocks, one kernel each way). Reported: the bytes moved per
    second each way, against a plain pinned-memory copy of the same byte count by the copy engines
    (the host link's practical peak on this machine, measured in the same run)."""
    import numpy as np
    import torch
    from paged_block_quantized_b200 import pkv
    from paged_block_quantized_b200 import workloads as W
    from paged_block_quantized_b200.step import DeviceStep

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = W.make(args.config, seed=args.seed + rank)
    g = DeviceStep(w, device=dev, poison=None)
    g.prefill()
    bs = w.block_size
    seqs = list(range(0, w.num_seqs, 4))
    ids = sorted(set(int(b) for s_ in seqs for b in w.block_tables[s_, :(int(w.context_lens[s_]) + bs - 1) // bs]))
    n = len(ids)
    host = pkv.DevicePool.allocate(n, bs, w.num_kv_heads, w.head_dim, w.k_dtype, w.v_dtype, pinned_host=True)
    out_map = torch.tensor(list(zip(ids, range(n))), dtype=torch.int32, device=dev)
    in_map = torch.tensor(list(zip(range(n), ids)), dtype=torch.int32, device=dev)
    nbytes = host.nbytes()
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        pkv.pkv_swap_blocks(g.pool.desc, host.desc, out_map, n, pkv.PKV_SWAP_OUT, g.dev_error)
        pkv.pkv_swap_blocks(g.pool.desc, host.desc, in_map, n, pkv.PKV_SWAP_IN, g.dev_error)
    torch.cuda.synchronize(dev)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for i in range(K):
        ev[i][0].record(stream)
        pkv.pkv_swap_blocks(g.pool.desc, host.desc, out_map, n, pkv.PKV_SWAP_OUT, g.dev_error)
        ev[i][1].record(stream)
        pkv.pkv_swap_blocks(g.pool.desc, host.desc, in_map, n, pkv.PKV_SWAP_IN, g.dev_error)
        ev[i][2].record(stream)
    torch.cuda.synchronize(dev)
    assert g.error() == 0
    out_s = statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(K)) / 1e3
    in_s = statistics.mean(ev[i][1].elapsed_time(ev[i][2]) for i in range(K)) / 1e3
    # the copy engines on one contiguous pinned buffer of the same size, each way
    hbuf = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dbuf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    for _ in range(3):
        dbuf.copy_(hbuf, non_blocking=True)
        hbuf.copy_(dbuf, non_blocking=True)
    torch.cuda.synchronize(dev)
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    e[0].record(stream)
    for _ in range(K):
        hbuf.copy_(dbuf, non_blocking=True)
    e[1].record(stream)
    for _ in range(K):
        dbuf.copy_(hbuf, non_blocking=True)
    e[2].record(stream)
    torch.cuda.synchronize(dev)
    d2h_peak = nbytes * K / (e[0].elapsed_time(e[1]) / 1e3) / 1e9
    h2d_peak = nbytes * K / (e[1].elapsed_time(e[2]) / 1e3) / 1e9
    out_gbs, in_gbs = nbytes / out_s / 1e9, nbytes / in_s / 1e9
    return {
        "metric": "block swap GB/s (device pool <-> pinned host pool)", "value": (2 * nbytes) / (out_s + in_s) / 1e9,
        "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": (out_s + in_s) * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": dtype_label(w), "data": "synthetic",
        "config": {"workload": f"{w.name}: every block of {len(seqs)} of {w.num_seqs} sequences ({n} scattered blocks, "
                               f"{nbytes} bytes with scales and zero points)", "parallelism": f"dp{world}"},
        "swap_out_gbs": out_gbs, "swap_in_gbs": in_gbs,
        "roofline": {"bound": "host link", "kernel": "swap_blocks_kernel", "achieved": (out_gbs + in_gbs) / 2,
                     "peak": (d2h_peak + h2d_peak) / 2, "unit": "GB/s",
                     "frac": ((out_gbs / d2h_peak) + (in_gbs / h2d_peak)) / 2,
                     "traffic": ncu_traffic("swap_blocks_mixed", "swap_source_sha256_16",
                                            lambda: _source_hash(("swap.cu", "common.cuh")))[0]
                     if args.config == "mixed" else None,
                     "peak_source": f"measured in this run: pinned copies by the copy engines, "
                                    f"device->host {d2h_peak:.1f} GB/s, host->device {h2d_peak:.1f} GB/s"},
        "gpu_launches": 2 * K,
    }


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: each step decodes a bounded sample of the workload."""
    if rank != 0:
        return None
    import numpy as np
    import oracle
    from paged_block_quantized_b200 import workloads as W

    w = W.make(args.config, seed=args.seed)
    threads = os.cpu_count() or 1
    per_step_budget = max(0.5, 150.0 / max(args.steps + args.warmup, 1))
    o1 = oracle_pool_for(w, [0])
    t0 = time.perf_counter()
    oracle.decode(o1["cache"], o1["q"], o1["tables"], w.context_lens[:1], w.softmax_scale,
                  max_context_len=w.max_context_len, num_threads=threads)
    per_tok = max((time.perf_counter() - t0) / int(w.context_lens[0]), 1e-9)
    n = 1
    while n < w.num_seqs and per_tok * w.context_lens[:n + 1].sum() < per_step_budget:
        n += 1
    o = oracle_pool_for(w, list(range(n)))
    lens = w.context_lens[o["seqs"]]
    run = lambda: oracle.decode(o["cache"], o["q"], o["tables"], lens, w.softmax_scale,
                                max_context_len=w.max_context_len, num_threads=threads)
    for _ in range(args.warmup):
        run()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        run()
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = int(lens.sum()) * args.steps / total
    sample = (f"{n} of {w.num_seqs} sequences ({int(lens.sum())} KV tokens) per step, binary64 oracle decode, "
              f"OpenMP over (sequence, head), {threads} threads")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total * 1e3 / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**config_block(w, None, "decode (oracle, sampled sequences)"), "parallelism": "rank 0 only"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    rank, world, local = dist_setup(args)
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
        elif args.op == "swap":
            line = run_swap(args, rank, world, local)
        elif args.config == "prefill":
            line = run_prefill(args, rank, world, local)
        else:
            line = run_pkv(args, rank, world, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1 and args.impl == "pkv":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
