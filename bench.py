"""Benchmark of one engine step of paged attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 3] [--impl ours|reference]

A step is one pass of the hot path over one batch: ``pa_cache_append`` of the
step's new K/V rows, then attention (``pa_decode`` for a decode batch,
``pa_prefill_chunk`` for the mixed batch).  Block tables and slots come from
the host allocator before timing.  The default workload is the Llama-3.3-70B-
like attention layer at concurrency 128 (64 query heads, 8 KV heads, head_dim
128, 16-token blocks, lognormal contexts with median 1500 clipped to
[16, 8192]).

Prints one JSON line.  ``value`` is KV GB/s: the KV bytes the step must read
(every cached token once, K and V, all KV heads) times the number of ranks,
over the device time per step (CUDA events, max over ranks).  ``e2e`` repeats
the step through the same C-ABI calls with host buffers: the per-step inputs
are copied from pinned host memory and the output back inside the timed
region.  ``roofline`` rates the dominant kernel (attention) from its own
per-launch CUDA-event times against the measured HBM copy bandwidth.

Multi-GPU: one process per GPU (torchrun); each rank runs its own batch (weak
scaling, no collective on the data path; an all-reduce of the timings only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 4 * L2_BYTES  # written between timed steps when a step's KV would fit in L2
PROFILE_DIR = os.path.join(ROOT, "profiles")


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


KERNEL_SOURCES = {  # the files whose text decides each kernel's code
    "pa_rows_kernel": ("pa_rows.cu", "pa_device.cuh"),
    "pa_chunk_kernel": ("pa_chunk.cu", "pa_device.cuh", "pa_umma.cuh"),
    "pa_verify_kernel": ("pa_verify.cu", "pa_device.cuh", "pa_umma.cuh"),
}


def code_tokens(text: str) -> str:
    """C/CUDA source without comments and with whitespace runs collapsed: an
    edit of comments or layout leaves it (and the compiled kernel) unchanged.
    The sources hold no string literal with a comment marker in it."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(kernel: str) -> str:
    """Hash of the code (comments and whitespace aside) of the files that
    decide a kernel's binary."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_445_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update((name + "\n" + code_tokens(f.read())).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str, variant: str = ""):
    """dram read+write bytes per launch from a committed ncu summary, if it was
    taken on the current kernel sources; else None."""
    path = os.path.join(PROFILE_DIR, f"{kernel}_{workload}{variant}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    t = re.search(r"dram_bytes_per_launch_full_size:\s*([0-9.e+]+)", text)
    if not m or not t or m.group(1) != kernel_source_hash(kernel):
        return None
    return float(t.group(1))


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device: int, period_s: float = 0.02):
        self.period = period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_device)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            try:
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(torch_device)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: the line says so
            log(f"clock sampling unavailable: {e}")

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = get_reasons(self.h)
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):  # may be entered again: the samples accumulate
        self._stop.clear()
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------- distributed
def dist_setup(n_gpus: int, backend: str = "nccl"):
    """One process per GPU: read RANK / LOCAL_RANK / WORLD_SIZE from the
    environment torchrun sets and join the process group (NCCL on GPUs; the
    CPU tests use gloo)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}: launch N>1 with torchrun")
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=120)
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timeout)
    elif backend == "nccl":
        import torch
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_over_ranks(x: float, world: int, op: str = "max", device: str = "cuda") -> float:
    """MAX or SUM of one number over all ranks (every rank gets the result)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    return reduce_over_ranks(x, world, "max", device)


def rank_seed(workload: int, rank: int) -> int:
    """Each rank runs its own batch of the same workload (weak scaling)."""
    return 445 + workload + 1000 * rank


def step_launches(w, chunk_head_dims=(128,), chunk_groups=(1, 2, 4, 8, 16), verify_max_seqs=512) -> int:
    """Kernel launches of one unfused step: the append and the rows kernel;
    for a varlen batch at head_dim 128 with a supported group also the tcgen05
    chunk kernel and the two multi-row kernels (32 and 64 columns), which
    pa_prefill_chunk launches whatever the batch holds (each returns at once
    when it has no work)."""
    n = 2
    if not w.is_decode and w.head_dim in chunk_head_dims and (w.num_q_heads // w.num_kv_heads) in chunk_groups:
        n += 1 + (2 if w.num_seqs <= verify_max_seqs else 0)
    return n


def plan_launches(words) -> int:
    """Kernel launches of a planned pa_prefill_chunk_planned call: one per
    kernel that has work (the plan's flags: 32- and 64-column verification,
    chunk, rows)."""
    return bin(words[1] & 15).count("1")


def plan_split(words):
    """SMs of the decode rows beside the chunk kernel (0: one after the other)."""
    return int(words[2])


def verify_batch(w, max_cols=64, max_seqs=512) -> bool:
    """Every sequence of the batch has 2 .. max_cols/G query rows: the
    multi-row (verification) kernel does all the attention work."""
    g = w.num_q_heads // w.num_kv_heads
    qlen = np.diff(np.asarray(w.query_start))
    return (not w.is_decode and w.head_dim == 128 and w.num_seqs <= max_seqs and bool(np.all(qlen >= 2))
            and bool(np.all(qlen * g <= max_cols)))


def compose_value(total_kv_bytes: float, ms_step_max: float) -> float:
    """Whole-job KV GB/s: the bytes all ranks read over the slowest rank's step."""
    return total_kv_bytes / (ms_step_max * 1e-3) / 1e9


# --------------------------------------------------------------------- workload
def l2_flush_needed(unique_kv_bytes: int) -> bool:
    """Whether the KV one step reads (each distinct byte once) could stay in
    the 126 MB L2 until the next step; then the timed steps run with L2
    flushed in between, so HBM, not L2, serves the cache."""
    return unique_kv_bytes < 2 * L2_BYTES


def l2_note(flush: bool, kv_bytes: int, unique_kv_bytes: int) -> str:
    if flush:
        return (f"flushed: a {FLUSH_BYTES >> 20} MiB buffer is written before every timed step, outside its events "
                f"(the step's {unique_kv_bytes / 1e6:.0f} MB of distinct KV would otherwise stay in the 126 MB L2)")
    return f"no flush: every step reads {kv_bytes / 1e9:.2f} GB of KV, larger than the 126 MB L2"


def step_bytes(w):
    from paged_kv_cache_445_b200 import roofline
    kv = roofline.decode_kv_bytes(w.context_lens, w.num_kv_heads, w.head_dim)
    attn = roofline.attention_algorithmic_bytes(w.context_lens, w.query_start, w.num_q_heads, w.num_kv_heads,
                                                w.head_dim, w.block_size)
    app = roofline.append_algorithmic_bytes(len(w.slot_mapping), w.num_kv_heads, w.head_dim)
    flops = roofline.prefill_flops(w.context_lens, w.query_start, w.num_q_heads, w.head_dim)
    return kv, attn, app, flops


class GpuStep:
    """One workload resident on the GPU.  A decode batch runs its step as one
    fused launch (pa_decode_append) unless fused=False; a mixed batch runs
    pa_cache_append then pa_prefill_chunk."""

    def __init__(self, w, device, fused=True, cascade=True, fp8=False, plan=True):
        import torch

        import paged_kv_cache_445_b200 as pa
        self.pa, self.torch, self.w = pa, torch, w

        def bf(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)

        def i32(a):
            return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)

        self.k_cache, self.v_cache = bf(w.k_cache), bf(w.v_cache)
        self.k_new, self.v_new, self.q = bf(w.k_new), bf(w.v_new), bf(w.q)
        self.block_tables, self.context_lens = i32(w.block_tables), i32(w.context_lens)
        self.query_start, self.slot_mapping = i32(w.query_start), i32(w.slot_mapping)
        self.out = torch.empty_like(self.q)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.decode = w.is_decode
        self.fused = self.decode and fused
        self.fp8 = fp8
        if fp8:  # E4M3 codes with per-tensor scales (decode batches only)
            if not self.decode:
                raise SystemExit("--kv-dtype fp8 is a decode path")
            kc, vc, self.k_scale, self.v_scale = workloads_fp8_caches(w)
            self.k_cache, self.v_cache = torch.from_numpy(kc).to(device), torch.from_numpy(vc).to(device)
        groups = w.prefix_groups() if self.decode and cascade else None
        self.cascade = groups is not None
        if self.cascade:  # shared prefixes read once per group (pa_decode_cascade)
            self.group_start, self.group_prefix = i32(groups[0]), i32(groups[1])
            self.workspace = pa.make_cascade_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                                       w.block_tables.shape[1], w.block_size, device)
        else:
            self.workspace = pa.make_workspace(w.num_query_tokens, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                               w.block_tables.shape[1], w.block_size, device)
        # a varlen batch: the host plan (made before timing from the host copies
        # of query_start and context_lens, as a scheduler would) picks the
        # kernels with work and how decode rows and chunk rows share the SMs
        self.plan = None
        if not self.decode and plan:
            self.plan = pa.pa_plan_batch(w.query_start, w.context_lens, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                         w.block_size, w.block_tables.shape[1])
        # kernel launches per step
        if self.cascade:
            self.launches = 2 if self.fused else 3
        elif self.plan is not None:
            self.launches = 1 + plan_launches(list(self.plan.words))
        else:
            self.launches = 1 if self.fused else step_launches(w)
        # host-to-device inputs of one step (what e2e copies)
        self.inputs = ["q", "k_new", "v_new", "block_tables", "context_lens"]
        if not self.fused:
            self.inputs.append("slot_mapping")
        if not self.decode:
            self.inputs.append("query_start")

    def append(self):
        if self.fused:
            return  # part of the attention launch
        if self.fp8:
            self.pa.pa_cache_append_fp8(self.k_new, self.v_new, self.k_cache, self.v_cache, self.slot_mapping,
                                        self.k_scale, self.v_scale, self.status)
            return
        self.pa.pa_cache_append(self.k_new, self.v_new, self.k_cache, self.v_cache, self.slot_mapping, self.status)

    def attend(self):
        if self.fp8:
            self.pa.pa_decode_fp8(self.out, self.q, self.k_cache, self.v_cache, self.block_tables, self.context_lens,
                                  self.w.scale, self.k_scale, self.v_scale, self.workspace,
                                  k_new=self.k_new if self.fused else None, v_new=self.v_new if self.fused else None,
                                  dev_status=self.status)
        elif self.cascade:
            self.pa.pa_decode_cascade(self.out, self.q, self.k_cache, self.v_cache, self.block_tables,
                                      self.context_lens, self.w.scale, self.group_start, self.group_prefix,
                                      self.workspace, k_new=self.k_new if self.fused else None,
                                      v_new=self.v_new if self.fused else None, dev_status=self.status)
        elif self.fused:
            self.pa.pa_decode_append(self.out, self.q, self.k_new, self.v_new, self.k_cache, self.v_cache,
                                     self.block_tables, self.context_lens, self.w.scale, self.workspace, self.status)
        elif self.decode:
            self.pa.pa_decode(self.out, self.q, self.k_cache, self.v_cache, self.block_tables, self.context_lens,
                              self.w.scale, self.workspace, self.status)
        elif self.plan is not None:
            self.pa.pa_prefill_chunk_planned(self.out, self.q, self.query_start, self.k_cache, self.v_cache,
                                             self.block_tables, self.context_lens, self.w.scale, self.workspace,
                                             self.plan, self.status)
        else:
            self.pa.pa_prefill_chunk(self.out, self.q, self.query_start, self.k_cache, self.v_cache,
                                     self.block_tables, self.context_lens, self.w.scale, self.workspace, self.status)


def workloads_fp8_caches(w):
    from paged_kv_cache_445_b200 import workloads
    return workloads.fp8_caches(w, seed=445)


def measure(args, peaks, workload, rank, world, local, *, cascade, fp8, plan=True, cpu_seconds=None):
    """Time one workload's step (device events, then end to end through the
    C ABI with host buffers) and return its JSON line as a dict."""
    import torch

    from paged_kv_cache_445_b200 import workloads
    device = torch.device("cuda", local)
    t0 = time.time()
    w = workloads.standard(workload, seed=rank_seed(workload, rank))
    log(f"[rank {rank}] workload {w.name}: {w.num_seqs} seqs, {w.num_query_tokens} query rows, "
        f"{int(w.context_lens.sum())} keys, pool {w.num_blocks} blocks ({time.time() - t0:.1f}s to generate)")
    g = GpuStep(w, device, fused=not args.separate_append, cascade=cascade, fp8=fp8, plan=plan)
    kv_bytes, attn_bytes, app_bytes, flops = step_bytes(w)
    if g.fp8:  # one byte per cached element instead of two; the appended rows are written as bytes too
        attn_bytes -= kv_bytes // 2
        app_bytes -= len(w.slot_mapping) * w.num_kv_heads * w.head_dim * 2
        kv_bytes //= 2
    stream = torch.cuda.current_stream()
    from paged_kv_cache_445_b200 import roofline as _rl
    unique_kv = _rl.unique_kv_bytes(w.block_tables, w.context_lens, w.block_size, w.num_kv_heads, w.head_dim)
    if g.fp8:
        unique_kv //= 2
    flush = l2_flush_needed(unique_kv)

    for _ in range(args.warmup):
        g.append()
        g.attend()
    torch.cuda.synchronize()
    if int(g.status.item()) != 0:
        raise SystemExit(f"device status {int(g.status.item())} after warm-up")

    graph = None
    if args.graph:  # the whole step (all its launches) as one CUDA graph, replayed per step
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            g.append()
            g.attend()
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()
        if int(g.status.item()) != 0:
            raise SystemExit(f"device status {int(g.status.item())} after graph warm-up")

    # ---- device-timed region
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    with sampler:
        # the K timed steps, back to back with nothing between them (an event
        # recorded between two launches would cost the overlap of one launch's
        # tail with the next one's start)
        start.record(stream)
        for i in range(args.steps):
            if graph is not None:
                graph.replay()
                continue
            g.append()
            g.attend()
        end.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        # the kernel's own launch time, for the roofline: the same steps again
        # with an event pair around each attention call
        torch.cuda.synchronize()
        for i in range(args.steps):
            if graph is not None:  # append + attention inside one replay: the events bracket both
                ev[i][0].record(stream)
                graph.replay()
                ev[i][1].record(stream)
                continue
            g.append()
            ev[i][0].record(stream)
            g.attend()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_total = start.elapsed_time(end)
    attn_ms = [a.elapsed_time(b) for a, b in ev]
    warm_ms_step = None
    if flush:
        # the same steps with L2 flushed before each; only the steps are timed
        warm_ms_step = max_over_ranks(ms_total / args.steps, world)
        scratch = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=g.out.device)
        whole = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
        barrier(world)
        torch.cuda.synchronize()
        with sampler:
            for i in range(args.steps):
                scratch.fill_(i & 255)
                whole[i][0].record(stream)
                if graph is not None:
                    ev[i][0].record(stream)
                    graph.replay()
                    ev[i][1].record(stream)
                else:
                    g.append()
                    ev[i][0].record(stream)
                    g.attend()
                    ev[i][1].record(stream)
                whole[i][1].record(stream)
            torch.cuda.synchronize()
        barrier(world)
        ms_total = sum(a.elapsed_time(b) for a, b in whole)
        attn_ms = [a.elapsed_time(b) for a, b in ev]
        del scratch
    ms_step = max_over_ranks(ms_total / args.steps, world)
    attn_avg_ms = max_over_ranks(sum(attn_ms) / len(attn_ms), world)
    if int(g.status.item()) != 0:
        raise SystemExit(f"device status {int(g.status.item())} after timing")

    # ---- end to end through the public calls with host buffers.  Every step
    # copies its inputs from pinned host memory and its output back.  As a
    # serving loop does, the copies run on their own streams, double-buffered,
    # so that step i's inputs travel while step i - 1 computes (steps whose KV
    # must be flushed from L2 run one after another instead, below).
    pin = {name: getattr(g, name).cpu().pin_memory() for name in g.inputs}
    out_host = torch.empty(g.out.shape, dtype=g.out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = out_host.numel() * out_host.element_size()
    sets = [{**{k: getattr(g, k) for k in g.inputs}, "out": g.out},
            {**{k: getattr(g, k).clone() for k in g.inputs}, "out": torch.empty_like(g.out)}]

    def use(b):
        for k in g.inputs:
            setattr(g, k, b[k])
        g.out = b["out"]

    def e2e_step():  # one step, every copy on the compute stream
        use(sets[0])
        for k, t in pin.items():
            getattr(g, k).copy_(t, non_blocking=True)
        g.append()
        g.attend()
        out_host.copy_(g.out, non_blocking=True)

    in_s, out_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_pipelined(i):
        b = sets[i % 2]
        with torch.cuda.stream(in_s):
            if i >= 2:
                in_s.wait_event(ev_done[i % 2])  # step i - 2 has read its inputs
            for k, t in pin.items():
                b[k].copy_(t, non_blocking=True)
            ev_in[i % 2].record(in_s)
        stream.wait_event(ev_in[i % 2])
        if i >= 2:
            stream.wait_event(ev_out[i % 2])  # step i - 2's output has left the buffer
        use(b)
        g.append()
        g.attend()
        ev_done[i % 2].record(stream)
        with torch.cuda.stream(out_s):
            out_s.wait_event(ev_done[i % 2])
            out_host.copy_(b["out"], non_blocking=True)
            ev_out[i % 2].record(out_s)

    for i in range(max(2, args.warmup)):
        e2e_pipelined(i)
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e_start.record(in_s)
    for i in range(args.steps):
        e2e_pipelined(i)
    e_end.record(out_s)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end) / args.steps, world)
    e2e_mode = "pipelined: inputs of step i copied while step i - 1 computes (two buffer sets, copy streams)"
    if flush:  # as above: L2 flushed before each step, the steps alone timed
        scratch = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=g.out.device)
        whole = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
        barrier(world)
        torch.cuda.synchronize()
        for i in range(args.steps):
            scratch.fill_(i & 255)
            whole[i][0].record(stream)
            e2e_step()
            whole[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in whole) / args.steps, world)
        e2e_mode = "one step at a time, L2 flushed before each (copies on the compute stream)"
        del scratch
    use(sets[0])
    total_kv = reduce_over_ranks(float(kv_bytes), world, "sum")
    total_seqs = reduce_over_ranks(float(w.num_seqs), world, "sum")

    # ---- CPU baseline: the oracle on this host's cores, rank 0 at N = 1 only
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_baseline(w, args.cpu_seconds if cpu_seconds is None else cpu_seconds, fp8=g.fp8)

    clocks = sampler.summary()
    hbm, bf16_burst, bf16_sust, peak_src = peaks
    app_in_launch = app_bytes if (g.fused or graph is not None) else 0
    logical_launch_bytes = attn_bytes + app_in_launch
    if unique_kv < kv_bytes:  # blocks shared between sequences (a shared prefix) need cross HBM only once
        attn_bytes = attn_bytes - kv_bytes + unique_kv
    # the timed launch (or replay) also appends when fused or replayed as a graph
    launch_bytes = attn_bytes + app_in_launch
    achieved = launch_bytes / (attn_avg_ms * 1e-3) / 1e9
    verify = verify_batch(w)
    traffic = (profiled_traffic("pa_verify_kernel", w.name) if verify else
               profiled_traffic("pa_rows_kernel", w.name, "-fp8" if g.fp8 else ""))
    line = {
        "metric": "paged-attn decode KV GB/s + seq-steps/s (70B layer, bs128); % of HBM peak",
        "value": round(compose_value(total_kv, ms_step), 2),
        "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8-e4m3 cache, bf16 q/out" if g.fp8 else "bf16",
        "data": "synthetic (seeded PCG64, bf16 N(0,1) K/V, q N(0,0.5^2)); no weights",
        "config": {
            "workload": w.name, "num_seqs": w.num_seqs, "num_q_heads": w.num_q_heads,
            "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size,
            "num_blocks": w.num_blocks, "query_rows": w.num_query_tokens,
            "context_tokens": int(w.context_lens.sum()), "kv_bytes_per_step": kv_bytes,
            "unique_kv_bytes_per_step": unique_kv,
            "l2": l2_note(flush, kv_bytes, unique_kv),
            "parallelism": f"dp{world} (independent batch per GPU)",
            "cuda_graph": graph is not None,
            "host_plan": None if g.plan is None else {"launches": plan_launches(list(g.plan.words)),
                                                       "decode_sms": plan_split(list(g.plan.words))},
        },
        "seq_steps_per_s": round(total_seqs / (ms_step * 1e-3), 1),
        "frac_of_hbm_peak": round(compose_value(total_kv, ms_step) / hbm / world, 4),
        "frac_of_8tbs_nominal": round(compose_value(total_kv, ms_step) / 8000.0 / world, 4),
        "roofline": {
            "kernel": ("pa_rows_kernel, FP8 E4M3 cache (append + attention, one launch)" if g.fp8 else
                       "pa_verify_kernel (timed as the whole pa_prefill_chunk call: its launches of the "
                       "chunk and rows kernels find no work)" if verify else
                       ("pa_prefill_chunk_planned call: decode rows (rows kernel, %d SMs) beside the tcgen05 "
                        "chunk kernel (the other SMs)" % plan_split(list(g.plan.words))
                        if g.plan is not None and plan_split(list(g.plan.words)) > 0 else
                        "pa_prefill_chunk call (chunk kernel + rows kernel, one after the other)")
                       if not w.is_decode else
                       "pa_cascade_kernel + pa_rows_kernel (shared prefixes once, then the private keys)"
                       if g.cascade else
                       "pa_rows_kernel (append + attention, one launch)" if g.fused else "pa_rows_kernel (attention)"),
            "bound": _rl.bound(flops, launch_bytes, bf16_burst * 1e12, hbm * 1e9),
            "intensity_flop_per_byte": round(flops / launch_bytes, 2),
            "ridge_flop_per_byte": round(_rl.ridge_point(bf16_burst * 1e12, hbm * 1e9), 1),
            "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
            if peak_src == "measured" else "fallback 6.65 TB/s",
            "traffic": traffic, "algorithmic_bytes_per_launch": launch_bytes,
            "avg_launch_ms": round(attn_avg_ms, 5),
            **({"logical_bytes_per_launch": logical_launch_bytes,
                "achieved_logical": round(logical_launch_bytes / (attn_avg_ms * 1e-3) / 1e9, 1)}
               if logical_launch_bytes != launch_bytes else {}),
        },
        "append": {"algorithmic_bytes": app_bytes},
        "e2e": {"value": round(compose_value(total_kv, e2e_ms), 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "mode": e2e_mode},
        "gpu_launches": g.launches * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    if warm_ms_step is not None:  # the same steps back to back, the KV left in L2 by the step before
        line["l2_warm"] = {"value": round(compose_value(total_kv, warm_ms_step), 2), "unit": "GB/s",
                           "ms_per_step": round(warm_ms_step, 5)}
    if not w.is_decode:
        line["roofline_tensor"] = {"flops_per_step": flops, "achieved_tflops": round(flops / (attn_avg_ms * 1e-3) / 1e12, 1),
                                   "peak": bf16_sust, "unit": "TFLOP/s"}
        # both kernels at once: the step cannot beat the slower of the two rooflines
        bound_ms = max(kv_bytes / (hbm * 1e9), flops / (bf16_burst * 1e12)) * 1e3
        line["overlap_bound"] = {"ms": round(bound_ms, 5), "frac": round(bound_ms / attn_avg_ms, 4),
                                 "what": "max(decode KV bytes / measured HBM, chunk FLOPs / measured bf16 burst) "
                                         "over the timed call"}
    del g
    torch.cuda.empty_cache()
    return line


SUB_RECORDS = [  # (key, workload, cascade, fp8): the other workloads of the default run, at N = 1
    ("grpo-shared-prefix", 4, False, False),
    ("grpo-shared-prefix-cascade", 4, True, False),
    ("grpo-long-prefix", 7, False, False),
    ("grpo-long-prefix-cascade", 7, True, False),
    ("mixed-chunk-decode", 5, False, False),
    ("llama3.3-70b-layer-decode-b128-fp8", 3, False, True),
]


def calibrate(args):
    """Per-SM streaming rates for the decode split (pa_calibrate), once per run."""
    if args.no_calibrate:
        return {"weighted": False}
    import paged_kv_cache_445_b200 as pa
    t0 = time.time()
    w = np.asarray(pa.pa_calibrate(), dtype=np.float64)
    rel = w / np.median(w)
    log(f"calibrated {len(w)} SMs in {time.time() - t0:.2f}s: shares {rel.min():.2f} .. {rel.max():.2f} of the median")
    return {"weighted": True, "sms": int(len(w)), "share_vs_median": {"min": round(float(rel.min()), 3),
                                                                      "max": round(float(rel.max()), 3)}}


def run_ours(args, peaks):
    rank, world, local = dist_setup(args.gpus)
    split = calibrate(args)
    line = measure(args, peaks, args.workload, rank, world, local, cascade=args.cascade,
                   fp8=args.kv_dtype == "fp8", plan=not args.no_plan)
    line["config"]["sm_split"] = split
    if world == 1 and not args.no_sub_records and args.workload == 3 and args.kv_dtype == "bf16" \
            and not args.cascade and not args.graph:
        # the other workloads, each with its own roofline, clocks and short CPU baseline
        subs = {}
        for key, wl, casc, f8 in SUB_RECORDS:
            sub = measure(args, peaks, wl, rank, world, local, cascade=casc, fp8=f8, cpu_seconds=args.sub_cpu_seconds)
            sub["config"]["sm_split"] = split
            for k in ("metric", "n_gpus", "steps", "warmup", "higher_is_better", "scaling", "vs_baseline", "data"):
                sub.pop(k, None)
            subs[key] = sub
        line["workloads"] = subs
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()




# --------------------------------------------------------------------- oracle
def oracle_sample(w, max_rows: int):
    """The first sequences of the batch (all heads), up to max_rows query rows."""
    import oracle
    rows = []
    qs = w.query_start
    for s in range(w.num_seqs):
        for t in range(int(qs[s]), int(qs[s + 1])):
            rows.append((s, t))
        if len(rows) >= max_rows:
            break
    seqs = sorted({s for s, _ in rows})
    only = np.array([(t, h) for _, t in rows for h in range(w.num_q_heads)], dtype=np.int32)
    keys = sum(int(w.context_lens[s]) for s in seqs)
    from paged_kv_cache_445_b200 import roofline
    return oracle, only, seqs, roofline.kv_cache_bytes(1, w.num_kv_heads, w.head_dim, keys)


def oracle_step(oracle, w, only, kc, vc, scales=None):
    slots = oracle.slot_mapping(w.block_tables, w.context_lens, w.query_start, w.block_size, w.num_blocks)
    if scales is not None:  # E4M3 cache: (k_scale, v_scale)
        oracle.cache_append_fp8(w.k_new, w.v_new, kc, vc, slots, *scales)
        oracle.paged_attention_fp8(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale, *scales,
                                   only=only)
        return
    oracle.cache_append(w.k_new, w.v_new, kc, vc, slots)
    oracle.paged_attention(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale, only=only)


def oracle_baseline(w, seconds: float, max_rows: int = 16, fp8: bool = False):
    oracle, only, seqs, sample_bytes = oracle_sample(w, max_rows)
    scales = None
    if fp8:
        kc, vc, k_scale, v_scale = workloads_fp8_caches(w)
        scales, sample_bytes = (k_scale, v_scale), sample_bytes // 2
    else:
        kc, vc = w.k_cache, w.v_cache  # appended in place: the same rows every step
    def timed(budget_s):
        n, t0 = 0, time.perf_counter()
        while True:
            oracle_step(oracle, w, only, kc, vc, scales)
            n += 1
            if time.perf_counter() - t0 >= budget_s:
                break
        return n, (time.perf_counter() - t0) / n

    cores = oracle.num_threads()
    n, dt = timed(seconds)
    what = (f"{len(seqs)} sequences x {w.num_q_heads} heads of the same workload (append of all "
            f"{len(w.slot_mapping)} rows + attention of the sampled rows)")
    line = {"value": round(sample_bytes / dt / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{what}, {n} steps in {n * dt:.1f} s"}
    if cores > 1:  # the same sample on one core
        oracle.set_num_threads(1)
        try:
            n1, dt1 = timed(seconds / 4)
        finally:
            oracle.set_num_threads(cores)
        line["single_core"] = {"value": round(sample_bytes / dt1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                               "sample": f"{what}, {n1} steps in {n1 * dt1:.1f} s"}
    return line


def run_reference(args):
    """The oracle as the reference arm: rank 0 only, on host cores.  Each step
    is a bounded sample (the first query rows of the batch, all heads, sized so
    that warm-up plus timed steps take about --reference-seconds)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from paged_kv_cache_445_b200 import roofline, workloads
    import oracle
    w = workloads.standard(args.workload)
    kc, vc = w.k_cache, w.v_cache
    # calibrate: seconds per (row, head) item on the first sequence
    probe = np.array([(int(w.query_start[0]), h) for h in range(w.num_q_heads)], dtype=np.int32)
    t0 = time.perf_counter()
    oracle_step(oracle, w, probe, kc, vc)
    per_item = max((time.perf_counter() - t0) / len(probe), 1e-6)
    budget = args.reference_seconds / (args.steps + args.warmup)
    n_items = int(max(1, min(len(probe), budget / per_item)))
    only = probe[:n_items]
    kv_heads = sorted({int(h) // (w.num_q_heads // w.num_kv_heads) for _, h in only})
    sample_bytes = roofline.kv_cache_bytes(1, len(kv_heads), w.head_dim, int(w.context_lens[0]))
    for _ in range(args.warmup):
        oracle_step(oracle, w, only, kc, vc)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(oracle, w, only, kc, vc)
    dt = (time.perf_counter() - t0) / args.steps
    value = round(sample_bytes / dt / 1e9, 6)
    sample = (f"sequence 0 ({int(w.context_lens[0])} keys), {n_items} of {w.num_q_heads} query heads "
              f"({len(kv_heads)} KV heads), plus the append of all {len(w.slot_mapping)} new rows, per step")
    line = {
        "impl": "reference",
        "metric": "paged-attn decode KV GB/s + seq-steps/s (70B layer, bs128); % of HBM peak",
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded PCG64)",
        "config": {"workload": w.name, "num_seqs": w.num_seqs, "num_q_heads": w.num_q_heads,
                   "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size},
        "cpu_baseline": {"value": value, "unit": "GB/s", "kind": "oracle", "cores": oracle.num_threads(),
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", type=int, default=3, choices=[1, 2, 3, 4, 5, 6, 7])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--reference-seconds", type=float, default=90.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kv-dtype", default="bf16", choices=["bf16", "fp8"],
                    help="fp8: the cache holds E4M3 codes with per-tensor scales (decode workloads)")
    ap.add_argument("--graph", action="store_true",
                    help="capture one step (all its launches) in a CUDA graph and time its replays")
    ap.add_argument("--cascade", action="store_true",
                    help="shared-prefix batches: pa_decode_cascade (each shared prefix read once per group) "
                         "instead of plain decode")
    ap.add_argument("--no-calibrate", action="store_true",
                    help="leave out pa_calibrate: the decode kernel splits its work equally between warps")
    ap.add_argument("--no-plan", action="store_true",
                    help="varlen batches: pa_prefill_chunk without the host plan (every kernel launched, one after "
                         "the other on the whole GPU)")
    ap.add_argument("--no-sub-records", action="store_true",
                    help="the default run: leave out the other workloads' records (GRPO plain and cascade, mixed, FP8)")
    ap.add_argument("--sub-cpu-seconds", type=float, default=4.0,
                    help="oracle seconds of each sub-record's CPU baseline")
    ap.add_argument("--separate-append", action="store_true",
                    help="decode batches: pa_cache_append + pa_decode instead of the fused pa_decode_append")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
        return
    from paged_kv_cache_445_b200.csrc import build as pabuild
    pabuild.build()
    run_ours(args, measured_peaks())


if __name__ == "__main__":
    main()
