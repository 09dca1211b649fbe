"""Benchmark: one paged decode step per iteration on the batch-256 GQA layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload NAME] [--partition P]

A step is one pass of the whole hot path over one batch: copy_blocks (when
the workload has copy-on-write pairs), reshape_and_cache of the step's new
K/V, and paged decode attention (plus its split-KV merge when split).  Inputs
are resident in HBM when the timed region starts; the KV pool (2.5 GB for the
default workload) is larger than the 126 MB L2, so no flush is needed between
steps.  Timing: W untimed steps, then K steps between CUDA events on the
launching stream, bracketed by a barrier and device synchronisation; the
maximum over ranks is reported.  Under torchrun every rank runs its own
replica of the workload (independent sequences, no collective on the data
path): weak scaling.

value  = algorithmic bytes of the step / step time (GB/s): unique KV bytes
         read (2 * num_kv_heads * head_size * 2 per distinct cached token, the
         per-block formula of the KV-cache manager) + q + fp32 out + used
         block-table entries + context lengths + the cache write (new K/V in,
         rows out, slots) + copy-on-write bytes when present.
roofline = the decode-attention kernel alone: its algorithmic bytes per launch
         / its average CUDA-event duration, against the measured HBM peak.
e2e    = the same metric through the public API with host buffers: per step
         the step's inputs go host->device from pinned memory, the output
         comes back device->host, all inside the timed region.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = ("paged decode attn: KV GB/s and % of HBM peak; seq-tokens/s at "
          "batch 256")
DEFAULT_WORKLOAD = "llama2_70b_gqa_b256"
FALLBACK_HBM_GBS = 6650.0
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "dram_traffic_by_workload.txt")
_CSRC = os.path.join(ROOT, "paged_kv_cache_435_b200", "csrc")
# Sources whose change invalidates a recorded DRAM-traffic figure, per kernel.
KERNEL_SOURCES = {
    "paged_decode_kernel": ["pa_decode.cu", "pa_common.cuh", "pa_decode.cuh"],
    "paged_multi_row_kernel": ["pa_multi_row.cu", "pa_common.cuh", "pa_split.cuh",
                               "pa_cascade.cuh", "pa_multi_row.cuh"],
    "paged_multi_query_tc_kernel": ["pa_multi_query_tc.cu", "pa_common.cuh",
                                    "pa_split.cuh", "pa_multi_query.cuh"],
}


# ---------------------------------------------------------------- accounting
def attention_bytes(case, seqs=None) -> int:
    """Algorithmic bytes of one decode-attention call."""
    w = case.workload
    lens = case.lens_np if seqs is None else case.lens_np[seqs]
    B = len(lens)
    uniq = case.unique_tokens if seqs is None else int(lens.sum())
    kv = uniq * 2 * w.num_kv_heads * w.head_size * 2
    nq = B if case.query_lens_np is None else int(
        (case.query_lens_np if seqs is None else case.query_lens_np[seqs]).sum())
    q = nq * w.num_heads * w.head_size * 2
    out = nq * w.num_heads * w.head_size * 4
    tables = int((-(-lens // w.block_size)).sum()) * 4
    return kv + q + out + tables + B * 4


def attention_flops(case) -> int:
    """Dense flops of the attention: 4 * Hq * D per (query, visible token)
    pair (QK^T and PV multiply-adds)."""
    w = case.workload
    if case.query_lens_np is None:
        pairs = int(case.lens_np.sum())
    else:
        L, k = case.lens_np, case.query_lens_np
        pairs = int((k * (L - k) + k * (k + 1) // 2).sum())
    return pairs * 4 * w.num_heads * w.head_size


def step_bytes(case) -> int:
    w = case.workload
    row = w.num_kv_heads * w.head_size * 2
    live = int((case.slot_mapping.cpu() >= 0).sum())
    write = 2 * live * row * 2 + case.slot_mapping.numel() * 8
    cow = 0
    if case.copy_pairs.shape[0]:
        blk = w.block_size * row
        cow = case.copy_pairs.shape[0] * (2 * blk * 2 + 16)
    return attention_bytes(case) + write + cow


def kernel_sha(kernel: str = "paged_decode_kernel") -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(_CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def dominant_kernel(case, shared_prefix: bool) -> str:
    """The kernel whose DRAM traffic the roofline line reports."""
    if case.query_start_loc is not None:
        k = int(case.query_lens_np.max()) * (case.workload.num_heads //
                                             case.workload.num_kv_heads)
        return ("paged_multi_query_tc_kernel" if k >= 128 and case.workload.head_size == 128
                else "paged_multi_row_kernel")
    return "paged_multi_row_kernel" if shared_prefix else "paged_decode_kernel"


def read_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary: records of `key = value` lines separated by blank lines, used
    only while the record's kernel_sha matches the current kernel sources."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    records, cur = [], {}
    with open(PROFILE_TRAFFIC) as f:
        for line in f:
            line = line.strip()
            if not line:
                if cur:
                    records.append(cur)
                cur = {}
                continue
            if "=" in line and not line.startswith("#"):
                k, v = line.split("=", 1)
                cur[k.strip()] = v.strip()
    if cur:
        records.append(cur)
    for r in records:
        if (r.get("workload") == workload and r.get("kernel") == kernel and
                r.get("kernel_sha") == kernel_sha(kernel)):
            try:
                return float(r["dram_bytes_per_launch"])
            except (KeyError, ValueError):
                return None
    return None


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def tensor_peak():
    """Dense bf16 TFLOP/s for a kernel timed inside a long loop (sustained)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and throttle reasons via NVML while the timed region runs."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    }

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM))
                self.reasons |= int(n.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nvml is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._nvml is not None:
            self._t.join()

    def absorb(self, other: "ClockSampler"):
        """Add another sampler's record (a second timed region)."""
        self.samples.extend(other.samples)
        self.reasons |= other.reasons
        if self.max_mhz is None:
            self.max_mhz = other.max_mhz

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0}
        names = [v for k, v in self.REASONS.items()
                 if self.reasons & k and k != 0x1]
        return {"sm_mhz": float(np.median(self.samples)),
                "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ---------------------------------------------------------------- distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return dist
    return None


def barrier(dist):
    if dist is not None:
        dist.barrier()


def max_over_ranks(dist, x: float, device) -> float:
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- GPU arm
class Step:
    """Device buffers and the library calls of one decode step."""

    def __init__(self, case, partition_size: int, shared_prefix: bool = False):
        import paged_kv_cache_435_b200 as pa
        self.pa = pa
        self.case = case
        w = case.workload
        B = w.num_seqs
        _, Hq, D = case.q.shape
        self.out = torch.empty(case.q.shape, dtype=torch.float32,
                               device=case.q.device)
        self.maxlen = case.max_context_len
        self.partition = pa.pa_decode_partition_size(
            B, Hq, w.num_kv_heads, D, w.block_size, self.maxlen, partition_size)
        self.partition_arg = partition_size
        # Groups of sequences sharing prompt blocks: the shared-prefix call.
        self.shared_prefix = shared_prefix and case.group_start is not None
        size_fn = (pa.pa_shared_prefix_workspace_size if self.shared_prefix
                   else pa.pa_decode_workspace_size)
        nbytes = size_fn(B, Hq, w.num_kv_heads, D, w.block_size, self.maxlen,
                         partition_size)
        self.ws = (torch.empty(nbytes, dtype=torch.uint8, device=case.q.device)
                   if nbytes else None)
        self.flags = torch.zeros(1, dtype=torch.int32, device=case.q.device)

    def cache_ops(self):
        c = self.case
        if c.copy_pairs.shape[0]:
            self.pa.pa_copy_blocks([c.k_cache], [c.v_cache], c.copy_pairs,
                                   error_flags=self.flags)
        self.pa.pa_reshape_and_cache(c.new_key, c.new_value, c.k_cache,
                                     c.v_cache, c.slot_mapping,
                                     error_flags=self.flags)

    def attention(self):
        c = self.case
        if c.query_start_loc is not None:
            self.pa.pa_multi_query_attention(
                self.out, c.q, c.k_cache, c.v_cache, c.block_tables,
                c.context_lens, c.query_start_loc, self.maxlen,
                int(c.query_lens_np.max()), c.scale, error_flags=self.flags)
            return
        if self.shared_prefix:
            self.pa.pa_decode_attention_shared_prefix(
                self.out, c.q, c.k_cache, c.v_cache, c.block_tables,
                c.context_lens, c.group_start, c.prefix_lens, self.maxlen,
                c.max_group_size, c.scale, self.ws,
                partition_size=self.partition_arg, error_flags=self.flags)
            return
        self.pa.pa_decode_attention(
            self.out, c.q, c.k_cache, c.v_cache, c.block_tables, c.context_lens,
            self.maxlen, c.scale, partition_size=self.partition_arg,
            workspace=self.ws, error_flags=self.flags)


def run_gpu(args):
    import paged_kv_cache_435_b200 as pa
    from paged_kv_cache_435_b200 import inputs

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    pa.raw()  # fail loudly if the library is missing

    case = inputs.make_case(args.workload, device=dev, num_seqs=args.seqs)
    w = case.workload
    part = args.partition if args.partition is not None else w.partition_size
    step = Step(case, part, shared_prefix=not args.plain_decode)
    stream = torch.cuda.current_stream(dev)

    # in-run copy bandwidth (read + write bytes of a 1 GiB device copy)
    # and in-run read-only stream bandwidth (a 1 GiB fp32-accumulated sum:
    # the decode kernel only reads its big operand, which a copy peak, half
    # of whose bytes are writes, can understate)
    copy_best = read_best = None
    if not args.kernel_only:
        a = torch.ones(1 << 29, dtype=torch.bfloat16, device=dev)
        b = torch.empty_like(a)
        copy_best = read_best = 0.0
        for _ in range(6):
            e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
            e0.record(stream); b.copy_(a); e1.record(stream); e1.synchronize()
            copy_best = max(copy_best, 2 * a.numel() * 2 /
                            (e0.elapsed_time(e1) * 1e-3) / 1e9)
            e0.record(stream); a.sum(dtype=torch.float32); e1.record(stream)
            e1.synchronize()
            read_best = max(read_best, a.numel() * 2 /
                            (e0.elapsed_time(e1) * 1e-3) / 1e9)
        del a, b

    for _ in range(args.warmup):
        step.cache_ops(); step.attention()
    torch.cuda.synchronize(dev)

    K = args.steps
    ev_attn = [(torch.cuda.Event(True), torch.cuda.Event(True)) for _ in range(K)]
    t0, t1 = torch.cuda.Event(True), torch.cuda.Event(True)
    with ClockSampler(local) as clk:
        barrier(dist)
        torch.cuda.synchronize(dev)
        n0 = pa.pa_launch_count()
        t0.record(stream)
        for i in range(K):
            step.cache_ops()
            ev_attn[i][0].record(stream)
            step.attention()
            ev_attn[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        launches = pa.pa_launch_count() - n0
        barrier(dist)
    ms_total = t0.elapsed_time(t1)
    attn_ms = sum(s.elapsed_time(e) for s, e in ev_attn) / K
    flags = int(step.flags.item())

    # e2e: host buffers through the public API
    e2e = None
    if not args.kernel_only:
        e2e, e2e_clk = run_e2e(case, step, args, dist, dev)
        clk.absorb(e2e_clk)


    ms_total = max_over_ranks(dist, ms_total, dev)
    attn_ms_max = max_over_ranks(dist, attn_ms, dev)
    sb = step_bytes(case)
    ab = attention_bytes(case)
    ms_step = ms_total / K
    value = world * sb / (ms_step * 1e-3) / 1e9
    peak, peak_kind = hbm_peak()
    tpeak, tpeak_kind = tensor_peak()
    flops = attention_flops(case)
    ridge = tpeak * 1e12 / (peak * 1e9)          # flop per byte
    tensor_bound = flops / ab > ridge
    achieved = ab / (attn_ms_max * 1e-3) / 1e9
    achieved_tflops = flops / (attn_ms_max * 1e-3) / 1e12
    dom = dominant_kernel(case, step.shared_prefix)
    traffic = read_traffic(w.name, dom)
    if tensor_bound:
        roof = {"bound": "tensor", "achieved": round(achieved_tflops, 1),
                "peak": tpeak,
                "peak_source": f"{tpeak_kind} (MEASURED_PEAKS.json bf16_tflops_sustained)",
                "unit": "TFLOP/s", "frac": round(achieved_tflops / tpeak, 4)}
    else:
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                               if peak_kind == "measured" else "fallback 6.65 TB/s",
                "unit": "GB/s", "frac": round(achieved / peak, 4)}
    kernel_name = (dom if case.query_start_loc is not None
                   else ("paged_multi_row_kernel (group pass) + " if step.shared_prefix
                         else "") + "paged_decode_kernel" +
                   (" + reduce" if step.partition < case.max_context_len else ""))

    result = None
    if rank == 0:
        cpu = (cpu_baseline(args) if world == 1 and not args.kernel_only
               and case.query_start_loc is None else None)
        clocks = clk.summary()
        result = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": round(ms_step, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16, random scattered block tables)",
            "config": {
                "workload": w.name,
                "description": w.description,
                "num_seqs": w.num_seqs, "num_heads": w.num_heads,
                "num_kv_heads": w.num_kv_heads, "head_size": w.head_size,
                "block_size": w.block_size,
                "num_blocks": int(case.k_cache.shape[0]),
                "context_tokens": case.logical_tokens,
                "unique_kv_tokens": case.unique_tokens,
                "partition_size": step.partition,
                "step": ("copy_blocks + " if case.copy_pairs.shape[0] else "") +
                        "reshape_and_cache + " +
                        ("paged_multi_query_attention" if case.query_start_loc is not None
                         else "paged_decode_attention_shared_prefix" if step.shared_prefix
                         else "paged_decode_attention"),
                "query_tokens_per_seq": (1 if case.query_lens_np is None
                                         else w.query_len),
                "l2": "no flush: inputs larger than L2 (KV pool "
                      f"{2 * case.k_cache.numel() * 2 / 1e9:.2f} GB > 126 MB)",
                "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            },
            "seq_tokens_per_s": round(world * (w.num_seqs if case.query_lens_np is None else int(case.query_lens_np.sum())) / (ms_step * 1e-3), 1),
            "context_tokens_per_s": round(world * case.logical_tokens / (ms_step * 1e-3), 1),
            "pct_hbm_peak": round(100 * value / (world * peak), 2),
            "step_bytes": sb,
            "in_run_copy_gbs": None if copy_best is None else round(copy_best, 1),
            "in_run_read_gbs": None if read_best is None else round(read_best, 1),
            "roofline": dict(
                kernel=kernel_name, **roof,
                frac_of_in_run_copy=(None if copy_best is None or tensor_bound
                                     else round(achieved / copy_best, 4)),
                frac_of_in_run_read=(None if read_best is None or tensor_bound
                                     else round(achieved / read_best, 4)),
                traffic=traffic,
                traffic_kernel=dom,
                algorithmic_bytes_per_launch=ab,
                flops_per_launch=flops,
                achieved_gbs=round(achieved, 1),
                achieved_tflops=round(achieved_tflops, 2),
                avg_launch_ms=round(attn_ms_max, 5)),
            "e2e": e2e,
            "gpu_launches": int(launches),
            "device_error_flags": flags,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return result


def run_e2e(case, step, args, dist, dev):
    """Per step: pinned host -> device copies of the step's inputs, the
    library calls, device -> host copy of the output.  Inputs travel on one
    copy stream and outputs on another (the two directions use separate copy
    engines and overlap), double-buffered, so step i+1's inputs travel while
    step i computes and step i's output returns while step i+1 computes;
    every step's copies are inside the timed region.  The KV pool is written
    and read only on the compute stream, in step order.  Returns the e2e
    record and the clock sampler of its timed region."""
    import paged_kv_cache_435_b200 as pa
    c = case
    names = ["q", "new_key", "new_value", "slot_mapping", "block_tables",
             "context_lens"] + (["copy_pairs"] if c.copy_pairs.shape[0] else []) \
        + (["query_start_loc"] if c.query_start_loc is not None else []) \
        + (["group_start", "prefix_lens"] if step.shared_prefix else [])
    host_in = {n: getattr(c, n).cpu().pin_memory() for n in names}
    dev_in = [{n: torch.empty_like(getattr(c, n)) for n in names} for _ in range(2)]
    outs = [torch.empty_like(step.out) for _ in range(2)]
    host_out = [torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
                for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = host_out[0].numel() * host_out[0].element_size()
    comp = torch.cuda.current_stream(dev)
    up = torch.cuda.Stream(dev)     # host -> device
    down = torch.cuda.Stream(dev)   # device -> host
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready = [ev(), ev()]     # inputs of buffer b landed
    in_free = [ev(), ev()]      # compute finished reading buffer b
    out_ready = [ev(), ev()]    # output of buffer b computed
    out_free = [ev(), ev()]     # output of buffer b copied to the host
    for e in in_free + out_free:
        e.record(comp)

    def stage_inputs(b):
        with torch.cuda.stream(up):
            up.wait_event(in_free[b])
            for n in names:
                dev_in[b][n].copy_(host_in[n], non_blocking=True)
            in_ready[b].record(up)

    def compute(b):
        d = dev_in[b]
        comp.wait_event(in_ready[b])
        comp.wait_event(out_free[b])
        if c.copy_pairs.shape[0]:
            pa.pa_copy_blocks([c.k_cache], [c.v_cache], d["copy_pairs"],
                              error_flags=step.flags, stream=comp)
        pa.pa_reshape_and_cache(d["new_key"], d["new_value"], c.k_cache,
                                c.v_cache, d["slot_mapping"],
                                error_flags=step.flags, stream=comp)
        if c.query_start_loc is not None:
            pa.pa_multi_query_attention(
                outs[b], d["q"], c.k_cache, c.v_cache, d["block_tables"],
                d["context_lens"], d["query_start_loc"], step.maxlen,
                int(c.query_lens_np.max()), c.scale, error_flags=step.flags,
                stream=comp)
        elif step.shared_prefix:
            pa.pa_decode_attention_shared_prefix(
                outs[b], d["q"], c.k_cache, c.v_cache, d["block_tables"],
                d["context_lens"], d["group_start"], d["prefix_lens"],
                step.maxlen, c.max_group_size, c.scale, step.ws,
                partition_size=step.partition_arg, error_flags=step.flags,
                stream=comp)
        else:
            pa.pa_decode_attention(outs[b], d["q"], c.k_cache, c.v_cache,
                                   d["block_tables"], d["context_lens"],
                                   step.maxlen, c.scale,
                                   partition_size=step.partition_arg,
                                   workspace=step.ws, error_flags=step.flags,
                                   stream=comp)
        in_free[b].record(comp)
        out_ready[b].record(comp)

    def return_output(b):
        with torch.cuda.stream(down):
            down.wait_event(out_ready[b])
            host_out[b].copy_(outs[b], non_blocking=True)
            out_free[b].record(down)

    def run(n):
        stage_inputs(0)
        for i in range(n):
            if i + 1 < n:
                stage_inputs((i + 1) % 2)
            compute(i % 2)
            return_output(i % 2)

    run(args.warmup)
    torch.cuda.synchronize(dev)
    K = args.steps
    t0, t1 = torch.cuda.Event(True), torch.cuda.Event(True)
    with ClockSampler(dev.index) as clk:
        barrier(dist)
        torch.cuda.synchronize(dev)
        t0.record(comp)
        run(K)
        comp.wait_stream(down)  # the last output has reached the host
        t1.record(comp)
        torch.cuda.synchronize(dev)
        barrier(dist)
    ms = max_over_ranks(dist, t0.elapsed_time(t1), dev) / K

    # Breakdown: each direction's copies alone, K steps' worth, on its stream.
    def copy_ms(stream, fn):
        e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        with torch.cuda.stream(stream):
            for i in range(K):
                fn(i % 2)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / K

    h2d_ms = copy_ms(up, lambda b: [dev_in[b][n].copy_(host_in[n], non_blocking=True)
                                    for n in names])
    d2h_ms = copy_ms(down, lambda b: host_out[b].copy_(outs[b], non_blocking=True))
    world = dist.get_world_size() if dist is not None else 1
    return {"value": round(world * step_bytes(case) / (ms * 1e-3) / 1e9, 2),
            "unit": "GB/s", "ms_per_step": round(ms, 5),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "h2d_ms_per_step_alone": round(h2d_ms, 5),
            "d2h_ms_per_step_alone": round(d2h_ms, 5),
            "overlap": "double-buffered on two copy streams (inputs up, "
                       "outputs down): step i+1's inputs and step i's output "
                       "cross PCIe while step i / i+1 compute"}, clk


# ---------------------------------------------------------------- CPU (oracle)
def oracle_sample(workload: str, n_seqs: int):
    """A bounded sample of the workload built on the host: the first n_seqs
    sequences of its seeded length draw, same shapes, its own pool."""
    from paged_kv_cache_435_b200 import inputs
    w = inputs.WORKLOADS[workload]
    if w.lengths == "shared":
        full = inputs.make_case(workload)  # host-sized (0.3 GB pool)
        return full, np.arange(min(n_seqs, w.num_seqs))
    rng = np.random.default_rng(1000 + w.wid)
    lens = inputs.draw_lengths(w.lengths, w.num_seqs, rng)[:n_seqs]
    sub = dataclasses.replace(w, num_seqs=len(lens), name=w.name + "_sample")
    return inputs.build_case(sub, lens, seed=4242), None


def time_oracle(case, seqs, threads):
    import oracle
    q, tables, lens = case.q, case.tables_np, case.lens_np.astype(np.int32)
    if seqs is not None:
        q = q[torch.from_numpy(seqs)]
        tables, lens = tables[seqs], lens[seqs]
    t = time.perf_counter()
    oracle.paged_decode_attention(q, case.k_cache, case.v_cache, tables, lens,
                                  case.scale, case.workload.num_kv_heads,
                                  threads=threads)
    return time.perf_counter() - t


def sample_bytes(case, seqs):
    if seqs is None:
        return attention_bytes(case)
    # a shared-prefix sample: count the distinct cached tokens it reads
    w = case.workload
    bs = w.block_size
    slots = set()
    for s in seqs:
        L = int(case.lens_np[s])
        row = case.tables_np[s]
        slots.update(int(row[t // bs]) * bs + t % bs for t in range(L))
    B = len(seqs)
    lens = case.lens_np[seqs]
    kv = len(slots) * 2 * w.num_kv_heads * w.head_size * 2
    tables = int((-(-lens // bs)).sum()) * 4
    return kv + B * w.num_heads * w.head_size * 6 + tables + B * 4


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(args, budget_s: float = 10.0, budget_1core_s: float = 8.0):
    """The fp64 oracle on the host: all threads on a 64-sequence sample for
    about budget_s, then one thread on the first 8 of those sequences for
    about budget_1core_s."""
    import oracle
    oracle.build()
    threads = oracle.default_threads()
    case, seqs = oracle_sample(args.workload, 64)
    nbytes = sample_bytes(case, seqs)
    reps, elapsed = 0, 0.0
    while elapsed < budget_s or reps == 0:
        elapsed += time_oracle(case, seqs, threads)
        reps += 1
    n = case.workload.num_seqs if seqs is None else len(seqs)

    case1, seqs1 = oracle_sample(args.workload, 8)
    nbytes1 = sample_bytes(case1, seqs1)
    reps1, elapsed1 = 0, 0.0
    while elapsed1 < budget_1core_s or reps1 == 0:
        elapsed1 += time_oracle(case1, seqs1, 1)
        reps1 += 1
    n1 = case1.workload.num_seqs if seqs1 is None else len(seqs1)
    return {"value": round(reps * nbytes / elapsed / 1e9, 4), "unit": "GB/s",
            "cores": threads, "kind": "oracle",
            "sample": f"{n} sequences of {args.workload} (same shapes and "
                      f"length draw, host-built pool), {reps} passes, "
                      f"{elapsed:.1f} s, fp64 C oracle on {threads} threads; "
                      f"1 thread: {n1} sequences, {reps1} passes, {elapsed1:.1f} s",
            "seq_tokens_per_s": round(reps * n / elapsed, 2),
            "value_1core": round(reps1 * nbytes1 / elapsed1 / 1e9, 4),
            "seq_tokens_per_s_1core": round(reps1 * n1 / elapsed1, 2),
            "os_cpu_count": os.cpu_count(),
            "cpu_model": cpu_model()}


def run_reference(args):
    """The oracle as the reference arm: each step one bounded sample."""
    world, rank, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    oracle.build()
    threads = oracle.default_threads()
    # size one step's sample so warm-up + timed steps take about two minutes
    probe, pseqs = oracle_sample(args.workload, 4)
    per_seq = time_oracle(probe, pseqs, threads) / 4
    budget = min(2.0, 120.0 / (args.steps + args.warmup))
    from paged_kv_cache_435_b200 import inputs
    n = int(max(1, min(inputs.WORKLOADS[args.workload].num_seqs,
                       round(budget / max(per_seq, 1e-6)))))
    case, seqs = oracle_sample(args.workload, n)
    nbytes = sample_bytes(case, seqs)
    for _ in range(args.warmup):
        time_oracle(case, seqs, threads)
    t = 0.0
    for _ in range(args.steps):
        t += time_oracle(case, seqs, threads)
    ms = 1e3 * t / args.steps
    value = nbytes / (ms * 1e-3) / 1e9
    n = case.workload.num_seqs if seqs is None else len(seqs)
    from paged_kv_cache_435_b200 import inputs
    w = inputs.WORKLOADS[args.workload]
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16, random scattered block tables)",
        "config": {"workload": w.name, "description": w.description,
                   "sample_seqs_per_step": n},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s",
                         "cores": threads, "kind": "oracle",
                         "os_cpu_count": os.cpu_count(), "cpu_model": cpu_model(),
                         "sample": f"{n} sequences of {w.name} per step, fp64 C "
                                   f"oracle on {threads} threads"},
        "e2e": {"value": round(value, 4), "unit": "GB/s",
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_swap(args):
    """swap_blocks bandwidth: 4096 blocks of the batch-256 GQA pool shape
    (K and V, 32 KB each) to pinned host memory and back, against a plain
    pinned-memory copy of the same bytes in each direction."""
    import paged_kv_cache_435_b200 as pa
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    nb_gpu, n, shape = 8192, 4096, (16, 8, 128)
    gen = torch.Generator(device=dev).manual_seed(5)
    gpu = [torch.randn(nb_gpu, *shape, device=dev, generator=gen).to(torch.bfloat16)
           for _ in range(2)]
    cpu = [torch.empty(n, *shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    rng = np.random.default_rng(9)
    src = rng.permutation(nb_gpu)[:n]
    out_pairs = torch.from_numpy(np.stack([src, np.arange(n)], 1).astype(np.int64)).to(dev)
    in_pairs = torch.from_numpy(np.stack([np.arange(n), src], 1).astype(np.int64)).to(dev)
    nbytes = 2 * n * gpu[0][0].numel() * 2
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / args.steps

    ms_out = timed(lambda: pa.pa_swap_blocks(gpu, cpu, out_pairs))
    ms_in = timed(lambda: pa.pa_swap_blocks(cpu, gpu, in_pairs))
    flat_g = torch.empty(nbytes // 2, dtype=torch.bfloat16, device=dev)
    flat_h = torch.empty(nbytes // 2, dtype=torch.bfloat16).pin_memory()
    ms_d2h = timed(lambda: flat_h.copy_(flat_g, non_blocking=True))
    ms_h2d = timed(lambda: flat_g.copy_(flat_h, non_blocking=True))
    gbs = lambda ms: round(nbytes / (ms * 1e-3) / 1e9, 1)  # noqa: E731
    return {"metric": "swap_blocks GB/s (GPU <-> pinned host)",
            "blocks": n, "bytes_per_direction": nbytes,
            "swap_out_gbs": gbs(ms_out), "swap_in_gbs": gbs(ms_in),
            "pinned_copy_d2h_gbs": gbs(ms_d2h), "pinned_copy_h2d_gbs": gbs(ms_h2d),
            "frac_out": round(ms_d2h / ms_out, 4), "frac_in": round(ms_h2d / ms_in, 4),
            "steps": args.steps, "warmup": args.warmup}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--partition", type=int, default=None)
    ap.add_argument("--seqs", type=int, default=None,
                    help="keep only the first N sequences of the workload")
    ap.add_argument("--swap", action="store_true",
                    help="measure swap_blocks bandwidth instead (own JSON line)")
    ap.add_argument("--plain-decode", action="store_true",
                    help="attend workloads with shared-prefix groups with the "
                         "plain decode call (no group pass)")
    ap.add_argument("--kernel-only", action="store_true",
                    help="time the device step only: no e2e leg, no in-run "
                         "copy peak, no CPU baseline (profiling runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.swap:
        res = run_swap(args)
    else:
        res = run_reference(args) if args.impl == "reference" else run_gpu(args)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
