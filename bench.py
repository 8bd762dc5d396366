#!/usr/bin/env python
"""Decode-step throughput of retrieval block-sparse attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one whole decode step of the 128K-context GQA workload
(infllm-decode-128k: batch 1, 32 q / 8 kv heads, head_dim 128, 131072 past
tokens in 128-token blocks with 4 representative keys each; top-32 blocks
per kv head + 128 sink + 4096 window tokens): block scores -> top-k ->
attention over sink U selected blocks U window (the persistent kernel, which
starts while the selection runs) -> merge, all in librba.so.  Representations are memorised
once before timing (memorisation is not part of a decode step).

Measurement: W untimed warm-up steps, then exactly K steps replayed from CUDA
graphs, bracketed by a barrier and a device synchronise, timed with CUDA
events on the launching stream (max over ranks).  Steps rotate over R
replicas of the store so that R x bytes-per-step >= 4 x L2: every step reads
HBM, not L2.  Under torchrun each rank runs its own replica set on its own
GPU (replicas only: the path has no exchange step), and the value is the
total steps/s of all ranks.

--impl reference times the fp64 CPU oracle on this host on bounded samples of
the same workload (see run_reference).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "retrieval-attention decode steps/sec & achieved HBM GB/s (% roofline) at 128K ctx"
UNIT = "steps/s"
WORKLOAD = "infllm-decode-128k"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
KERNEL_SOURCES = {
    "attend_decode_kernel": ["csrc/attend.cu", "csrc/attend_impl.cuh", "csrc/rba_internal.cuh"],
    "decode_fused_kernel": ["csrc/decode_fused.cu", "csrc/attend_impl.cuh",
                            "csrc/rba_internal.cuh"],
    "decode_mma_kernel": ["csrc/decode_fused.cu", "csrc/decode_persist.cuh",
                          "csrc/attend_impl.cuh", "csrc/rba_internal.cuh", "csrc/tmap.cu"],
    "decode_step_kernel": ["csrc/decode_step.cu", "csrc/decode_persist.cuh",
                           "csrc/attend_impl.cuh", "csrc/rba_internal.cuh", "csrc/tmap.cu"],
}


# ---------------------------------------------------------------------------
# plumbing


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="bound on the oracle CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-config measurements (other decode configs, prefill)")
    ap.add_argument("--config-seconds", type=float, default=0.5,
                    help="timed GPU seconds per extra config")
    ap.add_argument("--workload", default=WORKLOAD, help=argparse.SUPPRESS)
    # measure one entry of the configs block only (for profiling runs)
    ap.add_argument("--only-config", default=None, help=argparse.SUPPRESS)
    ap.add_argument("--replicas", type=int, default=0, help=argparse.SUPPRESS)
    return ap.parse_args(argv)


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(value: float, device) -> float:
    """Max of a per-rank value over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, bf16_tflops_sustained=1400.0, source="fallback")


def _code_only(text):
    """Source text without comments and blank space: edits to comments do not
    change a kernel, so they do not invalidate its recorded counters."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def source_hash(kernel):
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES.get(kernel, []):
        with open(os.path.join(ROOT, "retrieval_block_sparse_b200", rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def traffic_lookup(kernel, workload, path=None):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current source of the kernel (else None)."""
    p = path or os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None
    want = source_hash(kernel)
    with open(p) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel \
                    and parts[1] == want and parts[2] == workload:
                return float(parts[3])
    return None


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML while running."""

    NAMES = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
             0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
             0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, torch_device: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml as nv
            import torch
            nv.nvmlInit()
            pr = torch.cuda.get_device_properties(torch_device)
            try:
                bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
                self.h = nv.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = nv.nvmlDeviceGetHandleByIndex(torch_device)
            self.nv = nv
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: clocks reported as unavailable
            self.err = str(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((time.time(), sm, rs, pw))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"unavailable": getattr(self, "err", "nvml")}
        sel = [s for s in self.samples if t0 <= s[0] <= t1] or self.samples[-3:]
        reasons = set()
        for _, _, rs, _ in sel:
            for bit, name in self.NAMES.items():
                if rs & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": float(np.median([s[1] for s in sel])) if sel else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons), "samples": len(sel),
                "power_w_max": max((s[3] for s in sel), default=None), "source": "nvml"}


# ---------------------------------------------------------------------------
# workload bookkeeping (sizes only; no method arithmetic)


def attended_counts(idx, T, bs, sink, window):
    """Tokens attended per (b, kv head) for block selection idx [B][Hkv][k]."""
    w0 = max(T - window, 0)
    base = min(sink, w0) + (T - w0)
    lo = np.maximum(idx.astype(np.int64) * bs, sink)
    hi = np.minimum((idx.astype(np.int64) + 1) * bs, w0)
    return base + np.clip(hi - lo, 0, None).sum(axis=-1)


def step_bytes(w, nc, idx):
    es = 2 if w.dtype == "bf16" else 4
    rep_es = 4 if w.rep_mode == "mean" else es
    rep = w.batch * w.n_kv_heads * nc * w.n_rep * w.head_dim * rep_es
    gathered = int(attended_counts(idx, w.context, w.block_size, w.sink, w.window).sum()) \
        * w.head_dim * es * 2
    return rep, gathered


def count_kernel_nodes(graph):
    """Kernel nodes in a captured torch CUDA graph (None if not introspectable)."""
    try:
        from cuda.bindings import runtime as rt
    except Exception:
        try:
            from cuda import cudart as rt
        except Exception:
            return None
    try:
        raw = graph.raw_cuda_graph()
        err, _, n = rt.cudaGraphGetNodes(raw, 0)
        err, nodes, n = rt.cudaGraphGetNodes(raw, n)
        kinds = 0
        for node in nodes:
            e, t = rt.cudaGraphNodeGetType(node)
            if t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                kinds += 1
        return kinds
    except Exception:
        return None


def prefill_pairs(w, idx):
    """(query, key) pairs a prefill step attends: every row of a chunk sees the
    retrieved past tokens of its selection and its own chunk causally.
    idx: [n_chunks][n_sel][k] (n_sel = 1: one selection shared by all heads)."""
    counts = attended_counts(idx, w.context, w.block_size, w.sink, w.window)
    heads_per_sel = w.n_q_heads if idx.shape[1] == 1 else w.n_q_heads // w.n_kv_heads
    past = int(counts.sum()) * heads_per_sel * w.chunk_len
    own = w.n_chunks * w.n_q_heads * w.chunk_len * (w.chunk_len + 1) // 2
    return past + own


# ---------------------------------------------------------------------------
# our implementation


def run_ours(args):
    import torch
    import torch.distributed as dist

    import retrieval_block_sparse_b200 as rba
    from retrieval_block_sparse_b200 import synth

    rank, world, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    w = synth.WORKLOADS[args.workload]
    x = synth.decode_inputs(w)

    def to_dev(a):
        if w.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(
                torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)

    def new_store():
        return rba.Store(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                         head_dim=w.head_dim, block_size=w.block_size, capacity_tokens=w.context,
                         dtype=w.dtype, mode=w.rep_mode, n_rep=w.n_rep, device=dev)

    master = new_store()
    master.k.copy_(to_dev(x["K"]))
    master.v.copy_(to_dev(x["V"]))
    aux = None
    if w.rep_mode == "topr_attn":
        aux = to_dev(x["probe"])
    elif w.rep_mode == "external":
        aux = to_dev(x["landmarks"]).reshape(w.batch, w.n_kv_heads, w.n_blocks, 1, w.head_dim)
    master.memorize(None, None, first_block=0, n_blocks=w.n_blocks, aux=aux)
    q = to_dev(x["q"])
    first, nc = master.candidates(w.context, w.sink, w.window)
    idx0, _, _ = master.decode_step(q, w.top_k, w.context, w.sink, w.window)
    master.check()
    rep_b, gath_b = step_bytes(w, nc, idx0.cpu().numpy())
    bytes_step = rep_b + gath_b

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = args.replicas or max(2, math.ceil(4 * l2 / bytes_step))
    stores = [master] + [new_store() for _ in range(R - 1)]
    for s in stores[1:]:
        s.k.copy_(master.k)
        s.v.copy_(master.v)
        if master.rep is not None:
            s.rep.copy_(master.rep)
    ws = [s.decode_workspace(w.top_k, w.context, w.sink, w.window) for s in stores]
    outs = [torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=torch.float32, device=dev)
            for _ in stores]
    lses = [torch.empty((w.batch, w.n_q_heads), dtype=torch.float32, device=dev) for _ in stores]
    idxs = [torch.empty((w.batch, w.n_kv_heads, w.top_k), dtype=torch.int32, device=dev)
            for _ in stores]

    def step(r):
        stores[r].decode_step(q, w.top_k, w.context, w.sink, w.window, workspace=ws[r],
                              out=outs[r], lse=lses[r], idx=idxs[r])

    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for r in range(R):  # eager warm-up of every replica before capture
            step(r)
    torch.cuda.synchronize(dev)

    def capture(n, start=0):
        """One CUDA graph of n decode steps over the replicas, from replica `start`."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                step((start + i) % R)
        return g

    # The timed region is exactly args.steps steps, replayed from graphs of at
    # most CHUNK steps (a multiple of R, so every replay starts at replica 0),
    # enqueued behind an untimed pre-roll of R steps: the GPU never waits for
    # the host to launch the next graph, at any step count.
    chunk = min(args.steps, max(R, (1024 // R) * R))
    g_chunk = capture(chunk)
    n_chunks, rem = divmod(args.steps, chunk)
    g_rem = capture(rem) if rem else None
    g_pre = capture(R)
    g_one = capture(1)
    plan = master.decode_plan(w.top_k, w.context, w.sink, w.window)
    # score + top-k (one kernel for rows <= 8192 candidates, four above) + attention
    # as the library reports
    kern_per_step = master.decode_launches(w.top_k, w.context, w.sink, w.window)
    n_nodes = count_kernel_nodes(g_one)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):  # W untimed warm-up steps
            step(i % R)
    torch.cuda.synchronize(dev)

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.05)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    with torch.cuda.stream(stream):
        g_pre.replay()  # untimed: keeps the GPU busy while the timed graphs are enqueued
        with torch.cuda.nvtx.range("bench_timed"):
            ev0.record(stream)
            for _ in range(n_chunks):
                g_chunk.replay()
            if g_rem is not None:
                g_rem.replay()
            ev1.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)
    for s in stores:
        s.check()
    ms_max = reduce_max(ms, dev)
    steps_per_s = world * args.steps / (ms_max / 1e3)

    # dominant kernel alone: attention over the selected blocks (rba_attend:
    # the persistent kernel where the plan is 1, else split-K)
    aws = [s.attend_workspace(w.top_k, w.context, w.sink, w.window) for s in stores]

    def att(r):
        stores[r].attend(q, idxs[r], w.context, w.sink, w.window, out=outs[r], lse=lses[r],
                         workspace=aws[r])
    with torch.cuda.stream(stream):
        for r in range(R):
            att(r)
    g_att = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_att, stream=stream):
        for r in range(R):
            att(r)
    reps_att = max(1, 2000 // R)
    with torch.cuda.stream(stream):
        for _ in range(3):
            g_att.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps_att):
            g_att.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    att_us = e0.elapsed_time(e1) * 1e3 / (reps_att * R)
    # score kernel alone (rep-key stream)
    scs = [torch.empty((w.batch, w.n_kv_heads, nc), dtype=torch.float32, device=dev)
           for _ in stores]
    g_sc = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        for r in range(R):
            stores[r].score(q, w.context, w.sink, w.window, out=scs[r])
    with torch.cuda.graph(g_sc, stream=stream):
        for r in range(R):
            stores[r].score(q, w.context, w.sink, w.window, out=scs[r])
    with torch.cuda.stream(stream):
        for _ in range(3):
            g_sc.replay()
        e0.record(stream)
        for _ in range(reps_att):
            g_sc.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    score_us = e0.elapsed_time(e1) * 1e3 / (reps_att * R)

    pk = peaks()
    att_gbs = gath_b / (att_us * 1e-6) / 1e9
    step_us = ms_max * 1e3 / args.steps
    step_gbs = bytes_step / (step_us * 1e-6) / 1e9
    if plan == 3:
        # the whole step is one kernel: its algorithmic bytes over the average
        # step of the timed region (launch gaps included)
        dom = "decode_step_kernel"
        dom_bytes, dom_us, dom_gbs = bytes_step, step_us, step_gbs
    else:
        dom = {1: "decode_fused_kernel", 2: "decode_mma_kernel"}.get(plan,
                                                                     "attend_decode_kernel")
        dom_bytes, dom_us, dom_gbs = gath_b, att_us, att_gbs
    traffic = traffic_lookup(dom, args.workload)

    # end to end through the host-buffer entry point
    e2e = None
    if args.e2e_steps > 0:
        q_host = torch.empty_like(q, device="cpu").pin_memory()
        q_host.copy_(q.cpu())
        out_h = torch.empty(outs[0].shape, dtype=torch.float32).pin_memory()
        lse_h = torch.empty(lses[0].shape, dtype=torch.float32).pin_memory()
        idx_h = torch.empty(idxs[0].shape, dtype=torch.int32).pin_memory()
        q_devs = [torch.empty_like(q) for _ in stores]

        def e2e_step(i):
            r = i % R
            stores[r].decode_step_host(q_host, w.top_k, w.context, w.sink, w.window,
                                       q_dev=q_devs[r], idx_dev=idxs[r], out_dev=outs[r],
                                       lse_dev=lses[r], out_host=out_h, lse_host=lse_h,
                                       idx_host=idx_h, workspace=ws[r])
        with torch.cuda.stream(stream):
            for i in range(min(20, args.e2e_steps)):
                e2e_step(i)
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize(dev)
            e0.record(stream)
            for i in range(args.e2e_steps):
                e2e_step(i)
            e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = reduce_max(e0.elapsed_time(e1), dev)
        e2e = {"value": round(world * args.e2e_steps / (e_ms / 1e3), 2), "unit": UNIT,
               "h2d_bytes_per_step": q.numel() * q.element_size(),
               "d2h_bytes_per_step": out_h.numel() * 4 + lse_h.numel() * 4 + idx_h.numel() * 4,
               "steps": args.e2e_steps, "call": "rba_decode_step_host (pinned host buffers)"}

    configs = None
    if world == 1 and not args.no_configs:
        configs = measure_configs(dev, args.config_seconds)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, x, args.cpu_seconds, args.workload)

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return None
    launches = kern_per_step
    line = {
        "metric": METRIC, "value": round(steps_per_s, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_us / 1e3, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded generator; K,V~N(0,1), planted per-head bias, 16-query probe)",
        "config": {**workload_config(args.workload, w, nc),
                   "l2": f"inputs larger than L2: {R} store replicas rotated "
                         f"({R} x {bytes_step / 1e6:.1f} MB >= 4 x {l2 / 1e6:.0f} MB L2)",
                   "parallelism": f"replicas x{world} (no exchange step)",
                   "timed_region": f"{args.steps} steps in CUDA graphs of <= {chunk} steps, "
                                   f"behind an untimed {R}-step pre-roll"},
        "roofline": {"bound": "hbm", "kernel": dom,
                     "achieved": round(dom_gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": round(dom_gbs / pk["hbm_gbs"], 4),
                     "peak_source": f"{pk['source']} (MEASURED_PEAKS.json hbm_gbs)"
                     if pk["source"] == "measured" else "fallback 6650 GB/s",
                     "traffic": traffic, "algorithmic_bytes": dom_bytes,
                     "launch_us": round(dom_us, 3)},
        "step": {"algorithmic_bytes": bytes_step, "rep_key_bytes": rep_b,
                 "gathered_kv_bytes": gath_b, "us": round(step_us, 3),
                 "achieved_gbs": round(step_gbs, 1),
                 "frac_of_hbm": round(step_gbs / pk["hbm_gbs"], 4),
                 "attend_kernel_alone_us": round(att_us, 3),
                 "attend_kernel_alone_gbs": round(att_gbs, 1),
                 "score_kernel_alone_us": round(score_us, 3),
                 "score_kernel_alone_gbs": round(rep_b / (score_us * 1e-6) / 1e9, 1)},
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": launches * args.steps,
        "kernels_per_step": launches,
        "graph_kernel_nodes_per_step": n_nodes,
        "path": ("one cooperative launch: score slices -> per-head top-k -> tensor-core "
                 "attention" if plan == 3 else
                 "score -> top-k -> persistent attention (programmatic dependent launches; "
                 + ("whole-block tensor-core kernel)" if plan == 2 else "CUDA-core kernel)")
                 if plan in (1, 2) else f"score -> top-k -> split-K attention (plan {plan})"),
        "cpu_baseline": cpu,
        "configs": configs,
    }
    return line


def _to_dev(a, dtype, dev):
    import torch
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(
            torch.bfloat16).to(dev)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)


def _time_graph(g, stream, seconds, min_iters=5):
    """Average ms per replay of CUDA graph g, over about `seconds` of replays."""
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
        e0.record(stream)
        for _ in range(min_iters):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    est = e0.elapsed_time(e1) / min_iters
    n = max(min_iters, int(seconds * 1e3 / max(est, 1e-3)))
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(n):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n, n


def measure_decode_config(name, dev, seconds, pk, score_reduce="sum", workload=None,
                          one_launch=False):
    """Decode-step throughput of one decode config (graph-replayed steps; L2
    defeated by rotating store replicas, or by an L2-sized write between
    steps whose own time is subtracted when replicas would not fit).
    score_reduce="max": the max-over-representative-keys score variant;
    one_launch: the step as one cooperative launch where eligible."""
    import torch
    import retrieval_block_sparse_b200 as rba
    from retrieval_block_sparse_b200 import synth
    w = workload if workload is not None else synth.WORKLOADS[name]
    x = synth.decode_inputs(w)

    def new_store():
        s = rba.Store(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                      head_dim=w.head_dim, block_size=w.block_size, capacity_tokens=w.context,
                      dtype=w.dtype, mode=w.rep_mode, n_rep=w.n_rep, device=dev,
                      score_reduce=score_reduce)
        if one_launch:
            s.set_decode_step_one_launch(True)
        return s
    st = new_store()
    st.kv_rows(st.k).copy_(_to_dev(x["K"], w.dtype, dev))
    st.kv_rows(st.v).copy_(_to_dev(x["V"], w.dtype, dev))
    aux = None
    if w.rep_mode == "topr_attn":
        aux = _to_dev(x["probe"], w.dtype, dev)
    elif w.rep_mode == "external":
        aux = _to_dev(x["landmarks"], w.dtype, dev).reshape(w.batch, w.n_kv_heads, w.n_blocks,
                                                             1, w.head_dim)
    if w.rep_mode != "identity":
        st.memorize(None, None, first_block=0, n_blocks=w.n_blocks, aux=aux)
    del x["K"], x["V"]
    q = _to_dev(x["q"], w.dtype, dev)
    first, nc = st.candidates(w.context, w.sink, w.window)
    idx0, _, _ = st.decode_step(q, w.top_k, w.context, w.sink, w.window)
    st.check()
    rep_b, gath_b = step_bytes(w, nc, idx0.cpu().numpy())
    nbytes = rep_b + gath_b
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    store_bytes = st.k.numel() * st.k.element_size() * 2 + (
        st.rep.numel() * st.rep.element_size() if st.rep is not None else 0)
    R = max(1, math.ceil(4 * l2 / nbytes))
    use_flush = R > 16 or R * store_bytes > 48e9
    stores = [st]
    if not use_flush:
        for _ in range(R - 1):
            s2 = new_store()
            s2.k.copy_(st.k)
            s2.v.copy_(st.v)
            if st.rep is not None:
                s2.rep.copy_(st.rep)
            stores.append(s2)
    ws = [s.decode_workspace(w.top_k, w.context, w.sink, w.window) for s in stores]
    outs = [torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=torch.float32, device=dev)
            for _ in stores]
    lses = [torch.empty((w.batch, w.n_q_heads), dtype=torch.float32, device=dev)
            for _ in stores]
    idxs = [torch.empty((w.batch, w.n_kv_heads, w.top_k), dtype=torch.int32, device=dev)
            for _ in stores]
    flush = torch.empty(max(4 * l2, 1 << 20), dtype=torch.uint8, device=dev) if use_flush \
        else None

    def step(r):
        stores[r].decode_step(q, w.top_k, w.context, w.sink, w.window, workspace=ws[r],
                              out=outs[r], lse=lses[r], idx=idxs[r])
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for r in range(len(stores)):
            step(r)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for r in range(len(stores)):
            if use_flush:
                flush.fill_(1)
            step(r)
    ms, n = _time_graph(g, stream, seconds)
    ms /= len(stores)
    if use_flush:
        gf = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gf, stream=stream):
            flush.fill_(1)
        ms_f, _ = _time_graph(gf, stream, seconds / 4)
        ms -= ms_f
    for s in stores:
        s.check()
    us = ms * 1e3
    gbs = nbytes / (us * 1e-6) / 1e9
    plan = st.decode_plan(w.top_k, w.context, w.sink, w.window)
    return {"workload": name, "head_dim": w.head_dim, "score_reduce": score_reduce,
            "steps_per_s": round(1e6 / us, 2), "us_per_step": round(us, 3),
            "algorithmic_bytes": nbytes, "rep_key_bytes": rep_b, "gathered_kv_bytes": gath_b,
            "achieved_gbs": round(gbs, 1), "frac_of_hbm": round(gbs / pk["hbm_gbs"], 4),
            "path": {1: "pipelined, persistent attention (CUDA cores)",
                     2: "pipelined, persistent attention (whole-block, tensor cores)",
                     3: "one cooperative launch (score, top-k, tensor-core attention)"}.get(
                         plan, "split-K attention"),
            "kernels_per_step": st.decode_launches(w.top_k, w.context, w.sink, w.window),
            "steps_timed": n * len(stores),
            "l2": (f"L2-sized write between steps, its time subtracted" if use_flush else
                   f"{len(stores)} store replicas rotated ({len(stores)} x {nbytes / 1e6:.1f} MB"
                   f" >= 4 x L2)")}


def measure_prefill_config(name, dev, seconds, pk, workload=None):
    """Chunked-prefill step of one prefill config: selection (score + top-k)
    and the retrieval-causal tensor-core attention, timed apart."""
    import torch
    import retrieval_block_sparse_b200 as rba
    from retrieval_block_sparse_b200 import synth
    w = workload if workload is not None else synth.WORKLOADS[name]
    x = synth.prefill_inputs(w)
    mode = "embed_cosine" if w.score_mode == "cosine" else (
        "identity" if w.block_size == 1 else "mean")
    st = rba.Store(batch=1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                   block_size=w.block_size, capacity_tokens=w.context, dtype=w.dtype, mode=mode,
                   d_ret=w.d_ret, device=dev)
    st.kv_rows(st.k).copy_(_to_dev(x["K"], w.dtype, dev))
    st.kv_rows(st.v).copy_(_to_dev(x["V"], w.dtype, dev))
    del x["K"], x["V"]
    nb = w.context // w.block_size
    if mode == "embed_cosine":
        st.memorize(None, None, first_block=0, n_blocks=nb,
                    aux=torch.from_numpy(x["bank_embed"]).to(dev).reshape(1, nb, w.d_ret))
    elif mode == "mean":
        st.memorize(None, None, first_block=0, n_blocks=nb)
    Q = _to_dev(x["Q"], w.dtype, dev)
    Kc, Vc = _to_dev(x["chunk_K"], w.dtype, dev), _to_dev(x["chunk_V"], w.dtype, dev)
    first, nc = st.candidates(w.context, w.sink, w.window)
    qsel = torch.from_numpy(x["query_embed"]).to(dev) if mode == "embed_cosine" else Q
    n_sel = 1 if mode == "embed_cosine" else w.n_kv_heads
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream())
    sc = st.score(qsel, w.context, w.sink, w.window)
    idx = rba.topk(sc.reshape(-1, nc), w.top_k, index_base=first).reshape(w.n_chunks, n_sel,
                                                                           w.top_k)
    out = torch.empty(Q.shape, dtype=torch.float32, device=dev)
    lse = torch.empty(Q.shape[:3], dtype=torch.float32, device=dev)
    ws = st.prefill_workspace(w.n_chunks, w.chunk_len, n_sel, w.top_k, w.context, w.sink,
                              w.window)
    rows = sc.numel() // nc
    topk_ws = torch.empty(max(rba.lib().rba_topk_workspace_size(rows, nc, w.top_k), 16),
                          dtype=torch.uint8, device=dev)

    def select():
        st.score(qsel, w.context, w.sink, w.window, out=sc)
        rba.topk(sc.reshape(-1, nc), w.top_k, index_base=first, out=idx.reshape(-1, w.top_k),
                 workspace=topk_ws)

    def attend():
        st.attend_prefill(Q, idx, Kc, Vc, w.context, w.sink, w.window, out=out, lse=lse,
                          workspace=ws)
    with torch.cuda.stream(stream):
        select()
        attend()
    torch.cuda.synchronize()
    st.check()
    gs, ga = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(gs, stream=stream):
        select()
    with torch.cuda.graph(ga, stream=stream):
        attend()
    ms_s, _ = _time_graph(gs, stream, seconds / 2)
    ms_a, n_a = _time_graph(ga, stream, seconds)
    st.check()
    pairs = prefill_pairs(w, idx.cpu().numpy())
    flops = 4 * w.head_dim * pairs
    tflops = flops / (ms_a * 1e-3) / 1e12
    scan = None if mode == "embed_cosine" else (
        w.n_kv_heads * nc * w.head_dim * 2 if mode == "identity" else
        w.n_kv_heads * nc * w.head_dim * 4)
    del topk_ws
    res = {"workload": name, "head_dim": w.head_dim, "attend_us": round(ms_a * 1e3, 2),
           "attend_calls_timed": n_a,
           "pairs": pairs, "flops": flops, "attend_tflops": round(tflops, 1),
           "attend_frac_of_bf16_peak": round(tflops / pk["bf16_tflops"], 4),
           "bf16_peak_tflops": pk["bf16_tflops"], "select_us": round(ms_s * 1e3, 2),
           "l2": "inputs larger than L2 (K/V of the retrieved set + chunk + Q)"}
    if scan is not None:
        res["select_scan_bytes"] = scan
        res["select_gbs"] = round(scan / (ms_s * 1e-3) / 1e9, 1)
        res["select_frac_of_hbm"] = round(scan / (ms_s * 1e-3) / 1e9 / pk["hbm_gbs"], 4)
    return res


def measure_approx_config(dev, seconds, pk, group=64, kept=256):
    """Two-stage approximate token retrieval (RetrievalAttention summary,
    "proposed method") on the 1M-token decode shape with drift keys (nearby
    keys resemble each other; the regime a group-mean index exploits): per
    step rba_approx_select + rba_attend, graph-replayed with an L2-sized write
    between steps whose own time is subtracted.  Reports recall of its tokens
    against the exact top-k of the same store (rba_score + rba_topk), keys and
    bytes read per step, and the exact step on the same store for contrast."""
    import torch
    import retrieval_block_sparse_b200 as rba
    from retrieval_block_sparse_b200 import synth
    w = synth.WORKLOADS["token-retrieval-decode-1m"].scaled(recipe="drift")
    x = synth.decode_inputs(w)
    st = rba.Store(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   head_dim=w.head_dim, block_size=1, capacity_tokens=w.context,
                   dtype=w.dtype, mode="identity", device=dev)
    st.k.copy_(_to_dev(x["K"], w.dtype, dev))
    st.v.copy_(_to_dev(x["V"], w.dtype, dev))
    del x["K"], x["V"]
    q = _to_dev(x["q"], w.dtype, dev)
    means = st.group_means(group)
    BH = w.batch * w.n_kv_heads
    idx = torch.empty((w.batch, w.n_kv_heads, w.top_k), dtype=torch.int32, device=dev)
    groups = torch.empty((w.batch, w.n_kv_heads, kept), dtype=torch.int32, device=dev)
    scanned = torch.empty((w.batch, w.n_kv_heads), dtype=torch.int32, device=dev)
    out = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=torch.float32, device=dev)
    lse = torch.empty((w.batch, w.n_q_heads), dtype=torch.float32, device=dev)
    n = rba.lib().rba_approx_select_workspace_size(st.handle, w.context, w.sink, w.window,
                                                   group, kept, w.top_k)
    sel_ws = torch.zeros(max(n, 16), dtype=torch.uint8, device=dev)
    att_ws = st.attend_workspace(w.top_k, w.context, w.sink, w.window)
    step_ws = st.decode_workspace(w.top_k, w.context, w.sink, w.window)
    eidx = torch.empty_like(idx)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(4 * l2, dtype=torch.uint8, device=dev)

    def approx_step():
        st.approx_select(q, w.context, w.sink, w.window, group, kept, w.top_k, means, idx=idx,
                         groups_out=groups, scanned=scanned, workspace=sel_ws)
        st.attend(q, idx, w.context, w.sink, w.window, out=out, lse=lse, workspace=att_ws)

    def exact_step():
        st.decode_step(q, w.top_k, w.context, w.sink, w.window, workspace=step_ws, idx=eidx,
                       out=out, lse=lse)
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        approx_step()
        exact_step()
    torch.cuda.synchronize()
    st.check()
    a_idx, e_idx = idx.cpu().numpy(), eidx.cpu().numpy()
    recall = float(np.mean([len(set(a_idx[b, h]) & set(e_idx[b, h])) / w.top_k
                            for b in range(w.batch) for h in range(w.n_kv_heads)]))
    graphs = {}
    for name, fn in (("approx", approx_step), ("exact", exact_step), ("flush", None)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            flush.fill_(1)
            if fn is not None:
                fn()
        graphs[name] = g
    ms_f, _ = _time_graph(graphs["flush"], stream, seconds / 4)
    ms_a, n_a = _time_graph(graphs["approx"], stream, seconds)
    ms_e, _ = _time_graph(graphs["exact"], stream, seconds)
    st.check()
    us_a, us_e = (ms_a - ms_f) * 1e3, (ms_e - ms_f) * 1e3
    keys_read = int(scanned.cpu().numpy().astype(np.int64).sum())
    first, nc = st.candidates(w.context, w.sink, w.window)
    n_groups = int(count_groups(w, group))
    es = 2 if w.dtype == "bf16" else 4
    att_tokens = w.top_k + min(w.sink, w.context - w.window) + w.window
    bytes_a = BH * (n_groups * w.head_dim * 4 + kept * group * w.head_dim * es) + \
        BH * att_tokens * w.head_dim * es * 2
    bytes_e = BH * nc * w.head_dim * es + BH * att_tokens * w.head_dim * es * 2
    return {"workload": "token-retrieval-decode-1m (drift keys)", "group": group,
            "groups_kept": kept, "recall_vs_exact_top_k": round(recall, 4),
            "keys_read_per_step": keys_read,
            "keys_read_frac": round(keys_read / (BH * nc), 4),
            "us_per_step": round(us_a, 2), "steps_per_s": round(1e6 / us_a, 1),
            "algorithmic_bytes": bytes_a,
            "achieved_gbs": round(bytes_a / (us_a * 1e-6) / 1e9, 1),
            "frac_of_hbm": round(bytes_a / (us_a * 1e-6) / 1e9 / pk["hbm_gbs"], 4),
            "exact_us_per_step": round(us_e, 2), "exact_algorithmic_bytes": bytes_e,
            "speedup_vs_exact": round(us_e / us_a, 2), "steps_timed": n_a,
            "l2": "L2-sized write between steps, its time subtracted",
            "index": "group means (fp32) built once by rba_group_means, not timed"}


def count_groups(w, group):
    """Candidate groups of `group` tokens (full groups meeting [sink, T - window))."""
    w0 = max(w.context - w.window, 0)
    lo = w.sink // group
    hi = min(-(-w0 // group), w.context // group)
    return max(hi - lo, 0)


def measure_memory_update(name, dev, trials, pk):
    """Dynamic memory update (MemLong section 2.3.2) of the full store of
    workload `name`: synthetic retrieval counters, the page's 10% / 10% / 50%
    proportions over the blocks after the sink, in-place compaction.  Each
    trial restores the store from a copy and reads a 256 MB buffer (untimed:
    the copy, larger than L2, evicts it, and the read writes back the lines
    the copy left dirty), then times one update with CUDA events on the
    stream.

    Algorithmic bytes: every kept entry moves (the oldest entries are dropped,
    so each kept one shifts), read + write of its K/V rows over the unit's kv
    heads, its representation, positions and counter, plus one read of the
    counters by the selection and the keep map written."""
    import torch
    import retrieval_block_sparse_b200 as rba
    from retrieval_block_sparse_b200 import synth
    w = synth.WORKLOADS[name]
    cosine = getattr(w, "score_mode", "dot") == "cosine"
    if cosine:
        mode, r, d_ret, batch = "embed_cosine", 1, w.d_ret, 1
    else:
        mode, r, d_ret, batch = w.rep_mode, w.n_rep, 0, w.batch
    st = rba.Store(batch=batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   head_dim=w.head_dim, block_size=w.block_size, capacity_tokens=w.context,
                   dtype=w.dtype, mode=mode, n_rep=r, d_ret=d_ret, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)
    for t in (st.k, st.v, st.rep):
        if t is not None:
            t.copy_(torch.randn(t.shape, generator=gen, device=dev, dtype=torch.float32))
    if st.rep_pos is not None:
        st.rep_pos.random_(0, w.block_size, generator=gen)
    U = st.memory_units()
    counts = synth.retrieval_counts(w.seed, U, st.cap_blocks)
    counters = torch.from_numpy(counts.view(np.int32)).to(dev)
    T, bs = w.context, w.block_size
    nb = T // bs
    pinned = -(-w.sink // bs) if w.sink else 0
    newest, oldest, total = rba.memory_rule(nb - pinned)
    keep_map = torch.empty((U, max(total, 1)), dtype=torch.int32, device=dev)
    saved = [t.clone() for t in (st.k, st.v, st.rep, st.rep_pos, counters) if t is not None]
    live = [t for t in (st.k, st.v, st.rep, st.rep_pos, counters) if t is not None]
    stream = torch.cuda.current_stream()
    # the restore writes the store through L2; reading a buffer twice the L2's
    # size afterwards writes those dirty lines back before the timed region
    # (an update that follows decode steps finds an L2 of clean lines)
    scrub = torch.empty(256 << 20, dtype=torch.uint8, device=dev).view(torch.int32)
    scrub.zero_()
    times = []
    for i in range(trials + 2):
        for a, b in zip(live, saved):
            a.copy_(b)
        scrub.sum()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        t_new, _ = st.memory_update(T, counters, pinned_blocks=pinned, keep_map=keep_map)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= 2:
            times.append(e0.elapsed_time(e1) * 1e3)
    st.check()
    es = 2 if w.dtype == "bf16" else 4
    heads = w.n_kv_heads if cosine else 1
    kv_b = heads * 2 * bs * w.head_dim * es
    rep_b = 0 if st.rep is None else \
        st.rep.numel() // (U * st.cap_blocks) * st.rep.element_size()
    pos_b = 4 * r if st.rep_pos is not None else 0
    moved = U * total * 2 * (kv_b + rep_b + pos_b + 4)
    algo = moved + U * (nb - pinned - newest - oldest) * 4 + U * total * 4
    us = float(np.median(times))
    gbs = algo / (us * 1e-6) / 1e9
    rounds = -(-total // max(oldest, 1))
    return {"workload": name, "units": U, "entries": nb - pinned, "pinned_blocks": pinned,
            "keep_newest": newest, "drop_oldest": oldest, "keep_total": total,
            "T_new": t_new, "launches": 1 + rounds + 1, "trials": trials,
            "update_us": round(us, 2), "algorithmic_bytes": algo,
            "achieved_gbs": round(gbs, 1), "frac_of_hbm": round(gbs / pk["hbm_gbs"], 4),
            "timing": "median of trials; store restored from a copy between trials, then "
                      "a 256 MB read writes the copy's dirty L2 lines back (untimed)"}


def measure_configs(dev, seconds):
    pk = peaks()
    out = {}
    for name in ("tiny-decode-f32", "landmark-decode-b16", "token-retrieval-decode-1m"):
        out[name] = measure_decode_config(name, dev, seconds, pk)
    out["infllm-decode-128k:max-over-rep-keys"] = measure_decode_config(
        "infllm-decode-128k", dev, seconds, pk, score_reduce="max")
    out["infllm-decode-128k:one-launch"] = measure_decode_config(
        "infllm-decode-128k", dev, seconds, pk, one_launch=True)
    for name in ("memlong-cosine-prefill", "token-retrieval-prefill-1m"):
        out[name] = measure_prefill_config(name, dev, seconds, pk)
    # head dim 100 (MemLong's OpenLLaMA-3B: 32 heads of 100), pool rows padded to 128
    from retrieval_block_sparse_b200 import synth
    out["infllm-decode-128k:head-dim-100"] = measure_decode_config(
        "infllm-decode-128k", dev, seconds, pk,
        workload=synth.WORKLOADS["infllm-decode-128k"].scaled(head_dim=100))
    out["memlong-cosine-prefill:head-dim-100"] = measure_prefill_config(
        "memlong-cosine-prefill", dev, seconds, pk,
        workload=synth.WORKLOADS["memlong-cosine-prefill"].scaled(head_dim=100))
    for name in ("memlong-cosine-prefill", "infllm-decode-128k"):
        out["memory-update:" + name] = measure_memory_update(name, dev, 10, pk)
    out["token-retrieval-decode-1m:two-stage"] = measure_approx_config(dev, seconds, pk)
    return out


# ---------------------------------------------------------------------------
# CPU baseline / reference arm: the fp64 oracle, as it stands


def _blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = [i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def _oracle_units(w, x):
    """One (batch, kv head) unit of the decode step, as the oracle computes it."""
    import oracle as O
    probe = O.widen(x["probe"], w.dtype) if "probe" in x else None
    reps = None
    if w.rep_mode != "identity":
        reps = np.zeros((w.batch, w.n_kv_heads, w.n_blocks, w.n_rep, w.head_dim))
        for b in range(w.batch):
            for h in range(w.n_kv_heads):
                if w.rep_mode == "external":
                    reps[b, h, :, 0] = O.widen(x["landmarks"][b, h], w.dtype)
                    continue
                K = O.widen(x["K"][b, h, :w.n_blocks * w.block_size], w.dtype)
                reps[b, h] = O.memorize(K, w.rep_mode, w.block_size, w.n_rep,
                                        probe=None if probe is None else probe[h])[0]
    g = w.n_q_heads // w.n_kv_heads
    units = [(b, h) for b in range(w.batch) for h in range(w.n_kv_heads)]

    def unit(i):
        b, h = units[i % len(units)]
        O.decode(x["q"][b:b + 1, h * g:(h + 1) * g], x["K"][b:b + 1, h:h + 1],
                 x["V"][b:b + 1, h:h + 1], None if reps is None else reps[b:b + 1, h:h + 1],
                 dtype=w.dtype,
                 block_size=w.block_size, sink=w.sink, window=w.window, top_k_blocks=w.top_k)
    return unit, len(units)


def _host_cpu():
    """Host core count and CPU model (reported beside the threads the oracle used)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model}


def cpu_baseline(w, x, seconds, workload=WORKLOAD):
    unit, per_step = _oracle_units(w, x)
    unit(0)
    n, t0 = 0, time.perf_counter()
    while True:
        unit(n)
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds and n >= per_step:
            break
    return {"value": round(n / el / per_step, 4), "unit": UNIT, "cores": _blas_threads(),
            "kind": "oracle", **_host_cpu(),
            "sample": f"{n} (batch, kv head) units = {n / per_step:.2f} decode steps of {workload} "
                      f"(score + top-k + attend, fp64 numpy; memorise excluded), {el:.1f} s; "
                      f"cores = BLAS threads used"}


def workload_config(name, w, nc):
    """The workload part of a bench line's config (the same in both arms)."""
    return {"workload": name, "batch": w.batch, "q_heads": w.n_q_heads,
            "kv_heads": w.n_kv_heads, "head_dim": w.head_dim, "context": w.context,
            "block_size": w.block_size, "rep_keys": w.n_rep, "top_k": w.top_k,
            "sink": w.sink, "window": w.window, "candidates": nc}


def run_reference(args):
    """The oracle as the reference arm: each reference step is a bounded sample
    of whole decode steps (every (batch, kv head) unit of the workload), sized
    from the warm-up to take about one second, so that K steps take about K
    seconds whatever the host."""
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    from retrieval_block_sparse_b200 import synth
    import oracle as O
    w = synth.WORKLOADS[args.workload]
    x = synth.decode_inputs(w)
    nc = int(O.candidate_blocks(w.context, w.block_size, w.sink, w.window).size)
    unit, per_step = _oracle_units(w, x)
    t0 = time.perf_counter()
    n_warm = max(args.warmup, 1) * per_step
    for i in range(n_warm):
        unit(i)
    t_step = (time.perf_counter() - t0) / max(args.warmup, 1)
    # decode steps per reference step: about one second each, fewer when K such
    # samples would exceed the 240 s bound of the whole timed run
    budget = 240.0
    sample = max(1, int(round(1.0 / max(t_step, 1e-6))))
    sample = max(1, min(sample, int(budget / max(args.steps * t_step, 1e-6))))
    t0 = time.perf_counter()
    done = 0
    while done < args.steps:
        for i in range(sample * per_step):
            unit(i)
        done += 1
        if time.perf_counter() - t0 > budget:
            break
    el = time.perf_counter() - t0
    n_dec = done * sample
    value = n_dec / el
    desc = (f"{done} samples of {sample} whole decode steps of {args.workload} "
            f"({sample * per_step} (batch, kv head) units each: score + top-k + attend, fp64 "
            f"numpy; memorise excluded), {el:.1f} s; cores = BLAS threads used" +
            (f"; stopped at the {budget:.0f} s bound before {args.steps}" if done < args.steps
             else ""))
    cores = _blas_threads()
    return {"metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
            "steps": done, "warmup": args.warmup,
            "ms_per_step": round(el * 1e3 / n_dec, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded generator)", "impl": "reference",
            "config": workload_config(args.workload, w, nc),
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores,
                             "kind": "oracle", "sample": desc, **_host_cpu()},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main(argv=None):
    args = parse(argv)
    if args.only_config:
        import torch
        torch.cuda.set_device(0)
        dev = torch.device("cuda", 0)
        from retrieval_block_sparse_b200 import synth
        if args.only_config == "token-retrieval-decode-1m:two-stage":
            print(json.dumps({"config": measure_approx_config(dev, args.config_seconds,
                                                              peaks())}), flush=True)
            return
        if args.only_config.startswith("memory-update:"):
            res = measure_memory_update(args.only_config.split(":", 1)[1], dev, 10, peaks())
            print(json.dumps({"config": res}), flush=True)
            return
        w = synth.WORKLOADS[args.only_config]
        fn = measure_decode_config if isinstance(w, synth.DecodeWorkload) else \
            measure_prefill_config
        print(json.dumps({"config": fn(args.only_config, dev, args.config_seconds, peaks())}),
              flush=True)
        return
    line = run_reference(args) if args.impl == "reference" else run_ours(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
