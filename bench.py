"""Benchmark of the B200 suffix attention (one JSON line on rank 0).

A step is one dm05_suffix_attn call over one batch of synthetic input of the
named workload (default: the base-model chunk, B=1, P=1024 bucket with 900
valid rows, S=50, 8/4 heads, D=256).  Timing: W untimed warm-up calls, then
exactly K calls replayed from CUDA graphs and bracketed by a barrier and a
device synchronise, timed with CUDA events on the launching stream, max over
ranks.  Every call reads a different one of R rotating input sets whose total
size is more than twice the L2, so each call streams its K/V from HBM.

Multi-GPU: the path has no exchange step; each rank runs independent
replicas on its own GPU (no collective on the data path) and `value` is the
whole job's time per call, max-over-ranks time / (K * N).

--impl reference times the fp64 CPU oracle on the host cores (each step one
bounded sample of query rows of the same workload, scaled to a full call).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "suffix-attn µs/call & achieved HBM GB/s (frac of roofline), P=1024 S=50 B=1"
UNIT = "us/call"
KV_ROW_BYTES_PER_HEAD = 2 * 256 * 2   # K and V rows of one KV head, bf16, D=256
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="base_chunk",
                    choices=("base_chunk", "libero_tiny", "history_loop", "batched_mask", "bucket_sweep"))
    ap.add_argument("--splits", type=int, default=0, help="force CTAs per (sample, KV head); 0 = auto")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-baseline sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true", help="skip the per-workload table")
    ap.add_argument("--prefix-static", action="store_true",
                    help="declare the prefix cache static (DM05_FLAG_PREFIX_STATIC) in the timed calls")
    return ap.parse_args()


def workload_inputs(name):
    from gqa_prefix_suffix_b200 import inputs as gen
    w = gen.WORKLOADS[name]()
    if isinstance(w, list):
        # the history loop reuses one prefix; the sweep: take its largest bucket
        w = w[0] if name == "history_loop" else w[-1]
    return w


def algorithmic_bytes(inp):
    """K/V bytes the method must move: visible prefix rows plus the S suffix
    rows, K and V, every KV head, bf16 (rows past valid_len and hidden rows
    are not counted)."""
    import torch
    total_rows = 0
    for b in range(inp.B):
        vl = inp.P if inp.prefix_valid_len is None else max(0, min(inp.P, int(inp.prefix_valid_len[b])))
        vis = vl if inp.prefix_mask is None else int((inp.prefix_mask[b, :vl] != 0).sum())
        total_rows += vis + inp.S
    kv = total_rows * inp.Hkv * KV_ROW_BYTES_PER_HEAD
    G = inp.Hq // inp.Hkv
    flops = 4 * total_rows * inp.Hkv * G * inp.S * inp.D
    del torch
    return kv, flops


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash():
    """Hash of the kernel's device code (the launch plan is checked apart)."""
    h = hashlib.sha256()
    for rel in ("gqa_prefix_suffix_b200/csrc/suffix_attn_kernel.cuh", "gqa_prefix_suffix_b200/csrc/sm100_ptx.cuh"):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload, plan):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel device code with the same launch plan (splits per
    head, query blocks, tile rows); else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            j = json.load(f)
        e = j.get(workload)
        if (e and e.get("kernel_device_source_hash") == kernel_source_hash()
                and tuple(e.get("plan", ())) == tuple(plan)):
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while running."""

    def __init__(self, torch_device):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self._nv = pynvml
            try:  # the same physical GPU as the torch device, whatever CUDA_VISIBLE_DEVICES says
                uuid = str(torch.cuda.get_device_properties(torch_device).uuid)
                self._h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(torch_device.index or 0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self._ok = False

    def _run(self):
        nv = self._nv
        names = {
            "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
            "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
            "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for k, bit in names.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self._ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


def max_over_ranks(dist, value, device):
    """The largest of the ranks' values (each rank passes its own); the value
    itself when there is no process group."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_us_per_call(max_ms, calls_per_rank, world):
    """Whole-job time per call: the slowest rank's time over every call that
    all replicas made."""
    return max_ms * 1e3 / (calls_per_rank * world)


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ----------------------------------------------------------------------------- CPU side

def host_bits(inp):
    """The workload's tensors as numpy arrays (bf16 as uint16 bit patterns),
    converted once so that timed oracle calls do no marshalling copies."""
    import types

    import numpy as np
    import torch

    def bits(t):
        return None if t is None else np.ascontiguousarray(t.contiguous().view(torch.int16).numpy().view(np.uint16))

    def plain(t):
        return None if t is None else np.ascontiguousarray(t.numpy())

    return types.SimpleNamespace(
        name=inp.name, B=inp.B, Hq=inp.Hq, Hkv=inp.Hkv, P=inp.P, S=inp.S, D=inp.D,
        q=bits(inp.q), k_prefix=bits(inp.k_prefix), v_prefix=bits(inp.v_prefix), k_suffix=bits(inp.k_suffix),
        v_suffix=bits(inp.v_suffix), prefix_valid_len=plain(inp.prefix_valid_len), prefix_mask=plain(inp.prefix_mask))


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cover_launch():
    """A short device-side wait (~50 us, torch's spin kernel) on the current
    stream just ahead of the start event: the first graph replay is then
    already queued when the event fires, so the timed region holds device work
    only, not the host's launch of the first replay."""
    import torch
    sleep = getattr(torch.cuda, "_sleep", None)
    if sleep is not None:
        sleep(100_000)


def warm_graphs(graphs, stream, min_passes=3, min_ms=200.0):
    """Untimed replays of the captured graphs before the timed pass: at least
    `min_passes` passes over all of them and at least `min_ms` of GPU time
    (the first replays after capture run measurably slower)."""
    import torch
    spent, passes = 0.0, 0
    while passes < min_passes or spent < min_ms:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for g in graphs:
                g.replay()
            e1.record(stream)
        stream.synchronize()
        spent += e0.elapsed_time(e1)
        passes += 1
        if passes > 1000:
            break
    return passes


def time_calls(calls, K, W, dev, stream, bd, l2, rotate=True):
    """Device time per call of K dm05_suffix_attn calls that cycle through
    `calls` (a list of input sets, one call each), captured as CUDA graphs of
    up to 1000 calls and timed with CUDA events on the launching stream.
    With `rotate`, the list is copied until the copies hold more than twice
    the L2, so every call streams its K/V from HBM; a call list that shares
    one prefix (the history loop, warm) is timed as is."""
    import torch
    one = sum(t.numel() * t.element_size() for c in calls for t in c.tensors().values() if t is not None)
    copies = max(2, int(2 * l2 // max(1, one)) + 2) if rotate else 1
    # one device copy of each call (calls that share a prefix cache keep
    # sharing it), then on-device clones, as the headline measurement does
    base, prefix_dev = [], {}
    for c in calls:
        key = (c.k_prefix.data_ptr(), c.v_prefix.data_ptr())
        if key not in prefix_dev:
            prefix_dev[key] = (c.k_prefix.to(dev), c.v_prefix.to(dev))
        mv = lambda t: None if t is None else t.to(dev)
        base.append((key, dict(q=mv(c.q), prefix_valid_len=mv(c.prefix_valid_len), prefix_mask=mv(c.prefix_mask),
                               k_suffix=mv(c.k_suffix), v_suffix=mv(c.v_suffix)),
                     (c.B, c.Hq, c.Hkv, c.P, c.S, c.D)))
    sets = []
    for _ in range(copies):
        prefix_copy = {k: (kp.clone(), vp.clone()) for k, (kp, vp) in prefix_dev.items()} if rotate else prefix_dev
        for key, t, dims in base:
            B, Hq, Hkv, P, S, D = dims
            kp, vp = prefix_copy[key]
            sets.append(dict(q=t["q"].clone(), k_prefix=kp, v_prefix=vp,
                             prefix_valid_len=None if t["prefix_valid_len"] is None else t["prefix_valid_len"].clone(),
                             prefix_mask=None if t["prefix_mask"] is None else t["prefix_mask"].clone(),
                             k_suffix=t["k_suffix"].clone(), v_suffix=t["v_suffix"].clone(),
                             out=torch.empty((B, Hq, S, D), dtype=torch.bfloat16, device=dev),
                             lse=torch.empty((B, Hq, S), dtype=torch.float32, device=dev), dims=dims))
    del base, prefix_dev
    torch.cuda.synchronize()
    ptr = lambda x: None if x is None else x.data_ptr()

    def call(t):
        B, Hq, Hkv, P, S, D = t["dims"]
        rc = bd.dm05_suffix_attn(ptr(t["q"]), ptr(t["k_prefix"]), ptr(t["v_prefix"]), ptr(t["prefix_valid_len"]),
                                 ptr(t["prefix_mask"]), ptr(t["k_suffix"]), ptr(t["v_suffix"]), ptr(t["out"]),
                                 ptr(t["lse"]), B, Hq, Hkv, P, S, D, stream.cuda_stream)
        if rc != 0:
            raise bd.Dm05Error(rc, "dm05_suffix_attn")

    n = len(sets)
    for d in {t["dims"] for t in sets}:
        rc = bd.dm05_suffix_attn_reserve(*d, stream.cuda_stream)
        if rc != 0:
            raise bd.Dm05Error(rc, "reserve")
    with torch.cuda.stream(stream):
        for i in range(max(3, W)):
            call(sets[i % n])
    stream.synchronize()
    chunk = min(K, 1000)
    graphs = []
    done = 0
    while done < K:
        m = min(chunk, K - done)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(m):
                call(sets[(done + i) % n])
        graphs.append((g, m))
        done += m
    warm_graphs([g for g, _ in graphs], stream)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(graphs) + 1)]
    with torch.cuda.stream(stream):
        cover_launch()
        evs[0].record(stream)
        for i, (g, _) in enumerate(graphs):
            g.replay()
            evs[i + 1].record(stream)
    stream.synchronize()
    us = evs[0].elapsed_time(evs[-1]) * 1e3 / K
    del graphs, sets
    return us, copies


def prefill_flops(inp):
    """Algorithmic FLOPs of a prefix-prefill call: every computed query row
    i (below its sample's valid length) against its i + 1 visible keys, QK^T
    and PV at 2 flops per multiply-add."""
    total = 0
    for b in range(inp.B):
        vl = inp.P if inp.valid_len is None else max(0, min(inp.P, int(inp.valid_len[b])))
        total += 4 * inp.D * inp.Hq * vl * (vl + 1) // 2
    return total


def time_prefill(inp, K, W, dev, stream, bd, l2):
    """Device time per dm05_prefix_prefill_attn call, the same protocol as
    time_calls (rotating on-device copies over 2 x L2, graphs of up to 1000
    calls, CUDA events on the launching stream)."""
    import torch
    one = sum(t.numel() * t.element_size() for t in inp.tensors().values() if t is not None)
    copies = max(2, int(2 * l2 // max(1, one)) + 2)
    d0 = inp.to(dev)
    sets = []
    for _ in range(copies):
        sets.append(dict(q=d0.q.clone(), k=d0.k.clone(), v=d0.v.clone(),
                         vl=None if d0.valid_len is None else d0.valid_len.clone(),
                         out=torch.empty_like(d0.q),
                         lse=torch.empty((inp.B, inp.Hq, inp.P), dtype=torch.float32, device=dev)))
    ptr = lambda x: None if x is None else x.data_ptr()
    rc = bd.dm05_prefix_prefill_reserve(inp.B, inp.Hq, inp.Hkv, inp.P, inp.D, stream.cuda_stream)
    if rc != 0:
        raise bd.Dm05Error(rc, "dm05_prefix_prefill_reserve")

    def call(t):
        rc = bd.dm05_prefix_prefill_attn(ptr(t["q"]), ptr(t["k"]), ptr(t["v"]), ptr(t["vl"]), ptr(t["out"]),
                                         ptr(t["lse"]), inp.B, inp.Hq, inp.Hkv, inp.P, inp.D, stream.cuda_stream)
        if rc != 0:
            raise bd.Dm05Error(rc, "dm05_prefix_prefill_attn")

    with torch.cuda.stream(stream):
        for i in range(max(3, W)):
            call(sets[i % copies])
    stream.synchronize()
    graphs, done = [], 0
    while done < K:
        m = min(1000, K - done)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(m):
                call(sets[(done + i) % copies])
        graphs.append(g)
        done += m
    warm_graphs(graphs, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        cover_launch()
        e0.record(stream)
        for g in graphs:
            g.replay()
        e1.record(stream)
    stream.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / K
    del graphs, sets
    return us, copies


def time_prologue(inp, K, W, dev, stream, bd, l2):
    """Device time per dm05_suffix_qkv_prologue call: rotating on-device copies
    of the inputs over 2 x L2, graphs of up to 1000 calls, CUDA events."""
    import torch
    one = sum(t.numel() * t.element_size() for t in inp.tensors().values())
    copies = max(2, int(2 * l2 // max(1, one)) + 2)
    d0 = inp.to(dev)
    sets = []
    for _ in range(copies):
        sets.append(dict(x=d0.x.clone(), w=d0.w.clone(), qw=d0.qw.clone(), kw=d0.kw.clone(), pos=d0.pos.clone(),
                         q=torch.empty((inp.B, inp.Hq, inp.S, inp.D), dtype=torch.bfloat16, device=dev),
                         k=torch.empty((inp.B, inp.Hkv, inp.S, inp.D), dtype=torch.bfloat16, device=dev),
                         v=torch.empty((inp.B, inp.Hkv, inp.S, inp.D), dtype=torch.bfloat16, device=dev)))

    def call(t):
        rc = bd.dm05_suffix_qkv_prologue(t["x"].data_ptr(), t["w"].data_ptr(), t["qw"].data_ptr(),
                                         t["kw"].data_ptr(), t["pos"].data_ptr(), t["q"].data_ptr(),
                                         t["k"].data_ptr(), t["v"].data_ptr(), inp.B, inp.S, inp.H, inp.Hq,
                                         inp.Hkv, inp.D, 1e-6, 10000.0, stream.cuda_stream)
        if rc != 0:
            raise bd.Dm05Error(rc, "dm05_suffix_qkv_prologue")

    with torch.cuda.stream(stream):
        for i in range(max(3, W)):
            call(sets[i % copies])
    stream.synchronize()
    graphs, done = [], 0
    while done < K:
        m = min(1000, K - done)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(m):
                call(sets[(done + i) % copies])
        graphs.append(g)
        done += m
    warm_graphs(graphs, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        cover_launch()
        e0.record(stream)
        for g in graphs:
            g.replay()
        e1.record(stream)
    stream.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / K
    del graphs, sets
    return us, copies


def history_steps(calls, K, dev, stream, bd):
    """The 10 denoising-step calls of the history loop over one prefix cache:
    (a) one dm05_suffix_attn_steps launch of the 10 calls (a graph the library
    captured once, static-prefix flag set), (b) the same 10 calls issued one by
    one with dm05_suffix_attn (no graph).  Both time whole 10-step loops with
    CUDA events on the launching stream (the prefix stays warm across steps,
    as specified)."""
    import torch
    ds = [c.to(dev) for c in calls]
    d0 = ds[0]
    outs = [torch.empty_like(d.q) for d in ds]
    lses = [torch.empty(d.q.shape[:3], dtype=torch.float32, device=dev) for d in ds]
    ptr = lambda x: None if x is None else x.data_ptr()
    steps = [(ptr(d.q), ptr(d.k_suffix), ptr(d.v_suffix), ptr(o), ptr(l)) for d, o, l in zip(ds, outs, lses)]
    B, Hq, Hkv, P, S, D = d0.B, d0.Hq, d0.Hkv, d0.P, d0.S, d0.D
    handles = {}
    for name, flags in (("steps_one_launch", 0), ("steps_one_launch_static_prefix", bd.DM05_FLAG_PREFIX_STATIC)):
        rc, h = bd.dm05_suffix_attn_steps_create(steps, ptr(d0.k_prefix), ptr(d0.v_prefix),
                                                 ptr(d0.prefix_valid_len), None, B, Hq, Hkv, P, S, D, flags)
        if rc != 0:
            raise bd.Dm05Error(rc, "dm05_suffix_attn_steps_create")
        handles[name] = h
    loops = max(20, K // 10)

    def timed(fn, n):
        for _ in range(max(3, n // 10)):
            fn()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            cover_launch()
            e0.record(stream)
            for _ in range(n):
                fn()
            e1.record(stream)
        stream.synchronize()
        return e0.elapsed_time(e1) * 1e3 / n

    def one_launch(h):
        def go():
            if bd.dm05_suffix_attn_steps_launch(h, stream.cuda_stream) != 0:
                raise RuntimeError("dm05_suffix_attn_steps_launch failed")
        return go

    def separate():
        for d, o, l in zip(ds, outs, lses):
            if bd.dm05_suffix_attn(ptr(d.q), ptr(d0.k_prefix), ptr(d0.v_prefix), ptr(d0.prefix_valid_len), None,
                                   ptr(d.k_suffix), ptr(d.v_suffix), ptr(o), ptr(l), B, Hq, Hkv, P, S, D,
                                   stream.cuda_stream) != 0:
                raise RuntimeError("dm05_suffix_attn failed")

    n = len(calls)
    res = {}
    try:
        for name, h in handles.items():
            t = timed(one_launch(h), loops)
            res[name] = {"per_10_steps": t * 10 / n, "us_per_call": t / n, "loops": loops,
                         "api": "dm05_suffix_attn_steps_launch (the 10 calls captured once)"
                                + (", DM05_FLAG_PREFIX_STATIC" if "static" in name else "")}
        t_sep = timed(separate, loops)
    finally:
        for h in handles.values():
            bd.dm05_suffix_attn_steps_destroy(h)
    res["separate_calls"] = {"per_10_steps": t_sep * 10 / n, "us_per_call": t_sep / n, "loops": loops,
                             "api": "10 x dm05_suffix_attn, no graph"}
    return res


def time_post(inp, K, W, dev, stream, bd, l2):
    """Device time per dm05_post_attention call (five launches), the same
    rotating-copy and graph protocol as the other workloads."""
    import torch
    one = sum(t.numel() * t.element_size() for t in inp.tensors().values())
    copies = max(2, int(2 * l2 // max(1, one)) + 2)
    d0 = inp.to(dev)
    sets = [dict({k: v.clone() for k, v in d0.tensors().items()},
                 out=torch.empty((inp.B * inp.S, inp.Hd), dtype=torch.bfloat16, device=dev)) for _ in range(copies)]
    rc = bd.dm05_post_attention_reserve(inp.B, inp.S, inp.Hq, inp.D, inp.Hd, inp.F, stream.cuda_stream)
    if rc != 0:
        raise bd.Dm05Error(rc, "dm05_post_attention_reserve")

    def call(t):
        rc = bd.dm05_post_attention(t["attn"].data_ptr(), t["h"].data_ptr(), t["scale"].data_ptr(),
                                    t["shift"].data_ptr(), t["gate"].data_ptr(), t["wo"].data_ptr(),
                                    t["wgu"].data_ptr(), t["wd"].data_ptr(), t["out"].data_ptr(), inp.B, inp.S,
                                    inp.Hq, inp.D, inp.Hd, inp.F, 1e-6, stream.cuda_stream)
        if rc != 0:
            raise bd.Dm05Error(rc, "dm05_post_attention")

    with torch.cuda.stream(stream):
        for i in range(max(3, W)):
            call(sets[i % copies])
    stream.synchronize()
    n = max(1, min(K, 400))
    graphs, done = [], 0
    while done < n:
        m = min(200, n - done)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(m):
                call(sets[(done + i) % copies])
        graphs.append(g)
        done += m
    warm_graphs(graphs, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        cover_launch()
        e0.record(stream)
        for g in graphs:
            g.replay()
        e1.record(stream)
    stream.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / n
    del graphs, sets
    return us, copies


def measured_tensor_peak():
    """Dense bf16 tensor peak in TFLOP/s: the measured burst figure when the
    driver's MEASURED_PEAKS.json is present, else the recipe's fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def workload_table(args, dev, stream, bd, l2, peak):
    """Every workload of the benchmark timed with the same protocol as the
    headline (rotating input sets over 2 x L2, K calls from CUDA graphs):
    µs per call, algorithmic K/V GB/s and its fraction of the HBM peak, and
    the work plan."""
    from gqa_prefix_suffix_b200 import inputs as gen
    K, W = args.steps, args.warmup

    def row(calls, rotate=True, note=None):
        us, copies = time_calls(calls, K, W, dev, stream, bd, l2, rotate=rotate)
        kv = sum(algorithmic_bytes(c)[0] for c in calls) / len(calls)
        c0 = calls[0]
        _, sp, tr, rb = bd.dm05_suffix_attn_plan(c0.B, c0.Hq, c0.Hkv, c0.P, c0.S, c0.D)
        gbs = kv / (us * 1e-6) / 1e9
        r = {"us_per_call": us, "algorithmic_bytes": kv, "achieved_gbs": gbs, "frac": gbs / peak,
             "plan": {"splits_per_head": sp, "row_blocks": rb, "tile_rows": tr}, "calls": K,
             "l2": (f"{copies} copies of {len(calls)} input sets" if rotate
                    else "one shared prefix, L2-warm by design")}
        if note:
            r["note"] = note
        return r

    out = {}
    out["libero_tiny"] = row([gen.libero_tiny()])
    sweep = gen.bucket_sweep()
    by_p = {}
    for c in sweep:
        by_p.setdefault(c.P, []).append(c)
    out["bucket_sweep"] = {str(P): row(g) for P, g in sorted(by_p.items())}
    hist = gen.history_loop()
    cold = row(hist, rotate=True, note="prefix cache rotated through more than 2 x L2 (cold)")
    warm = row(hist, rotate=False, note="one prefix cache, 10 fresh suffix sets per 10 steps (warm, as specified)")
    cold["per_10_steps"] = 10 * cold["us_per_call"]
    warm["per_10_steps"] = 10 * warm["us_per_call"]
    out["history_loop"] = {"cold": cold, "warm": warm, **history_steps(hist, K, dev, stream, bd)}
    out["batched_mask"] = row([gen.batched_mask()])
    # the prefix-prefill attention (prefix-causal mask) on the base chunk's and
    # the history demo's prefixes: a dense contraction, bound by the tensor cores
    tpeak, tkind = measured_tensor_peak()
    for inp in (gen.prefill_base(), gen.prefill_history()):
        us, copies = time_prefill(inp, K, W, dev, stream, bd, l2)
        fl = prefill_flops(inp)
        _, sp, qb, rb = bd.dm05_prefix_prefill_plan(inp.B, inp.Hq, inp.Hkv, inp.P, inp.D)
        tf = fl / (us * 1e-6) / 1e12
        out[inp.name] = {"us_per_call": us, "algorithmic_flops": fl, "achieved_tflops": tf,
                         "roofline": {"bound": "tensor", "peak": tpeak, "peak_source": tkind, "frac": tf / tpeak},
                         "plan": {"splits_per_head": sp, "query_block": qb, "row_blocks": rb}, "calls": K,
                         "l2": f"{copies} rotating copies"}
    # the post-attention block (output projection, Adarms, GEGLU, MLP down):
    # weight-bound at B = 1, tensor-bound at B = 32
    for inp in (gen.post_base(), gen.post_batched()):
        us, copies = time_post(inp, K, W, dev, stream, bd, l2)
        T = inp.B * inp.S
        wbytes = 2 * (inp.Hd * inp.Hq * inp.D + 2 * inp.F * inp.Hd + inp.Hd * inp.F)
        nbytes = wbytes + 2 * (T * inp.Hq * inp.D + 2 * T * inp.Hd) + 6 * inp.B * inp.Hd
        fl = 2 * T * (inp.Hd * inp.Hq * inp.D + 2 * inp.F * inp.Hd + inp.Hd * inp.F)
        t_hbm, t_tc = nbytes / (peak * 1e9), fl / (tpeak * 1e12)
        bound = "hbm" if t_hbm >= t_tc else "tensor"
        out[inp.name] = {"us_per_call": us, "algorithmic_bytes": nbytes, "algorithmic_flops": fl,
                         "achieved_gbs": nbytes / (us * 1e-6) / 1e9, "achieved_tflops": fl / (us * 1e-6) / 1e12,
                         "roofline": {"bound": bound, "frac": (t_hbm if bound == "hbm" else t_tc) / (us * 1e-6)},
                         "calls": K, "l2": f"{copies} rotating copies", "launches_per_call": 5}
    # the suffix prologue (QKV projection + QK-Norm + RoPE): the weight stream
    # bounds it at B = 1, the tensor cores at B = 32
    for inp in (gen.prologue_base(), gen.prologue_batched()):
        us, copies = time_prologue(inp, K, W, dev, stream, bd, l2)
        F = (inp.Hq + 2 * inp.Hkv) * inp.D
        T = inp.B * inp.S
        nbytes = 2 * (F * inp.H + T * inp.H + T * F) + 4 * T
        fl = 2 * T * F * inp.H
        gbs, tf = nbytes / (us * 1e-6) / 1e9, fl / (us * 1e-6) / 1e12
        t_hbm, t_tc = nbytes / (peak * 1e9), fl / (tpeak * 1e12)
        bound = "hbm" if t_hbm >= t_tc else "tensor"
        out[inp.name] = {"us_per_call": us, "algorithmic_bytes": nbytes, "algorithmic_flops": fl,
                         "achieved_gbs": gbs, "achieved_tflops": tf,
                         "roofline": {"bound": bound, "frac": (t_hbm if bound == "hbm" else t_tc) / (us * 1e-6),
                                      "peak": peak if bound == "hbm" else tpeak,
                                      "unit": "GB/s" if bound == "hbm" else "TFLOP/s"},
                         "calls": K, "l2": f"{copies} rotating copies"}
    return out


def cpu_oracle_rate(inp, seconds, threads):
    """Times the fp64 oracle on bounded samples of query rows of this workload
    and scales to a full call.  Returns (us per full call, rows timed, calls)."""
    import oracle
    orc = oracle.default()
    inp = host_bits(inp)
    n_rows = inp.B * inp.Hq * inp.S
    chunk = max(1, threads)
    t_total, rows_done, calls, start = 0.0, 0, 0, 0
    while t_total < seconds:
        lo = start % n_rows
        hi = min(n_rows, lo + chunk)
        t0 = time.perf_counter()
        orc.inputs_call(inp, nthreads=threads, row_range=(lo, hi))
        t_total += time.perf_counter() - t0
        rows_done += hi - lo
        calls += 1
        start = hi
    return t_total / rows_done * n_rows * 1e6, rows_done, calls


def run_reference(args, world, rank):
    """The reference arm: the fp64 CPU oracle, as it stands, on the host cores."""
    if rank != 0:
        return 0
    import oracle
    full = workload_inputs(args.workload)
    inp = host_bits(full)
    threads = oracle.max_threads()
    orc = oracle.default()
    n_rows = inp.B * inp.Hq * inp.S
    rows_per_step = max(1, threads)
    for i in range(args.warmup):
        lo = (i * rows_per_step) % n_rows
        orc.inputs_call(inp, nthreads=threads, row_range=(lo, min(n_rows, lo + rows_per_step)))
    t0 = time.perf_counter()
    rows = 0
    for i in range(args.steps):
        lo = (i * rows_per_step) % n_rows
        hi = min(n_rows, lo + rows_per_step)
        orc.inputs_call(inp, nthreads=threads, row_range=(lo, hi))
        rows += hi - lo
    dt = time.perf_counter() - t0
    us_per_call = dt / rows * n_rows * 1e6
    kv, _ = algorithmic_bytes(full)
    sample = (f"each step: {rows_per_step} query rows (of {n_rows} per call) of {inp.name}, "
              f"fp64 oracle; value scaled to a full call")
    line = {
        "impl": "reference", "metric": METRIC, "value": us_per_call, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(full, None),
        "cpu_baseline": {"value": us_per_call, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": us_per_call, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "achieved_kv_gbs": kv / (us_per_call * 1e-6) / 1e9,
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(inp, extra):
    vl = None if inp.prefix_valid_len is None else [int(x) for x in inp.prefix_valid_len.tolist()]
    cfg = {"workload": inp.name, "B": inp.B, "Hq": inp.Hq, "Hkv": inp.Hkv, "P": inp.P, "S": inp.S, "D": inp.D,
           "valid_len": vl if vl is None or len(vl) <= 4 else f"{len(vl)} values, mean {sum(vl) / len(vl):.1f}",
           "prefix_mask": inp.prefix_mask is not None}
    if extra:
        cfg.update(extra)
    return cfg


# ----------------------------------------------------------------------------- GPU side

def main():
    args = parse()
    world, rank, local = dist_setup()
    if args.impl == "reference":
        return run_reference(args, world, rank)

    import torch
    from gqa_prefix_suffix_b200 import binding as bd

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    bd.lib()  # fails loudly if the CUDA library is missing
    inp = workload_inputs(args.workload)
    B, Hq, Hkv, P, S, D = inp.B, inp.Hq, inp.Hkv, inp.P, inp.S, inp.D
    kv_bytes, flops = algorithmic_bytes(inp)

    # rotating input sets: total footprint > 2 x L2
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    set_bytes = sum(t.numel() * t.element_size() for t in inp.tensors().values() if t is not None)
    set_bytes += B * Hq * S * (D * 2 + 4)
    R = max(2, int(2 * l2 // set_bytes) + 2)
    base = inp.to(dev)
    sets = []
    for r in range(R):
        t = {k: (None if v is None else v.clone()) for k, v in base.tensors().items()}
        t["out"] = torch.empty((B, Hq, S, D), dtype=torch.bfloat16, device=dev)
        t["lse"] = torch.empty((B, Hq, S), dtype=torch.float32, device=dev)
        sets.append(t)
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)
    sh = stream.cuda_stream
    if bd.dm05_set_split_override(args.splits) != 0:
        raise SystemExit("bad --splits")
    rc = bd.dm05_suffix_attn_reserve(B, Hq, Hkv, P, S, D, sh)
    if rc != 0:
        raise bd.Dm05Error(rc, "reserve")
    rc, splits, tile_rows, row_blocks = bd.dm05_suffix_attn_plan(B, Hq, Hkv, P, S, D)

    flags = bd.DM05_FLAG_PREFIX_STATIC if args.prefix_static else 0

    def call(t, s=sh):
        ptr = lambda x: None if x is None else x.data_ptr()
        rc = bd.dm05_suffix_attn_ex(ptr(t["q"]), ptr(t["k_prefix"]), ptr(t["v_prefix"]), ptr(t["prefix_valid_len"]),
                                    ptr(t["prefix_mask"]), ptr(t["k_suffix"]), ptr(t["v_suffix"]), ptr(t["out"]),
                                    ptr(t["lse"]), B, Hq, Hkv, P, S, D, flags, s)
        if rc != 0:
            raise bd.Dm05Error(rc, "dm05_suffix_attn")

    # warm-up (untimed)
    with torch.cuda.stream(stream):
        for i in range(max(3, args.warmup)):
            call(sets[i % R])
    stream.synchronize()

    # the K timed steps, captured as graphs of up to `chunk` calls each
    K = args.steps
    chunk = min(K, 1000)
    n_full, rem = divmod(K, chunk)

    def capture(n, offset):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                call(sets[(offset + i) % R])
        return g

    g_full = capture(chunk, 0) if n_full else None
    g_rem = capture(rem, n_full * chunk) if rem else None
    # untimed replays of each graph (part of the warm-up: the first replays
    # after capture run slower)
    warm_graphs([g for g in (g_full, g_rem) if g is not None], stream)

    # one event between consecutive replays: the total spans all K calls, and
    # each replay gives one sample of the per-call time for the spread
    replays = [(g_full, chunk)] * n_full + ([(g_rem, rem)] if g_rem is not None else [])
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(replays) + 1)]
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev)
    with sampler:
        with torch.cuda.stream(stream):
            cover_launch()
            evs[0].record(stream)
            for i, (g, _) in enumerate(replays):
                g.replay()
                evs[i + 1].record(stream)
        stream.synchronize()
    torch.cuda.synchronize()
    if pg is not None:
        pg.barrier()
    t_ms = evs[0].elapsed_time(evs[-1])
    per_replay = sorted(evs[i].elapsed_time(evs[i + 1]) * 1e3 / n for i, (_, n) in enumerate(replays))
    t_ms = max_over_ranks(pg, t_ms, dev)
    rc, word = bd.dm05_get_error_word(sh)
    if word != 0:
        raise SystemExit(f"kernel error word {word:#x}")

    def pct(xs, q):
        return xs[min(len(xs) - 1, max(0, int(round(q * (len(xs) - 1)))))]

    latency = {"median": statistics.median(per_replay), "p10": pct(per_replay, 0.1), "p90": pct(per_replay, 0.9),
               "replays": len(per_replay), "unit": UNIT}
    # a single call launched on its own (no graph, no neighbour to overlap with)
    singles = []
    for i in range(20):
        ea = torch.cuda.Event(enable_timing=True)
        eb = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            ea.record(stream)
            call(sets[i % R])
            eb.record(stream)
        stream.synchronize()
        singles.append(ea.elapsed_time(eb) * 1e3)
    latency["eager_single"] = statistics.median(singles)
    # the launch floor of this machine: a graph of 1000 one-element kernels
    z = torch.zeros(1, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(3):
            z.add_(1.0)
    stream.synchronize()
    g_floor = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_floor, stream=stream):
        for _ in range(1000):
            z.add_(1.0)
    with torch.cuda.stream(stream):
        g_floor.replay()
        ea = torch.cuda.Event(enable_timing=True)
        eb = torch.cuda.Event(enable_timing=True)
        ea.record(stream)
        for _ in range(3):
            g_floor.replay()
        eb.record(stream)
    stream.synchronize()
    latency["launch_floor"] = ea.elapsed_time(eb) * 1e3 / 3000
    del g_floor

    us_per_call_device = t_ms * 1e3 / K          # one GPU's time per call
    value = whole_job_us_per_call(t_ms, K, world)  # whole-job time per call
    achieved = kv_bytes / (us_per_call_device * 1e-6) / 1e9
    peak, peak_kind = measured_peaks()

    extra = {}
    if not args.no_workloads:
        extra["workloads"] = workload_table(args, dev, stream, bd, l2, peak)

    # ---- end to end through the public API: one dm05_suffix_attn_host call per
    # step copies the pinned host inputs in, runs the kernel and copies O and
    # the LSE back to pinned host memory
    host = {k: (None if v is None else v.pin_memory()) for k, v in inp.tensors().items()}
    out_h = torch.empty((B, Hq, S, D), dtype=torch.bfloat16).pin_memory()
    lse_h = torch.empty((B, Hq, S), dtype=torch.float32).pin_memory()
    vl_h = host["prefix_valid_len"]
    rc, h2d, d2h = bd.dm05_suffix_attn_host_copy_bytes(None if vl_h is None else vl_h.data_ptr(),
                                                       host["prefix_mask"] is not None, True, B, Hq, Hkv, P, S, D)
    if rc != 0:
        raise RuntimeError(f"dm05_suffix_attn_host_copy_bytes: {bd.dm05_status_string(rc)}")
    E = max(1, min(args.e2e_steps, K))

    def e2e_step():
        bd.suffix_attn_host(host["q"], host["k_prefix"], host["v_prefix"], host["k_suffix"], host["v_suffix"],
                            prefix_valid_len=vl_h, prefix_mask=host["prefix_mask"], out=out_h, lse=lse_h,
                            stream=stream)

    for _ in range(3):
        e2e_step()
    stream.synchronize()
    if pg is not None:
        pg.barrier()
    # The copies cross PCIe, which other jobs on the host share: time the E
    # steps in back-to-back chunks and report the median chunk (every step of
    # every chunk still includes its copies in and out).
    n_chunks = max(1, min(10, E // 10))
    per = max(1, E // n_chunks)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_chunks + 1)]
    evs[0].record(stream)
    for c in range(n_chunks):
        for _ in range(per):
            e2e_step()
        evs[c + 1].record(stream)
    stream.synchronize()
    chunk_us = sorted(evs[c].elapsed_time(evs[c + 1]) * 1e3 / per for c in range(n_chunks))
    e2e_us = max_over_ranks(pg, chunk_us[len(chunk_us) // 2], dev)
    e2e_value = whole_job_us_per_call(e2e_us / 1e3, 1, world)
    E = per * n_chunks

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        threads = oracle.max_threads()
        us, rows, n = cpu_oracle_rate(inp, args.cpu_seconds, threads)
        cpu = {"value": us, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{rows} query rows of {inp.name} in {n} oracle calls (~{args.cpu_seconds:.0f} s), "
                         f"fp64, scaled to a full call of {B * Hq * S} rows"}
        one_s = min(3.0, args.cpu_seconds)
        us1, rows1, _ = cpu_oracle_rate(inp, one_s, 1)
        cpu["value_1_thread"] = us1
        cpu["sample_1_thread"] = f"{rows1} query rows on 1 thread (~{one_s:.0f} s), scaled the same way"
        cpu["cpu_model"] = cpu_model()

    clocks = sampler.summary()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": value / 1e3, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": workload_config(inp, {
                "splits_per_head": splits, "row_blocks": row_blocks, "tile_rows": tile_rows,
                "parallelism": f"replicas x{world}",
                "l2": f"{R} rotating input sets, {R * set_bytes / 1e6:.0f} MB > 2 x L2 ({l2 / 1e6:.0f} MB)",
                "graph_calls": chunk, "prefix_static": bool(args.prefix_static)}),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": profiled_traffic(args.workload, (splits, row_blocks, tile_rows)),
                         "peak_source": peak_kind, "algorithmic_bytes": kv_bytes,
                         "tensor_tflops": flops / (us_per_call_device * 1e-6) / 1e12},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": E, "chunks": n_chunks, "chunk_min": chunk_us[0] / world,
                    "chunk_max": chunk_us[-1] / world, "statistic": "median over chunks",
                    "api": "dm05_suffix_attn_host (pinned host buffers in and out)"},
            "gpu_launches": K,
            "clocks": clocks,
            "latency": latency,
        }
        line.update(extra)
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    del g_full, g_rem
    if pg is not None:
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
