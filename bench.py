#!/usr/bin/env python
"""Routed-attention forward throughput (index + route + attend) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference]
                    [--workload scaling32k]

One step = one mdr_forward (rotary + summaries + codes, posting lists,
probe/rerank/top-R, selected-set attention) over one sequence of the
workload, inputs resident in HBM.  Each GPU (one process per GPU under
torchrun) runs its own sequence: weak scaling, no collective on the data path.
L2 is flushed before every step, outside the timed events: a 256 MiB write,
then a read of the same buffer, so that no dirty lines of the flush are left
to be written back inside the timed region.
Rank 0 prints one JSON line.  Beside the forward's throughput, roofline,
clocks, CPU baseline and end-to-end number it carries, each measured in the
same run (each can be left out with its --no-* flag):
  decode         one-token steps with the incremental index at 32K (latency);
  controls       target-block hit rates of the planted-block workload: route,
                 forced route, local-only;
  calibration    codebook calibration rounds on the long workload's key
                 summaries, and a held-out sequence's overflow and maximum
                 load before and after; the same rounds on 2^20 records;
  backward       dq, dk, dv of the attention with the route held fixed at 32K;
  scaling_sweep  the forward from 4K to 128K tokens with log-log slopes, and
                 the CPU oracle's index + route slope at 4K-32K (N = 1 only).

--impl reference times the CPU oracle (oracle/mdr_oracle.py) as it stands on
the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
# libmdr kernels one forward launches: summaries, codes, posting lists, route, attention.
KERNELS_PER_FORWARD = 5
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from workloads import SCALING_SWEEP, ALL, make_codebooks, make_grad, make_inputs, make_keys  # noqa: E402

METRIC = "routed-attention fwd tokens/s (index+route+attend) at 32K; % HBM roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def workload(name):
    for w in list(ALL.values()) + SCALING_SWEEP:
        if w.name == name:
            return w
    raise SystemExit(f"unknown workload {name}")


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def init_dist(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, dist, world: int, device) -> float:
    """The largest value over all ranks (every rank gets it)."""
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    return tokens_per_rank * world / (ms_max / 1e3)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense bf16 tensor-core peak in TFLOP/s: the measured burst figure (a
    kernel timed alone), else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured (burst)"
    return FALLBACK_BF16_TFLOPS, "fallback (burst)"


class ClockSampler:
    """SM clock, power and clock-event reasons of this process's GPU during
    the timed region, read through NVML by a thread every ~2 ms (the timed
    region is tens of milliseconds, too short for nvidia-smi's own loop).
    The GPU is matched by PCI domain/bus/device, so a remapped
    CUDA_VISIBLE_DEVICES does not matter; reason names come from NVML's own
    bit constants.  Reads only."""

    NAMES = {"GpuIdle": "gpu_idle", "ApplicationsClocksSetting": "applications_clocks",
             "SwPowerCap": "sw_power_cap", "HwSlowdown": "hw_slowdown", "SyncBoost": "sync_boost",
             "SwThermalSlowdown": "sw_thermal_slowdown", "HwThermalSlowdown": "hw_thermal_slowdown",
             "HwPowerBrakeSlowdown": "hw_power_brake_slowdown", "DisplayClockSetting": "display_clock"}

    def __init__(self, dev):
        self.dev, self.samples, self.err, self.thread = dev, [], None, None

    def __enter__(self):
        import threading
        import torch
        try:
            import pynvml as nv
            nv.nvmlInit()
            pr = torch.cuda.get_device_properties(self.dev)
            want = (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
            self.h = None
            for i in range(nv.nvmlDeviceGetCount()):
                h = nv.nvmlDeviceGetHandleByIndex(i)
                pci = nv.nvmlDeviceGetPciInfo(h)
                if (pci.domain, pci.bus, pci.device) == want:
                    self.h = h
            if self.h is None:
                raise RuntimeError(f"no NVML device at PCI {want}")
            self.nv = nv
            self.bits = {getattr(nv, "nvmlClocksEventReason" + k): v for k, v in self.NAMES.items()}
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.stop, first = threading.Event(), threading.Event()

            def run():
                while not self.stop.is_set():
                    self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                         nv.nvmlDeviceGetCurrentClocksEventReasons(self.h),
                                         nv.nvmlDeviceGetPowerUsage(self.h)))
                    first.set()
                    self.stop.wait(0.002)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            first.wait(timeout=5)          # sampling has begun before the timed steps are issued
        except Exception as e:             # no NVML: the line says why instead of carrying clocks
            self.err = repr(e)
        return self

    def __exit__(self, *a):
        if self.thread:
            self.stop.set()
            self.thread.join(timeout=5)
            self.nv.nvmlShutdown()

    def summary(self):
        if not self.samples:
            return {"error": self.err or "no samples"}
        reasons = set()
        for _, bits, _ in self.samples:
            reasons |= {n for b, n in self.bits.items() if bits & b}
        return {"sm_mhz": statistics.median(x[0] for x in self.samples), "sm_max_mhz": self.max_mhz,
                "power_w": statistics.median(x[2] for x in self.samples) / 1e3,
                "samples": len(self.samples), "source": "NVML, every 2 ms",
                "reasons": sorted(reasons - {"gpu_idle"})}


# Committed ncu summaries that carry a per-launch DRAM traffic figure: kernel
# sources they were taken from, and the workload they were taken on.
PROFILED_TRAFFIC = {
    "attend": ("profiles/attend_tc_scaling32k.txt", "scaling32k",
               ("learned_product_hash_b200/csrc/k_attend_tc.cu", "learned_product_hash_b200/csrc/attend_tc_common.cuh",
                "learned_product_hash_b200/csrc/tc_ptx.cuh")),
}


def profiled_traffic(kernel: str, workload_name: str):
    """dram__bytes_read.sum + dram__bytes_write.sum per launch of `kernel` from
    its committed ncu summary; None for another workload or once the kernel's
    sources no longer hash to the value recorded at capture time."""
    import hashlib
    entry = PROFILED_TRAFFIC.get(kernel)
    if entry is None or entry[1] != workload_name:
        return None
    path, _, srcs = entry
    try:
        text = open(os.path.join(ROOT, path)).read()
        h = hashlib.sha256()
        for src in srcs:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
    except OSError:
        return None
    rec = {k.strip(): v.strip() for k, v in
           (line.split(":", 1) for line in text.splitlines() if line.startswith(("source_sha256:", "traffic_bytes_per_launch:")))}
    if rec.get("source_sha256") != h.hexdigest():
        return None
    try:
        return int(rec["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def oracle_group_seconds(w, inp, h):
    """CPU oracle forward of one KV-head group: KV head h of sequence 0 and
    its query heads, all query blocks.  Returns seconds."""
    from oracle import mdr_oracle as O
    g = w.Hq // w.Hkv
    p = O.Params.of(w.with_(B=1, Hq=g, Hkv=1))
    q = inp.q[:1, :, h * g:(h + 1) * g]
    k, v = inp.k[:1, :, h:h + 1], inp.v[:1, :, h:h + 1]
    t0 = time.perf_counter()
    O.forward(q, k, v, inp.codebooks, p)
    return time.perf_counter() - t0


def oracle_sample(w, seed, max_seconds):
    """Time whole KV-head groups until max_seconds; tokens/s of the full
    workload (B sequences, all groups) at that speed."""
    inp = make_inputs(w, seed)
    secs = []
    for h in range(w.Hkv):
        secs.append(oracle_group_seconds(w, inp, h))
        if sum(secs) >= max_seconds:
            break
    t_full = statistics.mean(secs) * w.Hkv * w.B
    return w.B * w.S / t_full, sum(secs), len(secs)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return 1


def run_reference(args, w):
    """The CPU oracle as it stands, on the host's cores (BLAS pool = all
    cores), on this arm's workload: each step is one whole forward of one
    sequence (all KV-head groups), unless (warm-up + steps) whole forwards
    would take over REF_BUDGET_S, in which case each step times as many whole
    KV-head groups as fit and is scaled to the full forward (the line's
    sample says which)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    inp = make_inputs(w, 1000)
    ncpu = os.cpu_count() or 1
    t_group = oracle_group_seconds(w, inp, 0)                  # sizing run, not timed
    groups_total = w.Hkv * w.B
    per_step = groups_total
    n_steps = args.warmup + args.steps
    if n_steps * t_group * groups_total > REF_BUDGET_S:
        per_step = max(1, int(REF_BUDGET_S / (n_steps * t_group)))
        per_step = min(per_step, groups_total)
    secs = []
    for it in range(n_steps):
        t = sum(oracle_group_seconds(w, inp, (it * per_step + i) % w.Hkv) for i in range(per_step))
        if it >= args.warmup:
            secs.append(t)
    t_full = statistics.mean(secs) * groups_total / per_step
    tps = w.B * w.S / t_full
    g = w.Hq // w.Hkv
    sample = (f"each step: one whole forward of one sequence ({w.Hkv} KV-head groups of {g} query heads, "
              f"all {w.nb} query blocks)" if per_step == groups_total else
              f"each step: {per_step} of {groups_total} KV-head groups ({g} query heads, all {w.nb} query "
              f"blocks each), scaled to the full forward")
    line = {"impl": "reference", "metric": METRIC, "value": tps, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_full * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, args),
            "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": ncpu, "kind": "oracle",
                             "blas_threads": blas_threads(), "sample": sample},
            "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(w, args):
    return {"workload": w.name, "B": w.B, "S": w.S, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "block": w.block,
            "P": w.P, "K": w.K, "cap": w.cap, "probes": w.probes, "R": w.R, "L": w.L, "keys": w.keys,
            "l2": "flushed between steps (256 MiB write + read back, outside the timed events)",
            "parallelism": f"one sequence per GPU x {args.gpus}"}


REF_BUDGET_S = 240.0               # the reference arm's whole run stays within about four minutes
FP32_LANES_PER_SM = 128            # B200: 128 FP32 lanes per SM, one FMA (2 flops) each per clock


def loglog_exponent(sizes, times) -> float:
    """Least-squares slope of log(time) against log(size): 1 for linear
    scaling (the Report's Finite-range scaling fit)."""
    return float(np.polyfit(np.log(np.asarray(sizes, dtype=np.float64)),
                            np.log(np.asarray(times, dtype=np.float64)), 1)[0])


def oracle_route_seconds(w, seed: int, reps: int = 1) -> list:
    """Seconds of each of reps calls of the CPU oracle's index build + route
    (no attention) on the same inputs of workload w."""
    from oracle import mdr_oracle as O
    inp = make_inputs(w, seed)
    out = []
    for _ in range(reps):
        t0 = time.perf_counter()
        O.forward(inp.q, inp.k, inp.v, inp.codebooks, O.Params.of(w), attention=False)
        out.append(time.perf_counter() - t0)
    return out


def backward_flops(sel: np.ndarray, bs: int, D: int) -> int:
    """Flops of the four gradient products of the attention backward (dv =
    P^T dO, dP = dO V^T, dq = dS K, dk = dS^T Q), 2*D each per visible
    (query token, key token) pair: bs*bs pairs for a remote block, bs*(bs+1)/2
    for the query block's own block; -1 entries and ids past the query block
    add nothing."""
    nb = sel.shape[2]
    j = np.arange(nb)[None, None, :, None]
    full = ((sel >= 0) & (sel < j)).sum()
    own = (sel == j).sum()
    pairs = int(full) * bs * bs + int(own) * bs * (bs + 1) // 2
    return 8 * D * pairs


def backward_bytes(w, sel: np.ndarray, es: int) -> int:
    """Algorithmic bytes of one attention backward, the forward's byte model
    carried over: q, k, v and dout read once, dq, dk, dv written once in
    float32, and per valid (route, selected block) pair the four tiles the
    gradient needs -- the block's K and V (for dq) and the query block's Q and
    dO (for dk, dv), bs x D each."""
    nb = sel.shape[2]
    j = np.arange(nb)[None, None, :, None]
    pairs = int(((sel >= 0) & (sel <= j)).sum())
    tok = w.B * w.S
    once = tok * w.D * (2 * w.Hq + 2 * w.Hkv) * es + tok * w.D * (w.Hq + 2 * w.Hkv) * 4
    return once + pairs * 4 * w.block * w.D * es


def forward_bytes(w, nsel: int, es: int) -> dict:
    """Algorithmic bytes of one forward (the path's byte model): the
    summary pass reads q and k once; the attention reads q, gathers K and V of
    every valid selected block and writes the output.  The summary pass's
    rotated copies (written once, read by the attention) are not algorithmic
    bytes: they are reported beside, as what this design adds."""
    routes = w.B * w.Hq * w.nb
    summ = (w.Hq + w.Hkv) * w.S * w.D * es * w.B
    attn = routes * 2 * w.block * w.D * es + nsel * w.block * 2 * w.D * es
    return {"summaries": summ, "attention": attn, "path": summ + attn, "rotated_copies_written": summ}


def gqa_union(sel_t, w):
    """Valid selected ids of a KV-head group's query heads, summed per
    (sequence, KV head, query block) as the union of the group's rows and as
    the sum of the rows: how many K/V block gathers one gather per group
    (instead of one per query head) would save."""
    import torch
    g = w.Hq // w.Hkv
    n = w.R + w.L
    x = sel_t.view(w.B, w.Hkv, g, w.nb, n).permute(0, 1, 3, 2, 4).reshape(w.B, w.Hkv, w.nb, g * n)
    xs, _ = torch.sort(x.long(), dim=-1)
    first = xs[..., :1] >= 0
    new = (xs[..., 1:] != xs[..., :-1]) & (xs[..., 1:] >= 0)
    union = int(first.sum().item() + new.sum().item())
    total = int((x >= 0).sum().item())
    return {"group_size": g, "per_head_blocks": total, "union_blocks": union,
            "union_fraction": union / total if total else None}


def measure_forward(mdr, w, q, k, v, cb, dev, stream, flush_l2, reps=10, warm=3):
    """Median of reps L2-flushed mdr_forward calls (CUDA events on the
    launching stream), per-kernel times from as many calls with an event at
    every kernel boundary, the §8(d) byte model from the returned selection,
    overflow and (for grouped heads) the union of each group's selections."""
    import torch
    cfg = mdr.make_config(w)
    idx, rt, ws = mdr.Index.empty(cfg, dev), mdr.RouteOut.empty(cfg, dev), mdr.workspace(cfg, dev)
    out = torch.empty_like(q)
    times = []
    for it in range(warm + reps):
        flush_l2()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        mdr.mdr_forward(cfg, q, k, v, cb, idx, rt, out, ws)
        e1.record(stream)
        e1.synchronize()
        if it >= warm:
            times.append(e0.elapsed_time(e1))
    assert mdr.mdr_read_device_status(ws) == 0
    kevs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(reps)]
    for e in kevs:
        flush_l2()
        mdr.mdr_forward_profiled(cfg, q, k, v, cb, idx, rt, out, ws, e)
    torch.cuda.synchronize()
    ker = {n: statistics.median(e[i].elapsed_time(e[i + 1]) for e in kevs)
           for i, n in enumerate(("summarize", "lists", "route", "attend"))}
    es = 2 if w.dtype == "bf16" else 4
    nsel = int((rt.sel >= 0).sum().item())
    by = forward_bytes(w, nsel, es)
    ms = statistics.median(times)
    peak, peak_kind = peaks()
    res = {"ms_per_forward": ms, "tokens_per_s": w.B * w.S / (ms / 1e3), "selected_blocks": nsel,
           "selected_blocks_per_route": nsel / (w.B * w.Hq * w.nb),
           "bytes": by, "path_roofline_frac": by["path"] / (ms / 1e3) / 1e9 / peak,
           "kernels_ms": ker,
           "attention_roofline_frac": by["attention"] / (ker["attend"] / 1e3) / 1e9 / peak,
           "summaries_roofline_frac": by["summaries"] / (ker["summarize"] / 1e3) / 1e9 / peak,
           "peak_gbs": peak, "peak_kind": peak_kind,
           "overflow": int(idx.overflow.sum().item()), "max_load": int(idx.maxload.max().item())}
    if w.Hq != w.Hkv:
        res["gqa"] = gqa_union(rt.sel, w)
    del idx, rt, ws, out
    return res


def batched_decode(mdr, w, B, dev, stream, dist, world, peak):
    """Decode steps with B sequences per GPU of the workload's shape: a
    prefill of all but the last block (k, v ~ N(0, 1) drawn on the device),
    then one token of every sequence per step through the last block (no
    block completes), timed with CUDA events over consecutive steps after
    three warm-up steps.  Bytes per step: K and V of every selected token
    (tokens s <= t of the selected blocks, per sequence and query head), the
    new query, key and value, and the output."""
    import ctypes
    import torch
    if B <= 1:
        return None
    wb = w.with_(B=B)
    cfg = mdr.make_config(wb)
    S0 = w.S - w.block
    gen = torch.Generator(device=dev)
    gen.manual_seed(8000)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    es = 2 if w.dtype == "bf16" else 4
    cb = torch.from_numpy(make_codebooks(w, 8000)).to(dev)
    dst = mdr.DecodeState.empty(cfg, dev)
    dws = mdr.decode_workspace(cfg, dev)
    k0 = torch.randn(B, S0, w.Hkv, w.D, generator=gen, device=dev).to(dt)
    v0 = torch.randn(B, S0, w.Hkv, w.D, generator=gen, device=dev).to(dt)
    mdr.mdr_decode_prefill(cfg, S0, k0, v0, cb, dst, dws)
    torch.cuda.synchronize()
    del k0, v0
    n_dec = min(60, w.block - 1)
    qs = torch.randn(n_dec, B, w.Hq, w.D, generator=gen, device=dev).to(dt)
    ks = torch.randn(n_dec, B, w.Hkv, w.D, generator=gen, device=dev).to(dt)
    vs = torch.randn(n_dec, B, w.Hkv, w.D, generator=gen, device=dev).to(dt)
    out_t = torch.empty(B, w.Hq, w.D, dtype=dt, device=dev)
    sel_t = torch.empty(B, w.Hq, w.R + w.L, dtype=torch.int32, device=dev)
    warm = 3
    fn = mdr.lib().mdr_decode_step
    cfg_r, st_r = ctypes.byref(cfg), ctypes.byref(dst.c())
    sp = stream.cuda_stream
    calls = [(cfg_r, S0 + i, qs[i].data_ptr(), ks[i].data_ptr(), vs[i].data_ptr(), cb.data_ptr(), st_r,
              out_t.data_ptr(), sel_t.data_ptr(), None, dws.data_ptr(), dws.numel(), sp) for i in range(n_dec)]
    for c_args in calls[:warm]:
        if fn(*c_args) != mdr.MDR_OK:
            raise RuntimeError("mdr_decode_step failed")
    torch.cuda.synchronize()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for c_args in calls[warm:]:
        if fn(*c_args) != mdr.MDR_OK:
            raise RuntimeError("mdr_decode_step failed")
    d1.record(stream)
    d1.synchronize()
    assert mdr.mdr_read_device_status(dws) == 0
    n_t = n_dec - warm
    d_ms = d0.elapsed_time(d1) / n_t
    t_last = S0 + n_dec - 1
    sl = sel_t.cpu().numpy()
    ntok = int(sum(min(w.block, t_last + 1 - int(blk) * w.block) for blk in sl.ravel() if blk >= 0))
    d_bytes = ntok * 2 * w.D * es + 2 * B * w.Hq * w.D * es + 2 * B * w.Hkv * w.D * es
    d_ms_max = max_over_ranks(d_ms, dist, world, dev)
    del dst, dws
    return {"batch_per_gpu": B, "value": d_ms_max * 1e3, "unit": "us/step",
            "tokens_per_s": B * world / (d_ms_max / 1e3), "steps": n_t,
            "position": f"tokens {S0 + warm}..{t_last} ({S0 // w.block} blocks indexed)",
            "gpu_launches": 3 * n_t, "inputs": "k, v, q ~ N(0, 1) drawn on the device (torch, seeded)",
            "roofline": {"bound": "hbm", "achieved": d_bytes / (d_ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": d_bytes / (d_ms / 1e3) / 1e9 / peak, "algorithmic_bytes_per_step": d_bytes}}


def cpu_baseline(w, max_seconds):
    """The CPU oracle as it stands on this host at 1 thread, 4 threads (the
    Report's setup) and all cores: its BLAS pool limited by threadpoolctl
    (the route and attention loops themselves are Python, one thread).  Each
    setting times whole KV-head groups of one sequence for about
    max_seconds/3 and scales to the full forward.  value = all cores."""
    from threadpoolctl import threadpool_limits
    ncpu = os.cpu_count() or 1
    by = {}
    for n in sorted({1, 4, ncpu}):
        with threadpool_limits(limits=n):
            tps, secs, groups = oracle_sample(w, 1000, max_seconds=max_seconds / 3)
        by[str(n)] = {"tokens_per_s": tps, "seconds": secs, "groups_timed": groups}
    top = by[str(ncpu)]
    return {"value": top["tokens_per_s"], "unit": "tokens/s", "cores": ncpu, "kind": "oracle", "nproc": ncpu,
            "by_threads": by,
            "sample": f"per thread setting, whole KV-head groups (of {w.Hkv}) of one sequence, all {w.nb} query "
                      f"blocks, about {max_seconds / 3:.0f} s each, scaled to the full forward; threads = the "
                      f"BLAS pool (threadpoolctl); the oracle's loops run on one Python thread"}


def device_inputs(w, seed, dev):
    """q, v ~ N(0, 1) drawn on the device by torch's seeded generator (the
    workloads' recipe for q and v, without the host round trip); k by the
    workload's own key recipe (gaussian or clusters) on the host; codebooks
    seeded random unit vectors.  Stored as the workload's dtype."""
    import torch
    from workloads import make_keys
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q = torch.randn(w.B, w.S, w.Hq, w.D, generator=gen, device=dev).to(dt)
    v = torch.randn(w.B, w.S, w.Hkv, w.D, generator=gen, device=dev).to(dt)
    if w.keys == "gaussian":
        k = torch.randn(w.B, w.S, w.Hkv, w.D, generator=gen, device=dev).to(dt)
    else:
        kb = make_keys(w, seed)[1]
        k = (torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16) if w.dtype == "bf16"
             else torch.from_numpy(kb)).to(dev)
    cb = torch.from_numpy(make_codebooks(w, seed)).to(dev)
    return q, k, v, cb


def run_mine(args, w):
    import torch
    from learned_product_hash_b200 import mdr
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dist = init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    es = 2 if w.dtype == "bf16" else 4

    inp = make_inputs(w, 1000 + rank)
    conv = (lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)) if w.dtype == "bf16" \
        else torch.from_numpy
    q_h, k_h, v_h = (conv(x) for x in (inp.q_store, inp.k_store, inp.v_store))
    cb_h = torch.from_numpy(inp.codebooks)
    q, k, v, cb = (t.to(dev) for t in (q_h, k_h, v_h, cb_h))
    cfg = mdr.make_config(w)
    idx = mdr.Index.empty(cfg, dev)
    rt = mdr.RouteOut.empty(cfg, dev)
    out = torch.empty_like(q)
    ws = mdr.workspace(cfg, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def flush_l2():
        flush.zero_()
        flush.max()

    def step(evs):
        flush_l2()
        mdr.mdr_forward_profiled(cfg, q, k, v, cb, idx, rt, out, ws, evs)

    for _ in range(args.warmup):
        step([None] * 5)
    torch.cuda.synchronize()
    assert mdr.mdr_read_device_status(ws) == 0
    # Timed steps: events before the first and after the last kernel only
    # (an event between two kernels would hold the next one back until the
    # previous has drained, undoing the overlap of their launches).
    evs = [[torch.cuda.Event(enable_timing=True), None, None, None, torch.cuda.Event(enable_timing=True)]
           for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for s in range(args.steps):
            step(evs[s])
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    assert mdr.mdr_read_device_status(ws) == 0
    tot = [e[0].elapsed_time(e[4]) for e in evs]
    # Per-kernel breakdown: separate steps with an event at every kernel boundary.
    kevs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(min(args.steps, 20))]
    for e in kevs:
        step(e)
    torch.cuda.synchronize()
    ker = {n: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in kevs)
           for i, n in enumerate(("summarize", "lists", "route", "attend"))}
    ms_max = max_over_ranks(statistics.mean(tot), dist, world, dev)
    tokens = w.B * w.S * world
    value = throughput(w.B * w.S, world, ms_max)

    # Roofline of the attention kernel: q read + gathered K/V of valid
    # selected blocks + out write, per (b, hq, j) route.
    sel = rt.sel.cpu().numpy()
    nsel = int((sel >= 0).sum())
    by = forward_bytes(w, nsel, es)
    attn_bytes = by["attention"]
    peak, peak_kind = peaks()
    achieved = attn_bytes / (ker["attend"] / 1e3) / 1e9
    total_bytes = by["path"]
    kernels = {
        "summarize": {"ms": ker["summarize"], "algorithmic_bytes": by["summaries"],
                      "frac": by["summaries"] / (ker["summarize"] / 1e3) / 1e9 / peak,
                      "also_written_bytes": by["rotated_copies_written"],
                      "note": "reads q, k once (the byte model); also writes the rotated copies the "
                              "attention reads, which the byte model does not count"},
        "lists": {"ms": ker["lists"], "note": "one CTA per (sequence, KV head); < 1 % of the bytes"},
        "route": {"ms": ker["route"], "note": "reads list slots and key summaries (L2); < 1 % of the bytes"},
        "attend": {"ms": ker["attend"], "algorithmic_bytes": attn_bytes, "frac": achieved / peak}}

    # Decoding: the state of the first nb-1 blocks (prefill), then one token
    # per sequence at a time through the last block, timed with CUDA events
    # over consecutive steps (no block completes inside the timed steps).
    decode = None
    if not args.no_decode:
        dst = mdr.DecodeState.empty(cfg, dev)
        dws = mdr.decode_workspace(cfg, dev)
        S0 = w.S - w.block
        mdr.mdr_decode_prefill(cfg, S0, k[:, :S0].contiguous(), v[:, :S0].contiguous(), cb, dst, dws)
        n_dec = min(60, w.block - 1)
        toks = [(q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous()) for t in range(S0, S0 + n_dec)]
        out_t = torch.empty(w.B, w.Hq, w.D, dtype=q.dtype, device=dev)
        sel_t = torch.empty(w.B, w.Hq, w.R + w.L, dtype=torch.int32, device=dev)
        for i in range(3):
            mdr.mdr_decode_step(cfg, S0 + i, *toks[i], cb, dst, out_t, sel_t, dws)
        torch.cuda.synchronize()
        # The C entry point with its arguments marshalled once, so that the
        # host stays ahead of the GPU and the events time the device work.
        import ctypes
        fn = mdr.lib().mdr_decode_step
        cfg_r, st_r = ctypes.byref(cfg), ctypes.byref(dst.c())
        sp = stream.cuda_stream
        calls = [(cfg_r, S0 + i, qq.data_ptr(), kk.data_ptr(), vv.data_ptr(), cb.data_ptr(), st_r,
                  out_t.data_ptr(), sel_t.data_ptr(), None, dws.data_ptr(), dws.numel(), sp)
                 for i, (qq, kk, vv) in enumerate(toks)]
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for c_args in calls:
            if fn(*c_args) != mdr.MDR_OK:
                raise RuntimeError("mdr_decode_step failed")
        d1.record(stream)
        d1.synchronize()
        assert mdr.mdr_read_device_status(dws) == 0
        d_ms = d0.elapsed_time(d1) / n_dec
        t_last = S0 + n_dec - 1
        sl = sel_t.cpu().numpy()
        ntok = int(sum(min(w.block, t_last + 1 - int(blk) * w.block) for blk in sl.ravel() if blk >= 0))
        d_bytes = ntok * 2 * w.D * es + 2 * w.B * w.Hq * w.D * es     # gathered K, V + q, out
        d_ms_max = max_over_ranks(d_ms, dist, world, dev)
        decode = {"metric": "decode step latency (one token per sequence: key append, route, attend) at 32K",
                  "value": d_ms_max * 1e3, "unit": "us/step", "tokens_per_s": w.B * world / (d_ms_max / 1e3),
                  "batch_per_gpu": w.B, "steps": n_dec, "position": f"tokens {S0}..{t_last} ({S0 // w.block} blocks indexed)",
                  "l2": "not flushed between steps", "gpu_launches": 3 * n_dec,
                  "roofline": {"bound": "hbm", "achieved": d_bytes / (d_ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                               "frac": d_bytes / (d_ms / 1e3) / 1e9 / peak, "algorithmic_bytes_per_step": d_bytes}}
        del dst, dws
        decode["batched"] = batched_decode(mdr, w, args.decode_batch, dev, stream, dist, world, peak)

    # Controls on the planted-block workload (untimed): how often the route
    # selects each sequence's planted block for its last query block, with
    # the random unit codebooks (the untrained router), with the planted
    # block forced in, and with no remote blocks at all (R = 0).
    controls = None
    if not args.no_controls:
        wa = workload("ar")
        ia = make_inputs(wa, 2000 + rank)
        conv_a = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        qa, ka = conv_a(ia.q_store), conv_a(ia.k_store)
        cba = torch.from_numpy(ia.codebooks).to(dev)
        tg = np.full((wa.B, wa.Hq, wa.nb), -1, dtype=np.int32)
        tg[:, :, wa.nb - 1] = ia.planted[:, None]
        tg = torch.from_numpy(tg).to(dev)
        counts = torch.empty(2, dtype=torch.int32, device=dev)
        rates = {}
        for name, wc, forced in (("route", wa, False), ("forced", wa, True), ("local_only", wa.with_(R=0), False)):
            ca = mdr.make_config(wc)
            ixa, rta, wsa = mdr.Index.empty(ca, dev), mdr.RouteOut.empty(ca, dev), mdr.workspace(ca, dev)
            mdr.mdr_build_index(ca, ka, cba, ixa, wsa)
            if forced:
                mdr.mdr_route_forced(ca, qa, cba, ixa, tg, rta, wsa)
            else:
                mdr.mdr_route(ca, qa, cba, ixa, rta, wsa)
            mdr.mdr_target_hits(ca, rta.sel, tg, counts)
            n_t, n_h = (int(x) for x in counts.cpu())
            rates[name] = n_h / n_t
        controls = {"workload": f"{wa.name}: B={wa.B}, H={wa.Hq}, S={wa.S}, block {wa.block}, R={wa.R}, L={wa.L}, "
                                "one planted block per sequence, random unit codebooks",
                    "routes_with_target": n_t, "target_hit_rate": rates}

    # Codebook calibration on the long workload (the Report's Figure 3
    # analogue): the key summaries of one training sequence, computed by
    # mdr_build_index, calibrate the random codebooks for 20 rounds (timed);
    # then a held-out sequence is indexed with the codebooks before and after.
    calibration = None
    if not args.no_calibration:
        wl = workload("long")
        cl = mdr.make_config(wl)
        cb0 = torch.from_numpy(make_codebooks(wl, 3000 + rank)).to(dev)
        ixl, wsl = mdr.Index.empty(cl, dev), mdr.workspace(cl, dev)
        conv_b = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
        mdr.mdr_build_index(cl, conv_b(make_keys(wl, 3001 + rank)[1]), cb0, ixl, wsl)
        rec = ixl.kbar.clone()                                   # [1, Hkv, nb, D] = [N, D]
        N = rec.numel() // wl.D
        cws = mdr.calibrate_workspace(N, wl.D, wl.P, wl.K, dev)
        cb1 = torch.empty_like(cb0)
        rounds = 20
        mdr.mdr_calibrate_codebooks(rec, cb0, cb1, 2, cws)       # warm-up
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        mdr.mdr_calibrate_codebooks(rec, cb0, cb1, rounds, cws)
        c1.record(stream)
        c1.synchronize()
        c_ms = c0.elapsed_time(c1) / rounds
        kh = conv_b(make_keys(wl, 3002 + rank)[1])
        held = {}
        for name, cbx in (("before", cb0), ("after", cb1)):
            mdr.mdr_build_index(cl, kh, cbx, ixl, wsl)
            held[name] = {"overflow": int(ixl.overflow.sum().item()), "max_load": int(ixl.maxload.max().item())}
        c_bytes = 2 * N * wl.D * 4 + 2 * N * wl.P * 4           # records read by assign and update, assignment
        peak_c, _ = peaks()
        calibration = {"workload": f"{wl.name}: key summaries of one training sequence ({N} records of {wl.D}), "
                                   f"P={wl.P}, K={wl.K}, {rounds} rounds from random unit codebooks",
                       "us_per_round": c_ms * 1e3, "launches_per_round": 3,
                       "l2": "not flushed: the 4 MB of records stay in L2 across rounds, as in a calibration loop",
                       "roofline": {"bound": "hbm", "achieved": c_bytes / (c_ms / 1e3) / 1e9, "peak": peak_c,
                                    "unit": "GB/s", "frac": c_bytes / (c_ms / 1e3) / 1e9 / peak_c,
                                    "algorithmic_bytes_per_round": c_bytes},
                       "held_out": held, "capacity": wl.cap}
        del ixl, wsl, cws, rec
        # The same rounds on a record set far larger than L2 (2^20 unit
        # records, 512 MB): the bandwidth regime, where the 8K-record loop
        # above is bound by its three launches per round.
        NL, rounds_l = 1 << 20, 5
        gl = torch.Generator(device=dev)
        gl.manual_seed(3100 + rank)
        recl = torch.randn(NL, wl.D, generator=gl, device=dev)
        recl /= recl.norm(dim=1, keepdim=True)
        cwl = mdr.calibrate_workspace(NL, wl.D, wl.P, wl.K, dev)
        mdr.mdr_calibrate_codebooks(recl, cb0, cb1, 1, cwl)      # warm-up
        c0.record(stream)
        mdr.mdr_calibrate_codebooks(recl, cb0, cb1, rounds_l, cwl)
        c1.record(stream)
        c1.synchronize()
        cl_ms = c0.elapsed_time(c1) / rounds_l
        cl_bytes = 2 * NL * wl.D * 4 + 2 * NL * wl.P * 4
        calibration["large"] = {
            "records": NL, "rounds": rounds_l, "us_per_round": cl_ms * 1e3,
            "inputs": "unit vectors (torch's seeded generator on the device, normalised)",
            "l2": "the records (512 MB) exceed L2",
            "roofline": {"bound": "hbm", "achieved": cl_bytes / (cl_ms / 1e3) / 1e9, "peak": peak_c, "unit": "GB/s",
                         "frac": cl_bytes / (cl_ms / 1e3) / 1e9 / peak_c, "algorithmic_bytes_per_round": cl_bytes}}
        del recl, cwl

    # Backward of the attention with the forward's route held fixed: dq, dk,
    # dv (float32) for a seeded upstream gradient, timed with CUDA events.
    backward = None
    if not args.no_backward:
        do = torch.from_numpy(make_grad(w, 4000 + rank)[1].view(np.int16)).view(torch.bfloat16).to(dev) \
            if w.dtype == "bf16" else torch.from_numpy(make_grad(w, 4000 + rank)[1]).to(dev)
        dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
        dk = torch.empty(k.shape, dtype=torch.float32, device=dev)
        dv = torch.empty(v.shape, dtype=torch.float32, device=dev)
        bws = mdr.backward_workspace(cfg, dev)
        for _ in range(2):
            mdr.mdr_attend_backward(cfg, q, k, v, rt.sel, do, dq, dk, dv, bws)
        torch.cuda.synchronize()
        nb_it = 5
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        for _ in range(nb_it):
            mdr.mdr_attend_backward(cfg, q, k, v, rt.sel, do, dq, dk, dv, bws)
        b1.record(stream)
        b1.synchronize()
        assert mdr.mdr_read_device_status(bws) == 0
        b_ms = b0.elapsed_time(b1) / nb_it
        b_ms_max = max_over_ranks(b_ms, dist, world, dev)
        fl = backward_flops(sel, w.block, w.D)
        if w.dtype == "bf16":
            tpk, tpk_kind = tensor_peak()
            roof = {"bound": "tensor", "achieved": fl / (b_ms / 1e3) / 1e12, "peak": tpk, "unit": "TFLOP/s",
                    "frac": fl / (b_ms / 1e3) / 1e12 / tpk, "peak_kind": tpk_kind,
                    "algorithmic_flops_per_call": fl,
                    "note": "flops of the four gradient products; the kernels also recompute S twice, "
                            "dP twice and O once (about 2.25x the algorithmic MMA work)"}
            arith = "bf16 operands on the tensor cores (tcgen05), float32 accumulation in tensor memory"
            launches = 4
        else:
            alu_peak = torch.cuda.get_device_properties(dev).multi_processor_count * FP32_LANES_PER_SM * 2 * \
                (clk.summary() or {}).get("sm_max_mhz", 1965) * 1e6 / 1e12
            roof = {"bound": "alu", "achieved": fl / (b_ms / 1e3) / 1e12, "peak": alu_peak, "unit": "TFLOP/s",
                    "frac": fl / (b_ms / 1e3) / 1e12 / alu_peak,
                    "peak_kind": "derived: SMs x 128 FP32 lanes x 2 flops x max SM clock",
                    "algorithmic_flops_per_call": fl}
            arith = "float32 on CUDA cores"
            launches = 4
        # With the forward's output and row normalisers saved (training: the
        # forward ran mdr_forward_train), the dq kernel skips its statistics pass.
        saved = None
        if w.dtype == "bf16":
            o_s = torch.empty_like(q)
            lse_s = torch.empty(w.B, w.Hq, w.S, dtype=torch.float32, device=dev)
            mdr.mdr_attend_train(cfg, q, k, v, rt.sel, o_s, lse_s, ws)
            for _ in range(2):
                mdr.mdr_attend_backward_saved(cfg, q, k, v, rt.sel, o_s, lse_s, do, dq, dk, dv, bws)
            torch.cuda.synchronize()
            b0.record(stream)
            for _ in range(nb_it):
                mdr.mdr_attend_backward_saved(cfg, q, k, v, rt.sel, o_s, lse_s, do, dq, dk, dv, bws)
            b1.record(stream)
            b1.synchronize()
            assert mdr.mdr_read_device_status(bws) == 0
            s_ms = max_over_ranks(b0.elapsed_time(b1) / nb_it, dist, world, dev)
            tpk_s, tpk_kind_s = tensor_peak()
            saved = {"entry_point": "mdr_attend_backward_saved (output and row normalisers of mdr_attend_train)",
                     "ms_per_call": s_ms, "value": throughput(w.B * w.S, world, s_ms), "unit": "tokens/s",
                     "roofline": {"bound": "tensor", "achieved": fl / (s_ms / 1e3) / 1e12, "peak": tpk_s,
                                  "unit": "TFLOP/s", "frac": fl / (s_ms / 1e3) / 1e12 / tpk_s,
                                  "peak_kind": tpk_kind_s}}
            del o_s, lse_s
        bb = backward_bytes(w, sel, es)
        hpk, hpk_kind = peaks()
        roof_bytes = {"bound": "hbm", "achieved": bb / (b_ms / 1e3) / 1e9, "peak": hpk, "unit": "GB/s",
                      "frac": bb / (b_ms / 1e3) / 1e9 / hpk, "peak_kind": hpk_kind,
                      "algorithmic_bytes_per_call": bb,
                      "note": "the bytes side of the same call: at ~34 flops per byte the gradient sits far below "
                              "the ridge of either peak; the kernels take in ~2.7 GB (the dq kernel gathers K, V "
                              "twice: a statistics pass and a gradient pass)"}
        backward = {"metric": "attention backward (dq, dk, dv for a fixed route) at 32K",
                    "value": throughput(w.B * w.S, world, b_ms_max), "unit": "tokens/s", "ms_per_call": b_ms_max,
                    "launches_per_call": launches, "arithmetic": arith,
                    "l2": "not flushed between calls: q, k, v, dout, the rotated copies and the float32 "
                          "gradients (~0.8 GB) exceed L2",
                    "roofline": roof, "roofline_bytes": roof_bytes, "saved_statistics": saved}
        del bws, dq, dk, dv, do

    # Scaling of the forward from 4K to 128K tokens (one GPU): the median of
    # 10 L2-flushed mdr_forward calls per length, inputs drawn on the device
    # by torch's seeded generator (q, k, v ~ N(0, 1), the recipe of the
    # scaling workloads), and the log-log slope over 4K-32K (the Report's
    # range) and 4K-128K; beside it, the CPU oracle's index build + route at
    # 4K-32K (one warm-up, median of 3, as the Report times it).
    scaling_obj = None
    if world == 1 and not args.no_sweep:
        try:
            pts, sweep_bytes = {}, {}
            for wsw in SCALING_SWEEP:
                csw = mdr.make_config(wsw)
                gen = torch.Generator(device=dev)
                gen.manual_seed(5000 + wsw.S)
                mk = lambda H: torch.randn(wsw.B, wsw.S, H, wsw.D, generator=gen, device=dev).to(torch.bfloat16)
                qs_, ks_, vs_ = mk(wsw.Hq), mk(wsw.Hkv), mk(wsw.Hkv)
                cbs = torch.from_numpy(make_codebooks(wsw, 5000)).to(dev)
                ixs, rts, wss = mdr.Index.empty(csw, dev), mdr.RouteOut.empty(csw, dev), mdr.workspace(csw, dev)
                outs = torch.empty_like(qs_)
                times = []
                for it in range(13):
                    flush_l2()
                    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    s0.record(stream)
                    mdr.mdr_forward(csw, qs_, ks_, vs_, cbs, ixs, rts, outs, wss)
                    s1.record(stream)
                    s1.synchronize()
                    if it >= 3:
                        times.append(s0.elapsed_time(s1))
                assert mdr.mdr_read_device_status(wss) == 0
                pts[wsw.S] = statistics.median(times)
                nsel_sw = int((rts.sel >= 0).sum().item())
                by_sw = forward_bytes(wsw, nsel_sw, 2)
                sweep_bytes[wsw.S] = {"selected_blocks_per_route": nsel_sw / (wsw.B * wsw.Hq * wsw.nb),
                                      "path_bytes": by_sw["path"],
                                      "path_roofline_frac": by_sw["path"] / (pts[wsw.S] / 1e3) / 1e9 / peak,
                                      "kv_bytes": 2 * wsw.B * wsw.S * wsw.Hkv * wsw.D * 2}
                del qs_, ks_, vs_, ixs, rts, wss, outs
            Ss = sorted(pts)
            short = [S for S in Ss if S <= 32768]
            scaling_obj = {"workload": "scaling: B=1, H=8, D=128 bf16, block 64, K=32, cap 64, p=4, R=8, L=2",
                           "ms_per_forward": {str(S): pts[S] for S in Ss},
                           "tokens_per_s": {str(S): S / (pts[S] / 1e3) for S in Ss},
                           "per_length": {str(S): sweep_bytes[S] for S in Ss},
                           "l2_bytes": torch.cuda.get_device_properties(dev).L2_cache_size,
                           "exponent_4k_32k": loglog_exponent(short, [pts[S] for S in short]),
                           "exponent_4k_128k": loglog_exponent(Ss, [pts[S] for S in Ss])}
            if rank == 0 and not args.no_cpu:
                cpu_pts = {}
                for wsw in [x for x in SCALING_SWEEP if x.S <= 32768]:
                    cpu_pts[wsw.S] = statistics.median(oracle_route_seconds(wsw, 6000, 4)[1:])   # 1 warm-up, median of 3
                Sc = sorted(cpu_pts)
                scaling_obj["cpu_oracle_index_route"] = {
                    "seconds": {str(S): cpu_pts[S] for S in Sc}, "cores": blas_threads(),
                    "threads": "the BLAS pool as it stands; the route itself is a Python loop (one thread)",
                    "exponent_4k_32k": loglog_exponent(Sc, [cpu_pts[S] for S in Sc])}
        except Exception as e:                   # the line still carries every other number
            scaling_obj = {"error": repr(e)}

    # The forward on the other workload shapes (one GPU): the planted-block,
    # capacity and long-context workloads, each with its byte model,
    # roofline fractions, overflow and (grouped heads) the union of each
    # group's selections.
    workloads_obj = None
    if world == 1 and not args.no_workloads:
        workloads_obj = {}
        for name in ("ar", "capacity", "long"):
            try:
                wx = workload(name)
                if name == "long":
                    qx, kx, vx, cbx = device_inputs(wx, 7000, dev)
                    recipe = "q, v ~ N(0,1) drawn on the device (torch, seeded); keys: the Zipf cluster recipe"
                else:
                    ix = make_inputs(wx, 7000)
                    qx, kx, vx = (conv(x).to(dev) for x in (ix.q_store, ix.k_store, ix.v_store))
                    cbx = torch.from_numpy(ix.codebooks).to(dev)
                    recipe = f"the {wx.keys} recipe of the workload generator"
                r = measure_forward(mdr, wx, qx, kx, vx, cbx, dev, stream, flush_l2)
                r["config"] = {k_: v_ for k_, v_ in config_of(wx, argparse.Namespace(gpus=1)).items()
                               if k_ not in ("l2", "parallelism")}
                r["inputs"] = recipe
                workloads_obj[name] = r
                del qx, kx, vx, cbx
            except Exception as e:                  # the line still carries every other number
                workloads_obj[name] = {"error": repr(e)}
        torch.cuda.empty_cache()

    # End to end through the C ABI with host buffers.
    e2e = None
    if not args.no_e2e:
        qp, kp, vp = (x.pin_memory() for x in (q_h, k_h, v_h))
        cbp = cb_h.pin_memory()
        outp = torch.empty_like(qp).pin_memory()
        selp = torch.empty(sel.shape, dtype=torch.int32).pin_memory()
        ovp = torch.empty(w.B, w.Hkv, dtype=torch.int32).pin_memory()
        mxp = torch.empty(w.B, w.Hkv, dtype=torch.int32).pin_memory()
        dws = torch.empty(mdr.mdr_host_workspace_bytes(cfg), dtype=torch.uint8, device=dev)
        nE = max(3, min(args.steps, 10))
        times = []
        for it in range(2 + nE):
            flush_l2()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            mdr.mdr_forward_host(cfg, qp, kp, vp, cbp, outp, selp, ovp, mxp, dws)
            e1.record(stream)
            e1.synchronize()
            if it >= 2:
                times.append(e0.elapsed_time(e1))
        te_ms = max_over_ranks(statistics.mean(times), dist, world, dev)
        h2d = sum(x.numel() * x.element_size() for x in (qp, kp, vp, cbp))
        d2h = sum(x.numel() * x.element_size() for x in (outp, selp, ovp, mxp))
        e2e = {"value": throughput(w.B * w.S, world, te_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": te_ms}
        del dws

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(w, args.cpu_seconds)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
                "config": config_of(w, argparse.Namespace(gpus=world)),
                "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                             "frac": achieved / peak, "traffic": profiled_traffic("attend", w.name),
                             "peak_kind": peak_kind,
                             "kernel": "attend", "algorithmic_bytes_per_launch": attn_bytes},
                "path_roofline_frac": total_bytes / (ms_max / 1e3) / 1e9 / peak,
                "path_bytes": total_bytes, "kernels": kernels,
                "kernels_ms": ker, "cpu_baseline": cpu, "e2e": e2e, "decode": decode,
                "controls": controls, "calibration": calibration, "backward": backward,
                "scaling_sweep": scaling_obj, "workloads": workloads_obj,
                "gpu_launches": KERNELS_PER_FORWARD * args.steps, "clocks": clk.summary(),
                "overflow": int(idx.overflow.sum().item()), "selected_blocks": nsel}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="mine", choices=["mine", "reference"])
    ap.add_argument("--workload", default="scaling32k")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-controls", action="store_true")
    ap.add_argument("--no-calibration", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-workloads", action="store_true")
    ap.add_argument("--decode-batch", type=int, default=32)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args()
    w = workload(args.workload)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_mine(args, w)


if __name__ == "__main__":
    main()
