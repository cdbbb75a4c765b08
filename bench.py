#!/usr/bin/env python
"""Throughput of the MLA hot path on B200: one JSON line on stdout.

A step is one pass of the whole hot path on seeded synthetic inputs that are
resident in HBM: the Kimi-K2-shape causal prefill (B=1, T=2048, H=64,
R=512, N=128, P=64, V=128, YaRN) followed by the absorbed decode over a
latent cache (B=64, cache lengths uniform in [1000, 32768], Kimi-K2 heads).
The headline ``value`` is the prefill's TFLOP/s (algorithmic FLOPs over the
prefill's device time in each step); the decode's HBM GB/s is reported in
the ``decode`` object of the same line. Between steps L2 is flushed by
writing a 256 MiB buffer outside the per-step events.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload on the host cores instead (the reference arm).

Multi-GPU: the path does not shard across GPUs here (one process per GPU runs
an independent replica; no collective on the data path); ``value`` sums the
replicas' work over the slowest rank's time ("scaling": "weak").
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from decode_latent_rmsnorm_b200 import mla  # noqa: E402
from decode_latent_rmsnorm_b200 import workloads as W  # noqa: E402

METRIC = "MLA causal prefill TFLOP/s (frac of BF16 peak); absorbed decode HBM GB/s"


# ---------------------------------------------------------------- algorithmic work

def prefill_flops(wl) -> dict:
    """Algorithmic FLOPs: up-projection 2*T*R*H*(N+V); attention over the
    unmasked causal pairs only, 2*H*(D+V) per pair."""
    T = sum(wl.seqlens)
    H, R, N, P, V = wl.num_heads, wl.kv_lora_rank, wl.qk_nope, wl.qk_rope, wl.v_head
    up = 2.0 * T * R * H * (N + V)
    pairs = sum(L * (L + 1) / 2 for L in wl.seqlens)
    attn = 2.0 * H * (N + P + V) * pairs
    return dict(up=up, attn=attn, total=up + attn)


def decode_bytes(wl, lens) -> dict:
    """Algorithmic HBM bytes: every cached row once, kv_b_proj once, q and out."""
    H, R, N, P, V = wl.num_heads, wl.kv_lora_rank, wl.qk_nope, wl.qk_rope, wl.v_head
    es = 2 if wl.dtype == "bf16" else 4
    B = len(lens)
    cache = float(sum(lens)) * (R + P) * es
    weight = float(H) * (N + V) * R * es
    io = float(B) * H * (N + P) * es + float(B) * H * V * es
    flops = 2.0 * sum(lens) * H * ((R + P) + R)
    return dict(cache=cache, weight=weight, io=io, total=cache + weight + io, flops=flops)


def chunk_bytes(wl, prefix, n_new) -> dict:
    """Cache rows of a chunk call: each chunk token reads its sequence's rows
    up to its own (the absorbed form runs one decode row per token), and the
    unique rows are each sequence's prefix plus its chunk."""
    row = (wl.kv_lora_rank + wl.qk_rope) * 2
    attended = sum(p * n_new + n_new * (n_new + 1) // 2 for p in prefix)
    unique = sum(p + n_new for p in prefix)
    return dict(attended=float(attended) * row, unique=float(unique) * row)


# ---------------------------------------------------------------- environment

def recorded_traffic(kernel: str):
    """DRAM bytes per launch of ``kernel`` from the committed ncu capture
    (profiles/traffic.json), or None when there is none or the kernel's
    source changed since it was taken."""
    from decode_latent_rmsnorm_b200.kernel_sources import source_digest
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel)
    except (OSError, ValueError):
        return None
    if not isinstance(rec, dict) or rec.get("source_digest") != source_digest(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sustained=p["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """SM clock and clock-event reasons sampled while the timed region runs.

    NVML is polled from a thread every ``period_s`` (the timed region of a
    default run lasts only tens of milliseconds, too short for
    ``nvidia-smi -lms``); if NVML cannot be loaded, ``nvidia-smi`` is used."""

    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("sw_power_cap", 0x4),
               ("hw_power_brake_slowdown", 0x80))

    def __init__(self, device: torch.device, period_s: float = 0.0005):
        self.device = device
        self.period_s = period_s
        self.samples = []          # (sm_mhz, reason mask)
        self.max_mhz = None
        self._nvml = None
        self._handle = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None
        self._lines = []

    def _open_nvml(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device)
        uuid = str(props.uuid)
        if not uuid.startswith("GPU-"):
            uuid = "GPU-" + uuid
        self._handle = pynvml.nvmlDeviceGetHandleByUUID(uuid)
        self._nvml = pynvml
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self._handle, pynvml.NVML_CLOCK_SM))

    def _sample_nvml(self):
        nv = self._nvml
        mhz = nv.nvmlDeviceGetClockInfo(self._handle, nv.NVML_CLOCK_SM)
        mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._handle)
        self.samples.append((float(mhz), int(mask)))

    def _poll(self):
        while not self._stop.is_set():
            try:
                self._sample_nvml()
            except Exception:  # a failed read drops one sample
                pass
            time.sleep(self.period_s)

    def __enter__(self):
        try:
            self._open_nvml()
            self._sample_nvml()
            self._thread = threading.Thread(target=self._poll, daemon=True)
            self._thread.start()
        except Exception:
            self._nvml = None
            self._start_smi()
        return self

    def _start_smi(self):
        fields = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.sw_power_cap")
        idx = self.device.index if self.device.index is not None else 0
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(idx), "--query-gpu=" + fields,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._thread = threading.Thread(target=self._read_smi, daemon=True)
            self._thread.start()
        except OSError:
            self._proc = None

    def _read_smi(self):
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        bits = dict(self.REASONS)
        for line in self._proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 6:
                continue
            try:
                mhz, self.max_mhz = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            mask = 0
            for n, v in zip(names, parts[2:]):
                if v.lower() == "active":
                    mask |= bits[n]
            self.samples.append((mhz, mask))

    def __exit__(self, *exc):
        self._stop.set()
        if self._nvml is not None:
            try:
                self._sample_nvml()
            except Exception:
                pass
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
        if self._thread is not None:
            self._thread.join(timeout=5)
        return False

    def summary(self):
        sm = [s[0] for s in self.samples]
        reasons = sorted({n for _, m in self.samples for n, b in self.REASONS if m & b})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sm),
                "source": "nvml" if self._nvml is not None else "nvidia-smi"}


# ---------------------------------------------------------------- CPU oracle timing

def oracle_prefill_sample(wl, inp, budget_s: float):
    """Time the fp64 oracle on whole heads of the prefill workload until
    ``budget_s`` is spent; returns (TFLOP/s, sample text, threads)."""
    import numpy as np
    import oracle as O
    from threadpoolctl import threadpool_info
    rope = O.RopeConfig(**wl.rope)
    shape = O.MlaShape(wl.num_heads, wl.kv_lora_rank, wl.qk_nope, wl.qk_rope, wl.v_head,
                       eps=wl.eps, interleaved=wl.interleaved)
    scale = O.softmax_scale(rope, shape.qk_head_dim)
    cos, sin = O.rope_tables(rope, W.max_position(wl))
    a = {k: (v.double().numpy() if v.is_floating_point() else v.numpy()) for k, v in inp.items()}
    heads_done, t_spent, h = 0, 0.0, 0
    while t_spent < budget_s and h < wl.num_heads:
        t0 = time.perf_counter()
        O.prefill(a["latent"], a["q"], a["w_kvb"], a["w_norm"], a["positions"], a["cu_seqlens"], cos, sin,
                  shape, scale, heads=[h])
        t_spent += time.perf_counter() - t0
        heads_done += 1
        h += 1
    fl = prefill_flops(wl)["total"] * heads_done / wl.num_heads
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return fl / t_spent / 1e12, "%s: %d of %d heads, all rows (%.1f s)" % (
        wl.name, heads_done, wl.num_heads, t_spent), threads


# ---------------------------------------------------------------- GPU bench

def max_over_ranks(x: float, world: int) -> float:
    """The largest value of ``x`` over the job's ranks (identity at one rank).
    The reduction tensor lives where the process group's backend wants it."""
    if world == 1:
        return x
    dist = torch.distributed
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(work_per_rank: float, world: int, slowest_ms: float) -> float:
    """Whole-job rate: the work of all ranks (replicas) over the slowest rank's time."""
    return world * work_per_rank / (slowest_ms * 1e-3)


def workload_config(world, lens):
    """The config object both arms print."""
    return dict(workload="kimi_k2_prefill_bf16 + absorbed_decode_bf16",
                prefill="B=1 T=2048 H=64 R=512 N=128 P=64 V=128 YaRN(base 5e4, factor 32); "
                        "kv_b_proj prepared once",
                decode="B=64 H=64 R=512 N=128 P=64 V=128, cache lens U[1000,32768] sum=%d" % sum(lens),
                global_batch=world * (1 + len(lens)), parallelism="replicas x%d" % world,
                l2="flushed between steps (256 MiB write outside per-step events)")


def run_ours(args, rank, world, device):
    torch.cuda.set_device(device)
    peaks = measured_peaks()
    pwl = W.KIMI
    dwl = W.DECODE
    # inputs, resident in HBM
    pin = W.prefill_inputs(pwl)
    din = W.decode_inputs(dwl)
    lens = [int(x) for x in din["cache_lens"]]
    rope_p = mla.rope_for(pwl)
    dims_p = mla.dims_for(pwl, mla.mla_softmax_scale(rope_p, pwl.qk_head_dim))
    dims_d = mla.dims_for(dwl, mla.mla_softmax_scale(mla.rope_for(dwl), dwl.qk_head_dim))
    max_pos = max(W.max_position(pwl), W.max_position(dwl))
    cos, sin = mla.mla_init_rope_tables(rope_p, max_pos)
    P = {k: v.to(device) for k, v in pin.items()}
    D = {k: v.to(device) for k, v in din.items()}
    T = sum(pwl.seqlens)
    p_out = torch.empty((T, pwl.num_heads, pwl.v_head), dtype=torch.bfloat16, device=device)
    p_ws = torch.empty(mla.mla_prefill_workspace_size(dims_p, T, len(pwl.seqlens)), dtype=torch.uint8,
                       device=device)
    B = dwl.batch
    max_len = max(lens)
    d_out = torch.empty((B, dwl.num_heads, dwl.v_head), dtype=torch.bfloat16, device=device)
    d_ws = torch.empty(mla.mla_decode_workspace_size(dims_d, B, max_len), dtype=torch.uint8, device=device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    # kv_b_proj is converted for the tensor cores once, as at model load
    w_prep = mla.mla_prepare_kv_b_proj(dims_p, P["w_kvb"])

    def prefill():
        mla.mla_prefill_prepared(dims_p, P["latent"], P["q"], w_prep, P["w_norm"], P["positions"],
                                 P["cu_seqlens"], max(pwl.seqlens), cos, sin, out=p_out, workspace=p_ws)

    def prefill_unprepared():
        mla.mla_prefill(dims_p, P["latent"], P["q"], P["w_kvb"], P["w_norm"], P["positions"],
                        P["cu_seqlens"], max(pwl.seqlens), cos, sin, out=p_out, workspace=p_ws)

    def decode():
        mla.mla_decode(dims_d, D["q"], D["cache"], D["cache_offsets"], D["cache_lens"], D["positions"],
                       max_len, D["w_kvb"], cos, sin, out=d_out, workspace=d_ws)

    for _ in range(args.warmup):
        flush.fill_(1)
        prefill()
        decode()
    torch.cuda.synchronize()
    mla.mla_check_device_status()

    # timed region: events around the prefill and the decode of each step (no
    # events between the kernels of one call, which would keep the next
    # kernel from starting while the previous one finishes)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    launches0 = mla.mla_launch_count()
    with ClockSampler(device) as clocks:
        for i in range(args.steps):
            flush.fill_(i & 0xff)
            ev[i][0].record()
            prefill()
            ev[i][1].record()
            decode()
            ev[i][2].record()
        torch.cuda.synchronize()
    launches = mla.mla_launch_count() - launches0
    # per-kernel breakdown: the same steps again, with events around every kernel
    kev_p, kev_d = [], []
    for i in range(args.steps):
        flush.fill_(i & 0xff)
        kp, kd = mla.KernelEvents(16), mla.KernelEvents(16)
        with kp:
            prefill()
        with kd:
            decode()
        kev_p.append(kp)
        kev_d.append(kd)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    mla.mla_check_device_status()
    p_ms = [e[0].elapsed_time(e[1]) for e in ev]
    d_ms = [e[1].elapsed_time(e[2]) for e in ev]
    step_ms = [a + b for a, b in zip(p_ms, d_ms)]

    def reduce_max(x):
        return max_over_ranks(x, world)

    p_mean = reduce_max(statistics.mean(p_ms))
    d_mean = reduce_max(statistics.mean(d_ms))
    s_mean = reduce_max(statistics.mean(step_ms))
    fl = prefill_flops(pwl)
    by = decode_bytes(dwl, lens)
    p_tflops = job_throughput(fl["total"], world, p_mean) / 1e12
    d_gbs = job_throughput(by["total"], world, d_mean) / 1e9

    # per-kernel mean durations (kernel names reported by the library)
    def kernel_means(kev):
        acc = {}
        for k in kev:
            for n, t in zip(k.names, k.durations_ms()):
                acc.setdefault(n, []).append(t)
        return {n: statistics.mean(v) for n, v in acc.items()}

    kp_ms, kd_ms = kernel_means(kev_p), kernel_means(kev_d)
    allk = {**{("prefill", n): t for n, t in kp_ms.items()}, **{("decode", n): t for n, t in kd_ms.items()}}
    (phase, top), top_ms = max(allk.items(), key=lambda kv: kv[1])
    if phase == "prefill":
        algo = fl["attn"] if "attention" in top else fl["up"] if "proj" in top else fl["total"]
        roof = dict(bound="tensor", achieved=algo / (top_ms * 1e-3) / 1e12, peak=peaks["bf16"],
                    unit="TFLOP/s")
    else:
        algo = by["cache"] if "attention" in top else by["total"]
        roof = dict(bound="hbm", achieved=algo / (top_ms * 1e-3) / 1e9, peak=peaks["hbm"], unit="GB/s")
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = recorded_traffic(top)
    roof["kernel"] = top
    roof["peak_source"] = peaks["source"]

    # the prefill with kv_b_proj converted inside the call (mla_prefill)
    unprep_ms = reduce_max(time_calls(args, prefill_unprepared, flush))
    chunk = run_chunk(args, din, D, device, world, reduce_max, peaks)
    chunk["long"] = run_chunk_long(args, device, world, reduce_max, peaks, flush)
    projections = run_projections(args, device, world, reduce_max, peaks)
    configs = run_configs(args, device, world, reduce_max, peaks, flush)

    # end to end through the same C-ABI with pinned host buffers
    e2e = run_e2e(args, pwl, dwl, pin, din, dims_p, dims_d, cos, sin, P, D, p_ws, d_ws, device, world,
                  reduce_max, fl, by, w_prep)

    res = dict(
        metric=METRIC, value=p_tflops, unit="TFLOP/s", n_gpus=world, steps=args.steps,
        warmup=args.warmup, ms_per_step=s_mean, higher_is_better=True, scaling="weak",
        vs_baseline=None, dtype="bf16", data="synthetic (seeded N(0,1) inputs, N(0,1/R) kv_b_proj)",
        config=workload_config(world, lens),
        prefill=dict(ms=p_mean, tflops=p_tflops, frac_of_bf16_peak=p_tflops / (world * peaks["bf16"]),
                     tokens_per_s=world * T / (p_mean * 1e-3), gflop=fl["total"] / 1e9,
                     weight="kv_b_proj prepared once (mla_prepare_kv_b_proj), mla_prefill_prepared timed",
                     unprepared=dict(call="mla_prefill (kv_b_proj converted inside every call)",
                                     ms=unprep_ms, tflops=world * fl["total"] / (unprep_ms * 1e-3) / 1e12)),
        decode=dict(metric="absorbed decode HBM GB/s", value=d_gbs, unit="GB/s", ms=d_mean,
                    frac_of_hbm=d_gbs / (world * peaks["hbm"]), tokens_per_s=world * B / (d_mean * 1e-3),
                    tflops=world * by["flops"] / (d_mean * 1e-3) / 1e12, bytes=by["total"]),
        kernels_ms=dict(prefill=kp_ms, decode=kd_ms), configs=configs, chunk=chunk, projections=projections,
        roofline=roof, e2e=e2e, gpu_launches=int(launches), clocks=clocks.summary(),
        peaks=dict(hbm_gbs=peaks["hbm"], bf16_tflops=peaks["bf16"], source=peaks["source"]),
    )
    return res, (pwl, pin)


def run_e2e(args, pwl, dwl, pin, din, dims_p, dims_d, cos, sin, P, D, p_ws, d_ws, device, world,
            reduce_max, fl, by, w_prep):
    """The same calls end to end: every step copies its inputs from pinned host
    memory and reads its result back. Weights, rotary tables and the latent
    cache stay resident (model state); the step inputs are the prefill's
    latent/q/positions/cu_seqlens and the decode's q/positions/lengths/offsets.

    Steps run as a serving pipeline on three streams with double-buffered
    device inputs and outputs: the upload of step i+1 and the download of
    step i-1 overlap the kernels of step i. The timed region spans all K
    steps, from the first upload to the last download; the reported time per
    step is that span over K. The same steps run one after another on one
    stream are reported under ``serial``."""
    hp = {k: pin[k].pin_memory() for k in ("latent", "q", "positions", "cu_seqlens")}
    hd = {k: din[k].pin_memory() for k in ("q", "positions", "cache_lens", "cache_offsets")}
    T = sum(pwl.seqlens)
    B = dwl.batch
    max_len = int(din["cache_lens"].max())
    nb = 2
    p_shape, d_shape = (T, pwl.num_heads, pwl.v_head), (B, dwl.num_heads, dwl.v_head)
    bufs = dict(
        prefill=dict(host_in=hp, dev_in=[{k: torch.empty_like(v, device=device) for k, v in hp.items()}
                                         for _ in range(nb)],
                     dev_out=[torch.empty(p_shape, dtype=torch.bfloat16, device=device) for _ in range(nb)],
                     host_out=[torch.empty(p_shape, dtype=torch.bfloat16).pin_memory() for _ in range(nb)]),
        decode=dict(host_in=hd, dev_in=[{k: torch.empty_like(v, device=device) for k, v in hd.items()}
                                        for _ in range(nb)],
                    dev_out=[torch.empty(d_shape, dtype=torch.bfloat16, device=device) for _ in range(nb)],
                    host_out=[torch.empty(d_shape, dtype=torch.bfloat16).pin_memory() for _ in range(nb)]))
    h2d = {k: sum(v.numel() * v.element_size() for v in b["host_in"].values()) for k, b in bufs.items()}
    d2h = {k: b["host_out"][0].numel() * 2 for k, b in bufs.items()}

    def compute(kind, s):
        x, out = bufs[kind]["dev_in"][s], bufs[kind]["dev_out"][s]
        if kind == "prefill":
            mla.mla_prefill_prepared(dims_p, x["latent"], x["q"], w_prep, P["w_norm"], x["positions"],
                                     x["cu_seqlens"], max(pwl.seqlens), cos, sin, out=out, workspace=p_ws)
        else:
            mla.mla_decode(dims_d, x["q"], D["cache"], x["cache_offsets"], x["cache_lens"], x["positions"],
                           max_len, D["w_kvb"], cos, sin, out=out, workspace=d_ws)

    def upload(kind, s):
        b = bufs[kind]
        for k, v in b["host_in"].items():
            b["dev_in"][s][k].copy_(v, non_blocking=True)

    def download(kind, s):
        bufs[kind]["host_out"][s].copy_(bufs[kind]["dev_out"][s], non_blocking=True)

    def pipelined(kind, steps):
        comp = torch.cuda.current_stream()
        up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
        in_free, out_free = [None] * nb, [None] * nb
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record(up)
        for i in range(steps):
            sl = i % nb
            if in_free[sl] is not None:
                up.wait_event(in_free[sl])
            with torch.cuda.stream(up):
                upload(kind, sl)
            uploaded = torch.cuda.Event()
            uploaded.record(up)
            comp.wait_event(uploaded)
            if out_free[sl] is not None:
                comp.wait_event(out_free[sl])
            compute(kind, sl)
            done = torch.cuda.Event()
            done.record(comp)
            in_free[sl] = done
            down.wait_event(done)
            with torch.cuda.stream(down):
                download(kind, sl)
            fetched = torch.cuda.Event()
            fetched.record(down)
            out_free[sl] = fetched
        end.record(down)
        torch.cuda.synchronize()
        return start.elapsed_time(end) / steps

    def serial(kind, steps):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for e in evs:
            e[0].record()
            upload(kind, 0)
            compute(kind, 0)
            download(kind, 0)
            e[1].record()
        torch.cuda.synchronize()
        return statistics.mean(e[0].elapsed_time(e[1]) for e in evs)

    res = {}
    for kind in ("prefill", "decode"):
        pipelined(kind, args.warmup)
        res[kind] = reduce_max(pipelined(kind, args.steps))
        serial(kind, args.warmup)
        res[kind + "_serial"] = reduce_max(serial(kind, args.steps))
    return dict(value=world * fl["total"] / (res["prefill"] * 1e-3) / 1e12, unit="TFLOP/s",
                h2d_bytes_per_step=h2d["prefill"] + h2d["decode"], d2h_bytes_per_step=d2h["prefill"] + d2h["decode"],
                prefill_ms=res["prefill"], decode_ms=res["decode"],
                decode_gbs=world * by["total"] / (res["decode"] * 1e-3) / 1e9,
                timing="pipelined steps (upload i+1 and download i-1 overlap the kernels of step i); "
                       "span of all steps over K",
                serial=dict(value=world * fl["total"] / (res["prefill_serial"] * 1e-3) / 1e12,
                            prefill_ms=res["prefill_serial"], decode_ms=res["decode_serial"],
                            decode_gbs=world * by["total"] / (res["decode_serial"] * 1e-3) / 1e9))


def time_calls(args, fn, flush):
    """Mean CUDA-event time (ms) of ``fn`` over ``args.steps`` calls after
    ``args.warmup`` untimed ones; L2 flushed (256 MiB write) before each
    timed call, outside its events."""
    for _ in range(args.warmup):
        fn()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for i, e in enumerate(evs):
        flush.fill_(i & 0xff)
        e[0].record()
        fn()
        e[1].record()
    torch.cuda.synchronize()
    mla.mla_check_device_status()
    return statistics.mean(e[0].elapsed_time(e[1]) for e in evs)


def run_configs(args, device, world, reduce_max, peaks, flush):
    """Throughput of the other prefill workloads of the pages' shapes (GLM-5
    B2 T4096 N192 V256, the packed varlen batch 1024/3000/7777/16384 with
    Kimi-K2 heads, and the tiny fp32 case), each timed alone through the
    C-ABI with the prepared kv_b_proj: TFLOP/s over the algorithmic FLOPs,
    tokens/s, and the fraction of the bf16 peak (the fp32 case runs the
    CUDA-core kernels: no tensor-core fraction)."""
    res = {}
    for wl in (W.GLM, W.VARLEN, W.TINY):
        inp = W.prefill_inputs(wl)
        d = {k: v.to(device) for k, v in inp.items()}
        dims = mla.dims_for(wl, mla.mla_softmax_scale(mla.rope_for(wl), wl.qk_head_dim))
        cos, sin = mla.mla_init_rope_tables(mla.rope_for(wl), W.max_position(wl))
        T = sum(wl.seqlens)
        out = torch.empty((T, wl.num_heads, wl.v_head), dtype=wl.torch_dtype, device=device)
        ws = torch.empty(mla.mla_prefill_workspace_size(dims, T, len(wl.seqlens)), dtype=torch.uint8, device=device)
        w_prep = mla.mla_prepare_kv_b_proj(dims, d["w_kvb"])

        def call():
            mla.mla_prefill_prepared(dims, d["latent"], d["q"], w_prep, d["w_norm"], d["positions"],
                                     d["cu_seqlens"], max(wl.seqlens), cos, sin, out=out, workspace=ws)

        ms = reduce_max(time_calls(args, call, flush))
        kev = mla.KernelEvents(16)
        flush.fill_(7)
        with kev:
            call()
        torch.cuda.synchronize()
        fl = prefill_flops(wl)
        tf = world * fl["total"] / (ms * 1e-3) / 1e12
        r = dict(shape="H=%d R=%d N=%d P=%d V=%d seqlens=%s %s" % (wl.num_heads, wl.kv_lora_rank, wl.qk_nope,
                                                                  wl.qk_rope, wl.v_head, list(wl.seqlens),
                                                                  wl.dtype),
                 ms=ms, tflops=tf, tokens_per_s=world * T / (ms * 1e-3), gflop=fl["total"] / 1e9,
                 dispatch=mla.mla_last_dispatch(), kernels_ms=dict(zip(kev.names, kev.durations_ms())))
        if wl.dtype == "bf16":
            r["frac_of_bf16_peak"] = tf / (world * peaks["bf16"])
            att = [t for n, t in r["kernels_ms"].items() if "attention" in n]
            if att:
                r["attention_tflops"] = fl["attn"] / (att[0] * 1e-3) / 1e12
        res[wl.name] = r
        del d, out, ws, w_prep
        torch.cuda.empty_cache()
    return res


def run_chunk(args, din, D, device, world, reduce_max, peaks, n_new=4):
    """Chunks of ``n_new`` new tokens continuing the decode workload's 64
    cached sequences (mla_prefill_cached): the chunk's rows are appended and
    every chunk token attends to its prefix, the chunk tokens before it and
    itself. The prefix rows are the decode cache's rows, copied on the device
    into regions with room for the chunk."""
    lens = [int(x) for x in din["cache_lens"]]
    offs_d = [int(x) for x in din["cache_offsets"]]
    B = len(lens)
    cwl = W.scaled(W.KIMI, seqlens=(n_new,) * B, seed=5, extra=dict(prefix_lens=(0,) * B))
    cin = W.chunk_inputs(cwl)
    dims = mla.dims_for(cwl, mla.mla_softmax_scale(mla.rope_for(cwl), cwl.qk_head_dim))
    max_total = max(lens) + n_new
    cos, sin = mla.mla_init_rope_tables(mla.rope_for(cwl), max_total)
    offs = [0] * B
    for b in range(1, B):
        offs[b] = offs[b - 1] + lens[b - 1] + n_new
    cache = torch.empty((offs[-1] + lens[-1] + n_new, D["cache"].shape[1]), dtype=torch.bfloat16, device=device)
    for b in range(B):
        cache[offs[b]:offs[b] + lens[b]].copy_(D["cache"][offs_d[b]:offs_d[b] + lens[b]])
    C = {k: cin[k].to(device) for k in ("latent", "q", "w_kvb", "w_norm", "cu_seqlens")}
    c_offs = torch.tensor(offs, dtype=torch.int64, device=device)
    c_pre = torch.tensor(lens, dtype=torch.int32, device=device)
    T = B * n_new
    out = torch.empty((T, cwl.num_heads, cwl.v_head), dtype=torch.bfloat16, device=device)
    ws = torch.empty(mla.mla_prefill_cached_workspace_size(dims, T, max_total), dtype=torch.uint8, device=device)

    def call():
        mla.mla_prefill_cached(dims, C["latent"], C["q"], C["w_kvb"], C["w_norm"], C["cu_seqlens"], c_offs, c_pre,
                               max_total, cos, sin, cache, out=out, workspace=ws)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    mla.mla_check_device_status()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for e in evs:
        e[0].record()
        call()
        e[1].record()
    torch.cuda.synchronize()
    kev = mla.KernelEvents(16)
    with kev:
        call()
    torch.cuda.synchronize()
    mla.mla_check_device_status()
    ms = reduce_max(statistics.mean(e[0].elapsed_time(e[1]) for e in evs))
    by = chunk_bytes(cwl, lens, n_new)
    att = world * by["attended"] / (ms * 1e-3) / 1e9
    return dict(workload="64 sequences, cached prefixes = the decode cache lengths, %d new tokens each" % n_new,
                ms=ms, tokens_per_s=world * T / (ms * 1e-3), attended_gbs=att,
                attended_frac_of_hbm=att / (world * peaks["hbm"]),
                unique_cache_gbs=world * by["unique"] / (ms * 1e-3) / 1e9,
                kernels_ms=dict(zip(kev.names, kev.durations_ms())))


def run_chunk_long(args, device, world, reduce_max, peaks, flush, nseq=4, prefix=16384, n_new=2048):
    """Long chunks over long cached prefixes: ``nseq`` sequences of ``prefix``
    cached rows, each continued by ``n_new`` new tokens in one
    mla_prefill_cached call (the library picks the eager form: every cached
    row's keys and values are expanded once by the up-projection GEMM and the
    chunk's queries attend to them causally in absolute positions). FLOPs:
    the up-projection of every key row plus the attention of every chunk token
    to its prefix, the chunk tokens before it and itself."""
    cwl = W.scaled(W.KIMI, kind="prefill", seqlens=(n_new,) * nseq, seed=7,
                   extra=dict(prefix_lens=(prefix,) * nseq))
    cin = W.chunk_inputs(cwl)
    dims = mla.dims_for(cwl, mla.mla_softmax_scale(mla.rope_for(cwl), cwl.qk_head_dim))
    max_total = int(cin["max_total_len"])
    cos, sin = mla.mla_init_rope_tables(mla.rope_for(cwl), max_total)
    C = {k: v.to(device) for k, v in cin.items() if isinstance(v, torch.Tensor)}
    T = nseq * n_new
    out = torch.empty((T, cwl.num_heads, cwl.v_head), dtype=torch.bfloat16, device=device)
    ws = torch.empty(mla.mla_prefill_cached_eager_workspace_size(dims, T, nseq, max_total), dtype=torch.uint8,
                     device=device)

    def call():
        mla.mla_prefill_cached(dims, C["latent"], C["q"], C["w_kvb"], C["w_norm"], C["cu_seqlens"],
                               C["cache_offsets"], C["prefix_lens"], max_total, cos, sin, C["cache"], out=out,
                               workspace=ws)

    ms = reduce_max(time_calls(args, call, flush))
    form = mla.mla_last_dispatch()
    kev = mla.KernelEvents(16)
    with kev:
        call()
    torch.cuda.synchronize()
    mla.mla_check_device_status()
    H, R, N, V = cwl.num_heads, cwl.kv_lora_rank, cwl.qk_nope, cwl.v_head
    D = N + cwl.qk_rope
    keys = nseq * (prefix + n_new)
    pairs = nseq * (n_new * prefix + n_new * (n_new + 1) // 2)
    flops = 2.0 * keys * R * H * (N + V) + 2.0 * pairs * H * (D + V)
    tflops = world * flops / (ms * 1e-3) / 1e12
    unique = keys * (R + cwl.qk_rope) * 2
    return dict(workload="%d sequences of %d cached rows, %d new tokens each" % (nseq, prefix, n_new),
                form=form, ms=ms, tokens_per_s=world * T / (ms * 1e-3), gflop=flops / 1e9, tflops=tflops,
                frac_of_bf16_peak=tflops / (world * peaks["bf16"]),
                unique_cache_gbs=world * unique / (ms * 1e-3) / 1e9,
                kernels_ms=dict(zip(kev.names, kev.durations_ms())))


def run_projections(args, device, world, reduce_max, peaks, n=2048, hidden=7168, q_rank=1536):
    """The projections on either side of the path at the Kimi-K2 prefill size
    (hidden size 7168 and query rank 1536 of the Kimi-K2 model): the joint
    down-projection with the cache append, the query path and o_proj, each
    timed alone with CUDA events; a 256 MiB write before each timed call
    (outside its events) flushes L2."""
    wl = W.KIMI
    inp = W.projection_inputs(wl, n, hidden, q_rank)
    d = {k: v.to(device) for k, v in inp.items()}
    dims = mla.dims_for(wl, mla.mla_softmax_scale(mla.rope_for(wl), wl.qk_head_dim))
    cos, sin = mla.mla_init_rope_tables(mla.rope_for(wl), n)
    H, R, N, P, V = wl.num_heads, wl.kv_lora_rank, wl.qk_nope, wl.qk_rope, wl.v_head
    latent = torch.empty((n, R + P), dtype=torch.bfloat16, device=device)
    cache = torch.empty((n, R + P), dtype=torch.bfloat16, device=device)
    rows = torch.arange(n, dtype=torch.int64, device=device)
    q = torch.empty((n, H, N + P), dtype=torch.bfloat16, device=device)
    q_ws = torch.empty(mla.mla_q_proj_workspace_size(dims, q_rank, n), dtype=torch.uint8, device=device)
    kv_ws = torch.empty(mla.mla_kv_down_append_workspace_size(dims, n), dtype=torch.uint8, device=device)
    out = torch.empty((n, hidden), dtype=torch.bfloat16, device=device)
    calls = dict(
        kv_a_proj_and_append=(lambda: mla.mla_kv_down_append(dims, d["hidden"], d["w_kva"], latent, d["w_norm"],
                                                             d["positions"], cos, sin, cache, rows,
                                                             workspace=kv_ws),
                              2.0 * n * hidden * (R + P)),
        q_proj=(lambda: mla.mla_q_proj(dims, d["hidden"], d["w_qa"], d["w_qnorm"], d["w_qb"], q, q_ws),
                2.0 * n * hidden * q_rank + 2.0 * n * q_rank * H * (N + P)),
        o_proj=(lambda: mla.mla_o_proj(dims, d["attn"], d["w_o"], out), 2.0 * n * H * V * hidden))
    res = dict(workload="Kimi-K2 heads, %d tokens, hidden %d, query rank %d" % (n, hidden, q_rank),
               l2="flushed before each timed call")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    for name, (fn, flops) in calls.items():
        for _ in range(args.warmup):
            fn()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        for i, e in enumerate(evs):
            flush.fill_(i & 0xff)
            e[0].record()
            fn()
            e[1].record()
        torch.cuda.synchronize()
        ms = reduce_max(statistics.mean(e[0].elapsed_time(e[1]) for e in evs))
        tf = world * flops / (ms * 1e-3) / 1e12
        res[name] = dict(ms=ms, tflops=tf, frac_of_bf16_peak=tf / (world * peaks["bf16"]), gflop=flops / 1e9)
    mla.mla_check_device_status()
    return res


def cpu_baseline(budget_s=15.0):
    pin = W.prefill_inputs(W.KIMI)
    v, sample, threads = oracle_prefill_sample(W.KIMI, pin, budget_s)
    return dict(value=v, unit="TFLOP/s", cores=threads, kind="oracle", sample=sample)


def oracle_decode_sample(wl, din, budget_s: float):
    """Time the fp64 absorbed-decode oracle on whole sequences of the decode
    workload until ``budget_s`` is spent; returns (GB/s of algorithmic bytes,
    sample text, seconds spent)."""
    import oracle as O
    rope = O.RopeConfig(**wl.rope)
    shape = O.MlaShape(wl.num_heads, wl.kv_lora_rank, wl.qk_nope, wl.qk_rope, wl.v_head,
                       eps=wl.eps, interleaved=wl.interleaved)
    scale = O.softmax_scale(rope, shape.qk_head_dim)
    cos, sin = O.rope_tables(rope, W.max_position(wl))
    q = din["q"].double().numpy()
    w = din["w_kvb"].double().numpy()
    lens = [int(x) for x in din["cache_lens"]]
    offs = [int(x) for x in din["cache_offsets"]]
    done, t_spent, rows = 0, 0.0, 0
    for b in range(len(lens)):
        if t_spent >= budget_s:
            break
        rows_b = din["cache"][offs[b]:offs[b] + lens[b]].double().numpy()
        t0 = time.perf_counter()
        O.decode_absorbed(q[b:b + 1], rows_b, [0], [lens[b]], din["positions"][b:b + 1].numpy(), w, cos, sin,
                          shape, scale)
        t_spent += time.perf_counter() - t0
        done += 1
        rows += lens[b]
    by = decode_bytes(wl, lens[:done])
    return by["total"] / t_spent / 1e9, "%s: %d of %d sequences (%d cache rows, %.1f s)" % (
        wl.name, done, len(lens), rows, t_spent), t_spent


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle as it stands, on host cores. Each
    step times a bounded sample of the same two workloads: whole heads of the
    Kimi-K2 prefill (about 2 s) and whole sequences of the absorbed decode
    (about 1 s). ``value`` is the prefill's TFLOP/s (the headline metric), the
    ``decode`` object its GB/s, and ``ms_per_step`` the wall time of the
    sample one step runs (not an extrapolation to the full workload)."""
    if rank != 0:
        return None
    pin = W.prefill_inputs(W.KIMI)
    din = W.decode_inputs(W.DECODE)
    vals, dvals, step_s = [], [], []
    sample = dsample = ""
    threads = 1
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        v, sample, threads = oracle_prefill_sample(W.KIMI, pin, budget_s=2.0)
        dv, dsample, _ = oracle_decode_sample(W.DECODE, din, budget_s=1.0)
        if i >= args.warmup:
            vals.append(v)
            dvals.append(dv)
            step_s.append(time.perf_counter() - t0)
    v = statistics.mean(vals)
    return dict(metric=METRIC, value=v, unit="TFLOP/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
                ms_per_step=statistics.mean(step_s) * 1e3, higher_is_better=True, scaling="weak",
                vs_baseline=None, dtype="f64", data="synthetic", impl="reference",
                config=workload_config(world, [int(x) for x in W.decode_cache_lens(W.DECODE)]),
                step="a bounded sample of each workload per step: " + sample + "; " + dsample,
                decode=dict(metric="absorbed decode HBM GB/s (algorithmic bytes)", value=statistics.mean(dvals),
                            unit="GB/s"),
                cpu_baseline=dict(kind="oracle", cores=threads, sample=sample + "; " + dsample, value=v,
                                  unit="TFLOP/s"),
                e2e=dict(value=v, unit="TFLOP/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.cuda.set_device(device)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    res, _ = run_ours(args, rank, world, device)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline()
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
