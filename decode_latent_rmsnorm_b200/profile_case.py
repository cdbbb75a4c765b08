"""Run one workload of the MLA path a few times, for a profiler to capture.

    python -m decode_latent_rmsnorm_b200.profile_case --case decode --reps 4

Cases: ``kimi_prefill`` (B=1 T=2048 H=64, YaRN), ``glm_prefill`` (B=2 T=4096,
N=192 V=256), ``decode`` (B=64 absorbed decode over latent caches of lengths
uniform in [1000, 32768]), ``all`` (Kimi prefill then decode). Inputs are the
seeded synthetic workloads; every call goes through the C-ABI library.
The last line printed is the mean device time of the calls after the first.
"""

from __future__ import annotations

import argparse
import statistics

import torch

from . import mla
from . import workloads as W


def _prefill_call(wl, device):
    inp = {k: v.to(device) for k, v in W.prefill_inputs(wl).items()}
    rope = mla.rope_for(wl)
    dims = mla.dims_for(wl, mla.mla_softmax_scale(rope, wl.qk_head_dim))
    cos, sin = mla.mla_init_rope_tables(rope, W.max_position(wl))
    T = sum(wl.seqlens)
    out = torch.empty((T, wl.num_heads, wl.v_head), dtype=torch.bfloat16, device=device)
    ws = torch.empty(mla.mla_prefill_workspace_size(dims, T, len(wl.seqlens)), dtype=torch.uint8,
                     device=device)

    def call():
        mla.mla_prefill(dims, inp["latent"], inp["q"], inp["w_kvb"], inp["w_norm"], inp["positions"],
                        inp["cu_seqlens"], max(wl.seqlens), cos, sin, out=out, workspace=ws)
    return call


def _decode_call(wl, device):
    inp = {k: v.to(device) for k, v in W.decode_inputs(wl).items()}
    rope = mla.rope_for(wl)
    dims = mla.dims_for(wl, mla.mla_softmax_scale(rope, wl.qk_head_dim))
    cos, sin = mla.mla_init_rope_tables(rope, W.max_position(wl))
    B = wl.batch
    max_len = int(inp["cache_lens"].max())
    out = torch.empty((B, wl.num_heads, wl.v_head), dtype=torch.bfloat16, device=device)
    ws = torch.empty(mla.mla_decode_workspace_size(dims, B, max_len), dtype=torch.uint8, device=device)

    def call():
        mla.mla_decode(dims, inp["q"], inp["cache"], inp["cache_offsets"], inp["cache_lens"],
                       inp["positions"], max_len, inp["w_kvb"], cos, sin, out=out, workspace=ws)
    return call


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", default="all", choices=["kimi_prefill", "glm_prefill", "decode", "all"])
    ap.add_argument("--reps", type=int, default=4)
    args = ap.parse_args()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    calls = []
    if args.case in ("kimi_prefill", "all"):
        calls.append(_prefill_call(W.KIMI, device))
    if args.case == "glm_prefill":
        calls.append(_prefill_call(W.GLM, device))
    if args.case in ("decode", "all"):
        calls.append(_decode_call(W.DECODE, device))
    times = []
    for _ in range(max(args.reps, 1)):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for c in calls:
            c()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    mla.mla_check_device_status()
    rest = times[1:] or times
    print("case=%s reps=%d mean_ms=%.4f" % (args.case, len(times), statistics.mean(rest)))


if __name__ == "__main__":
    main()
