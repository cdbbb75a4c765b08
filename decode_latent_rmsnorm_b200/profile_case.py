"""Run one workload of the MLA path a few times, for a profiler to capture.

    python -m decode_latent_rmsnorm_b200.profile_case --case decode --reps 4

Cases: ``kimi_prefill`` (B=1 T=2048 H=64, YaRN), ``glm_prefill`` (B=2 T=4096,
N=192 V=256), ``varlen_prefill`` (Kimi-K2 heads, sequences 1024/3000/7777/16384
packed), ``decode`` (B=64 absorbed decode over latent caches of lengths
uniform in [1000, 32768]), ``chunk`` (4 new tokens on each of 64 cached
sequences of 16384 rows, about 1.2 GB of cache), ``chunk_eager`` (2048 new
tokens on each of 2 cached sequences of 16384 rows, the eager form),
``projections`` (the joint
down-projection with the cache append, the query path and o_proj at 2048
tokens, hidden size 7168, query rank 1536), ``all`` (Kimi prefill then
decode). Inputs are the seeded synthetic workloads; every call goes through
the C-ABI library.
The prefills run with kv_b_proj prepared once (mla_prefill_prepared), as
the bench times them. The last line printed is the mean device time of the
calls after the first.
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
    w_prep = mla.mla_prepare_kv_b_proj(dims, inp["w_kvb"])

    def call():
        mla.mla_prefill_prepared(dims, inp["latent"], inp["q"], w_prep, inp["w_norm"], inp["positions"],
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


def _chunk_call(device, n_new=4, prefix=16384, batch=64, eager=False):
    wl = W.scaled(W.KIMI, seqlens=(n_new,) * batch, seed=5, extra=dict(prefix_lens=(prefix,) * batch))
    inp = W.chunk_inputs(wl)
    d = {k: v.to(device) for k, v in inp.items() if isinstance(v, torch.Tensor)}
    rope = mla.rope_for(wl)
    dims = mla.dims_for(wl, mla.mla_softmax_scale(rope, wl.qk_head_dim))
    cos, sin = mla.mla_init_rope_tables(rope, inp["max_total_len"])
    T = n_new * batch
    out = torch.empty((T, wl.num_heads, wl.v_head), dtype=torch.bfloat16, device=device)
    need = mla.mla_prefill_cached_workspace_size(dims, T, inp["max_total_len"])
    if eager:
        need = max(need, mla.mla_prefill_cached_eager_workspace_size(dims, T, batch, inp["max_total_len"]))
    ws = torch.empty(need, dtype=torch.uint8, device=device)

    def call():
        mla.mla_prefill_cached(dims, d["latent"], d["q"], d["w_kvb"], d["w_norm"], d["cu_seqlens"],
                               d["cache_offsets"], d["prefix_lens"], inp["max_total_len"], cos, sin, d["cache"],
                               out=out, workspace=ws)
    return call


def _projection_call(device, n=2048, hidden=7168, q_rank=1536):
    wl = W.KIMI
    d = {k: v.to(device) for k, v in W.projection_inputs(wl, n, hidden, q_rank).items()}
    rope = mla.rope_for(wl)
    dims = mla.dims_for(wl, mla.mla_softmax_scale(rope, wl.qk_head_dim))
    cos, sin = mla.mla_init_rope_tables(rope, n)
    latent = torch.empty((n, wl.kv_lora_rank + wl.qk_rope), dtype=torch.bfloat16, device=device)
    cache = torch.empty_like(latent)
    rows = torch.arange(n, dtype=torch.int64, device=device)
    q = torch.empty((n, wl.num_heads, wl.qk_head_dim), dtype=torch.bfloat16, device=device)
    q_ws = torch.empty(mla.mla_q_proj_workspace_size(dims, q_rank, n), dtype=torch.uint8, device=device)
    kv_ws = torch.empty(mla.mla_kv_down_append_workspace_size(dims, n), dtype=torch.uint8, device=device)
    out = torch.empty((n, hidden), dtype=torch.bfloat16, device=device)

    def call():
        mla.mla_kv_down_append(dims, d["hidden"], d["w_kva"], latent, d["w_norm"], d["positions"], cos, sin,
                               cache, rows, workspace=kv_ws)
        mla.mla_q_proj(dims, d["hidden"], d["w_qa"], d["w_qnorm"], d["w_qb"], q, q_ws)
        mla.mla_o_proj(dims, d["attn"], d["w_o"], out)
    return call


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", default="all",
                    choices=["kimi_prefill", "glm_prefill", "varlen_prefill", "decode", "chunk", "chunk_eager",
                             "projections", "all"])
    ap.add_argument("--reps", type=int, default=4)
    args = ap.parse_args()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    calls = []
    if args.case in ("kimi_prefill", "all"):
        calls.append(_prefill_call(W.KIMI, device))
    if args.case == "glm_prefill":
        calls.append(_prefill_call(W.GLM, device))
    if args.case == "varlen_prefill":
        calls.append(_prefill_call(W.VARLEN, device))
    if args.case in ("decode", "all"):
        calls.append(_decode_call(W.DECODE, device))
    if args.case == "chunk":
        calls.append(_chunk_call(device))
    if args.case == "chunk_eager":
        calls.append(_chunk_call(device, n_new=2048, prefix=16384, batch=2, eager=True))
    if args.case == "projections":
        calls.append(_projection_call(device))
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
