"""Shared helpers of the GPU parity tests: run the CUDA library and the fp64
oracle on the same seeded inputs and compare with the stated tolerances.

Tolerances: fp32 runs max-abs <= 1e-4; bf16 runs rel-L2 <= 5e-3 and
max-abs <= 2e-2 (on the evaluated elements).
"""

import json
import os

import numpy as np
import torch

import oracle as O
from decode_latent_rmsnorm_b200 import mla
from decode_latent_rmsnorm_b200 import workloads as W

FP32_MAX_ABS = 1e-4
BF16_REL_L2 = 5e-3
BF16_MAX_ABS = 2e-2


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def oracle_cfg(wl):
    rope = O.RopeConfig(**wl.rope)
    shape = O.MlaShape(wl.num_heads, wl.kv_lora_rank, wl.qk_nope, wl.qk_rope, wl.v_head,
                       eps=wl.eps, interleaved=wl.interleaved)
    return rope, shape, O.softmax_scale(rope, shape.qk_head_dim)


def compare(got, ref, dtype, what=""):
    """Compare on the entries the oracle evaluated (non-NaN); returns metrics."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    sel = ~np.isnan(ref)
    assert sel.any(), "nothing evaluated"
    g, r = got[sel], ref[sel]
    assert np.isfinite(g).all(), "%s: non-finite output" % what
    err = g - r
    max_abs = float(np.abs(err).max())
    rel_l2 = float(np.linalg.norm(err) / max(np.linalg.norm(r), 1e-300))
    m = dict(max_abs=max_abs, rel_l2=rel_l2, n=int(sel.sum()))
    log = os.environ.get("MLA_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps(dict(what=what, dtype=dtype, **m)) + "\n")
    if dtype == "fp32":
        assert max_abs <= FP32_MAX_ABS, "%s fp32 %s" % (what, m)
    else:
        assert rel_l2 <= BF16_REL_L2 and max_abs <= BF16_MAX_ABS, "%s bf16 %s" % (what, m)
    return m


def gpu_tables(wl, max_pos):
    return mla.mla_init_rope_tables(mla.rope_for(wl), max_pos)


def run_prefill(wl, inp, max_pos=None):
    dev = "cuda"
    rope, shape, scale = oracle_cfg(wl)
    dims = mla.dims_for(wl, mla.mla_softmax_scale(mla.rope_for(wl), shape.qk_head_dim))
    max_pos = max_pos or W.max_position(wl)
    cos, sin = gpu_tables(wl, max_pos)
    d = {k: v.to(dev) for k, v in inp.items()}
    max_len = int(max(wl.seqlens)) if wl.seqlens else 0
    out = mla.mla_prefill(dims, d["latent"], d["q"], d["w_kvb"], d["w_norm"], d["positions"],
                          d["cu_seqlens"], max_len, cos, sin)
    torch.cuda.synchronize()
    mla.mla_check_device_status()
    return out


def oracle_prefill(wl, inp, heads=None, rows=None):
    rope, shape, scale = oracle_cfg(wl)
    cos, sin = O.rope_tables(rope, W.max_position(wl))
    return O.prefill(f64(inp["latent"]), f64(inp["q"]), f64(inp["w_kvb"]), f64(inp["w_norm"]),
                     inp["positions"].numpy(), inp["cu_seqlens"].numpy(), cos, sin, shape, scale,
                     heads=heads, rows=rows)


def run_decode(wl, inp, max_pos=None):
    dev = "cuda"
    rope, shape, scale = oracle_cfg(wl)
    dims = mla.dims_for(wl, mla.mla_softmax_scale(mla.rope_for(wl), shape.qk_head_dim))
    max_pos = max_pos or W.max_position(wl)
    cos, sin = gpu_tables(wl, max_pos)
    d = {k: v.to(dev) for k, v in inp.items()}
    out = mla.mla_decode(dims, d["q"], d["cache"], d["cache_offsets"], d["cache_lens"],
                         d["positions"], int(inp["cache_lens"].max()), d["w_kvb"], cos, sin)
    torch.cuda.synchronize()
    mla.mla_check_device_status()
    return out


def oracle_decode(wl, inp, batches, heads=None, absorbed=False):
    """Per sampled sequence, on that sequence's own slice of the cache."""
    rope, shape, scale = oracle_cfg(wl)
    cos, sin = O.rope_tables(rope, W.max_position(wl))
    B, H = inp["q"].shape[0], wl.num_heads
    out = np.full((B, H, wl.v_head), np.nan)
    fn = O.decode_absorbed if absorbed else O.decode_eager
    q = f64(inp["q"])
    w = f64(inp["w_kvb"])
    for b in batches:
        o, n = int(inp["cache_offsets"][b]), int(inp["cache_lens"][b])
        rows = f64(inp["cache"][o:o + n])
        res = fn(q[b:b + 1], rows, np.array([0]), np.array([n]), inp["positions"][b:b + 1].numpy(),
                 w, cos, sin, shape, scale, heads=heads)
        out[b] = res[0]
    return out


def run_prefill_cached(wl, inp):
    """The chunk call on the GPU; returns (out, cache after the call)."""
    rope, shape, scale = oracle_cfg(wl)
    dims = mla.dims_for(wl, mla.mla_softmax_scale(mla.rope_for(wl), shape.qk_head_dim))
    cos, sin = gpu_tables(wl, inp["max_total_len"])
    d = {k: v.to("cuda") for k, v in inp.items() if isinstance(v, torch.Tensor)}
    out = mla.mla_prefill_cached(dims, d["latent"], d["q"], d["w_kvb"], d["w_norm"], d["cu_seqlens"],
                                 d["cache_offsets"], d["prefix_lens"], inp["max_total_len"], cos, sin, d["cache"])
    torch.cuda.synchronize()
    return out, d["cache"]


def oracle_prefill_cached(wl, inp, heads=None):
    rope, shape, scale = oracle_cfg(wl)
    cos, sin = O.rope_tables(rope, inp["max_total_len"])
    return O.prefill_cached(f64(inp["latent"]), f64(inp["q"]), f64(inp["cache"]), inp["cache_offsets"].numpy(),
                            inp["prefix_lens"].numpy(), inp["cu_seqlens"].numpy(), f64(inp["w_kvb"]),
                            f64(inp["w_norm"]), cos, sin, shape, scale, heads=heads)
