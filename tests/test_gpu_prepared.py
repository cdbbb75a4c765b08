"""GPU checks of the prefill with a prepared kv_b_proj, of the dispatch
report, and of repeated calls on one workspace (the persistent attention
kernel's work counter is reset by every call).

mla_prefill_prepared runs the same kernels on the same fp16 weight copy as
mla_prefill, so the two must agree bit for bit; both are also compared with
the fp64 oracle at the bf16 tolerance.
"""

import numpy as np
import pytest
import torch

from decode_latent_rmsnorm_b200 import mla
from decode_latent_rmsnorm_b200 import workloads as W
from _parity import compare, f64, gpu_tables, oracle_cfg, oracle_prefill

pytestmark = pytest.mark.gpu


def _setup(wl, inp):
    rope, shape, scale = oracle_cfg(wl)
    dims = mla.dims_for(wl, mla.mla_softmax_scale(mla.rope_for(wl), shape.qk_head_dim))
    cos, sin = gpu_tables(wl, W.max_position(wl))
    d = {k: v.to("cuda") for k, v in inp.items()}
    return dims, cos, sin, d


@pytest.mark.parametrize("wl", [W.scaled(W.KIMI, seqlens=(129, 1, 300), seed=41),
                                W.scaled(W.KIMI, seqlens=(0, 513, 255), seed=42),
                                W.scaled(W.GLM, seqlens=(300, 129), seed=43),
                                W.TINY], ids=["kimi_ragged", "kimi_empty_first", "glm", "tiny_fp32"])
def test_prepared_equals_unprepared(gpu_lib, wl):
    inp = W.prefill_inputs(wl)
    dims, cos, sin, d = _setup(wl, inp)
    L = max(wl.seqlens)
    ref = mla.mla_prefill(dims, d["latent"], d["q"], d["w_kvb"], d["w_norm"], d["positions"],
                          d["cu_seqlens"], L, cos, sin)
    prep = mla.mla_prepare_kv_b_proj(dims, d["w_kvb"])
    got = mla.mla_prefill_prepared(dims, d["latent"], d["q"], prep, d["w_norm"], d["positions"],
                                   d["cu_seqlens"], L, cos, sin)
    torch.cuda.synchronize()
    mla.mla_check_device_status()
    assert torch.equal(got, ref)
    compare(f64(got), oracle_prefill(wl, inp), wl.dtype, "prepared " + wl.name)


def test_prepared_size_and_errors(gpu_lib):
    wl = W.scaled(W.KIMI, seqlens=(64,), seed=44)
    inp = W.prefill_inputs(wl)
    dims, cos, sin, d = _setup(wl, inp)
    n = mla.mla_kv_b_proj_prepared_size(dims)
    assert n == 2 * 64 * 256 * 512            # fp16 [H (N + V), R]
    small = torch.empty(n - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(mla.MlaError) as e:
        mla.mla_prepare_kv_b_proj(dims, d["w_kvb"], small)
    assert e.value.status == 3
    # a weight beyond the fp16 range is flagged on the device
    w_big = d["w_kvb"].clone()
    w_big[5, 7] = 1.0e6
    mla.mla_prepare_kv_b_proj(dims, w_big)
    with pytest.raises(mla.MlaError) as e:
        mla.mla_check_device_status()
    assert e.value.status == 1
    mla.mla_check_device_status()             # the word was cleared


def test_dispatch_report(gpu_lib):
    wl = W.scaled(W.KIMI, seqlens=(200,), seed=45)
    inp = W.prefill_inputs(wl)
    dims, cos, sin, d = _setup(wl, inp)
    mla.mla_prefill(dims, d["latent"], d["q"], d["w_kvb"], d["w_norm"], d["positions"], d["cu_seqlens"], 200,
                    cos, sin)
    assert mla.mla_last_dispatch() == "tensor-core"
    # a q view that starts 2 bytes into its buffer is not 16-byte aligned
    qbuf = torch.empty(d["q"].numel() + 8, dtype=d["q"].dtype, device="cuda")
    q_off = qbuf[1:1 + d["q"].numel()].view(d["q"].shape)
    q_off.copy_(d["q"])
    out = mla.mla_prefill(dims, d["latent"], q_off, d["w_kvb"], d["w_norm"], d["positions"], d["cu_seqlens"],
                          200, cos, sin)
    assert mla.mla_last_dispatch().startswith("simt:") and "aligned" in mla.mla_last_dispatch()
    torch.cuda.synchronize()
    mla.mla_check_device_status()
    compare(f64(out), oracle_prefill(wl, inp), "bf16", "unaligned q (CUDA-core kernels)")
    tiny = W.prefill_inputs(W.TINY)
    dims_t, cos_t, sin_t, dt = _setup(W.TINY, tiny)
    mla.mla_prefill(dims_t, dt["latent"], dt["q"], dt["w_kvb"], dt["w_norm"], dt["positions"],
                    dt["cu_seqlens"], 32, cos_t, sin_t)
    assert mla.mla_last_dispatch().startswith("simt:")


def test_repeated_calls_one_workspace(gpu_lib):
    # the attention's work counter lives in the workspace: each call resets it
    wl = W.scaled(W.KIMI, seqlens=(700, 1, 1300), seed=46)
    inp = W.prefill_inputs(wl)
    dims, cos, sin, d = _setup(wl, inp)
    T = int(sum(wl.seqlens))
    ws = torch.empty(mla.mla_prefill_workspace_size(dims, T, len(wl.seqlens)), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        outs.append(mla.mla_prefill(dims, d["latent"], d["q"], d["w_kvb"], d["w_norm"], d["positions"],
                                    d["cu_seqlens"], max(wl.seqlens), cos, sin, workspace=ws))
    torch.cuda.synchronize()
    mla.mla_check_device_status()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    compare(f64(outs[2]), oracle_prefill(wl, inp), "bf16", "repeated calls")
