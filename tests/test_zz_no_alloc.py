"""The prefill entry point that allocates nothing (mla_prefill_noalloc).

Some callers cannot allocate device memory: a plugin running inside an
application whose framework already holds the GPU's memory in its own
caching allocator, or a latency-bound loop that must not call cudaMalloc
(which can wait for the whole device to go idle). For them the library
offers mla_prefill_noalloc, whose scratch is a static array inside the
library. This file checks, through the C-ABI, that it returns what
mla_prefill returns with a caller-provided workspace, on two calls in a row
(the second must not see stale state from the first), and that a call too
large for the static scratch is refused before anything is launched.

The file name makes pytest collect it last.
"""

import ctypes

import numpy as np
import pytest
import torch

from decode_latent_rmsnorm_b200 import mla
from decode_latent_rmsnorm_b200 import workloads as W
from _parity import compare, f64

pytestmark = pytest.mark.gpu


def _inputs(seqlens, seed):
    wl = W.scaled(W.KIMI, seqlens=seqlens, seed=seed)
    inp = {k: v.cuda() for k, v in W.prefill_inputs(wl).items()}
    dims = mla.dims_for(wl, mla.mla_softmax_scale(mla.rope_for(wl), wl.qk_head_dim))
    cos, sin = mla.mla_init_rope_tables(mla.rope_for(wl), W.max_position(wl))
    return wl, inp, dims, cos, sin


def test_noalloc_prefill_matches_workspace_prefill(gpu_lib):
    from _parity import oracle_prefill
    # the device error word must be clean before the first no-alloc call, so
    # that an error left by an earlier test is not blamed on this path
    mla.mla_check_device_status()
    for seqlens, seed in (((200,), 41), ((60, 50), 42)):
        wl, d, dims, cos, sin = _inputs(seqlens, seed)
        T = sum(seqlens)
        assert mla.mla_prefill_workspace_size(dims, T, len(seqlens)) <= mla.NOALLOC_SCRATCH_BYTES
        out = torch.full((T, wl.num_heads, wl.v_head), float("nan"), dtype=torch.bfloat16, device="cuda")
        mla.mla_prefill_noalloc(dims, d["latent"], d["q"], d["w_kvb"], d["w_norm"], d["positions"],
                                d["cu_seqlens"], max(seqlens), cos, sin, out)
        torch.cuda.synchronize()
        mla.mla_check_device_status()
        # a fresh workspace prefill after the no-alloc call: the same kernels on
        # the same inputs give the same bits, so stale scratch left by the
        # previous call (the first loop pass) would show as a difference here
        ref = mla.mla_prefill(dims, d["latent"], d["q"], d["w_kvb"], d["w_norm"], d["positions"],
                              d["cu_seqlens"], max(seqlens), cos, sin)
        torch.cuda.synchronize()
        mla.mla_check_device_status()
        assert torch.equal(out, ref), "no-alloc prefill differs from the workspace prefill (%s)" % (seqlens,)
        cpu = {k: v.cpu() for k, v in d.items()}
        compare(f64(out), oracle_prefill(wl, cpu), "bf16", "noalloc vs oracle")


def test_noalloc_prefill_rejects_oversized_work(gpu_lib):
    wl, d, dims, cos, sin = _inputs((200,), 43)
    T = 4096   # needs more scratch than the static array holds
    assert mla.mla_prefill_workspace_size(dims, T, 1) > mla.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x1000)
    lib = mla.load()
    rc = lib.mla_prefill_noalloc(ctypes.byref(dims), fake, fake, fake, fake, fake, fake, 1, T, T, fake, fake,
                                 T, fake, None)
    assert rc == 3
    assert "static scratch" in mla.mla_last_error_string()
