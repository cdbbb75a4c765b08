"""The seeded input recipe (decode_latent_rmsnorm_b200/workloads.py) and the
recorded profiler figures (profiles/traffic.json), checked on the CPU."""

import json
import os

import pytest
import torch

from decode_latent_rmsnorm_b200 import workloads as W
from decode_latent_rmsnorm_b200.kernel_sources import KERNEL_SOURCES

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_inputs_are_reproducible_and_seed_dependent():
    a, b = W.prefill_inputs(W.TINY), W.prefill_inputs(W.TINY)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    c = W.prefill_inputs(W.scaled(W.TINY, seed=99))
    assert not torch.equal(a["latent"], c["latent"])


def test_prefill_recipe_shapes_and_distributions():
    wl = W.KIMI
    inp = W.prefill_inputs(wl)
    T = 2048
    assert inp["latent"].shape == (T, 576) and inp["latent"].dtype == torch.bfloat16
    assert inp["q"].shape == (T, 64, 192)
    assert inp["w_kvb"].shape == (64 * 256, 512)
    assert inp["positions"].tolist() == list(range(T))
    assert inp["cu_seqlens"].tolist() == [0, T]
    lat = inp["latent"].float()
    assert abs(lat.mean().item()) < 0.01 and abs(lat.std().item() - 1.0) < 0.01
    w = inp["w_kvb"].float()
    assert abs(w.std().item() - (1.0 / 512) ** 0.5) < 0.001
    wn = inp["w_norm"].float()
    assert abs(wn.mean().item() - 1.0) < 0.02 and abs(wn.std().item() - 0.1) < 0.02


def test_varlen_positions_restart_per_sequence():
    inp = W.prefill_inputs(W.scaled(W.VARLEN, seqlens=(3, 5)))
    assert inp["positions"].tolist() == [0, 1, 2, 0, 1, 2, 3, 4]
    assert inp["cu_seqlens"].tolist() == [0, 3, 8]


def test_decode_recipe():
    lens = W.decode_cache_lens(W.DECODE)
    assert lens.numel() == 64 and int(lens.min()) >= 1000 and int(lens.max()) <= 32768
    assert int(lens.sum()) == 1120176
    small = W.scaled(W.DECODE, batch=3, cache_lens=(5, 1, 7))
    inp = W.decode_inputs(small)
    assert inp["cache"].shape == (13, 576)
    assert inp["cache_offsets"].tolist() == [0, 5, 6]
    assert inp["positions"].tolist() == [5, 1, 7]          # the new token sits after its cache


def test_chunk_recipe_regions():
    wl = W.scaled(W.KIMI, seqlens=(2, 0, 3), extra=dict(prefix_lens=(4, 1, 0)))
    inp = W.chunk_inputs(wl, gap=2)
    assert inp["cache_offsets"].tolist() == [0, 8, 11]      # prefix + chunk + gap per region
    assert inp["cu_seqlens"].tolist() == [0, 2, 2, 5]
    assert inp["max_total_len"] == 6
    c = inp["cache"]
    assert c.shape == (16, 576)
    assert torch.all(c[4:8] == 0) and torch.any(c[0:4] != 0)   # chunk rows and the gap start at zero


def test_recorded_traffic_is_well_formed():
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for kernel, r in rec.items():
        if kernel.startswith("_"):
            continue
        assert kernel in KERNEL_SOURCES, kernel
        assert r["dram_bytes_per_launch"] == r["dram_read_bytes"] + r["dram_write_bytes"]
        assert len(r["source_digest"]) == 64
        assert os.path.exists(os.path.join(ROOT, r["summary"])), r["summary"]


@pytest.mark.parametrize("kernel", sorted(KERNEL_SOURCES))
def test_kernel_source_lists_exist(kernel):
    for name in KERNEL_SOURCES[kernel]:
        assert os.path.exists(os.path.join(ROOT, "decode_latent_rmsnorm_b200", "csrc", name)), name
