"""The algorithmic work the bench divides by (the numerators of its rates and
of the roofline), checked against independent counts."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from decode_latent_rmsnorm_b200 import workloads as W  # noqa: E402


def test_prefill_flops_of_the_kimi_workload():
    fl = bench.prefill_flops(W.KIMI)
    # up-projection: 2 T R H (N + V); attention: 2 H (D + V) per unmasked pair
    assert fl["up"] == 2 * 2048 * 512 * 64 * 256
    assert fl["attn"] == 2 * 64 * (192 + 128) * (2048 * 2049 // 2)
    assert fl["total"] / 1e9 == pytest.approx(120.30, abs=0.01)


def test_causal_pairs_counted_by_loops():
    wl = W.scaled(W.KIMI, seqlens=(1, 5, 0, 17))
    pairs = sum(1 for L in wl.seqlens for i in range(L) for j in range(L) if j <= i)
    assert bench.prefill_flops(wl)["attn"] == 2 * 64 * 320 * pairs


def test_decode_bytes_of_the_decode_workload():
    lens = [int(x) for x in W.decode_cache_lens(W.DECODE)]
    by = bench.decode_bytes(W.DECODE, lens)
    assert sum(lens) == 1120176
    assert by["cache"] == 1120176 * 576 * 2
    assert by["weight"] == 64 * 256 * 512 * 2
    assert by["io"] == 64 * 64 * 192 * 2 + 64 * 64 * 128 * 2
    assert by["total"] / 1e9 == pytest.approx(1.3098, abs=1e-4)


def test_chunk_rows_counted_by_loops():
    prefix, n = [0, 3, 10], 4
    attended = sum(p + i + 1 for p in prefix for i in range(n))
    unique = sum(p + n for p in prefix)
    by = bench.chunk_bytes(W.KIMI, prefix, n)
    assert by["attended"] == attended * 576 * 2
    assert by["unique"] == unique * 576 * 2


def test_job_rate_is_all_ranks_work_over_the_slowest():
    assert bench.job_throughput(5.0, 4, 2.0) == pytest.approx(4 * 5.0 / 2e-3)
