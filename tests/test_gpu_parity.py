"""GPU parity: the CUDA library against the fp64 oracle on seeded inputs.

Small cases compare every element; the full-size workloads compare every
element the oracle evaluates (all of the Kimi-K2 prefill; sampled heads and
rows elsewhere). All calls go through the C-ABI via the ctypes binding.
"""

import numpy as np
import pytest
import torch

import oracle as O
from decode_latent_rmsnorm_b200 import mla
from decode_latent_rmsnorm_b200 import workloads as W
from _parity import (compare, f64, oracle_cfg, oracle_decode, oracle_prefill,
                     oracle_prefill_cached, run_decode, run_prefill, run_prefill_cached)

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------- rotary tables

@pytest.mark.parametrize("wl", [W.TINY, W.KIMI, W.GLM], ids=lambda w: w.name)
def test_rope_tables_match_oracle(gpu_lib, wl):
    rope, shape, _ = oracle_cfg(wl)
    max_pos = 40000
    cos, sin = mla.mla_init_rope_tables(mla.rope_for(wl), max_pos)
    rc, rs = O.rope_tables(rope, max_pos)
    m = O.rope_table_mscale(rope)
    assert np.abs(f64(cos) - rc).max() <= 1e-7 * m
    assert np.abs(f64(sin) - rs).max() <= 1e-7 * m


def test_rope_tables_yarn_mscale_ratio(gpu_lib):
    # mscale != mscale_all_dim: tables carry get_mscale(f, m) / get_mscale(f, m_all)
    rope = O.RopeConfig(rope_dim=64, base=50000.0, yarn=True, factor=32.0, mscale=0.707,
                        mscale_all_dim=0.0)
    cfg = mla.RopeCfg.make(64, 50000.0, yarn=True, factor=32.0, mscale=0.707, mscale_all_dim=0.0)
    cos, sin = mla.mla_init_rope_tables(cfg, 5000)
    rc, rs = O.rope_tables(rope, 5000)
    assert np.abs(f64(cos) - rc).max() <= 2e-7 and np.abs(f64(sin) - rs).max() <= 2e-7


# ---------------------------------------------------------------- prefill

def test_prefill_tiny_fp32(gpu_lib):
    inp = W.prefill_inputs(W.TINY)
    got = run_prefill(W.TINY, inp)
    compare(f64(got), oracle_prefill(W.TINY, inp), "fp32", "tiny")


@pytest.mark.parametrize("seqlens", [(1,), (127,), (129, 1, 300), (0, 200, 0, 77, 0)],
                         ids=lambda s: "x".join(map(str, s)))
def test_prefill_kimi_heads_ragged(gpu_lib, seqlens):
    wl = W.scaled(W.KIMI, seqlens=seqlens, seed=11)
    inp = W.prefill_inputs(wl)
    got = run_prefill(wl, inp)
    compare(f64(got), oracle_prefill(wl, inp), "bf16", "kimi ragged")


def test_prefill_glm_heads_small(gpu_lib):
    wl = W.scaled(W.GLM, seqlens=(300, 129), seed=12)
    inp = W.prefill_inputs(wl)
    got = run_prefill(wl, inp)
    compare(f64(got), oracle_prefill(wl, inp), "bf16", "glm small")


@pytest.mark.parametrize("nv", [(64, 64), (64, 128), (128, 64), (64, 192)], ids=lambda nv: "N%dV%d" % nv)
def test_prefill_bf16_other_head_geometry(gpu_lib, nv):
    # tensor-core geometries unlike the configs: 4 heads, rank 256, ragged lengths
    N, V = nv
    wl = W.Workload("geom_bf16", "prefill", 4, 256, N, 64, V, "bf16", W.KIMI_ROPE, 31 + N + V,
                    seqlens=(300, 129, 520, 1))
    inp = W.prefill_inputs(wl)
    got = run_prefill(wl, inp)
    compare(f64(got), oracle_prefill(wl, inp), "bf16", "geometry N%d V%d" % nv)


def test_prefill_fp32_other_geometry(gpu_lib):
    # fp32, half-split pairs, a geometry unlike the configs (H=3, N=32, P=16, V=24)
    wl = W.Workload("odd_fp32", "prefill", 3, 128, 32, 16, 24, "fp32", dict(W.KIMI_ROPE, rope_dim=16),
                    21, seqlens=(70, 33))
    inp = W.prefill_inputs(wl)
    got = run_prefill(wl, inp)
    compare(f64(got), oracle_prefill(wl, inp), "fp32", "odd fp32")


def test_prefill_kimi_full(gpu_lib):
    inp = W.prefill_inputs(W.KIMI)
    got = run_prefill(W.KIMI, inp)
    compare(f64(got), oracle_prefill(W.KIMI, inp), "bf16", "kimi full")


def test_prefill_glm_full_sampled_heads(gpu_lib):
    inp = W.prefill_inputs(W.GLM)
    got = run_prefill(W.GLM, inp)
    compare(f64(got), oracle_prefill(W.GLM, inp, heads=[0, 1, 31, 63]), "bf16", "glm full")


def _varlen_rows(seqlens, seed=0):
    """Sampled query rows of long sequences: first/last 32, rows around every
    128-row tile boundary, and seeded random rows (256 in all)."""
    rng = np.random.default_rng(seed)
    rows = {}
    for s, L in enumerate(seqlens):
        if L <= 4096:
            continue
        pick = set(range(32)) | set(range(L - 32, L))
        for t in range(128, L, 128 * 16):
            pick |= {t - 1, t}
        while len(pick) < 256:
            pick.add(int(rng.integers(0, L)))
        rows[s] = np.array(sorted(pick))
    return rows


def test_prefill_varlen_sampled(gpu_lib):
    wl = W.VARLEN
    inp = W.prefill_inputs(wl)
    got = run_prefill(wl, inp)
    ref = oracle_prefill(wl, inp, heads=[0, 1, 31, 63], rows=_varlen_rows(wl.seqlens))
    compare(f64(got), ref, "bf16", "varlen")


def test_prefill_longest_sampled(gpu_lib):
    """One sequence of 32 768 tokens (the longest length the configs use):
    256 key steps for the last query block, 128 blocks x 64 heads = 8192 work
    items for the persistent attention. Sampled rows (both ends, around tile
    edges, random) of the first and last head."""
    wl = W.scaled(W.KIMI, seqlens=(32768,), seed=29)
    inp = W.prefill_inputs(wl)
    got = run_prefill(wl, inp)
    assert mla.mla_last_dispatch().startswith("tensor-core"), mla.mla_last_dispatch()
    ref = oracle_prefill(wl, inp, heads=[0, 63], rows=_varlen_rows(wl.seqlens, seed=5))
    compare(f64(got), ref, "bf16", "prefill 32768")


def test_prefill_many_short_sequences(gpu_lib):
    """240 sequences whose lengths sit on and around the 128- and 256-row
    tile edges (1, 2, 127, 128, 129, 255, 256, 257 in turn): single-tile query
    blocks alternate with two-tile ones, so consecutive work items of the
    persistent attention change sequence, tile count and key-step count at
    nearly every claim. Every row of three heads is compared."""
    base = (1, 2, 127, 128, 129, 255, 256, 257)
    wl = W.scaled(W.KIMI, seqlens=tuple(base[(5 * i) % 8] for i in range(240)), seed=23)
    inp = W.prefill_inputs(wl)
    got = run_prefill(wl, inp)
    assert mla.mla_last_dispatch().startswith("tensor-core"), mla.mla_last_dispatch()
    ref = oracle_prefill(wl, inp, heads=[0, 21, 63])
    compare(f64(got), ref, "bf16", "many short sequences")


def test_prefill_output_guard_bytes(gpu_lib):
    # Writes stay inside `out`: guard regions around it keep their bytes.
    wl = W.scaled(W.KIMI, seqlens=(200, 57), seed=13)
    inp = W.prefill_inputs(wl)
    T = 257
    n = T * 64 * 128
    buf = torch.full((n + 2 * 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    out = buf[4096:4096 + n].view(T, 64, 128)
    rope, shape, _ = oracle_cfg(wl)
    dims = mla.dims_for(wl, mla.mla_softmax_scale(mla.rope_for(wl), 192))
    cos, sin = mla.mla_init_rope_tables(mla.rope_for(wl), 256)
    d = {k: v.cuda() for k, v in inp.items()}
    mla.mla_prefill(dims, d["latent"], d["q"], d["w_kvb"], d["w_norm"], d["positions"], d["cu_seqlens"],
                    200, cos, sin, out=out)
    torch.cuda.synchronize()
    assert torch.all(buf[:4096] == 7.0) and torch.all(buf[4096 + n:] == 7.0)


# ---------------------------------------------------------------- decode

def test_decode_small_all_heads(gpu_lib):
    wl = W.scaled(W.DECODE, batch=5, cache_lens=(1, 2, 63, 700, 2049), seed=14)
    inp = W.decode_inputs(wl)
    got = run_decode(wl, inp)
    ref = oracle_decode(wl, inp, batches=range(5))
    compare(f64(got), ref, "bf16", "decode small")


def test_decode_glm_heads_interleaved_b70(gpu_lib):
    # GLM-5 heads (qk_nope 192, v_head 256, interleaved rotary pairs), 70
    # sequences (a partial second batch block in the per-head GEMMs), lengths
    # around the 128-row tile edges
    lens = tuple((1, 127, 128, 129, 255, 256, 257)[i % 7] for i in range(70))
    wl = W.Workload("glm_decode_bf16", "decode", 64, 512, 192, 64, 256, "bf16", W.GLM_ROPE, 16,
                    interleaved=True, batch=70, cache_lens=lens)
    inp = W.decode_inputs(wl)
    got = run_decode(wl, inp)
    ref = oracle_decode(wl, inp, batches=[0, 1, 2, 3, 4, 5, 6, 33, 64, 65, 69], absorbed=True)
    compare(f64(got), ref, "bf16", "decode glm b70")


def test_decode_many_short_sequences(gpu_lib):
    # 400 short sequences around the 64-row tile edges: each CTA's row range
    # holds several sequences, so segments of one or two tiles follow each
    # other (a query block reloaded between back-to-back scores, segment ends
    # next to the first tile of the next segment, single-row sequences)
    lens = tuple((1, 2, 63, 64, 65, 127, 128, 129)[(7 * i) % 8] for i in range(400))
    wl = W.scaled(W.DECODE, batch=400, cache_lens=lens, seed=17)
    inp = W.decode_inputs(wl)
    got = run_decode(wl, inp)
    assert mla.mla_last_dispatch().startswith("tensor-core"), mla.mla_last_dispatch()
    picks = sorted(set(range(0, 400, 11)) | {1, 2, 3, 4, 5, 6, 7, 398, 399})
    ref = oracle_decode(wl, inp, batches=picks, absorbed=True)
    compare(f64(got), ref, "bf16", "decode 400 short")


@pytest.mark.parametrize("heads", [8, 16, 32])
def test_decode_fewer_heads_tensor_core(gpu_lib, heads):
    # one GPU's share of a head-sharded Kimi-K2 decode: the tensor-core
    # kernels pad the heads to 64 with zero queries and drop their outputs
    wl = W.Workload("kimi_decode_h%d" % heads, "decode", heads, 512, 128, 64, 128, "bf16", W.KIMI_ROPE,
                    20 + heads, batch=6, cache_lens=(1, 127, 129, 700, 2049, 5000))
    inp = W.decode_inputs(wl)
    got = run_decode(wl, inp)
    assert mla.mla_last_dispatch().startswith("tensor-core"), mla.mla_last_dispatch()
    ref = oracle_decode(wl, inp, batches=range(6))
    compare(f64(got), ref, "bf16", "decode %d heads" % heads)


def test_decode_fp32_tiny_geometry(gpu_lib):
    wl = W.Workload("tiny_decode_fp32", "decode", 2, 64, 16, 8, 16, "fp32", W.TINY_ROPE, 15,
                    batch=3, cache_lens=(1, 40, 333))
    inp = W.decode_inputs(wl)
    got = run_decode(wl, inp)
    compare(f64(got), oracle_decode(wl, inp, batches=range(3)), "fp32", "decode fp32")


def test_decode_full_sampled(gpu_lib):
    wl = W.DECODE
    inp = W.decode_inputs(wl)
    got = f64(run_decode(wl, inp))
    eager = oracle_decode(wl, inp, batches=[0, 9, 17, 25, 33, 41, 50, 63], heads=[0, 1, 31, 63])
    compare(got, eager, "bf16", "decode vs eager")
    absorbed = oracle_decode(wl, inp, batches=range(0, 64, 4), absorbed=True)
    compare(got, absorbed, "bf16", "decode vs absorbed")


def test_decode_longest_all_heads(gpu_lib):
    # the longest cache length of the decode workload (32768 rows) next to a
    # short one, every head checked against the oracle (its absorbed form,
    # which is the same fp64 value up to rounding at a fraction of the cost);
    # the long row spans many CTAs' row ranges, so its output merges many
    # partials
    wl = W.scaled(W.DECODE, batch=2, cache_lens=(32768, 3), seed=17)
    inp = W.decode_inputs(wl)
    got = f64(run_decode(wl, inp))
    ref = oracle_decode(wl, inp, batches=[0, 1], absorbed=True)
    compare(got, ref, "bf16", "decode L=32768 all heads")
    eager = oracle_decode(wl, inp, batches=[0], heads=[0, 63])
    compare(got, eager, "bf16", "decode L=32768 vs eager")


def test_cache_append_then_decode_matches_prefill_row(gpu_lib):
    # Append every token of two sequences to a latent cache on the GPU, then a
    # decode step for each sequence's last token must reproduce the oracle's
    # prefill output for that token.
    wl = W.scaled(W.KIMI, seqlens=(333, 1000), seed=16)
    inp = W.prefill_inputs(wl)
    rope, shape, scale = oracle_cfg(wl)
    dims = mla.dims_for(wl, mla.mla_softmax_scale(mla.rope_for(wl), 192))
    cos, sin = mla.mla_init_rope_tables(mla.rope_for(wl), 1000)
    d = {k: v.cuda() for k, v in inp.items()}
    T = 1333
    cache = torch.zeros((T, 576), dtype=torch.bfloat16, device="cuda")
    rows = torch.arange(T, dtype=torch.int64, device="cuda")
    mla.mla_cache_append(dims, d["latent"], d["w_norm"], d["positions"], cos, sin, cache, rows)
    torch.cuda.synchronize()
    # the appended rows themselves
    ocos, osin = O.rope_tables(rope, 1000)
    ref_rows = O.cache_append(f64(inp["latent"]), f64(inp["w_norm"]), inp["positions"].numpy(),
                              ocos, osin, shape)
    compare(f64(cache), ref_rows, "bf16", "cache rows")
    last = torch.tensor([332, 1332])
    qd = d["q"][last.cuda()].contiguous()
    offs = torch.tensor([0, 333], dtype=torch.int64, device="cuda")
    lens = torch.tensor([333, 1000], dtype=torch.int32, device="cuda")
    pos = torch.tensor([332, 999], dtype=torch.int32, device="cuda")
    got = mla.mla_decode(dims, qd, cache, offs, lens, pos, 1000, d["w_kvb"], cos, sin)
    torch.cuda.synchronize()
    rows_sel = {0: np.array([332]), 1: np.array([999])}
    ref = oracle_prefill(wl, inp, rows=rows_sel)
    compare(f64(got), ref[[332, 1332]], "bf16", "decode vs prefill row")


def test_device_status_clean(gpu_lib):
    mla.mla_check_device_status()


# ---------------------------------------------------------------- chunks over a cached prefix

def _chunk_wl(base, chunks, prefixes, seed, **kw):
    return W.scaled(base, kind="prefill", seqlens=tuple(chunks), seed=seed,
                    extra=dict(prefix_lens=tuple(prefixes)), **kw)


def _check_chunk(wl, heads=None, gap=3):
    inp = W.chunk_inputs(wl, gap=gap)
    got, cache = run_prefill_cached(wl, inp)
    mla.mla_check_device_status()
    ref, ref_cache = oracle_prefill_cached(wl, inp, heads=heads)
    dt = "fp32" if wl.dtype == "fp32" else "bf16"
    compare(f64(got), ref, dt, "chunk out %s" % wl.name)
    # the chunk's rows went into the cache; no other row changed
    new = np.zeros(cache.shape[0], bool)
    cu, offs, pre = inp["cu_seqlens"], inp["cache_offsets"], inp["prefix_lens"]
    for s in range(len(wl.seqlens)):
        r0 = int(offs[s]) + int(pre[s])
        new[r0:r0 + int(cu[s + 1] - cu[s])] = True
    if new.any():
        compare(f64(cache)[new], ref_cache[new], dt, "chunk cache rows %s" % wl.name)
    assert torch.equal(cache.cpu()[torch.from_numpy(~new)], inp["cache"][torch.from_numpy(~new)])


def test_prefill_cached_kimi_heads(gpu_lib):
    # prefixes from empty to several tiles, chunks from none to past a tile
    wl = _chunk_wl(W.KIMI, chunks=(5, 1, 0, 17, 130), prefixes=(0, 1, 127, 1000, 2999), seed=41)
    _check_chunk(wl, heads=[0, 5, 31, 63])


def test_prefill_cached_glm_heads_interleaved(gpu_lib):
    wl = _chunk_wl(W.GLM, chunks=(3, 64), prefixes=(700, 129), seed=42)
    _check_chunk(wl, heads=[0, 1, 62, 63])


def test_prefill_cached_fp32_tiny_geometry(gpu_lib):
    wl = _chunk_wl(W.TINY, chunks=(4, 9, 1), prefixes=(0, 30, 5), seed=43)
    _check_chunk(wl)


def test_prefill_cached_continues_a_prefill(gpu_lib):
    # Each sequence's first tokens go into the cache through mla_cache_append,
    # the rest run as a chunk: the chunk's outputs equal the oracle's prefill
    # of the whole sequences at those rows.
    wl = W.scaled(W.KIMI, seqlens=(333, 1000, 260), seed=44)
    inp = W.prefill_inputs(wl)
    split = (300, 999, 128)
    rope, shape, scale = oracle_cfg(wl)
    dims = mla.dims_for(wl, mla.mla_softmax_scale(mla.rope_for(wl), 192))
    cos, sin = mla.mla_init_rope_tables(mla.rope_for(wl), 1000)
    d = {k: v.cuda() for k, v in inp.items()}
    cu = inp["cu_seqlens"].tolist()
    first = torch.cat([torch.arange(cu[s], cu[s] + split[s]) for s in range(3)])
    rest = torch.cat([torch.arange(cu[s] + split[s], cu[s + 1]) for s in range(3)])
    cache = torch.zeros((sum(wl.seqlens), 576), dtype=torch.bfloat16, device="cuda")
    offs = torch.tensor(cu[:3], dtype=torch.int64)
    rows = torch.cat([offs[s] + torch.arange(split[s]) for s in range(3)])
    mla.mla_cache_append(dims, d["latent"][first.cuda()].contiguous(), d["w_norm"],
                         d["positions"][first.cuda()].contiguous(), cos, sin, cache, rows.cuda())
    cuq = torch.tensor([0] + list(np.cumsum([wl.seqlens[s] - split[s] for s in range(3)])), dtype=torch.int32)
    got = mla.mla_prefill_cached(dims, d["latent"][rest.cuda()].contiguous(), d["q"][rest.cuda()].contiguous(),
                                 d["w_kvb"], d["w_norm"], cuq.cuda(), offs.cuda(),
                                 torch.tensor(split, dtype=torch.int32, device="cuda"), 1000, cos, sin, cache)
    torch.cuda.synchronize()
    mla.mla_check_device_status()
    ref = oracle_prefill(wl, inp, heads=[0, 1, 31, 63])
    compare(f64(got), ref[rest.numpy()], "bf16", "chunk after cache append")


def test_prefill_cached_out_of_range_sequence_is_skipped(gpu_lib):
    # The last sequence's region is cut short (its rows would leave the
    # cache): its tokens are neither written nor attended, their outputs are
    # zero, the error word is set, and the other sequences are unaffected.
    wl = _chunk_wl(W.KIMI, chunks=(6, 4), prefixes=(50, 20), seed=45)
    inp = W.chunk_inputs(wl, gap=0)
    full_rows = inp["cache"].shape[0]
    inp_cut = dict(inp, cache=inp["cache"][:full_rows - 2].clone())
    got, cache = run_prefill_cached(wl, inp_cut)
    with pytest.raises(mla.MlaError):
        mla.mla_check_device_status()
    mla.mla_check_device_status()   # the error word was cleared
    assert torch.all(got[6:].float() == 0)
    assert torch.equal(cache[56:].cpu(), inp_cut["cache"][56:])
    ref, _ = oracle_prefill_cached(wl, inp, heads=[0, 63])
    compare(f64(got)[:6], ref[:6], "bf16", "chunk kept sequence")


# ---------------------------------------------------------------- projections on either side

# hidden size and query rank of the Kimi-K2 model (the pages name the
# projections but print neither size)
KIMI_HIDDEN, KIMI_QRANK = 7168, 1536


def _proj_case(wl, n, hid, qr, seed):
    inp = W.projection_inputs(wl, n, hid, qr, seed)
    rope, shape, _ = oracle_cfg(wl)
    dims = mla.dims_for(wl, mla.mla_softmax_scale(mla.rope_for(wl), shape.qk_head_dim))
    return inp, {k: v.cuda() for k, v in inp.items()}, dims, rope, shape


@pytest.mark.parametrize("hid", [KIMI_HIDDEN, 1000], ids=["tensor_cores", "cuda_cores"])
def test_kv_down_append_kimi_heads(gpu_lib, hid):
    n = 130
    inp, d, dims, rope, shape = _proj_case(W.KIMI, n, hid, 64, seed=1)
    cos, sin = mla.mla_init_rope_tables(mla.rope_for(W.KIMI), n)
    cache = torch.full((n + 9, 576), 3.0, dtype=torch.bfloat16, device="cuda")
    rows = torch.arange(n, dtype=torch.int64, device="cuda") + 5
    latent = mla.mla_kv_down_append(dims, d["hidden"], d["w_kva"], w_norm=d["w_norm"], positions=d["positions"],
                                    cos=cos, sin=sin, cache=cache, cache_rows=rows)
    torch.cuda.synchronize()
    mla.mla_check_device_status()
    lat_ref = O.kv_down_projection(f64(inp["hidden"]), f64(inp["w_kva"]))
    compare(f64(latent), lat_ref, "bf16", "kv_a_proj K=%d" % hid)
    ocos, osin = O.rope_tables(rope, n)
    rows_ref = O.cache_append(lat_ref, f64(inp["w_norm"]), inp["positions"].numpy(), ocos, osin, shape)
    compare(f64(cache[5:n + 5]), rows_ref, "bf16", "kv_a_proj cache rows K=%d" % hid)
    assert torch.all(cache[:5] == 3.0) and torch.all(cache[n + 5:] == 3.0)


@pytest.mark.parametrize("hid,qr", [(KIMI_HIDDEN, KIMI_QRANK), (1000, 200)], ids=["tensor_cores", "cuda_cores"])
def test_q_proj_kimi_heads(gpu_lib, hid, qr):
    n = 130
    inp, d, dims, rope, shape = _proj_case(W.KIMI, n, hid, qr, seed=2)
    q = mla.mla_q_proj(dims, d["hidden"], d["w_qa"], d["w_qnorm"], d["w_qb"])
    torch.cuda.synchronize()
    mla.mla_check_device_status()
    ref = O.q_projection(f64(inp["hidden"]), f64(inp["w_qa"]), f64(inp["w_qnorm"]), f64(inp["w_qb"]), shape)
    compare(f64(q), ref, "bf16", "q_proj K=%d/%d" % (hid, qr))


def test_projections_bench_size(gpu_lib):
    # the bench's 2048 tokens: the cache rows and q over millions of elements,
    # where the bf16 output's half-ulp (0.0156 at |x| >= 4) leaves the least room
    n = 2048
    inp, d, dims, rope, shape = _proj_case(W.KIMI, n, KIMI_HIDDEN, KIMI_QRANK, seed=0)
    cos, sin = mla.mla_init_rope_tables(mla.rope_for(W.KIMI), n)
    cache = torch.empty((n, 576), dtype=torch.bfloat16, device="cuda")
    rows = torch.arange(n, dtype=torch.int64, device="cuda")
    latent = mla.mla_kv_down_append(dims, d["hidden"], d["w_kva"], w_norm=d["w_norm"], positions=d["positions"],
                                    cos=cos, sin=sin, cache=cache, cache_rows=rows)
    q = mla.mla_q_proj(dims, d["hidden"], d["w_qa"], d["w_qnorm"], d["w_qb"])
    torch.cuda.synchronize()
    mla.mla_check_device_status()
    x = f64(inp["hidden"])
    lat_ref = O.kv_down_projection(x, f64(inp["w_kva"]))
    compare(f64(latent), lat_ref, "bf16", "kv_a_proj n=2048")
    ocos, osin = O.rope_tables(rope, n)
    compare(f64(cache), O.cache_append(lat_ref, f64(inp["w_norm"]), inp["positions"].numpy(), ocos, osin, shape),
            "bf16", "kv_a_proj cache rows n=2048")
    compare(f64(q), O.q_projection(x, f64(inp["w_qa"]), f64(inp["w_qnorm"]), f64(inp["w_qb"]), shape), "bf16",
            "q_proj n=2048")


def test_o_proj_kimi_heads(gpu_lib):
    n = 130
    inp, d, dims, rope, shape = _proj_case(W.KIMI, n, KIMI_HIDDEN, 64, seed=3)
    out = mla.mla_o_proj(dims, d["attn"], d["w_o"])
    torch.cuda.synchronize()
    mla.mla_check_device_status()
    compare(f64(out), O.o_projection(f64(inp["attn"]), f64(inp["w_o"])), "bf16", "o_proj")


def test_projections_fp32_tiny(gpu_lib):
    n, hid, qr = 37, 48, 24
    inp, d, dims, rope, shape = _proj_case(W.TINY, n, hid, qr, seed=4)
    latent = mla.mla_kv_down_append(dims, d["hidden"], d["w_kva"])
    q = mla.mla_q_proj(dims, d["hidden"], d["w_qa"], d["w_qnorm"], d["w_qb"])
    out = mla.mla_o_proj(dims, d["attn"], d["w_o"])
    torch.cuda.synchronize()
    mla.mla_check_device_status()
    x = f64(inp["hidden"])
    compare(f64(latent), O.kv_down_projection(x, f64(inp["w_kva"])), "fp32", "kv_a_proj fp32")
    compare(f64(q), O.q_projection(x, f64(inp["w_qa"]), f64(inp["w_qnorm"]), f64(inp["w_qb"]), shape), "fp32",
            "q_proj fp32")
    compare(f64(out), O.o_projection(f64(inp["attn"]), f64(inp["w_o"])), "fp32", "o_proj fp32")
