"""GPU parity of the eager form of chunks over a cached prefix.

Long chunks (at least 128 tokens per sequence on average) with a workspace
that holds the eager form expand the keys and values of every cached row and
run the two-tile attention with each sequence's prefix length as the query
offset. These tests check the form the library picked (mla_last_dispatch),
the outputs against the fp64 oracle's prefill_cached (sampled heads), the
cache rows the call appended, agreement with the absorbed form on the same
inputs, the continuation of a one-call prefill, and the handling of a
sequence whose rows leave the cache.
"""

import numpy as np
import pytest
import torch

import oracle as O
from decode_latent_rmsnorm_b200 import mla
from decode_latent_rmsnorm_b200 import workloads as W
from _parity import compare, f64, oracle_cfg, oracle_prefill, oracle_prefill_cached

pytestmark = pytest.mark.gpu


def _wl(chunks, prefixes, seed):
    return W.scaled(W.KIMI, kind="prefill", seqlens=tuple(chunks), seed=seed,
                    extra=dict(prefix_lens=tuple(prefixes)))


def _run(wl, inp, form="auto"):
    rope, shape, scale = oracle_cfg(wl)
    dims = mla.dims_for(wl, mla.mla_softmax_scale(mla.rope_for(wl), shape.qk_head_dim))
    cos, sin = mla.mla_init_rope_tables(mla.rope_for(wl), inp["max_total_len"])
    d = {k: v.to("cuda") for k, v in inp.items() if isinstance(v, torch.Tensor)}
    out = mla.mla_prefill_cached(dims, d["latent"], d["q"], d["w_kvb"], d["w_norm"], d["cu_seqlens"],
                                 d["cache_offsets"], d["prefix_lens"], inp["max_total_len"], cos, sin, d["cache"],
                                 form=form)
    torch.cuda.synchronize()
    return out, d["cache"], mla.mla_last_dispatch()


@pytest.mark.parametrize("chunks,prefixes", [((512, 300), (16000, 129)), ((2048,), (16384,))],
                         ids=["512+300_over_16000+129", "2048_over_16384"])
def test_eager_chunk_matches_oracle(gpu_lib, chunks, prefixes):
    wl = _wl(chunks, prefixes, seed=61 + len(chunks))
    inp = W.chunk_inputs(wl, gap=5)
    got, cache, how = _run(wl, inp)
    mla.mla_check_device_status()
    assert how.startswith("eager"), how
    ref, ref_cache = oracle_prefill_cached(wl, inp, heads=[0, 63])
    compare(f64(got), ref, "bf16", "eager chunk %s" % (chunks,))
    cu, offs, pre = inp["cu_seqlens"], inp["cache_offsets"], inp["prefix_lens"]
    new = np.zeros(cache.shape[0], bool)
    for s in range(len(chunks)):
        r0 = int(offs[s]) + int(pre[s])
        new[r0:r0 + int(cu[s + 1] - cu[s])] = True
    compare(f64(cache)[new], ref_cache[new], "bf16", "eager chunk cache rows")
    assert torch.equal(cache.cpu()[torch.from_numpy(~new)], inp["cache"][torch.from_numpy(~new)])


def test_eager_and_absorbed_agree(gpu_lib):
    wl = _wl((260, 400, 129), (777, 0, 1500), seed=64)
    inp = W.chunk_inputs(wl, gap=0)
    got_e, _, how_e = _run(wl, inp, form="eager")
    got_a, _, how_a = _run(wl, inp, form="absorbed")
    mla.mla_check_device_status()
    assert how_e.startswith("eager") and how_a.startswith("absorbed"), (how_e, how_a)
    ref, _ = oracle_prefill_cached(wl, inp, heads=[0, 17, 63])
    compare(f64(got_e), ref, "bf16", "eager vs oracle")
    compare(f64(got_a), ref, "bf16", "absorbed vs oracle")


def test_eager_chunk_continues_a_prefill(gpu_lib):
    # the first rows of each sequence enter the cache through mla_cache_append;
    # the long rest runs as an eager chunk and must equal the oracle's one-call
    # prefill of the whole sequences at those rows
    wl = W.scaled(W.KIMI, seqlens=(1500, 700), seed=65)
    inp = W.prefill_inputs(wl)
    split = (1100, 200)
    rope, shape, scale = oracle_cfg(wl)
    dims = mla.dims_for(wl, mla.mla_softmax_scale(mla.rope_for(wl), 192))
    cos, sin = mla.mla_init_rope_tables(mla.rope_for(wl), 1500)
    d = {k: v.cuda() for k, v in inp.items()}
    cu = inp["cu_seqlens"].tolist()
    first = torch.cat([torch.arange(cu[s], cu[s] + split[s]) for s in range(2)])
    rest = torch.cat([torch.arange(cu[s] + split[s], cu[s + 1]) for s in range(2)])
    cache = torch.zeros((sum(wl.seqlens), 576), dtype=torch.bfloat16, device="cuda")
    offs = torch.tensor(cu[:2], dtype=torch.int64)
    rows = torch.cat([offs[s] + torch.arange(split[s]) for s in range(2)])
    mla.mla_cache_append(dims, d["latent"][first.cuda()].contiguous(), d["w_norm"],
                         d["positions"][first.cuda()].contiguous(), cos, sin, cache, rows.cuda())
    cuq = torch.tensor([0] + list(np.cumsum([wl.seqlens[s] - split[s] for s in range(2)])), dtype=torch.int32)
    got = mla.mla_prefill_cached(dims, d["latent"][rest.cuda()].contiguous(), d["q"][rest.cuda()].contiguous(),
                                 d["w_kvb"], d["w_norm"], cuq.cuda(), offs.cuda(),
                                 torch.tensor(split, dtype=torch.int32, device="cuda"), 1500, cos, sin, cache)
    torch.cuda.synchronize()
    assert mla.mla_last_dispatch().startswith("eager")
    mla.mla_check_device_status()
    ref = oracle_prefill(wl, inp, heads=[0, 31, 63])
    compare(f64(got), ref[rest.numpy()], "bf16", "eager chunk after cache append")


def test_eager_out_of_range_sequence_is_skipped(gpu_lib):
    # the last sequence's region is cut short: its tokens are neither written
    # nor attended, their outputs are zero, the error word is set, and the
    # other sequence is unaffected
    wl = _wl((300, 200), (500, 100), seed=66)
    inp = W.chunk_inputs(wl, gap=0)
    full_rows = inp["cache"].shape[0]
    inp_cut = dict(inp, cache=inp["cache"][:full_rows - 2].clone())
    got, cache, how = _run(wl, inp_cut)
    assert how.startswith("eager"), how
    with pytest.raises(mla.MlaError):
        mla.mla_check_device_status()
    mla.mla_check_device_status()   # the error word was cleared
    assert torch.all(got[300:].float() == 0)
    ref, _ = oracle_prefill_cached(wl, inp, heads=[0, 63])
    compare(f64(got)[:300], ref[:300], "bf16", "eager chunk kept sequence")
