"""Seeded synthetic workloads of the MLA pages' shapes.

This module only draws random tensors and lays them out; it contains none of
the attention arithmetic. Tests feed the same tensors to the CUDA library and
to the CPU oracle; ``bench.py`` uses it for timing inputs.

Distributions (variance notation N(mean, var)):
  latent, q, decode cache rows ~ N(0, 1); kv_b_proj weight ~ N(0, 1/R);
  latent-norm weight = 1 + 0.1 * N(0, 1).
All values are drawn in fp32 from one CPU ``torch.Generator`` per workload,
in a fixed order, and then rounded to the run dtype.

Decode cache rows hold an already-normalized latent and an already-rotated
rotary key. They are drawn directly from N(0, 1): a RMS-normalized vector has
unit mean square and a rotation keeps an isotropic Gaussian isotropic, so the
draw has the statistics of a real cache without running any of the method.
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace

import torch

# Rotary settings of the Kimi-K2 pages: YaRN, base 50000, factor 32 over 4096
# original positions, beta_fast 32, beta_slow 1, mscale = mscale_all_dim = 1.
KIMI_ROPE = dict(rope_dim=64, base=50000.0, yarn=True, factor=32.0,
                 original_max_pos=4096, beta_fast=32.0, beta_slow=1.0,
                 mscale=1.0, mscale_all_dim=1.0)
# GLM-5: default (unscaled) rotary embedding, base 10000.
GLM_ROPE = dict(rope_dim=64, base=10000.0, yarn=False)
TINY_ROPE = dict(rope_dim=8, base=10000.0, yarn=False)


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                    # "prefill" or "decode"
    num_heads: int
    kv_lora_rank: int
    qk_nope: int
    qk_rope: int
    v_head: int
    dtype: str                   # "fp32" or "bf16"
    rope: dict
    seed: int
    interleaved: bool = False
    seqlens: tuple = ()          # prefill: per-sequence lengths
    batch: int = 0               # decode: sequences
    cache_len_range: tuple = (0, 0)   # decode: inclusive uniform range
    cache_lens: tuple = ()       # decode: explicit lengths (overrides the range)
    eps: float = 1e-6
    extra: dict = field(default_factory=dict)

    @property
    def qk_head_dim(self):
        return self.qk_nope + self.qk_rope

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16


TINY = Workload("tiny_fp32", "prefill", 2, 64, 16, 8, 16, "fp32", TINY_ROPE, 0,
                seqlens=(32,))
KIMI = Workload("kimi_k2_prefill_bf16", "prefill", 64, 512, 128, 64, 128, "bf16",
                KIMI_ROPE, 1, seqlens=(2048,))
GLM = Workload("glm5_prefill_bf16", "prefill", 64, 512, 192, 64, 256, "bf16",
               GLM_ROPE, 2, interleaved=True, seqlens=(4096, 4096))
VARLEN = Workload("varlen_prefill_bf16", "prefill", 64, 512, 128, 64, 128, "bf16",
                  KIMI_ROPE, 3, seqlens=(1024, 3000, 7777, 16384))
DECODE = Workload("absorbed_decode_bf16", "decode", 64, 512, 128, 64, 128, "bf16",
                  KIMI_ROPE, 4, batch=64, cache_len_range=(1000, 32768))

WORKLOADS = {w.name: w for w in (TINY, KIMI, GLM, VARLEN, DECODE)}


def scaled(wl: Workload, **kw) -> Workload:
    """A copy of ``wl`` with some fields replaced (smaller parity cases)."""
    return replace(wl, **kw)


def _randn(g, shape, dtype):
    return torch.randn(shape, generator=g, dtype=torch.float32).to(dtype)


def prefill_inputs(wl: Workload) -> dict:
    """CPU tensors for one prefill call.

    latent [Ttot, R + P], q [Ttot, H, N + P], w_kvb [H * (N + V), R],
    w_norm [R] in the run dtype; positions [Ttot] and cu_seqlens [nseq + 1]
    int32 (each sequence's positions restart at 0).
    """
    assert wl.kind == "prefill"
    g = torch.Generator().manual_seed(wl.seed)
    dt = wl.torch_dtype
    H, R, N, P, V = wl.num_heads, wl.kv_lora_rank, wl.qk_nope, wl.qk_rope, wl.v_head
    T = int(sum(wl.seqlens))
    latent = _randn(g, (T, R + P), dt)
    q = _randn(g, (T, H, N + P), dt)
    w_kvb = (torch.randn((H * (N + V), R), generator=g) * (1.0 / R) ** 0.5).to(dt)
    w_norm = (1.0 + 0.1 * torch.randn((R,), generator=g)).to(dt)
    cu = [0]
    for L in wl.seqlens:
        cu.append(cu[-1] + int(L))
    positions = torch.cat([torch.arange(int(L), dtype=torch.int32) for L in wl.seqlens]) \
        if T > 0 else torch.zeros(0, dtype=torch.int32)
    return dict(latent=latent, q=q, w_kvb=w_kvb, w_norm=w_norm,
                positions=positions, cu_seqlens=torch.tensor(cu, dtype=torch.int32))


def decode_cache_lens(wl: Workload) -> torch.Tensor:
    if wl.cache_lens:
        return torch.tensor(wl.cache_lens, dtype=torch.int32)
    g = torch.Generator().manual_seed(wl.seed)
    lo, hi = wl.cache_len_range
    return torch.randint(lo, hi + 1, (wl.batch,), generator=g, dtype=torch.int32)


def decode_inputs(wl: Workload) -> dict:
    """CPU tensors for one decode call.

    cache [sum(lens), R + P] packed sequence after sequence (cache_offsets
    [B] int64 gives each sequence's first row), cache_lens [B] int32,
    q [B, H, N + P], w_kvb [H * (N + V), R], positions [B] int32 (= the cache
    length: the new token sits right after its cached rows).
    """
    assert wl.kind == "decode"
    lens = decode_cache_lens(wl)
    B = lens.numel()
    g = torch.Generator().manual_seed(wl.seed + 1000)
    dt = wl.torch_dtype
    H, R, N, P, V = wl.num_heads, wl.kv_lora_rank, wl.qk_nope, wl.qk_rope, wl.v_head
    offsets = torch.zeros(B, dtype=torch.int64)
    if B > 1:
        offsets[1:] = torch.cumsum(lens.to(torch.int64), 0)[:-1]
    total = int(lens.to(torch.int64).sum())
    cache = torch.empty((total, R + P), dtype=dt)
    chunk = 1 << 16
    for r0 in range(0, total, chunk):
        r1 = min(total, r0 + chunk)
        cache[r0:r1] = _randn(g, (r1 - r0, R + P), dt)
    q = _randn(g, (B, H, N + P), dt)
    w_kvb = (torch.randn((H * (N + V), R), generator=g) * (1.0 / R) ** 0.5).to(dt)
    return dict(cache=cache, cache_offsets=offsets, cache_lens=lens, q=q, w_kvb=w_kvb,
                positions=lens.clone())


def chunk_inputs(wl: Workload, gap: int = 0) -> dict:
    """CPU tensors for one call of chunks that continue cached sequences.

    ``wl.seqlens`` gives each sequence's chunk tokens and
    ``wl.extra["prefix_lens"]`` its rows cached before the call. The cache
    [rows, R + P] gives sequence s a region of prefix + chunk rows followed
    by ``gap`` unused rows; the prefix rows are drawn N(0, 1) like the decode
    cache (the statistics of a normalized latent and a rotated key), and the
    chunk's rows and the unused rows start at zero. Also returns latent
    [Tq, R + P] (raw compressed_kv of the chunk tokens), q [Tq, H, N + P],
    w_kvb, w_norm, cu_seqlens int32 [nseq + 1], cache_offsets int64 [nseq],
    prefix_lens int32 [nseq] and max_total_len.
    """
    g = torch.Generator().manual_seed(wl.seed + 2000)
    dt = wl.torch_dtype
    H, R, N, P, V = wl.num_heads, wl.kv_lora_rank, wl.qk_nope, wl.qk_rope, wl.v_head
    chunks = [int(n) for n in wl.seqlens]
    prefix = [int(p) for p in wl.extra["prefix_lens"]]
    nseq = len(chunks)
    offsets, rows = [], 0
    for s in range(nseq):
        offsets.append(rows)
        rows += prefix[s] + chunks[s] + gap
    cache = torch.zeros((max(rows, 1), R + P), dtype=dt)
    for s in range(nseq):
        if prefix[s]:
            cache[offsets[s]:offsets[s] + prefix[s]] = _randn(g, (prefix[s], R + P), dt)
    T = sum(chunks)
    latent = _randn(g, (T, R + P), dt)
    q = _randn(g, (T, H, N + P), dt)
    w_kvb = (torch.randn((H * (N + V), R), generator=g) * (1.0 / R) ** 0.5).to(dt)
    w_norm = (1.0 + 0.1 * torch.randn((R,), generator=g)).to(dt)
    cu = [0]
    for n in chunks:
        cu.append(cu[-1] + n)
    return dict(latent=latent, q=q, w_kvb=w_kvb, w_norm=w_norm, cache=cache,
                cu_seqlens=torch.tensor(cu, dtype=torch.int32),
                cache_offsets=torch.tensor(offsets, dtype=torch.int64),
                prefix_lens=torch.tensor(prefix, dtype=torch.int32),
                max_total_len=max([p + n for p, n in zip(prefix, chunks)] + [1]))


def projection_inputs(wl: Workload, n: int, hidden_size: int, q_rank: int, seed: int = 0) -> dict:
    """CPU tensors for the projections on either side of the path, in the
    run dtype: hidden [n, hidden_size] and attn [n, H * V] ~ N(0, 1); the
    weights ~ N(0, 1/in) so each Linear keeps unit variance: w_kva
    [R + P, hidden_size], w_qa [q_rank, hidden_size], w_qb [H * (N + P),
    q_rank], w_o [hidden_size, H * V]; the RMSNorm weights w_norm [R] and
    w_qnorm [q_rank] = 1 + 0.1 * N(0, 1); positions [n] = 0 .. n - 1."""
    g = torch.Generator().manual_seed(wl.seed + 3000 + seed)
    dt = wl.torch_dtype
    H, R, N, P, V = wl.num_heads, wl.kv_lora_rank, wl.qk_nope, wl.qk_rope, wl.v_head

    def lin(out_f, in_f):
        return (torch.randn((out_f, in_f), generator=g) * (1.0 / in_f) ** 0.5).to(dt)

    hidden = _randn(g, (n, hidden_size), dt)
    attn = _randn(g, (n, H * V), dt)
    w_kva = lin(R + P, hidden_size)
    w_qa = lin(q_rank, hidden_size)
    w_qb = lin(H * (N + P), q_rank)
    w_o = lin(hidden_size, H * V)
    w_norm = (1.0 + 0.1 * torch.randn((R,), generator=g)).to(dt)
    w_qnorm = (1.0 + 0.1 * torch.randn((q_rank,), generator=g)).to(dt)
    return dict(hidden=hidden, attn=attn, w_kva=w_kva, w_qa=w_qa, w_qb=w_qb, w_o=w_o, w_norm=w_norm,
                w_qnorm=w_qnorm, positions=torch.arange(n, dtype=torch.int32))


def max_position(wl: Workload) -> int:
    """Smallest rotary-table length that covers every position used."""
    if wl.kind == "prefill":
        return max(int(max(wl.seqlens)) if wl.seqlens else 1, 1)
    return int(decode_cache_lens(wl).max()) + 1
