"""Plain fp64 CPU oracle of the multi-head latent attention (MLA) hot path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product library.

Everything is written out in numpy float64, step by step, in the order the
pages give it. A matrix product (``@``) is the only library primitive used as
a step; there is no tiling, fusion or online softmax here. Evaluating a subset
of heads or query rows (used to bound CPU time at large sizes) computes each
selected output exactly as the full definition would.

Sources (page title, then the section or excerpt on it):

* [EQ]   "Eager latent expansion" equation page -- "Read the equation" prose
         and its "Original context" code (latent split, kv_a_layernorm,
         kv_b_proj, view/transpose, split into k_nope and values).
* [KQ]   Kimi-K2 "Query content heads" page -- "Split content heads"
         (mla-queries excerpt) and "Join query parts" (mla-prefill excerpt).
* [GLM]  GLM-5 "Normalized key-value latent" page -- tensor card,
         "Key-value compression" (mla-init and mla-kv excerpts) and
         "KV cache" (kv-cache excerpt).
* [ROT]  Kimi-K2 "RoPE coefficients" page (decode mode) -- cos/sin tensor
         card, "Generate RoPE coefficients" (rope and model-args excerpts),
         "Query heads" (mla-init, mla-queries) and "Key heads" (mla-kv,
         mla-prefill excerpts).

The projections on either side of the path (q_a_proj, q_a_layernorm,
q_b_proj, kv_a_proj_with_mqa, o_proj) follow the [ROT] mla-init excerpt
(their nn.Linear shapes) and the mla-queries / mla-kv excerpts (their order).
They are taken without bias: the attention-bias option is outside this
build. The pages give no hidden size or query rank; both are arguments.

Readings taken where the pages are silent:

* RMSNorm body: y = w * x / sqrt(mean(x**2) + eps), no bias, no centring;
  eps = 1e-6 ([GLM] "Key-value compression" says the latent RMSNorms use the
  default 1e-6).
* apply_rotary_pos_emb body is not shown. A rotary pair (a, b) turns
  counter-clockwise by the angle pos * inv_freq[i]:
  (a, b) -> (a cos - b sin, b cos + a sin), written back to the same slots.
  Pairing: ``interleaved=False`` pairs element i with i + P/2 (the half-split
  layout implied by the duplicated cos/sin table ``cat(freqs, freqs)`` of the
  [ROT] rope excerpt); ``interleaved=True`` pairs 2i with 2i+1 (the GLM-5
  ``apply_rotary_pos_emb_interleave`` name). Parity of the rotation direction
  and pairing is unpinned by any printed value (the pages print none).
* The additive causal mask is 0 where key j <= query i of the same sequence
  and -inf elsewhere; packed sequences never see each other.
* Softmax runs in float64 (the pages upcast to fp32); dropout is the
  identity (inference).
* Decode cache rows hold [normalized latent (R) || rotated k_pe (P)], as the
  GLM-5 "KV cache" section describes; heads are expanded from every cached
  row; the query sits at ``positions[b]`` and attends to all cached rows.
* A chunk of new tokens that continues a cached sequence: the chunk's rows
  are written into the cache first (the GLM-5 "KV cache" order: update,
  then expand every cached row). Chunk token i of a sequence with p cached
  rows sits at position p + i, goes to the sequence's cache row p + i, and
  attends to cached rows 0 .. p + i (the causal mask in absolute positions).
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

__all__ = [
    "RopeConfig", "MlaShape",
    "yarn_find_correction_dim", "yarn_find_correction_range",
    "yarn_get_mscale", "yarn_linear_ramp_mask",
    "rope_inv_freq", "rope_table_mscale", "rope_tables", "softmax_scale",
    "rms_norm", "kv_up_projection", "apply_rope",
    "causal_attention_rows", "prefill", "decode_eager", "decode_absorbed",
    "cache_append", "prefill_cached",
    "kv_down_projection", "q_projection", "o_projection",
]


@dataclass(frozen=True)
class RopeConfig:
    """Rotary configuration; field names follow ``config.rope_scaling``.

    [ROT] "Generate RoPE coefficients": the YaRN class defaults are
    original_max_position_embeddings 4096, beta_fast 32, beta_slow 1,
    mscale 1, mscale_all_dim 0; ``yarn=False`` is the default (unscaled)
    rotary embedding that ``_init_rope`` picks when rope_scaling is None.
    """

    rope_dim: int
    base: float
    yarn: bool = False
    factor: float = 1.0
    original_max_pos: int = 4096
    beta_fast: float = 32.0
    beta_slow: float = 1.0
    mscale: float = 1.0
    mscale_all_dim: float = 0.0


@dataclass(frozen=True)
class MlaShape:
    """Head geometry ([ROT] "Query heads" mla-init; [GLM] mla-init)."""

    num_heads: int
    kv_lora_rank: int
    qk_nope: int
    qk_rope: int
    v_head: int
    eps: float = 1e-6
    interleaved: bool = False

    @property
    def qk_head_dim(self) -> int:
        return self.qk_nope + self.qk_rope


# --------------------------------------------------------------------------
# RoPE coefficients -- [ROT] "Generate RoPE coefficients", rope excerpt
# --------------------------------------------------------------------------

def yarn_find_correction_dim(num_rotations, dim, base, max_position_embeddings):
    """Rotary dimension whose pair turns ``num_rotations`` times over
    ``max_position_embeddings`` positions ([ROT] rope, yarn_find_correction_dim)."""
    return (dim * math.log(max_position_embeddings / (num_rotations * 2 * math.pi))) / (
        2 * math.log(base))


def yarn_find_correction_range(low_rot, high_rot, dim, base, max_position_embeddings):
    """Integer range [low, high] of pair indices that get blended
    ([ROT] rope, yarn_find_correction_range): floor of the first bound,
    ceil of the second, clamped to [0, dim - 1]."""
    low = math.floor(yarn_find_correction_dim(low_rot, dim, base, max_position_embeddings))
    high = math.ceil(yarn_find_correction_dim(high_rot, dim, base, max_position_embeddings))
    return max(low, 0), min(high, dim - 1)


def yarn_get_mscale(scale=1.0, mscale=1.0):
    """YaRN attention correction ([ROT] rope and [GLM] mla-init,
    yarn_get_mscale): 1 for scale <= 1, else 0.1 * mscale * ln(scale) + 1."""
    if scale <= 1:
        return 1.0
    return 0.1 * mscale * math.log(scale) + 1.0


def yarn_linear_ramp_mask(lo, hi, n):
    """Linear ramp over indices 0..n-1, 0 at ``lo`` and 1 at ``hi``, clamped
    ([ROT] rope, yarn_linear_ramp_mask). ``hi`` is nudged by 0.001 when the
    two bounds coincide, as the page does. Computed in float64 here."""
    if lo == hi:
        hi = hi + 0.001
    ramp = (np.arange(n, dtype=np.float64) - lo) / (hi - lo)
    return np.clip(ramp, 0.0, 1.0)


def rope_inv_freq(rope: RopeConfig) -> np.ndarray:
    """Per-pair angular frequency, shape [rope_dim / 2].

    Default rotary: base ** (-2i / dim) (the body of the default class is not
    shown; this is the ``freq_extra`` expression of the YaRN excerpt).
    YaRN ([ROT] rope, _set_cos_sin_cache): ``freq_inter = freq_extra / factor``
    and ``inv_freq = freq_inter * (1 - m) + freq_extra * m`` with
    ``m = 1 - ramp(low, high)`` over the correction range of
    (beta_fast, beta_slow).
    """
    dim = rope.rope_dim
    exponents = np.arange(0, dim, 2, dtype=np.float64) / dim
    freq_extra = 1.0 / (rope.base ** exponents)
    if not rope.yarn:
        return freq_extra
    freq_inter = 1.0 / (rope.factor * rope.base ** exponents)
    low, high = yarn_find_correction_range(
        rope.beta_fast, rope.beta_slow, dim, rope.base, rope.original_max_pos)
    inv_freq_mask = 1.0 - yarn_linear_ramp_mask(low, high, dim // 2)
    return freq_inter * (1.0 - inv_freq_mask) + freq_extra * inv_freq_mask


def rope_table_mscale(rope: RopeConfig) -> float:
    """Factor the cos/sin tables are multiplied by ([ROT] rope,
    _set_cos_sin_cache): get_mscale(factor, mscale) / get_mscale(factor,
    mscale_all_dim) under YaRN; 1 for the default rotary embedding."""
    if not rope.yarn:
        return 1.0
    return float(yarn_get_mscale(rope.factor, rope.mscale)
                 / yarn_get_mscale(rope.factor, rope.mscale_all_dim))


def rope_tables(rope: RopeConfig, max_pos: int):
    """cos/sin tables, shape [max_pos, rope_dim / 2] each, float64.

    [ROT] rope, _set_cos_sin_cache: angles ``outer(t, inv_freq)`` for
    t = 0..max_pos-1, times the table mscale. The page stores
    ``cat(freqs, freqs)`` (both members of pair i share angle i); one column
    per pair is kept here. The cos/sin card of the same page gives the
    per-position shape as 32 pairs for Kimi-K2.
    """
    inv_freq = rope_inv_freq(rope)
    t = np.arange(max_pos, dtype=np.float64)
    freqs = np.outer(t, inv_freq)
    m = rope_table_mscale(rope)
    return np.cos(freqs) * m, np.sin(freqs) * m


def softmax_scale(rope: RopeConfig, qk_head_dim: int) -> float:
    """Softmax scale ([ROT] model-args; [GLM] mla-init yarn_apply_mscale):
    qk_head_dim ** -0.5, times get_mscale(factor, mscale_all_dim) ** 2 when
    the rotary embedding is scaled and mscale_all_dim is non-zero."""
    scale = qk_head_dim ** (-0.5)
    if rope.yarn and rope.mscale_all_dim:
        m = yarn_get_mscale(rope.factor, rope.mscale_all_dim)
        scale = scale * m * m
    return scale


# --------------------------------------------------------------------------
# Latent normalisation and up-projection -- [EQ]; [ROT] "Key heads" mla-kv;
# [GLM] "Key-value compression" mla-kv
# --------------------------------------------------------------------------

def rms_norm(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    """kv_a_layernorm over the last axis: w * x / sqrt(mean(x^2) + eps)."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return w * (x / np.sqrt(ms + eps))


def kv_up_projection(c_hat: np.ndarray, W: np.ndarray, shape: MlaShape, heads=None):
    """kv_b_proj applied to normalized latent rows, split per head.

    ``c_hat`` [T, R]; ``W`` is the nn.Linear weight [H * (N + V), R], so the
    product is ``c_hat @ W.T``. The result is viewed [T, H, N + V], moved
    head-major and split into k_nope [H, T, N] and values [H, T, V]
    ([EQ] code; [ROT] "Key heads" mla-kv; [GLM] expand_kv).
    ``heads`` selects a subset of heads (default: all).
    """
    H, N, V = shape.num_heads, shape.qk_nope, shape.v_head
    if heads is None:
        heads = list(range(H))
    W_h = W.reshape(H, N + V, W.shape[1])[heads]            # [h, N+V, R]
    kv = np.einsum("tr,hjr->thj", c_hat, W_h)               # [T, h, N+V]
    kv = kv.transpose(1, 0, 2)                              # [h, T, N+V]
    return kv[:, :, :N], kv[:, :, N:]


def apply_rope(x: np.ndarray, cos_rows: np.ndarray, sin_rows: np.ndarray,
               interleaved: bool) -> np.ndarray:
    """Rotate the rotary part ``x`` [..., P] by per-pair angles whose cosines
    and sines are ``cos_rows``/``sin_rows`` [..., P/2] (broadcast against x).

    apply_rotary_pos_emb is named by [KQ]/[ROT] and
    apply_rotary_pos_emb_interleave by [GLM]; their bodies are not shown. The
    reading used (module docstring): pair (a, b) -> (a cos - b sin,
    b cos + a sin), results written back to the pair's own slots.
    """
    P = x.shape[-1]
    out = np.array(x, dtype=np.float64, copy=True)
    if interleaved:
        a, b = x[..., 0::2], x[..., 1::2]
        out[..., 0::2] = a * cos_rows - b * sin_rows
        out[..., 1::2] = b * cos_rows + a * sin_rows
    else:
        a, b = x[..., : P // 2], x[..., P // 2:]
        out[..., : P // 2] = a * cos_rows - b * sin_rows
        out[..., P // 2:] = b * cos_rows + a * sin_rows
    return out


# --------------------------------------------------------------------------
# Causal attention -- [KQ] "Join query parts" mla-prefill; [ROT] "Key heads"
# --------------------------------------------------------------------------

def causal_attention_rows(Q: np.ndarray, K: np.ndarray, Vv: np.ndarray,
                          q_index: np.ndarray, scale: float, return_probs=False):
    """One head of the eager attention for selected query rows.

    ``Q`` [n, D] are the queries at in-sequence indices ``q_index`` [n];
    ``K`` [L, D], ``Vv`` [L, dv] are all keys/values of the sequence.
    scores = Q K^T * scale; additive mask 0 for j <= i, -inf otherwise;
    softmax over keys in float64; output = P @ V.
    """
    scores = (Q @ K.T) * scale                                   # [n, L]
    j = np.arange(K.shape[0])
    mask = np.where(j[None, :] <= q_index[:, None], 0.0, -np.inf)
    scores = scores + mask
    scores = scores - scores.max(axis=-1, keepdims=True)
    e = np.exp(scores)
    probs = e / e.sum(axis=-1, keepdims=True)
    out = probs @ Vv
    return (out, probs) if return_probs else out


def prefill(latent, q, W, w_norm, positions, cu_seqlens, cos, sin,
            shape: MlaShape, scale: float, heads=None, rows=None,
            row_chunk: int = 2048):
    """Eager MLA prefill over packed sequences; returns out [Ttot, H, V].

    Inputs (float64 arrays, upcast from whatever the device sees):
    latent [Ttot, R + P] (compressed_kv before the split), q [Ttot, H, N + P],
    W [H * (N + V), R], w_norm [R], positions [Ttot], cu_seqlens [nseq + 1],
    cos/sin [max_pos, P/2].

    Steps, per sequence ([ROT] "Key heads" mla-kv then mla-prefill; [EQ];
    [KQ] "Join query parts"):
      1. split latent into c [L, R] and k_pe [L, P];
      2. c_hat = rms_norm(c);
      3. k_nope, V per head from kv_b_proj(c_hat);
      4. rotate q_pe of every head and the one shared k_pe at ``positions``;
      5. query = [q_nope || q_pe'], key_h = [k_nope_h || k_pe'] (k_pe' is
         broadcast to every head);
      6. scores * scale, causal mask, softmax, P @ V.

    ``heads``: subset of heads to evaluate (others stay NaN).
    ``rows``: optional dict {seq index: array of in-sequence query rows};
    sequences missing from it are evaluated in full. Unevaluated rows are NaN.
    Query rows are independent outputs; they are evaluated ``row_chunk`` at
    a time only to bound memory.
    """
    H, R, N, P, V = (shape.num_heads, shape.kv_lora_rank, shape.qk_nope,
                     shape.qk_rope, shape.v_head)
    Ttot = latent.shape[0]
    if heads is None:
        heads = list(range(H))
    out = np.full((Ttot, H, V), np.nan)
    nseq = len(cu_seqlens) - 1
    for s in range(nseq):
        a, b = int(cu_seqlens[s]), int(cu_seqlens[s + 1])
        L = b - a
        if L == 0:
            continue
        c, k_pe = latent[a:b, :R], latent[a:b, R:R + P]                 # step 1
        c_hat = rms_norm(c, w_norm, shape.eps)                          # step 2
        k_nope, v = kv_up_projection(c_hat, W, shape, heads)            # step 3
        pos = positions[a:b].astype(np.int64)
        k_pe_rot = apply_rope(k_pe, cos[pos], sin[pos], shape.interleaved)  # step 4
        q_sel = q[a:b][:, heads, :]                                     # [L, h, D]
        q_pe_rot = apply_rope(q_sel[:, :, N:], cos[pos][:, None, :],
                              sin[pos][:, None, :], shape.interleaved)
        sel = np.arange(L) if rows is None or s not in rows else np.asarray(rows[s])
        for hi, h in enumerate(heads):
            Q = np.concatenate([q_sel[:, hi, :N], q_pe_rot[:, hi, :]], axis=-1)  # step 5
            K = np.concatenate([k_nope[hi], k_pe_rot], axis=-1)
            for c0 in range(0, len(sel), row_chunk):
                idx = sel[c0:c0 + row_chunk]
                out[a + idx, h, :] = causal_attention_rows(                       # step 6
                    Q[idx], K, v[hi], idx, scale)
    return out


# --------------------------------------------------------------------------
# Decode over the latent cache -- [GLM] "KV cache"; [EQ] "Read the equation"
# --------------------------------------------------------------------------

def _cache_rows(cache, cache_offsets, cache_lens, b):
    o, n = int(cache_offsets[b]), int(cache_lens[b])
    return cache[o:o + n]


def decode_eager(q, cache, cache_offsets, cache_lens, positions, W, cos, sin,
                 shape: MlaShape, scale: float, batches=None, heads=None):
    """One query token per sequence over a latent cache, eager form.

    ``cache`` rows are [c_hat (R) || k_pe rotated (P)]; sequence b owns rows
    ``cache_offsets[b] .. cache_offsets[b] + cache_lens[b] - 1``. Following
    the GLM-5 "KV cache" section, k_nope and V of every cached row are
    expanded with kv_b_proj (expand_kv) and the cached rotated key is shared
    by all heads; the query's rotary part is turned at ``positions[b]``; all
    cached rows are attended (each precedes the query). Returns [B, H, V]
    (NaN where not evaluated).
    """
    H, R, N, V = shape.num_heads, shape.kv_lora_rank, shape.qk_nope, shape.v_head
    B = q.shape[0]
    batches = list(range(B)) if batches is None else batches
    heads = list(range(H)) if heads is None else heads
    out = np.full((B, H, V), np.nan)
    for b in batches:
        rows = _cache_rows(cache, cache_offsets, cache_lens, b)
        c_hat, k_rot = rows[:, :R], rows[:, R:]
        k_nope, v = kv_up_projection(c_hat, W, shape, heads)
        p = int(positions[b])
        q_pe_rot = apply_rope(q[b][heads, N:], cos[p][None, :], sin[p][None, :],
                              shape.interleaved)
        for hi, h in enumerate(heads):
            Q = np.concatenate([q[b, h, :N], q_pe_rot[hi]])
            K = np.concatenate([k_nope[hi], k_rot], axis=-1)
            s = (K @ Q) * scale
            s = s - s.max()
            e = np.exp(s)
            out[b, h] = (e / e.sum()) @ v[hi]
    return out


def decode_absorbed(q, cache, cache_offsets, cache_lens, positions, W, cos, sin,
                    shape: MlaShape, scale: float, batches=None, heads=None):
    """The same decode in absorbed form ([EQ] "Read the equation" contrasts
    the eager expansion with an absorbed path that contracts the projection
    weights with queries and latent aggregates).

    With W_UK_h = W[h(N+V) : h(N+V)+N] ([N, R]) and
    W_UV_h = W[h(N+V)+N : (h+1)(N+V)] ([V, R]):
      q_lat = W_UK_h^T q_nope;  s_t = scale (q_lat . c_hat_t + q_pe' . k_rot_t);
      o_lat = sum_t softmax(s)_t c_hat_t;  out = W_UV_h o_lat.
    Equal to ``decode_eager`` up to rounding.
    """
    H, R, N, V = shape.num_heads, shape.kv_lora_rank, shape.qk_nope, shape.v_head
    B = q.shape[0]
    batches = list(range(B)) if batches is None else batches
    heads = list(range(H)) if heads is None else heads
    Wh = W.reshape(H, N + V, R)[heads]
    W_UK, W_UV = Wh[:, :N, :], Wh[:, N:, :]                  # [h, N, R], [h, V, R]
    out = np.full((B, H, V), np.nan)
    for b in batches:
        rows = _cache_rows(cache, cache_offsets, cache_lens, b)
        c_hat, k_rot = rows[:, :R], rows[:, R:]
        p = int(positions[b])
        q_lat = np.einsum("hnr,hn->hr", W_UK, q[b, heads, :N])          # [h, R]
        q_pe_rot = apply_rope(q[b, heads, N:], cos[p][None, :], sin[p][None, :],
                              shape.interleaved)                         # [h, P]
        s = (c_hat @ q_lat.T + k_rot @ q_pe_rot.T) * scale               # [L, h]
        s = s - s.max(axis=0, keepdims=True)
        e = np.exp(s)
        probs = e / e.sum(axis=0, keepdims=True)                         # softmax over rows
        o_lat = probs.T @ c_hat                                          # [h, R]
        out[b, heads] = np.einsum("hvr,hr->hv", W_UV, o_lat)
    return out


def cache_append(latent, w_norm, positions, cos, sin, shape: MlaShape):
    """Cache rows for new tokens ([GLM] "KV cache" and "Key-value
    compression"): the latent is normalized (k_pass = kv_a_layernorm(kv_pass))
    and the shared rotary key is rotated at its position before both go into
    the cache. ``latent`` [n, R + P] -> [n, R + P]."""
    R = shape.kv_lora_rank
    c_hat = rms_norm(latent[:, :R], w_norm, shape.eps)
    pos = np.asarray(positions).astype(np.int64)
    k_rot = apply_rope(latent[:, R:], cos[pos], sin[pos], shape.interleaved)
    return np.concatenate([c_hat, k_rot], axis=-1)


def prefill_cached(latent, q, cache, cache_offsets, prefix_lens, cu_seqlens, W, w_norm,
                   cos, sin, shape: MlaShape, scale: float, heads=None):
    """A chunk of new tokens per sequence, continuing a latent cache.

    Sequence s owns cache rows ``cache_offsets[s]`` onwards; the first
    ``prefix_lens[s]`` of them are cached already. Its chunk is rows
    ``cu_seqlens[s] .. cu_seqlens[s+1] - 1`` of ``latent`` [Tq, R + P] (raw
    compressed_kv) and ``q`` [Tq, H, N + P].

    Steps per sequence, in the order of the [GLM] "KV cache" section:
      1. the chunk's cache rows, cache_append at positions p .. p + n - 1,
         are written to the sequence's rows p .. p + n - 1;
      2. k_nope and V of every cached row 0 .. p + n - 1 are expanded with
         kv_b_proj (expand_kv); the cached rotated key is shared by all heads;
      3. q_pe of chunk token i is rotated at position p + i;
      4. scores * scale, causal mask in absolute positions (token i sees
         cached rows j <= p + i), softmax, P @ V.

    Returns (out [Tq, H, V], the cache after step 1). ``heads``: subset of
    heads to evaluate (others stay NaN). The input cache is not modified.
    """
    H, R, N, V = shape.num_heads, shape.kv_lora_rank, shape.qk_nope, shape.v_head
    Tq = latent.shape[0]
    heads = list(range(H)) if heads is None else heads
    cache = np.array(cache, dtype=np.float64, copy=True)
    out = np.full((Tq, H, V), np.nan)
    for s in range(len(cu_seqlens) - 1):
        a, b = int(cu_seqlens[s]), int(cu_seqlens[s + 1])
        n, p, o = b - a, int(prefix_lens[s]), int(cache_offsets[s])
        if n == 0:
            continue
        pos = p + np.arange(n)
        cache[o + p:o + p + n] = cache_append(latent[a:b], w_norm, pos, cos, sin, shape)  # step 1
        rows = cache[o:o + p + n]
        c_hat, k_rot = rows[:, :R], rows[:, R:]
        k_nope, v = kv_up_projection(c_hat, W, shape, heads)                             # step 2
        q_sel = q[a:b][:, heads, :]
        q_pe_rot = apply_rope(q_sel[:, :, N:], cos[pos][:, None, :], sin[pos][:, None, :],
                              shape.interleaved)                                          # step 3
        for hi, h in enumerate(heads):
            Q = np.concatenate([q_sel[:, hi, :N], q_pe_rot[:, hi, :]], axis=-1)
            K = np.concatenate([k_nope[hi], k_rot], axis=-1)
            out[a:b, h, :] = causal_attention_rows(Q, K, v[hi], pos, scale)              # step 4
    return out, cache


# --------------------------------------------------------------------------
# Projections on either side of the path -- [ROT] "Query heads" mla-init and
# mla-queries, "Key heads" mla-kv
# --------------------------------------------------------------------------

def kv_down_projection(hidden, W_kva):
    """kv_a_proj_with_mqa: hidden [n, hidden_size] -> compressed_kv
    [n, R + P] = hidden @ W_kva.T, with W_kva the nn.Linear weight
    [R + P, hidden_size]. Its first R columns are the latent that
    kv_a_layernorm normalizes; the last P are the shared rotary key."""
    return hidden @ W_kva.T


def q_projection(hidden, W_qa, w_qnorm, W_qb, shape: MlaShape):
    """q = q_b_proj(q_a_layernorm(q_a_proj(hidden))), viewed [n, H, N + P].

    W_qa [q_rank, hidden_size], w_qnorm [q_rank] (an RMSNorm over the query
    rank, the same normalization as kv_a_layernorm), W_qb [H * (N + P),
    q_rank]; the view is q.view(bsz, q_len, H, q_head_dim) of mla-queries."""
    q_a = hidden @ W_qa.T
    q_an = rms_norm(q_a, w_qnorm, shape.eps)
    q = q_an @ W_qb.T
    return q.reshape(hidden.shape[0], shape.num_heads, shape.qk_head_dim)


def o_projection(attn, W_o):
    """o_proj: the attention output [n, H * V] (heads joined, as the path
    writes it) -> [n, hidden_size] = attn @ W_o.T, W_o [hidden_size, H * V]."""
    return attn @ W_o.T
