"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: values the
pages print (tests/golden/page_facts.txt), closed forms evaluated another way,
invariants, special cases that reduce to a library routine, and a brute-force
restatement written independently with explicit loops.
"""

import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def page_facts():
    facts = {}
    with open(os.path.join(GOLDEN, "page_facts.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = line.split()
                facts[k] = float(v)
    return facts


KIMI = O.RopeConfig(rope_dim=64, base=50000.0, yarn=True, factor=32.0, original_max_pos=4096,
                    beta_fast=32.0, beta_slow=1.0, mscale=1.0, mscale_all_dim=1.0)
GLM = O.RopeConfig(rope_dim=64, base=10000.0)


# ---------------------------------------------------------------- YaRN closed forms

@pytest.mark.parametrize("rot", [0.5, 1.0, 3.0, 32.0])
@pytest.mark.parametrize("base,maxpos", [(50000.0, 4096), (10000.0, 2048)])
def test_correction_dim_is_where_pair_turns_n_times(rot, base, maxpos):
    # Meaning of the closed form: pair index d (frequency base^(-2d/dim)) makes
    # exactly `rot` full turns over `maxpos` positions.
    dim = 64
    d = O.yarn_find_correction_dim(rot, dim, base, maxpos)
    turns = maxpos * base ** (-2.0 * d / dim) / (2 * math.pi)
    assert turns == pytest.approx(rot, rel=1e-12)


def test_correction_range_kimi_values():
    # beta_fast = 32 turns -> d = 8.91..., beta_slow = 1 turn -> d = 19.16...
    # (by hand: 64 ln(4096 / (2 pi r)) / (2 ln 50000)); floor/ceil give [8, 20].
    lo, hi = O.yarn_find_correction_range(32, 1, 64, 50000.0, 4096)
    assert (lo, hi) == (8, 20)


def test_correction_range_clamps():
    # A bound beyond the dimension range clamps to [0, dim - 1].
    lo, hi = O.yarn_find_correction_range(1e6, 1e-6, 64, 10000.0, 4096)
    assert lo == 0 and hi == 63


def test_mscale_closed_form():
    assert O.yarn_get_mscale(1.0, 5.0) == 1.0          # no correction at scale <= 1
    assert O.yarn_get_mscale(0.5, 5.0) == 1.0
    assert O.yarn_get_mscale(math.e, 1.0) == pytest.approx(1.1, abs=1e-15)
    assert O.yarn_get_mscale(math.e ** 10, 0.5) == pytest.approx(1.5, abs=1e-14)
    # Kimi: factor 32, ln 32 = 5 ln 2
    assert O.yarn_get_mscale(32.0, 1.0) == pytest.approx(1.0 + 0.5 * math.log(2.0), abs=1e-15)


def test_softmax_scale_page_values():
    f = page_facts()
    # GLM-5: printed 1/sqrt(256) with no YaRN correction under default RoPE.
    assert O.softmax_scale(GLM, int(f["glm5_qk_head_dim"])) == f["glm5_softmax_scale"]
    # Kimi-K2: 1/sqrt(192) times the square of the correction (1 + 0.5 ln 2).
    m = 1.0 + 0.5 * math.log(2.0)
    s = O.softmax_scale(KIMI, int(f["kimi_qk_head_dim"]))
    assert s == pytest.approx(m * m / math.sqrt(192.0), rel=1e-15)
    # mscale_all_dim = 0 switches the correction off.
    no_all = O.RopeConfig(rope_dim=64, base=50000.0, yarn=True, factor=32.0, mscale_all_dim=0.0)
    assert O.softmax_scale(no_all, 192) == pytest.approx(192 ** -0.5, rel=1e-15)


def test_yarn_defaults_match_page():
    f = page_facts()
    d = O.RopeConfig(rope_dim=64, base=10000.0, yarn=True)
    assert d.original_max_pos == f["yarn_default_original_max_pos"]
    assert d.beta_fast == f["yarn_default_beta_fast"]
    assert d.beta_slow == f["yarn_default_beta_slow"]
    assert d.mscale == f["yarn_default_mscale"]
    assert d.mscale_all_dim == f["yarn_default_mscale_all_dim"]


def test_ramp():
    r = O.yarn_linear_ramp_mask(8, 20, 32)
    assert r[:9].tolist() == [0.0] * 9
    assert r[20:].tolist() == [1.0] * 12
    assert r[14] == pytest.approx(0.5, abs=1e-15)
    assert np.all(np.diff(r) >= 0)
    s = O.yarn_linear_ramp_mask(5, 5, 8)     # coincident bounds: max nudged by 0.001
    assert s[5] == 0.0 and s[6] == 1.0 and s[4] == 0.0


def test_inv_freq_default_and_yarn_blend():
    i = np.arange(32)
    base_freq = 50000.0 ** (-2.0 * i / 64)
    inv = O.rope_inv_freq(KIMI)
    # high-frequency pairs (ramp 0) keep the original frequency ...
    np.testing.assert_allclose(inv[:9], base_freq[:9], rtol=1e-15)
    # ... low-frequency pairs (ramp 1) are interpolated by the factor ...
    np.testing.assert_allclose(inv[20:], base_freq[20:] / 32.0, rtol=1e-15)
    # ... and pair 14 (ramp 1/2) sits halfway between the two.
    assert inv[14] == pytest.approx(base_freq[14] * (0.5 + 0.5 / 32.0), rel=1e-15)
    assert inv[0] == 1.0
    np.testing.assert_allclose(O.rope_inv_freq(GLM), 10000.0 ** (-2.0 * i / 64), rtol=1e-15)


def test_rope_table_properties():
    f = page_facts()
    cos, sin = O.rope_tables(KIMI, 4096)
    assert cos.shape == (4096, int(f["kimi_rope_pairs"]))
    assert O.rope_table_mscale(KIMI) == 1.0            # mscale == mscale_all_dim
    np.testing.assert_array_equal(cos[0], 1.0)
    np.testing.assert_array_equal(sin[0], 0.0)
    np.testing.assert_allclose(cos ** 2 + sin ** 2, 1.0, atol=1e-14)
    # angle addition: row p+q from rows p and q
    p, q = 1000, 777
    np.testing.assert_allclose(cos[p + q], cos[p] * cos[q] - sin[p] * sin[q], atol=1e-12)
    np.testing.assert_allclose(sin[p + q], sin[p] * cos[q] + cos[p] * sin[q], atol=1e-12)
    # table mscale when mscale differs from mscale_all_dim
    odd = O.RopeConfig(rope_dim=64, base=50000.0, yarn=True, factor=32.0, mscale=1.0,
                       mscale_all_dim=0.0)
    c2, s2 = O.rope_tables(odd, 8)
    m = 1.0 + 0.5 * math.log(2.0)
    np.testing.assert_allclose(c2 ** 2 + s2 ** 2, m * m, rtol=1e-14)


# ---------------------------------------------------------------- RoPE apply

@pytest.mark.parametrize("interleaved", [False, True])
def test_rope_norm_identity_and_relative(interleaved):
    rng = np.random.default_rng(0)
    P = 64
    cos, sin = O.rope_tables(KIMI, 3000)
    x = rng.standard_normal(P)
    y = rng.standard_normal(P)
    # position 0 is the identity
    np.testing.assert_array_equal(O.apply_rope(x, cos[0], sin[0], interleaved), x)
    # pair norms preserved
    r = O.apply_rope(x, cos[1234], sin[1234], interleaved)
    if interleaved:
        pa, pr = x[0::2] ** 2 + x[1::2] ** 2, r[0::2] ** 2 + r[1::2] ** 2
    else:
        pa, pr = x[:32] ** 2 + x[32:] ** 2, r[:32] ** 2 + r[32:] ** 2
    np.testing.assert_allclose(pr, pa, rtol=1e-12)
    # q(m) . k(n) depends on m - n only
    def dot(m, n):
        return O.apply_rope(x, cos[m], sin[m], interleaved) @ O.apply_rope(y, cos[n], sin[n], interleaved)
    assert dot(900, 100) == pytest.approx(dot(2900, 2100), rel=1e-10)
    assert dot(5, 5) == pytest.approx(x @ y, rel=1e-12)


@pytest.mark.parametrize("interleaved", [False, True])
def test_rope_quarter_turn_direction_and_pairing(interleaved):
    # A quarter turn on pair 3 must send (a, b) to (-b, a) (counter-clockwise),
    # touch only that pair, and use the pairing of the reading.
    P = 16
    cos = np.ones(P // 2)
    sin = np.zeros(P // 2)
    cos[3], sin[3] = 0.0, 1.0
    x = np.arange(1.0, P + 1.0)
    r = O.apply_rope(x, cos, sin, interleaved)
    ia, ib = (6, 7) if interleaved else (3, 11)
    expect = x.copy()
    expect[ia], expect[ib] = -x[ib], x[ia]
    np.testing.assert_array_equal(r, expect)


# ---------------------------------------------------------------- RMSNorm, projection

def test_rmsnorm_constant_and_known_vector():
    R = 512
    w = np.linspace(0.5, 1.5, R)
    for a in (-3.0, 0.01, 7.5):
        y = O.rms_norm(np.full(R, a), w, 1e-6)
        np.testing.assert_allclose(y, w * a / math.sqrt(a * a + 1e-6), rtol=1e-14)
    # [3, 4, 0, ...]: mean square 25 / R
    x = np.zeros(R)
    x[0], x[1] = 3.0, 4.0
    y = O.rms_norm(x, np.ones(R), 0.0)
    assert y[0] == pytest.approx(3.0 / math.sqrt(25.0 / R), rel=1e-14)
    assert y[1] == pytest.approx(4.0 / math.sqrt(25.0 / R), rel=1e-14)
    # eps is the page's default
    assert page_facts()["eps"] == 1e-6


def test_kv_up_projection_layout():
    # With W a row selection (row o picks latent column (o * 7) mod R), the
    # projection output channel o = h (N+V) + j must land in k_nope[h, :, j]
    # for j < N and in V[h, :, j - N] otherwise.
    H, R, N, V = 3, 32, 4, 5
    shape = O.MlaShape(H, R, N, 2, V)
    W = np.zeros((H * (N + V), R))
    for o in range(H * (N + V)):
        W[o, (o * 7) % R] = 1.0
    c = np.random.default_rng(1).standard_normal((6, R))
    kn, v = O.kv_up_projection(c, W, shape)
    assert kn.shape == (H, 6, N) and v.shape == (H, 6, V)
    for h in range(H):
        for j in range(N + V):
            col = c[:, ((h * (N + V) + j) * 7) % R]
            got = kn[h, :, j] if j < N else v[h, :, j - N]
            np.testing.assert_array_equal(got, col)
    kn2, v2 = O.kv_up_projection(c, W, shape, heads=[2, 0])
    np.testing.assert_array_equal(kn2[0], kn[2])
    np.testing.assert_array_equal(v2[1], v[0])


# ---------------------------------------------------------------- attention

def test_softmax_rows_sum_to_one_and_first_row():
    rng = np.random.default_rng(2)
    L, D, dv = 37, 12, 5
    Q, K, V = rng.standard_normal((L, D)), rng.standard_normal((L, D)), rng.standard_normal((L, dv))
    out, probs = O.causal_attention_rows(Q, K, V, np.arange(L), 0.3, return_probs=True)
    np.testing.assert_allclose(probs.sum(-1), 1.0, atol=1e-14)
    assert np.all(np.triu(probs, 1) == 0.0)          # nothing above the diagonal
    np.testing.assert_array_equal(out[0], V[0])      # first causal row returns v0


def _small_case(seqlens, H=3, R=16, N=8, P=4, V=6, interleaved=False, seed=0, rope=None):
    rng = np.random.default_rng(seed)
    T = sum(seqlens)
    shape = O.MlaShape(H, R, N, P, V, interleaved=interleaved)
    rope = rope or O.RopeConfig(rope_dim=P, base=10000.0)
    d = dict(latent=rng.standard_normal((T, R + P)), q=rng.standard_normal((T, H, N + P)),
             W=rng.standard_normal((H * (N + V), R)) / math.sqrt(R),
             w_norm=1 + 0.1 * rng.standard_normal(R),
             positions=np.concatenate([np.arange(L) for L in seqlens]),
             cu=np.concatenate([[0], np.cumsum(seqlens)]))
    cos, sin = O.rope_tables(rope, max(seqlens) + 2)
    return shape, rope, d, cos, sin


def test_positions_zero_reduces_to_sdpa():
    # With every position 0 the rotation is the identity and the path is
    # plain causal scaled-dot-product attention on [q_nope||q_pe] and
    # [k_nope||k_pe]: compare with torch's SDPA in float64 on the CPU.
    shape, rope, d, cos, sin = _small_case([19])
    T, H, N, R = 19, shape.num_heads, shape.qk_nope, shape.kv_lora_rank
    pos0 = np.zeros(T, dtype=np.int64)
    scale = 0.37
    out = O.prefill(d["latent"], d["q"], d["W"], d["w_norm"], pos0, d["cu"], cos, sin, shape, scale)
    c_hat = O.rms_norm(d["latent"][:, :R], d["w_norm"], shape.eps)
    kn, v = O.kv_up_projection(c_hat, d["W"], shape)
    k = np.concatenate([kn, np.broadcast_to(d["latent"][None, :, R:], (H, T, shape.qk_rope))], -1)
    qq = d["q"].transpose(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qq), torch.from_numpy(np.ascontiguousarray(k)), torch.from_numpy(v),
        is_causal=True, scale=scale).numpy()
    np.testing.assert_allclose(out, ref.transpose(1, 0, 2), rtol=1e-12, atol=1e-12)


def _brute_force_prefill(latent, q, W, w_norm, positions, cu, inv_freq, shape, scale):
    """Independent restatement with explicit Python loops and an explicit
    [L, L] mask matrix (default-RoPE tables built from inv_freq inline)."""
    H, R, N, P, V = shape.num_heads, shape.kv_lora_rank, shape.qk_nope, shape.qk_rope, shape.v_head
    T = latent.shape[0]
    out = np.zeros((T, H, V))

    def rot(vec, pos):
        res = list(vec)
        for i in range(P // 2):
            a_i, b_i = (2 * i, 2 * i + 1) if shape.interleaved else (i, i + P // 2)
            ang = pos * inv_freq[i]
            res[a_i] = vec[a_i] * math.cos(ang) - vec[b_i] * math.sin(ang)
            res[b_i] = vec[b_i] * math.cos(ang) + vec[a_i] * math.sin(ang)
        return res

    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        L = b - a
        chat = []
        for t in range(a, b):
            ms = sum(latent[t, k] ** 2 for k in range(R)) / R
            chat.append([w_norm[k] * latent[t, k] / math.sqrt(ms + shape.eps) for k in range(R)])
        kpe = [rot(latent[t, R:], positions[t]) for t in range(a, b)]
        mask = [[0.0 if j <= i else -math.inf for j in range(L)] for i in range(L)]
        for h in range(H):
            K, Vh = [], []
            for t in range(L):
                kv = [sum(chat[t][k] * W[h * (N + V) + j, k] for k in range(R)) for j in range(N + V)]
                K.append(kv[:N] + kpe[t])
                Vh.append(kv[N:])
            for i in range(L):
                qi = list(q[a + i, h, :N]) + rot(q[a + i, h, N:], positions[a + i])
                sc = [sum(qi[x] * K[j][x] for x in range(N + P)) * scale + mask[i][j] for j in range(L)]
                m = max(sc)
                e = [math.exp(x - m) for x in sc]
                z = sum(e)
                for c in range(V):
                    out[a + i, h, c] = sum(e[j] / z * Vh[j][c] for j in range(L))
    return out


@pytest.mark.parametrize("interleaved", [False, True])
def test_brute_force_agreement(interleaved):
    seqlens = [5, 1, 7]
    shape, rope, d, cos, sin = _small_case(seqlens, H=2, R=8, N=4, P=4, V=3,
                                           interleaved=interleaved, seed=3)
    scale = 0.41
    out = O.prefill(d["latent"], d["q"], d["W"], d["w_norm"], d["positions"], d["cu"],
                    cos, sin, shape, scale)
    inv = [10000.0 ** (-2.0 * i / 4) for i in range(2)]
    ref = _brute_force_prefill(d["latent"], d["q"], d["W"], d["w_norm"], d["positions"],
                               d["cu"], inv, shape, scale)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_varlen_packing_invariance_and_first_rows():
    seqlens = [9, 4, 13]
    shape, rope, d, cos, sin = _small_case(seqlens, seed=4)
    scale = 0.3
    packed = O.prefill(d["latent"], d["q"], d["W"], d["w_norm"], d["positions"], d["cu"],
                       cos, sin, shape, scale)
    R = shape.kv_lora_rank
    for s in range(3):
        a, b = d["cu"][s], d["cu"][s + 1]
        alone = O.prefill(d["latent"][a:b], d["q"][a:b], d["W"], d["w_norm"],
                          d["positions"][a:b], np.array([0, b - a]), cos, sin, shape, scale)
        np.testing.assert_allclose(packed[a:b], alone, rtol=1e-13, atol=1e-14)
        # the first row of each sequence returns that sequence's v0
        c_hat = O.rms_norm(d["latent"][a:a + 1, :R], d["w_norm"], shape.eps)
        _, v = O.kv_up_projection(c_hat, d["W"], shape)
        np.testing.assert_allclose(packed[a], v[:, 0, :], rtol=1e-13, atol=1e-14)


def test_row_and_head_subsets_match_full():
    seqlens = [21]
    shape, rope, d, cos, sin = _small_case(seqlens, seed=5)
    full = O.prefill(d["latent"], d["q"], d["W"], d["w_norm"], d["positions"], d["cu"],
                     cos, sin, shape, 0.5)
    part = O.prefill(d["latent"], d["q"], d["W"], d["w_norm"], d["positions"], d["cu"],
                     cos, sin, shape, 0.5, heads=[2], rows={0: np.array([0, 7, 20])}, row_chunk=2)
    np.testing.assert_allclose(part[[0, 7, 20], 2], full[[0, 7, 20], 2], rtol=1e-14, atol=1e-15)
    assert np.isnan(part[1, 2]).all() and np.isnan(part[0, 0]).all()


# ---------------------------------------------------------------- decode

@pytest.mark.parametrize("interleaved", [False, True])
def test_decode_equals_last_prefill_row(interleaved):
    # A sequence of L+1 tokens: the prefill output of its last token equals a
    # decode step whose cache holds all L+1 appended rows (normalized latent,
    # rotated key) and whose query sits at position L.
    rope = O.RopeConfig(rope_dim=8, base=50000.0, yarn=True, factor=4.0, original_max_pos=16,
                        mscale=1.0, mscale_all_dim=1.0)
    seqlens = [12, 30]
    shape, rope, d, cos, sin = _small_case(seqlens, H=4, R=32, N=8, P=8, V=8,
                                           interleaved=interleaved, seed=6, rope=rope)
    scale = O.softmax_scale(rope, shape.qk_head_dim)
    pre = O.prefill(d["latent"], d["q"], d["W"], d["w_norm"], d["positions"], d["cu"],
                    cos, sin, shape, scale)
    cache = O.cache_append(d["latent"], d["w_norm"], d["positions"], cos, sin, shape)
    offs = d["cu"][:-1]
    lens = np.array(seqlens)
    last = d["cu"][1:] - 1
    qd = d["q"][last]
    pos = d["positions"][last]
    dec = O.decode_eager(qd, cache, offs, lens, pos, d["W"], cos, sin, shape, scale)
    np.testing.assert_allclose(dec, pre[last], rtol=1e-12, atol=1e-13)
    absd = O.decode_absorbed(qd, cache, offs, lens, pos, d["W"], cos, sin, shape, scale)
    np.testing.assert_allclose(absd, dec, rtol=1e-10, atol=1e-12)


def test_absorbed_equals_eager_kimi_geometry():
    rng = np.random.default_rng(7)
    shape = O.MlaShape(4, 512, 128, 64, 128)
    lens = np.array([50, 333])
    offs = np.array([0, 50])
    cache = rng.standard_normal((lens.sum(), 576))
    q = rng.standard_normal((2, 4, 192))
    W = rng.standard_normal((4 * 256, 512)) / math.sqrt(512)
    cos, sin = O.rope_tables(KIMI, 400)
    scale = O.softmax_scale(KIMI, 192)
    e = O.decode_eager(q, cache, offs, lens, lens, W, cos, sin, shape, scale)
    a = O.decode_absorbed(q, cache, offs, lens, lens, W, cos, sin, shape, scale)
    assert np.abs(a - e).max() <= 1e-10 * np.abs(e).max()


def test_cache_append_row():
    rng = np.random.default_rng(8)
    shape = O.MlaShape(2, 16, 4, 4, 4)
    x = rng.standard_normal((3, 20))
    w = np.ones(16)
    cos, sin = O.rope_tables(O.RopeConfig(rope_dim=4, base=10000.0), 10)
    rows = O.cache_append(x, w, [0, 3, 9], cos, sin, shape)
    np.testing.assert_allclose(np.mean(rows[:, :16] ** 2, -1), np.mean(x[:, :16] ** 2, -1)
                               / (np.mean(x[:, :16] ** 2, -1) + 1e-6), rtol=1e-13)
    np.testing.assert_array_equal(rows[0, 16:], x[0, 16:])       # position 0: unrotated
    np.testing.assert_allclose(np.linalg.norm(rows[:, 16:], axis=-1),
                               np.linalg.norm(x[:, 16:], axis=-1), rtol=1e-13)


# ---------------------------------------------------------------- chunks over a cached prefix

def _chunked_inputs(seqlens, splits, gap=3, **kw):
    """A small case whose sequences are cut at ``splits`` (cached prefix
    length per sequence). The cache holds each sequence in its own region,
    ``gap`` unused rows apart, so offsets are not a packed prefix sum."""
    shape, rope, d, cos, sin = _small_case(seqlens, **kw)
    offs = np.zeros(len(seqlens), dtype=np.int64)
    for s in range(1, len(seqlens)):
        offs[s] = offs[s - 1] + seqlens[s - 1] + gap
    rows = int(offs[-1] + seqlens[-1] + gap)
    return shape, rope, d, cos, sin, offs, rows


_YARN_SMALL = O.RopeConfig(rope_dim=4, base=50000.0, yarn=True, factor=4.0, original_max_pos=8,
                           mscale=0.9, mscale_all_dim=0.5)


@pytest.mark.parametrize("rope", [None, _YARN_SMALL], ids=["default_rope", "yarn"])
@pytest.mark.parametrize("interleaved", [False, True])
def test_prefill_cached_two_chunks_equal_one_prefill(interleaved, rope):
    # Splitting each sequence into a cached prefix and a chunk changes nothing:
    # chunk 1 (empty prefix) and chunk 2 (prefix = chunk 1) together give the
    # prefill of the whole sequence. An error in the chunk's positions, its
    # cache rows or the offset of the causal mask breaks this.
    seqlens, splits = [11, 6, 17], [4, 0, 16]
    shape, rope, d, cos, sin, offs, nrows = _chunked_inputs(seqlens, splits, H=3, R=16, N=8, P=4, V=6,
                                                            interleaved=interleaved, seed=21, rope=rope)
    scale = 0.35
    full = O.prefill(d["latent"], d["q"], d["W"], d["w_norm"], d["positions"], d["cu"], cos, sin, shape, scale)
    cu = d["cu"]
    idx1 = np.concatenate([np.arange(cu[s], cu[s] + splits[s]) for s in range(3)])
    idx2 = np.concatenate([np.arange(cu[s] + splits[s], cu[s + 1]) for s in range(3)])
    cu1 = np.concatenate([[0], np.cumsum(splits)])
    cu2 = np.concatenate([[0], np.cumsum(np.array(seqlens) - np.array(splits))])
    cache0 = np.full((nrows, shape.kv_lora_rank + shape.qk_rope), 7.5)
    out1, cache1 = O.prefill_cached(d["latent"][idx1], d["q"][idx1], cache0, offs, np.zeros(3, int), cu1,
                                    d["W"], d["w_norm"], cos, sin, shape, scale)
    out2, cache2 = O.prefill_cached(d["latent"][idx2], d["q"][idx2], cache1, offs, np.array(splits), cu2,
                                    d["W"], d["w_norm"], cos, sin, shape, scale)
    np.testing.assert_allclose(out1, full[idx1], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(out2, full[idx2], rtol=1e-12, atol=1e-13)
    # every sequence's region now holds its whole cache; the gaps are untouched
    appended = O.cache_append(d["latent"], d["w_norm"], d["positions"], cos, sin, shape)
    used = np.zeros(nrows, bool)
    for s in range(3):
        np.testing.assert_allclose(cache2[offs[s]:offs[s] + seqlens[s]], appended[cu[s]:cu[s + 1]], rtol=1e-15)
        used[offs[s]:offs[s] + seqlens[s]] = True
    assert np.all(cache2[~used] == 7.5) and np.all(cache0 == 7.5)


def test_prefill_cached_last_token_is_a_decode_step():
    # The chunk's last token attends to all p + n cached rows from position
    # p + n - 1: a decode step over the updated cache at that position.
    seqlens, splits = [9, 14], [5, 2]
    shape, rope, d, cos, sin, offs, nrows = _chunked_inputs(seqlens, splits, seed=22)
    scale = 0.3
    cu = d["cu"]
    pre = O.cache_append(d["latent"], d["w_norm"], d["positions"], cos, sin, shape)
    cache = np.zeros((nrows, pre.shape[1]))
    for s in range(2):
        cache[offs[s]:offs[s] + splits[s]] = pre[cu[s]:cu[s] + splits[s]]
    idx = np.concatenate([np.arange(cu[s] + splits[s], cu[s + 1]) for s in range(2)])
    cuq = np.concatenate([[0], np.cumsum(np.array(seqlens) - np.array(splits))])
    out, after = O.prefill_cached(d["latent"][idx], d["q"][idx], cache, offs, np.array(splits), cuq,
                                  d["W"], d["w_norm"], cos, sin, shape, scale)
    last = cuq[1:] - 1
    lens = np.array(seqlens)
    dec = O.decode_eager(d["q"][idx][last], after, offs, lens, lens - 1, d["W"], cos, sin, shape, scale)
    np.testing.assert_allclose(out[last], dec, rtol=1e-12, atol=1e-13)


def test_prefill_cached_without_prefix_is_prefill():
    seqlens = [7, 1, 12]
    shape, rope, d, cos, sin, offs, nrows = _chunked_inputs(seqlens, [0, 0, 0], interleaved=True, seed=23)
    scale = 0.45
    full = O.prefill(d["latent"], d["q"], d["W"], d["w_norm"], d["positions"], d["cu"], cos, sin, shape, scale)
    out, _ = O.prefill_cached(d["latent"], d["q"], np.zeros((nrows, shape.kv_lora_rank + shape.qk_rope)), offs,
                              np.zeros(3, int), d["cu"], d["W"], d["w_norm"], cos, sin, shape, scale)
    np.testing.assert_allclose(out, full, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- projections on either side

def _loop_linear(x, W):
    """x @ W.T with explicit loops (independent of numpy's matmul)."""
    out = np.zeros((x.shape[0], W.shape[0]))
    for t in range(x.shape[0]):
        for j in range(W.shape[0]):
            out[t, j] = math.fsum(x[t, k] * W[j, k] for k in range(x.shape[1]))
    return out


def test_projections_against_loops():
    rng = np.random.default_rng(31)
    shape = O.MlaShape(2, 8, 4, 2, 3)
    hid, qr = 12, 5
    x = rng.standard_normal((3, hid))
    W_kva = rng.standard_normal((8 + 2, hid))
    np.testing.assert_allclose(O.kv_down_projection(x, W_kva), _loop_linear(x, W_kva), rtol=1e-13, atol=1e-13)
    W_qa, W_qb = rng.standard_normal((qr, hid)), rng.standard_normal((2 * 6, qr))
    w_qn = 1 + 0.1 * rng.standard_normal(qr)
    qa = _loop_linear(x, W_qa)
    qan = np.array([[w_qn[k] * qa[t, k] / math.sqrt(sum(v * v for v in qa[t]) / qr + shape.eps)
                     for k in range(qr)] for t in range(3)])
    want = _loop_linear(qan, W_qb).reshape(3, 2, 6)
    np.testing.assert_allclose(O.q_projection(x, W_qa, w_qn, W_qb, shape), want, rtol=1e-12, atol=1e-12)
    attn = rng.standard_normal((3, 2 * 3))
    W_o = rng.standard_normal((hid, 6))
    np.testing.assert_allclose(O.o_projection(attn, W_o), _loop_linear(attn, W_o), rtol=1e-13, atol=1e-13)


def test_q_projection_layout_and_scale_invariance():
    # unit rows pick single inputs: q_a = the picked hidden values; the
    # RMSNorm makes the result independent of the hidden state's scale;
    # head h of the view is rows h*(N+P) .. (h+1)*(N+P) - 1 of W_qb
    shape = O.MlaShape(3, 8, 2, 2, 1)
    hid, qr = 10, 4
    W_qa = np.zeros((qr, hid))
    for k in range(qr):
        W_qa[k, 2 * k] = 1.0
    W_qb = np.zeros((3 * 4, qr))
    W_qb[1 * 4 + 3, 2] = 1.0                 # head 1, slot 3 <- q_an[2]
    x = np.arange(1.0, hid + 1.0)[None, :]
    q = O.q_projection(x, W_qa, np.ones(qr), W_qb, shape)
    qa = x[0, [0, 2, 4, 6]]
    expect = qa[2] / math.sqrt(np.mean(qa ** 2) + shape.eps)
    assert q.shape == (1, 3, 4)
    assert abs(q[0, 1, 3] - expect) < 1e-14 and np.count_nonzero(q) == 1
    q10 = O.q_projection(10 * x, W_qa, np.ones(qr), W_qb, shape)
    np.testing.assert_allclose(q10, q, rtol=1e-6)   # eps only breaks exact invariance


def test_kv_down_then_append_is_the_paths_cache_row():
    # compressed_kv from the down-projection, split, normalized and rotated:
    # the cache row the decode reads (GLM-5 "KV cache" order)
    rng = np.random.default_rng(32)
    shape = O.MlaShape(2, 16, 4, 4, 4)
    x = rng.standard_normal((2, 20))
    W = rng.standard_normal((20, 20)) / math.sqrt(20)
    cos, sin = O.rope_tables(O.RopeConfig(rope_dim=4, base=10000.0), 8)
    latent = O.kv_down_projection(x, W)
    rows = O.cache_append(latent, np.ones(16), [3, 5], cos, sin, shape)
    np.testing.assert_allclose(rows[:, :16], O.rms_norm(latent[:, :16], np.ones(16), shape.eps), rtol=1e-14)
    np.testing.assert_allclose(np.linalg.norm(rows[:, 16:], axis=-1), np.linalg.norm(latent[:, 16:], axis=-1),
                               rtol=1e-13)
