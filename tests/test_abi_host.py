"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before any launch."""

import ctypes
import math
import os
import re

import pytest

from decode_latent_rmsnorm_b200 import mla
import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

FAKE = ctypes.c_void_p(0x1000)   # never dereferenced: every call below fails on the host


def declared_functions():
    text = open(os.path.join(ROOT, "include", "mla.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol():
    lib = mla.load()
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
        assert n in mla.SIGNATURES, n
    assert mla.mla_version() >= 100


def kimi_dims(**kw):
    d = dict(num_heads=64, kv_lora_rank=512, qk_nope=128, qk_rope=64, v_head=128, dtype=0,
             rope_interleaved=0, eps=1e-6, softmax_scale=0.13)
    d.update(kw)
    return mla.Dims(**d)


def test_softmax_scale_matches_oracle():
    kimi = mla.RopeCfg.make(64, 50000.0, yarn=True, factor=32.0, original_max_pos=4096,
                            beta_fast=32.0, beta_slow=1.0, mscale=1.0, mscale_all_dim=1.0)
    glm = mla.RopeCfg.make(64, 10000.0)
    s = mla.mla_softmax_scale(kimi, 192)
    ref = O.softmax_scale(O.RopeConfig(64, 50000.0, True, 32.0, 4096, 32.0, 1.0, 1.0, 1.0), 192)
    assert s == pytest.approx(ref, rel=1e-7)
    assert mla.mla_softmax_scale(glm, 256) == 0.0625
    assert mla.mla_softmax_scale(mla.RopeCfg.make(8, 10000.0), 24) == pytest.approx(24 ** -0.5, rel=1e-7)


def test_rope_config_rejections():
    with pytest.raises(mla.MlaError) as e:
        mla.mla_softmax_scale(mla.RopeCfg.make(63, 10000.0), 128)
    assert e.value.status == 1
    with pytest.raises(mla.MlaError):
        mla.mla_softmax_scale(mla.RopeCfg.make(64, 1.0), 128)
    with pytest.raises(mla.MlaError):
        mla.mla_softmax_scale(mla.RopeCfg.make(64, 10000.0, yarn=True, factor=-1.0), 128)
    lib = mla.load()
    assert lib.mla_init_rope_tables(ctypes.byref(mla.RopeCfg.make(64, 1e4)), 0, FAKE, FAKE, None) == 1
    assert lib.mla_init_rope_tables(ctypes.byref(mla.RopeCfg.make(64, 1e4)), 8, None, FAKE, None) == 1


def _prefill(lib, dims, **over):
    a = dict(latent=FAKE, q=FAKE, w=FAKE, wn=FAKE, pos=FAKE, cu=FAKE, nseq=1, maxlen=16, T=16,
             cos=FAKE, sin=FAKE, maxpos=16, out=FAKE, ws=FAKE, wsb=1 << 40)
    a.update(over)
    return lib.mla_prefill(ctypes.byref(dims) if dims is not None else None, a["latent"], a["q"], a["w"],
                           a["wn"], a["pos"], a["cu"], a["nseq"], a["maxlen"], a["T"], a["cos"],
                           a["sin"], a["maxpos"], a["out"], a["ws"], a["wsb"], None)


def test_prefill_host_validation():
    lib = mla.load()
    assert _prefill(lib, None) == 1
    assert _prefill(lib, kimi_dims(dtype=7)) == 1
    assert _prefill(lib, kimi_dims(qk_rope=63)) == 1
    assert _prefill(lib, kimi_dims(kv_lora_rank=100)) == 2
    assert _prefill(lib, kimi_dims(v_head=260)) == 2
    assert _prefill(lib, kimi_dims(softmax_scale=float("nan"))) == 1
    assert _prefill(lib, kimi_dims(), latent=None) == 1
    assert _prefill(lib, kimi_dims(), cu=None) == 1
    assert _prefill(lib, kimi_dims(), maxlen=17) == 1          # longer than all tokens
    assert _prefill(lib, kimi_dims(), maxpos=0) == 1
    assert _prefill(lib, kimi_dims(), wsb=10) == 3
    assert "workspace" in mla.mla_last_error_string()
    assert _prefill(lib, kimi_dims(), ws=None) == 3
    # empty work is a successful no-op (nothing is launched)
    assert _prefill(lib, kimi_dims(), T=0, maxlen=0) == 0
    assert _prefill(lib, kimi_dims(), nseq=0) == 0


def test_decode_host_validation():
    lib = mla.load()
    d = kimi_dims()

    def call(**over):
        a = dict(q=FAKE, cache=FAKE, offs=FAKE, lens=FAKE, pos=FAKE, B=4, maxlen=100, w=FAKE, cos=FAKE,
                 sin=FAKE, maxpos=200, out=FAKE, ws=FAKE, wsb=1 << 40)
        a.update(over)
        return lib.mla_decode(ctypes.byref(d), a["q"], a["cache"], a.get("rows", 10 ** 6), a["offs"], a["lens"], a["pos"], a["B"],
                              a["maxlen"], a["w"], a["cos"], a["sin"], a["maxpos"], a["out"], a["ws"],
                              a["wsb"], None)

    assert call(B=-1) == 1
    assert call(B=0) == 0
    assert call(maxlen=0) == 1
    assert call(cache=None) == 1
    assert call(lens=None) == 1
    assert call(wsb=16) == 3
    assert call(rows=0) == 1


def test_workspace_sizes_are_monotone():
    d = kimi_dims()
    a = mla.mla_prefill_workspace_size(d, 1000, 1)
    b = mla.mla_prefill_workspace_size(d, 2000, 1)
    assert 0 < a < b
    # at least the bf16 k_nope, values and rotated key of every token
    assert b >= 2 * 2000 * (64 * (128 + 128) + 64)
    assert mla.mla_decode_workspace_size(d, 64, 32768) > mla.mla_decode_workspace_size(d, 8, 32768)
    with pytest.raises(mla.MlaError):
        mla.mla_prefill_workspace_size(d, -1, 1)


def test_prefill_cached_host_validation():
    lib = mla.load()
    d = kimi_dims()

    def call(**over):
        a = dict(lat=FAKE, q=FAKE, w=FAKE, wn=FAKE, cu=FAKE, nseq=2, T=5, offs=FAKE, pre=FAKE, maxlen=100,
                 cos=FAKE, sin=FAKE, maxpos=200, cache=FAKE, rows=10 ** 6, out=FAKE, ws=FAKE, wsb=1 << 40)
        a.update(over)
        return lib.mla_prefill_cached(ctypes.byref(d), a["lat"], a["q"], a["w"], a["wn"], a["cu"], a["nseq"], a["T"],
                                      a["offs"], a["pre"], a["maxlen"], a["cos"], a["sin"], a["maxpos"], a["cache"],
                                      a["rows"], a["out"], a["ws"], a["wsb"], None)

    assert call(T=0) == 0                    # no chunk tokens: nothing to do
    assert call(T=-1) == 1
    assert call(nseq=0) == 1                 # tokens but no sequence
    assert call(T=65536) == 2                # above the decode's batch limit
    assert call(maxlen=0) == 1
    assert call(maxpos=0) == 1
    assert call(rows=0) == 1
    assert call(pre=None) == 1
    assert call(cache=None) == 1
    assert call(wsb=16) == 3
    assert call(maxlen=256 * 2048 + 1) == 2  # the decode's length limit, before anything is launched
    # the workspace holds the per-token bookkeeping plus the decode's own
    need = mla.mla_prefill_cached_workspace_size(d, 5, 100)
    assert need >= mla.mla_decode_workspace_size(d, 5, 100) + 5 * 24
    assert call(wsb=need - 1) == 3
    with pytest.raises(mla.MlaError):
        mla.mla_prefill_cached_workspace_size(d, 65536, 100)


def test_projection_host_validation():
    lib = mla.load()
    d = kimi_dims()

    def kv(**o):
        a = dict(hid=7168, x=FAKE, w=FAKE, wn=FAKE, pos=FAKE, n=4, cos=FAKE, sin=FAKE, mp=10, lat=FAKE, cache=None,
                 rows=0, crows=None, ws=FAKE, wsb=1 << 40)
        a.update(o)
        return lib.mla_kv_down_append(ctypes.byref(d), a["hid"], a["x"], a["w"], a["wn"], a["pos"], a["n"], a["cos"],
                                      a["sin"], a["mp"], a["lat"], a["cache"], a["rows"], a["crows"], a["ws"],
                                      a["wsb"], None)

    assert kv(n=0) == 0
    assert kv(n=-1) == 1
    assert kv(n=(1 << 20) + 1) == 2
    assert kv(hid=0) == 1
    assert kv(x=None) == 1
    assert kv(lat=None) == 1
    assert kv(cache=FAKE) == 1                     # a cache without destination rows
    assert kv(cache=FAKE, crows=FAKE, wn=None) == 1
    assert kv(cache=FAKE, crows=FAKE, rows=0) == 1      # checked before the Linear runs
    assert kv(cache=FAKE, crows=FAKE, rows=10, mp=0) == 1
    assert kv(wsb=16) == 3                         # bf16 runs keep the Linear's result in fp32
    assert kv(ws=None) == 3
    assert mla.mla_kv_down_append_workspace_size(d, 100) >= 100 * 576 * 4
    assert mla.mla_kv_down_append_workspace_size(kimi_dims(dtype=1), 100) == 0

    def qp(**o):
        a = dict(hid=7168, qr=1536, x=FAKE, wa=FAKE, wn=FAKE, wb=FAKE, n=4, q=FAKE, ws=FAKE, wsb=1 << 40)
        a.update(o)
        return lib.mla_q_proj(ctypes.byref(d), a["hid"], a["qr"], a["x"], a["wa"], a["wn"], a["wb"], a["n"], a["q"],
                              a["ws"], a["wsb"], None)

    assert qp(n=0) == 0
    assert qp(qr=0) == 1
    assert qp(wn=None) == 1
    assert qp(wsb=16) == 3
    assert mla.mla_q_proj_workspace_size(d, 1536, 100) >= 100 * 1536 * (4 + 2) + 64 * 192 * 1536 * 2

    def op(**o):
        a = dict(hid=7168, x=FAKE, w=FAKE, n=4, out=FAKE)
        a.update(o)
        return lib.mla_o_proj(ctypes.byref(d), a["hid"], a["x"], a["w"], a["n"], a["out"], None)

    assert op(n=0) == 0
    assert op(hid=-3) == 1
    assert op(out=None) == 1
    assert op(n=(1 << 21)) == 2


def test_prepared_weight_and_selftest_host_validation():
    lib = mla.load()
    d = kimi_dims()
    assert mla.mla_kv_b_proj_prepared_size(d) == 2 * 64 * 256 * 512
    # outside the tensor-core shapes the prepared copy is the weight itself
    assert mla.mla_kv_b_proj_prepared_size(kimi_dims(dtype=1)) == 4 * 64 * 256 * 512
    assert lib.mla_prepare_kv_b_proj(ctypes.byref(d), FAKE, FAKE, 16, None) == 3
    assert lib.mla_prepare_kv_b_proj(ctypes.byref(d), None, FAKE, 1 << 40, None) == 1
    assert lib.mla_prepare_kv_b_proj(ctypes.byref(d), ctypes.c_void_p(0x1002), FAKE, 1 << 40, None) == 1  # alignment
    # mla_prefill_prepared: a NULL weight is an argument error
    rc = lib.mla_prefill_prepared(ctypes.byref(d), FAKE, FAKE, None, FAKE, FAKE, FAKE, 1, 10, 10, FAKE, FAKE, 10,
                                  FAKE, FAKE, 1 << 40, None)
    assert rc == 1
    assert lib.mla_selftest_wait_timeout(0, FAKE, None) == 1
    assert lib.mla_selftest_wait_timeout(2000000, FAKE, None) == 1
    assert lib.mla_selftest_wait_timeout(1000, None, None) == 1
    assert isinstance(mla.mla_last_dispatch(), str)
