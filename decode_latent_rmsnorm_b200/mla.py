"""Thin ctypes binding of ``libmla.so`` (C-ABI declared in ``include/mla.h``).

Argument marshalling only: each function checks that the torch tensors it is
given live on the GPU with the dtype and shape the C call expects, then passes
raw pointers and the current CUDA stream. Every step of the computation runs
in the library's kernels. The library is loaded on first use; if it is
missing or fails to load, an exception is raised (there is no fallback).
"""

from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

c_i32, c_i64, c_f32, c_f64, c_sz, c_vp = (ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                         ctypes.c_double, ctypes.c_size_t, ctypes.c_void_p)

MLA_BF16, MLA_FP32 = 0, 1
STATUS_NAMES = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED_SHAPE",
                3: "MLA_ERR_WORKSPACE_TOO_SMALL", 4: "MLA_ERR_CUDA", 5: "MLA_ERR_DEVICE_TIMEOUT"}

# Every symbol include/mla.h declares, with (restype, argtypes).
SIGNATURES = {
    "mla_softmax_scale": (c_i32, [c_vp, c_i32, ctypes.POINTER(c_f32)]),
    "mla_init_rope_tables": (c_i32, [c_vp, c_i32, c_vp, c_vp, c_vp]),
    "mla_prefill_workspace_size": (c_i32, [c_vp, c_i64, c_i32, ctypes.POINTER(c_sz)]),
    "mla_prefill": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_i32, c_i64,
                            c_vp, c_vp, c_i32, c_vp, c_vp, c_sz, c_vp]),
    "mla_decode_workspace_size": (c_i32, [c_vp, c_i32, c_i32, ctypes.POINTER(c_sz)]),
    "mla_decode": (c_i32, [c_vp, c_vp, c_vp, c_i64, c_vp, c_vp, c_vp, c_i32, c_i32, c_vp, c_vp,
                           c_vp, c_i32, c_vp, c_vp, c_sz, c_vp]),
    "mla_cache_append": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i64, c_vp, c_vp, c_i32, c_vp, c_i64,
                                 c_vp, c_vp]),
    "mla_prefill_cached_workspace_size": (c_i32, [c_vp, c_i64, c_i32, ctypes.POINTER(c_sz)]),
    "mla_prefill_cached": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_i64, c_vp, c_vp, c_i32,
                                   c_vp, c_vp, c_i32, c_vp, c_i64, c_vp, c_vp, c_sz, c_vp]),
    "mla_kv_down_append_workspace_size": (c_i32, [c_vp, c_i64, ctypes.POINTER(c_sz)]),
    "mla_kv_down_append": (c_i32, [c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_i64, c_vp, c_vp, c_i32, c_vp, c_vp,
                                   c_i64, c_vp, c_vp, c_sz, c_vp]),
    "mla_q_proj_workspace_size": (c_i32, [c_vp, c_i32, c_i64, ctypes.POINTER(c_sz)]),
    "mla_q_proj": (c_i32, [c_vp, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_i64, c_vp, c_vp, c_sz, c_vp]),
    "mla_o_proj": (c_i32, [c_vp, c_i32, c_vp, c_vp, c_i64, c_vp, c_vp]),
    "mla_check_device_status": (c_i32, [c_vp]),
    "mla_last_error_string": (ctypes.c_char_p, []),
    "mla_version": (c_i32, []),
    "mla_set_kernel_events": (c_i32, [c_vp, c_i32]),
    "mla_recorded_kernel_events": (c_i32, [ctypes.POINTER(c_i32)]),
    "mla_launch_count": (ctypes.c_uint64, []),
    "mla_recorded_kernel_name": (ctypes.c_char_p, [c_i32]),
    "mla_prefill_noalloc": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_i32, c_i64,
                                    c_vp, c_vp, c_i32, c_vp, c_vp]),
    "mla_kv_b_proj_prepared_size": (c_i32, [c_vp, ctypes.POINTER(c_sz)]),
    "mla_prepare_kv_b_proj": (c_i32, [c_vp, c_vp, c_vp, c_sz, c_vp]),
    "mla_prefill_prepared": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_i32, c_i64,
                                     c_vp, c_vp, c_i32, c_vp, c_vp, c_sz, c_vp]),
    "mla_last_dispatch": (ctypes.c_char_p, []),
    "mla_selftest_wait_timeout": (c_i32, [ctypes.c_uint32, c_vp, c_vp]),
    "mla_prefill_cached_eager_workspace_size": (c_i32, [c_vp, c_i64, c_i32, c_i32, ctypes.POINTER(c_sz)]),
    "mla_prefill_cached_form": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_i64, c_vp, c_vp, c_i32,
                                        c_vp, c_vp, c_i32, c_vp, c_i64, c_vp, c_vp, c_sz, c_i32, c_vp]),
}

# Bytes of the static scratch behind mla_prefill_noalloc (MLA_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


class RopeCfg(ctypes.Structure):
    """``mla_rope_cfg``."""
    _fields_ = [("rope_dim", c_i32), ("yarn", c_i32), ("original_max_pos", c_i32),
                ("reserved", c_i32), ("base", c_f64), ("factor", c_f64), ("beta_fast", c_f64),
                ("beta_slow", c_f64), ("mscale", c_f64), ("mscale_all_dim", c_f64)]

    @classmethod
    def make(cls, rope_dim, base, yarn=False, factor=1.0, original_max_pos=4096,
             beta_fast=32.0, beta_slow=1.0, mscale=1.0, mscale_all_dim=0.0):
        return cls(int(rope_dim), int(bool(yarn)), int(original_max_pos), 0, float(base),
                   float(factor), float(beta_fast), float(beta_slow), float(mscale),
                   float(mscale_all_dim))


class Dims(ctypes.Structure):
    """``mla_dims``."""
    _fields_ = [("num_heads", c_i32), ("kv_lora_rank", c_i32), ("qk_nope", c_i32),
                ("qk_rope", c_i32), ("v_head", c_i32), ("dtype", c_i32),
                ("rope_interleaved", c_i32), ("eps", c_f32), ("softmax_scale", c_f32)]

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == MLA_FP32 else torch.bfloat16


class MlaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s: %s" % (STATUS_NAMES.get(status, str(status)), message))
        self.status = status


_lib = None


def load() -> ctypes.CDLL:
    """Load the library (building it first if sources are newer)."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.LIB
    if _build.is_stale():
        _build.build()
    if not os.path.exists(path):
        raise RuntimeError("libmla.so is missing at %s and could not be built" % path)
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(rc: int):
    if rc != 0:
        raise MlaError(rc, load().mla_last_error_string().decode())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    return ctypes.c_void_p(t.data_ptr())


def mla_softmax_scale(rope: RopeCfg, qk_head_dim: int) -> float:
    out = c_f32()
    _check(load().mla_softmax_scale(ctypes.byref(rope), int(qk_head_dim), ctypes.byref(out)))
    return out.value


def mla_init_rope_tables(rope: RopeCfg, max_pos: int, device="cuda"):
    """Returns fp32 cos/sin tables [max_pos, rope_dim / 2] on ``device``."""
    cos = torch.empty((max_pos, rope.rope_dim // 2), dtype=torch.float32, device=device)
    sin = torch.empty_like(cos)
    _check(load().mla_init_rope_tables(ctypes.byref(rope), int(max_pos), _dev(cos, "cos"),
                                       _dev(sin, "sin"), _stream()))
    return cos, sin


def mla_prefill_workspace_size(dims: Dims, total_tokens: int, num_seqs: int) -> int:
    out = c_sz()
    _check(load().mla_prefill_workspace_size(ctypes.byref(dims), int(total_tokens), int(num_seqs),
                                             ctypes.byref(out)))
    return out.value


def mla_prefill(dims: Dims, latent, q, w_kvb, w_norm, positions, cu_seqlens, max_seqlen: int,
                cos, sin, out=None, workspace=None):
    """Causal MLA prefill; returns ``out`` [Ttot, H, V] (allocated if None)."""
    dt = dims.torch_dtype
    H, R, N, P, V = dims.num_heads, dims.kv_lora_rank, dims.qk_nope, dims.qk_rope, dims.v_head
    T = latent.shape[0]
    nseq = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((T, H, V), dtype=dt, device=latent.device)
    if workspace is None:
        workspace = torch.empty(max(mla_prefill_workspace_size(dims, T, nseq), 1), dtype=torch.uint8,
                                device=latent.device)
    _check(load().mla_prefill(
        ctypes.byref(dims), _dev(latent, "latent", dt, (T, R + P)), _dev(q, "q", dt, (T, H, N + P)),
        _dev(w_kvb, "w_kvb", dt, (H * (N + V), R)), _dev(w_norm, "w_norm", dt, (R,)),
        _dev(positions, "positions", torch.int32, (T,)), _dev(cu_seqlens, "cu_seqlens", torch.int32),
        int(nseq), int(max_seqlen), int(T), _dev(cos, "cos", torch.float32),
        _dev(sin, "sin", torch.float32), int(cos.shape[0]), _dev(out, "out", dt, (T, H, V)),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream()))
    return out


def mla_kv_b_proj_prepared_size(dims: Dims) -> int:
    out = c_sz()
    _check(load().mla_kv_b_proj_prepared_size(ctypes.byref(dims), ctypes.byref(out)))
    return out.value


def mla_prepare_kv_b_proj(dims: Dims, w_kvb, prepared=None):
    """The prepared copy of kv_b_proj for mla_prefill_prepared (a uint8
    device tensor; allocated if None). Done once per weight."""
    H, R, N, V = dims.num_heads, dims.kv_lora_rank, dims.qk_nope, dims.v_head
    n = mla_kv_b_proj_prepared_size(dims)
    if prepared is None:
        prepared = torch.empty(n, dtype=torch.uint8, device=w_kvb.device)
    _check(load().mla_prepare_kv_b_proj(
        ctypes.byref(dims), _dev(w_kvb, "w_kvb", dims.torch_dtype, (H * (N + V), R)), _dev(prepared, "prepared"),
        prepared.numel() * prepared.element_size(), _stream()))
    return prepared


def mla_prefill_prepared(dims: Dims, latent, q, w_prepared, w_norm, positions, cu_seqlens, max_seqlen: int,
                         cos, sin, out=None, workspace=None):
    """mla_prefill with the kv_b_proj copy from mla_prepare_kv_b_proj."""
    dt = dims.torch_dtype
    H, R, N, P, V = dims.num_heads, dims.kv_lora_rank, dims.qk_nope, dims.qk_rope, dims.v_head
    T = latent.shape[0]
    nseq = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((T, H, V), dtype=dt, device=latent.device)
    if workspace is None:
        workspace = torch.empty(max(mla_prefill_workspace_size(dims, T, nseq), 1), dtype=torch.uint8,
                                device=latent.device)
    if w_prepared.numel() * w_prepared.element_size() < mla_kv_b_proj_prepared_size(dims):
        raise ValueError("w_prepared is smaller than mla_kv_b_proj_prepared_size")
    _check(load().mla_prefill_prepared(
        ctypes.byref(dims), _dev(latent, "latent", dt, (T, R + P)), _dev(q, "q", dt, (T, H, N + P)),
        _dev(w_prepared, "w_prepared"), _dev(w_norm, "w_norm", dt, (R,)),
        _dev(positions, "positions", torch.int32, (T,)), _dev(cu_seqlens, "cu_seqlens", torch.int32),
        int(nseq), int(max_seqlen), int(T), _dev(cos, "cos", torch.float32),
        _dev(sin, "sin", torch.float32), int(cos.shape[0]), _dev(out, "out", dt, (T, H, V)),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream()))
    return out


def mla_selftest_wait_timeout(limit_us: int = 1000):
    """Runs the bounded-wait self-test kernel; returns the device int32 flag
    (1 once the wait has given up). Read the error word afterwards with
    mla_check_device_status (it reports MLA_ERR_DEVICE_TIMEOUT)."""
    flag = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    _check(load().mla_selftest_wait_timeout(int(limit_us), _dev(flag, "gave_up", torch.int32), _stream()))
    return flag


def mla_last_dispatch() -> str:
    """Which kernels this thread's last prefill / decode call ran."""
    return load().mla_last_dispatch().decode()


def mla_prefill_noalloc(dims: Dims, latent, q, w_kvb, w_norm, positions, cu_seqlens, max_seqlen: int,
                        cos, sin, out):
    """mla_prefill without a workspace, for callers that cannot allocate
    device memory: the library's static scratch array serves as workspace.
    ``out`` must be given (this call allocates nothing)."""
    dt = dims.torch_dtype
    H, R, N, P, V = dims.num_heads, dims.kv_lora_rank, dims.qk_nope, dims.qk_rope, dims.v_head
    T = latent.shape[0]
    nseq = cu_seqlens.numel() - 1
    _check(load().mla_prefill_noalloc(
        ctypes.byref(dims), _dev(latent, "latent", dt, (T, R + P)), _dev(q, "q", dt, (T, H, N + P)),
        _dev(w_kvb, "w_kvb", dt, (H * (N + V), R)), _dev(w_norm, "w_norm", dt, (R,)),
        _dev(positions, "positions", torch.int32, (T,)), _dev(cu_seqlens, "cu_seqlens", torch.int32),
        int(nseq), int(max_seqlen), int(T), _dev(cos, "cos", torch.float32),
        _dev(sin, "sin", torch.float32), int(cos.shape[0]), _dev(out, "out", dt, (T, H, V)), _stream()))
    return out


def mla_decode_workspace_size(dims: Dims, batch: int, max_cache_len: int) -> int:
    out = c_sz()
    _check(load().mla_decode_workspace_size(ctypes.byref(dims), int(batch), int(max_cache_len),
                                            ctypes.byref(out)))
    return out.value


def mla_decode(dims: Dims, q, cache, cache_offsets, cache_lens, positions, max_cache_len: int,
               w_kvb, cos, sin, out=None, workspace=None):
    """Absorbed decode; returns ``out`` [B, H, V] (allocated if None)."""
    dt = dims.torch_dtype
    H, R, N, P, V = dims.num_heads, dims.kv_lora_rank, dims.qk_nope, dims.qk_rope, dims.v_head
    B = q.shape[0]
    if out is None:
        out = torch.empty((B, H, V), dtype=dt, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(mla_decode_workspace_size(dims, B, max_cache_len), 1),
                                dtype=torch.uint8, device=q.device)
    if cache.dim() != 2 or cache.shape[1] != R + P:
        raise ValueError("cache must be [rows, R + P]")
    _check(load().mla_decode(
        ctypes.byref(dims), _dev(q, "q", dt, (B, H, N + P)), _dev(cache, "cache", dt),
        int(cache.shape[0]), _dev(cache_offsets, "cache_offsets", torch.int64, (B,)),
        _dev(cache_lens, "cache_lens", torch.int32, (B,)), _dev(positions, "positions", torch.int32, (B,)),
        int(B), int(max_cache_len), _dev(w_kvb, "w_kvb", dt, (H * (N + V), R)),
        _dev(cos, "cos", torch.float32), _dev(sin, "sin", torch.float32), int(cos.shape[0]),
        _dev(out, "out", dt, (B, H, V)), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream()))
    return out


def mla_cache_append(dims: Dims, latent, w_norm, positions, cos, sin, cache, cache_rows):
    """Writes RMSNorm(latent[:, :R]) || rope(latent[:, R:]) into ``cache`` rows."""
    dt = dims.torch_dtype
    R, P = dims.kv_lora_rank, dims.qk_rope
    n = latent.shape[0]
    if cache.dim() != 2 or cache.shape[1] != R + P:
        raise ValueError("cache must be [rows, R + P]")
    _check(load().mla_cache_append(
        ctypes.byref(dims), _dev(latent, "latent", dt, (n, R + P)), _dev(w_norm, "w_norm", dt, (R,)),
        _dev(positions, "positions", torch.int32, (n,)), int(n), _dev(cos, "cos", torch.float32),
        _dev(sin, "sin", torch.float32), int(cos.shape[0]), _dev(cache, "cache", dt),
        int(cache.shape[0]), _dev(cache_rows, "cache_rows", torch.int64, (n,)), _stream()))
    return cache


def mla_prefill_cached_workspace_size(dims: Dims, total_tokens: int, max_total_len: int) -> int:
    out = c_sz()
    _check(load().mla_prefill_cached_workspace_size(ctypes.byref(dims), int(total_tokens), int(max_total_len),
                                                    ctypes.byref(out)))
    return out.value


def mla_prefill_cached_eager_workspace_size(dims: Dims, total_tokens: int, num_seqs: int, max_total_len: int) -> int:
    out = c_sz()
    _check(load().mla_prefill_cached_eager_workspace_size(ctypes.byref(dims), int(total_tokens), int(num_seqs),
                                                          int(max_total_len), ctypes.byref(out)))
    return out.value


CHUNK_FORMS = {"auto": 0, "absorbed": 1, "eager": 2}


def mla_prefill_cached(dims: Dims, latent, q, w_kvb, w_norm, cu_seqlens, cache_offsets, prefix_lens,
                       max_total_len: int, cos, sin, cache, out=None, workspace=None, form="auto"):
    """Chunks of new tokens continuing cached sequences: appends the chunk's
    rows to ``cache`` and returns ``out`` [Tq, H, V] (allocated if None).
    ``form``: "auto" (the library picks by chunk length), "absorbed" or
    "eager". When ``workspace`` is None it is allocated for the forms the
    call may take."""
    dt = dims.torch_dtype
    H, R, N, P, V = dims.num_heads, dims.kv_lora_rank, dims.qk_nope, dims.qk_rope, dims.v_head
    T = latent.shape[0]
    nseq = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((T, H, V), dtype=dt, device=latent.device)
    if workspace is None:
        n = mla_prefill_cached_workspace_size(dims, T, max_total_len)
        if form == "eager" or (form == "auto" and nseq > 0 and T >= 128 * nseq):
            try:
                n = max(n, mla_prefill_cached_eager_workspace_size(dims, T, nseq, max_total_len))
            except MlaError:
                if form == "eager":
                    raise
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=latent.device)
    if cache.dim() != 2 or cache.shape[1] != R + P:
        raise ValueError("cache must be [rows, R + P]")
    _check(load().mla_prefill_cached_form(
        ctypes.byref(dims), _dev(latent, "latent", dt, (T, R + P)), _dev(q, "q", dt, (T, H, N + P)),
        _dev(w_kvb, "w_kvb", dt, (H * (N + V), R)), _dev(w_norm, "w_norm", dt, (R,)),
        _dev(cu_seqlens, "cu_seqlens", torch.int32), int(nseq), int(T),
        _dev(cache_offsets, "cache_offsets", torch.int64, (nseq,)),
        _dev(prefix_lens, "prefix_lens", torch.int32, (nseq,)), int(max_total_len),
        _dev(cos, "cos", torch.float32), _dev(sin, "sin", torch.float32), int(cos.shape[0]),
        _dev(cache, "cache", dt), int(cache.shape[0]), _dev(out, "out", dt, (T, H, V)),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), CHUNK_FORMS[form],
        _stream()))
    return out


def mla_kv_down_append_workspace_size(dims: Dims, n: int) -> int:
    out = c_sz()
    _check(load().mla_kv_down_append_workspace_size(ctypes.byref(dims), int(n), ctypes.byref(out)))
    return out.value


def mla_kv_down_append(dims: Dims, hidden, w_kva, latent=None, w_norm=None, positions=None, cos=None, sin=None,
                       cache=None, cache_rows=None, workspace=None):
    """kv_a_proj_with_mqa: returns ``latent`` [n, R + P]; with ``cache`` and
    ``cache_rows`` also appends the normalized, rotated rows to the cache."""
    dt = dims.torch_dtype
    R, P = dims.kv_lora_rank, dims.qk_rope
    n, hid = hidden.shape
    if latent is None:
        latent = torch.empty((n, R + P), dtype=dt, device=hidden.device)
    if workspace is None:
        workspace = torch.empty(max(mla_kv_down_append_workspace_size(dims, n), 1), dtype=torch.uint8,
                                device=hidden.device)
    append = cache is not None or cache_rows is not None
    if append:
        if cache is None or cache_rows is None or w_norm is None or positions is None or cos is None or sin is None:
            raise ValueError("appending needs cache, cache_rows, w_norm, positions, cos and sin")
        if cache.dim() != 2 or cache.shape[1] != R + P:
            raise ValueError("cache must be [rows, R + P]")
    none = ctypes.c_void_p(0)
    _check(load().mla_kv_down_append(
        ctypes.byref(dims), int(hid), _dev(hidden, "hidden", dt, (n, hid)), _dev(w_kva, "w_kva", dt, (R + P, hid)),
        _dev(w_norm, "w_norm", dt, (R,)) if append else none,
        _dev(positions, "positions", torch.int32, (n,)) if append else none, int(n),
        _dev(cos, "cos", torch.float32) if append else none, _dev(sin, "sin", torch.float32) if append else none,
        int(cos.shape[0]) if append else 0, _dev(latent, "latent", dt, (n, R + P)),
        _dev(cache, "cache", dt) if append else none, int(cache.shape[0]) if append else 0,
        _dev(cache_rows, "cache_rows", torch.int64, (n,)) if append else none, _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream()))
    return latent


def mla_q_proj_workspace_size(dims: Dims, q_rank: int, n: int) -> int:
    out = c_sz()
    _check(load().mla_q_proj_workspace_size(ctypes.byref(dims), int(q_rank), int(n), ctypes.byref(out)))
    return out.value


def mla_q_proj(dims: Dims, hidden, w_qa, w_qnorm, w_qb, q=None, workspace=None):
    """q = q_b_proj(q_a_layernorm(q_a_proj(hidden))); returns q [n, H, N + P]."""
    dt = dims.torch_dtype
    H, N, P = dims.num_heads, dims.qk_nope, dims.qk_rope
    n, hid = hidden.shape
    q_rank = w_qa.shape[0]
    if q is None:
        q = torch.empty((n, H, N + P), dtype=dt, device=hidden.device)
    if workspace is None:
        workspace = torch.empty(max(mla_q_proj_workspace_size(dims, q_rank, n), 1), dtype=torch.uint8,
                                device=hidden.device)
    _check(load().mla_q_proj(
        ctypes.byref(dims), int(hid), int(q_rank), _dev(hidden, "hidden", dt, (n, hid)),
        _dev(w_qa, "w_qa", dt, (q_rank, hid)), _dev(w_qnorm, "w_qnorm", dt, (q_rank,)),
        _dev(w_qb, "w_qb", dt, (H * (N + P), q_rank)), int(n), _dev(q, "q", dt, (n, H, N + P)),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream()))
    return q


def mla_o_proj(dims: Dims, attn, w_o, out=None):
    """o_proj: attn [n, H, V] or [n, H * V] -> out [n, hidden_size]."""
    dt = dims.torch_dtype
    H, V = dims.num_heads, dims.v_head
    n = attn.shape[0]
    hid = w_o.shape[0]
    if tuple(attn.shape[1:]) not in ((H, V), (H * V,)):
        raise ValueError("attn must be [n, H, V] or [n, H * V]")
    if out is None:
        out = torch.empty((n, hid), dtype=dt, device=attn.device)
    _check(load().mla_o_proj(
        ctypes.byref(dims), int(hid), _dev(attn, "attn", dt), _dev(w_o, "w_o", dt, (hid, H * V)), int(n),
        _dev(out, "out", dt, (n, hid)), _stream()))
    return out


def mla_check_device_status():
    _check(load().mla_check_device_status(_stream()))


def mla_last_error_string() -> str:
    return load().mla_last_error_string().decode()


def mla_version() -> int:
    return load().mla_version()


def mla_launch_count() -> int:
    return int(load().mla_launch_count())


class KernelEvents:
    """Records a CUDA event pair around each kernel the library launches
    while active (``mla_set_kernel_events``); ``durations_ms()`` after a
    synchronize gives one duration per recorded launch."""

    def __init__(self, pairs: int):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * pairs)]
        for e in self.events:   # torch creates the CUDA event on its first record
            e.record()
        self._handles = (c_vp * (2 * pairs))(*[e.cuda_event for e in self.events])
        self.pairs = pairs
        self.recorded = 0

    def __enter__(self):
        _check(load().mla_set_kernel_events(ctypes.cast(self._handles, c_vp), self.pairs))
        return self

    def __exit__(self, *exc):
        n = c_i32()
        _check(load().mla_recorded_kernel_events(ctypes.byref(n)))
        self.recorded = n.value
        self.names = [load().mla_recorded_kernel_name(i).decode() for i in range(self.recorded)]
        _check(load().mla_set_kernel_events(None, 0))
        return False

    def durations_ms(self):
        return [self.events[2 * i].elapsed_time(self.events[2 * i + 1]) for i in range(self.recorded)]


# ---------------------------------------------------------------- helpers

def dims_for(wl, softmax_scale: float) -> Dims:
    """``Dims`` of a ``workloads.Workload``."""
    return Dims(wl.num_heads, wl.kv_lora_rank, wl.qk_nope, wl.qk_rope, wl.v_head,
                MLA_FP32 if wl.dtype == "fp32" else MLA_BF16, int(wl.interleaved), float(wl.eps),
                float(softmax_scale))


def rope_for(wl) -> RopeCfg:
    return RopeCfg.make(**wl.rope)
