"""B200-native paged KV attention: Python binding of libpa.so (include/pa.h).

This module only marshals arguments: it checks tensor dtypes/shapes, passes
raw device pointers and the current CUDA stream to the C ABI, and turns a
non-zero status into an exception.  Every step of the computation runs in
the library's sm_100a kernels; there is no fallback path.  If the library
cannot be loaded the calls raise.

Calls (names as in the C ABI, without the ``pa_`` prefix):

* ``write_kv(k, v, slot_mapping, k_cache, v_cache)``
* ``attention_varlen(q, k_cache, v_cache, block_tables, seq_lens,
  query_start_loc, num_kv_heads, scale, causal, out)``
* ``attention_smallseq(q, k, v, cu_seqlens_kv, scale, out, weights=None)``
* ``attention_smallseq_bwd(q, k, v, dout, weights, cu_seqlens_kv, scale, dq, dk, dv)``
* ``get_error(workspace)`` / ``status_string(status)``
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

__all__ = [
    "PaError", "library_path", "load", "write_kv", "attention_varlen", "attention_smallseq",
    "attention_smallseq_bwd",
    "attention_varlen_static", "attention_varlen_spans", "STATIC_SCRATCH_BYTES",
    "varlen_workspace_size", "varlen_workspace", "error_workspace", "get_error",
    "status_string", "version", "set_wait_limit_ns", "EXPORTED_SYMBOLS", "PA_OK", "PA_ERR_INVALID_ARG",
    "PA_ERR_UNSUPPORTED", "PA_ERR_CUDA", "PA_ERR_DEVICE_INDEX", "PA_ERR_TIMEOUT",
    "DEVERR_SLOT", "DEVERR_BLOCK", "DEVERR_LENGTHS", "DEVERR_QLEN", "DEVERR_HINT",
    "DEVERR_TIMEOUT", "DEVERR_SPANS", "ERROR_WORD_BYTES", "DTYPE_BF16", "DTYPE_FP16",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
PA_OK = 0  # pa_status values of include/pa.h
PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_CUDA = 1, 2, 3
PA_ERR_DEVICE_INDEX, PA_ERR_TIMEOUT = 4, 5
DEVERR_SLOT, DEVERR_BLOCK, DEVERR_LENGTHS = 0x1, 0x2, 0x4
DEVERR_QLEN, DEVERR_HINT, DEVERR_TIMEOUT = 0x8, 0x10, 0x20
DEVERR_SPANS = 0x40
ERROR_WORD_BYTES = 256
STATIC_SCRATCH_BYTES = 32 << 20  # PA_STATIC_SCRATCH_BYTES

EXPORTED_SYMBOLS = (
    "pa_write_kv", "pa_attention_varlen_workspace_size", "pa_attention_varlen",
    "pa_attention_smallseq", "pa_get_error", "pa_status_string", "pa_version",
    "pa_attention_varlen_static", "pa_attention_varlen_spans", "pa_write_kv_ex",
    "pa_attention_varlen_ex", "pa_attention_smallseq_ex", "pa_attention_smallseq_bwd",
    "pa_write_kv_strided", "pa_attention_varlen_mods", "pa_set_wait_limit_ns",
)
DTYPE_BF16, DTYPE_FP16 = 0, 1

_lib = None
_lock = threading.Lock()


class PaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)}")
        self.status = status


def library_path() -> str:
    return os.path.join(_HERE, "libpa.so")


def load(build_if_missing: bool = True):
    """Load libpa.so (building it with nvcc first if it is missing or stale)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if build_if_missing:
            from . import _build
            try:
                _build.build()
            except Exception as e:  # the library must exist: no fallback
                if not os.path.exists(library_path()):
                    raise RuntimeError(f"libpa.so is missing and could not be built: {e}") from e
        try:
            lib = ctypes.CDLL(library_path())
        except OSError as e:
            raise RuntimeError(f"cannot load the CUDA library {library_path()}: {e}") from e
        p, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        lib.pa_write_kv.restype = ctypes.c_int
        lib.pa_write_kv.argtypes = [p, p, p, i64, i32, i32, p, p, i64, i32, p, p]
        lib.pa_attention_varlen_workspace_size.restype = ctypes.c_size_t
        lib.pa_attention_varlen_workspace_size.argtypes = [i32, i64, i32, i32, i32]
        lib.pa_attention_varlen.restype = ctypes.c_int
        lib.pa_attention_varlen.argtypes = [
            p, p, p, p, i32, p, p, i32, i64, i32, i32, i32, i32, i64, i32, i32,
            ctypes.c_float, i32, p, p, ctypes.c_size_t, p]
        lib.pa_attention_varlen_static.restype = ctypes.c_int
        lib.pa_attention_varlen_static.argtypes = [
            p, p, p, p, i32, p, p, i32, i64, i32, i32, i32, i32, i64, i32, i32,
            ctypes.c_float, i32, p, p]
        lib.pa_write_kv_ex.restype = ctypes.c_int
        lib.pa_write_kv_ex.argtypes = [p, p, p, i64, i32, i32, p, p, i64, i32, i64, i32, p, p]
        lib.pa_attention_varlen_ex.restype = ctypes.c_int
        lib.pa_attention_varlen_ex.argtypes = [
            p, p, p, p, i32, p, p, i32, i64, i32, i32, i32, i32, i64, i64, i32, i32, i32,
            ctypes.c_float, i32, p, p, i32, p, p, ctypes.c_size_t, p]
        lib.pa_write_kv_strided.restype = ctypes.c_int
        lib.pa_write_kv_strided.argtypes = [p, p, p, i64, i32, i32, p, p, i64, i32, p, i32, p, p]
        lib.pa_attention_varlen_mods.restype = ctypes.c_int
        lib.pa_attention_varlen_mods.argtypes = [
            p, p, p, p, i32, p, p, i32, i64, i32, i32, i32, i32, i64, i32, i32, i32,
            ctypes.c_float, i32, p, p, i32, p, p, p, p, ctypes.c_size_t, p]
        lib.pa_attention_varlen_spans.restype = ctypes.c_int
        lib.pa_attention_varlen_spans.argtypes = [
            p, p, p, p, i32, p, p, i32, i64, i32, i32, i32, i32, i64, i32, i32,
            ctypes.c_float, p, p, i32, p, p, ctypes.c_size_t, p]
        lib.pa_attention_smallseq_ex.restype = ctypes.c_int
        lib.pa_attention_smallseq_ex.argtypes = [p, p, p, p, i32, i32, i32, i32, i32,
                                                 ctypes.c_float, i32, p, p, i32, p, p]
        lib.pa_attention_smallseq_bwd.restype = ctypes.c_int
        lib.pa_attention_smallseq_bwd.argtypes = [p, p, p, p, p, i32, p, i32, i32, i32, i32, i32,
                                                  ctypes.c_float, i32, p, p, p, p, p]
        lib.pa_attention_smallseq.restype = ctypes.c_int
        lib.pa_attention_smallseq.argtypes = [p, p, p, p, i32, i32, i32, i32, i32,
                                              ctypes.c_float, p, p, p]
        lib.pa_get_error.restype = ctypes.c_int
        lib.pa_get_error.argtypes = [p, p, ctypes.POINTER(ctypes.c_uint32)]
        lib.pa_status_string.restype = ctypes.c_char_p
        lib.pa_status_string.argtypes = [ctypes.c_int]
        lib.pa_version.restype = ctypes.c_char_p
        lib.pa_version.argtypes = []
        lib.pa_set_wait_limit_ns.restype = None
        lib.pa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().pa_status_string(int(status)).decode()


def version() -> str:
    return load().pa_version().decode()


def set_wait_limit_ns(ns: int) -> None:
    """Test hook: bound every pipeline-barrier wait of prefill launches made
    from now on to `ns` nanoseconds (0 restores the 1 s default).  A short
    limit makes ordinary waits give up, raising DEVERR_TIMEOUT; only tests of
    that failure path should call this."""
    load().pa_set_wait_limit_ns(int(ns))


def _stream(stream, device=None) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(t: torch.Tensor, name: str, dtype, ndim: Optional[int] = None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def _same_device(device, **tensors):
    """Every tensor argument of a call lives on the device its kernels run on."""
    for name, t in tensors.items():
        if t is not None and t.device != device:
            raise ValueError(f"{name} is on {t.device}, the call's tensors on {device}")


def _raise(status: int, where: str):
    if status != PA_OK:
        raise PaError(status, where)


def error_workspace(device=None) -> torch.Tensor:
    """A zeroed workspace holding only the device error word."""
    return torch.zeros(ERROR_WORD_BYTES, dtype=torch.uint8, device=device or "cuda")


def varlen_workspace_size(num_seqs, num_q_tokens, num_q_heads, num_kv_heads, head_dim) -> int:
    return int(load().pa_attention_varlen_workspace_size(num_seqs, num_q_tokens, num_q_heads,
                                                         num_kv_heads, head_dim))


def varlen_workspace(num_seqs, num_q_tokens, num_q_heads, num_kv_heads, head_dim,
                     device=None) -> torch.Tensor:
    """A zero-initialised workspace for attention_varlen with these sizes."""
    n = varlen_workspace_size(num_seqs, num_q_tokens, num_q_heads, num_kv_heads, head_dim)
    return torch.zeros(max(n, ERROR_WORD_BYTES), dtype=torch.uint8, device=device or "cuda")


_DTYPES = {torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_FP16}


def _element_dtype(t, name):
    if t.dtype not in _DTYPES:
        raise TypeError(f"{name} must be bfloat16 or float16, got {t.dtype}")
    return t.dtype


class _Strides(ctypes.Structure):
    """pa_strides (include/pa.h)."""
    _fields_ = [("q_token", ctypes.c_int64), ("q_head", ctypes.c_int64),
                ("out_token", ctypes.c_int64), ("out_head", ctypes.c_int64),
                ("cache_block", ctypes.c_int64), ("cache_slot", ctypes.c_int64),
                ("cache_head", ctypes.c_int64)]


class _ScoreMods(ctypes.Structure):
    """pa_score_mods (include/pa.h)."""
    _fields_ = [("softcap", ctypes.c_float), ("alibi_slopes", ctypes.c_void_p),
                ("mask", ctypes.c_void_p), ("mask_head_stride", ctypes.c_int64),
                ("mask_token_stride", ctypes.c_int64), ("mask_len", ctypes.c_int64)]


def _check_caches(k_cache, v_cache, dtype):
    """Caches indexed [NB, BS, Hkv, D] with D contiguous and any block / slot /
    head strides (views of one [NB, 2, BS, Hkv, D] tensor, or a head-major
    [NB, Hkv, BS, D] tensor permuted to [NB, BS, Hkv, D], are fine).  Returns
    the (block, slot, head) element strides; the library checks the layout."""
    for t, name in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        if not isinstance(t, torch.Tensor) or t.dtype != dtype:
            raise TypeError(f"{name} must be a {dtype} tensor")
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.dim() != 4:
            raise ValueError(f"{name} must have 4 dims [NB, BS, Hkv, D]")
        if t.stride(3) != 1:
            raise ValueError(f"{name}: head_dim must be contiguous")
    if v_cache.shape != k_cache.shape or v_cache.stride() != k_cache.stride():
        raise ValueError("k_cache and v_cache must have the same shape and strides")
    return k_cache.stride(0), k_cache.stride(1), k_cache.stride(2)


def _dense_rows(cstr, hkv, d):
    return cstr[1] == hkv * d and cstr[2] == d


def _check_rows(t, name, dtype):
    """[T, H, D] with D contiguous and any token / head strides; returns them."""
    if not isinstance(t, torch.Tensor) or t.dtype != dtype:
        raise TypeError(f"{name} must be a {dtype} tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != 3 or t.stride(2) != 1:
        raise ValueError(f"{name} must be [T, H, D] with D contiguous")
    return t.stride(0), t.stride(1)


def write_kv(k, v, slot_mapping, k_cache, v_cache, workspace=None, stream=None):
    """Scatter k/v [T, Hkv, D] into the paged caches at slot_mapping (int64 [T]).

    k_cache / v_cache: indexed [NB, BS, Hkv, D], bf16 or fp16 like k and v;
    separate tensors, the two halves kv[:, 0] / kv[:, 1] of one
    [NB, 2, BS, Hkv, D] cache, or head-major caches [NB, Hkv, BS, D] passed
    as their .permute(0, 2, 1, 3) views.
    """
    dt = _element_dtype(k, "k")
    _check(k, "k", dt, 3)
    _check(v, "v", dt, 3)
    _check(slot_mapping, "slot_mapping", torch.int64, 1)
    cstr = _check_caches(k_cache, v_cache, dt)
    t, hkv, d = k.shape
    if v.shape != k.shape or slot_mapping.shape[0] != t:
        raise ValueError("k, v and slot_mapping disagree on the token count / shape")
    nb, bs, hkv_c, d_c = k_cache.shape
    if hkv_c != hkv or d_c != d:
        raise ValueError("cache shape does not match k/v")
    dev = k.device
    _same_device(dev, v=v, slot_mapping=slot_mapping, k_cache=k_cache, v_cache=v_cache,
                 workspace=workspace)
    ws = workspace.data_ptr() if workspace is not None else None
    with torch.cuda.device(dev):
        if _dense_rows(cstr, hkv, d):
            st = load().pa_write_kv_ex(k.data_ptr(), v.data_ptr(), slot_mapping.data_ptr(), t,
                                       hkv, d, k_cache.data_ptr(), v_cache.data_ptr(), nb, bs,
                                       cstr[0], _DTYPES[dt], ws, _stream(stream, dev))
            _raise(st, "pa_write_kv_ex")
            return
        strides = _Strides(0, 0, 0, 0, *cstr)
        st = load().pa_write_kv_strided(k.data_ptr(), v.data_ptr(), slot_mapping.data_ptr(), t,
                                        hkv, d, k_cache.data_ptr(), v_cache.data_ptr(), nb, bs,
                                        ctypes.byref(strides), _DTYPES[dt], ws,
                                        _stream(stream, dev))
    _raise(st, "pa_write_kv_strided")


def _score_mods(softcap, alibi_slopes, mask, hq, t, device):
    """pa_score_mods for the call, or None when every modifier is off.  The
    mask must hold a row for each of the call's t query tokens (and each
    query head, if 3-D): the library reads those rows and checks only their
    length."""
    if not softcap and alibi_slopes is None and mask is None:
        return None
    m = _ScoreMods(float(softcap or 0.0), None, None, 0, 0, 0)
    if alibi_slopes is not None:
        _check(alibi_slopes, "alibi_slopes", torch.float32, 1)
        if alibi_slopes.shape[0] != hq:
            raise ValueError("alibi_slopes must be [num_q_heads]")
        m.alibi_slopes = alibi_slopes.data_ptr()
    if mask is not None:
        if not isinstance(mask, torch.Tensor) or mask.dtype != torch.float32 or not mask.is_cuda:
            raise TypeError("mask must be a float32 CUDA tensor")
        if mask.device != device:
            raise ValueError("mask must be on q's device")
        if mask.dim() not in (2, 3) or mask.stride(-1) != 1:
            raise ValueError("mask must be [T, L] or [Hq, T, L] with L contiguous")
        if mask.dim() == 3 and mask.shape[0] != hq:
            raise ValueError("a 3-D mask must be [num_q_heads, T, L]")
        if mask.shape[-2] < t:
            raise ValueError("the mask needs a row for every query token")
        m.mask = mask.data_ptr()
        m.mask_token_stride = mask.stride(-2)
        m.mask_head_stride = mask.stride(0) if mask.dim() == 3 else 0
        m.mask_len = mask.shape[-1]
    return m


def _varlen_ex(q, k_cache, v_cache, block_tables, seq_lens, query_start_loc, num_kv_heads,
               scale, causal, span_offsets, spans, out, max_query_len, max_seq_len, workspace,
               stream, what, softcap=0.0, alibi_slopes=None, mask=None):
    dt = _element_dtype(q, "q")
    qstr = _check_rows(q, "q", dt)
    cstr = _check_caches(k_cache, v_cache, dt)
    _check(block_tables, "block_tables", torch.int32, 2)
    _check(seq_lens, "seq_lens", torch.int32, 1)
    _check(query_start_loc, "query_start_loc", torch.int32, 1)
    ostr = _check_rows(out, "out", dt)
    t, hq, d = q.shape
    nb, bs, hkv, d_c = k_cache.shape
    if hkv != num_kv_heads or d_c != d:
        raise ValueError("cache shape does not match q / num_kv_heads")
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    s = seq_lens.shape[0]
    if query_start_loc.shape[0] != s + 1 or block_tables.shape[0] != s:
        raise ValueError("seq_lens, query_start_loc and block_tables disagree on num_seqs")
    so_ptr, sp_ptr, n_spans = None, None, 0
    if span_offsets is not None:
        _check(span_offsets, "span_offsets", torch.int32, 1)
        _check(spans, "spans", torch.int32, 2)
        if span_offsets.shape[0] != s + 1 or (spans.numel() and spans.shape[1] != 2):
            raise ValueError("span_offsets must be [S+1] and spans [N, 2]")
        n_spans = spans.shape[0] if spans.numel() else 0
        so_ptr = span_offsets.data_ptr()
        sp_ptr = spans.data_ptr() if n_spans else None
    mb = block_tables.shape[1]
    mql = t if max_query_len is None else int(max_query_len)
    msl = mb * bs if max_seq_len is None else int(max_seq_len)
    dev = q.device
    _same_device(dev, k_cache=k_cache, v_cache=v_cache, block_tables=block_tables,
                 seq_lens=seq_lens, query_start_loc=query_start_loc, out=out,
                 span_offsets=span_offsets, spans=spans, workspace=workspace,
                 alibi_slopes=alibi_slopes, mask=mask)
    if workspace is None:
        workspace = varlen_workspace(s, t, hq, hkv, d, device=dev)
    mods = _score_mods(softcap, alibi_slopes, mask, hq, t, dev)
    dense = qstr == (hq * d, d) and ostr == (hq * d, d) and _dense_rows(cstr, hkv, d)
    with torch.cuda.device(dev):
        if dense and mods is None:
            st = load().pa_attention_varlen_ex(
                q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_tables.data_ptr(),
                mb, seq_lens.data_ptr(), query_start_loc.data_ptr(), s, t, hq, hkv, d, bs, nb,
                cstr[0], _DTYPES[dt], mql, msl, float(scale), int(bool(causal)), so_ptr, sp_ptr,
                n_spans, out.data_ptr(), workspace.data_ptr(),
                workspace.numel() * workspace.element_size(), _stream(stream, dev))
            _raise(st, what)
            return out
        strides = _Strides(*qstr, *ostr, *cstr)
        st = load().pa_attention_varlen_mods(
            q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_tables.data_ptr(), mb,
            seq_lens.data_ptr(), query_start_loc.data_ptr(), s, t, hq, hkv, d, bs, nb,
            _DTYPES[dt], mql, msl, float(scale), int(bool(causal)), so_ptr, sp_ptr, n_spans,
            ctypes.byref(strides), ctypes.byref(mods) if mods is not None else None,
            out.data_ptr(), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
            _stream(stream, dev))
    _raise(st, "pa_attention_varlen_mods")
    return out


def attention_varlen(q, k_cache, v_cache, block_tables, seq_lens, query_start_loc,
                     num_kv_heads, scale, causal, out, max_query_len=None, max_seq_len=None,
                     workspace=None, stream=None, softcap=0.0, alibi_slopes=None, mask=None):
    """Paged varlen attention; writes out [T, Hq, D] (q's dtype).

    max_query_len / max_seq_len are host-side hints (the metadata builder's
    maxima); when omitted the safe bounds (all tokens / the block table's
    reach) are used, which never forces a device synchronisation.  The caches
    may be separate tensors, the halves of one [NB, 2, BS, Hkv, D] cache, or
    head-major [NB, Hkv, BS, D] caches passed as .permute(0, 2, 1, 3) views;
    q and out may be head-major [Hq, T, D] tensors passed as
    .transpose(0, 1) views.  Score modifiers: softcap (> 0: s <- c tanh(s/c)),
    alibi_slopes (float32 [Hq]: s += slope_h (j - query position)), mask
    (float32 [T, L] or [Hq, T, L]: s += mask[h, t, j]).
    """
    return _varlen_ex(q, k_cache, v_cache, block_tables, seq_lens, query_start_loc,
                      num_kv_heads, scale, causal, None, None, out, max_query_len, max_seq_len,
                      workspace, stream, "pa_attention_varlen_ex", softcap, alibi_slopes, mask)


def attention_varlen_spans(q, k_cache, v_cache, block_tables, seq_lens, query_start_loc,
                           num_kv_heads, scale, span_offsets, spans, out, max_query_len=None,
                           max_seq_len=None, workspace=None, stream=None, softcap=0.0,
                           alibi_slopes=None, mask=None):
    """Paged varlen attention with full-attention spans inside causal sequences.

    span_offsets: int32 [S+1] (sequence s owns spans span_offsets[s] ..
    span_offsets[s+1]-1); spans: int32 [N, 2] (start, end) key positions.
    A query whose key position lies in a span [start, end) sees keys
    0 .. end-1; every other query is causal.  Writes out [T, Hq, D].  Layouts
    and score modifiers as attention_varlen.
    """
    if span_offsets is None or spans is None:
        raise ValueError("span_offsets and spans are required")
    return _varlen_ex(q, k_cache, v_cache, block_tables, seq_lens, query_start_loc,
                      num_kv_heads, scale, True, span_offsets, spans, out, max_query_len,
                      max_seq_len, workspace, stream, "pa_attention_varlen_ex", softcap,
                      alibi_slopes, mask)


def attention_varlen_static(q, k_cache, v_cache, block_tables, seq_lens, query_start_loc,
                            num_kv_heads, scale, causal, out, max_query_len=None,
                            max_seq_len=None, stream=None):
    """attention_varlen for callers that cannot allocate device memory.

    Takes no workspace: the library keeps the scratch in a fixed device array
    of STATIC_SCRATCH_BYTES (32 MiB) per GPU.  Meant for hosts that own all
    device memory through their own allocator, or paths where cudaMalloc would
    synchronise the device.  Sizes needing more scratch raise (status
    PA_ERR_UNSUPPORTED); calls that overlap on the GPU race on the shared
    array; device-side index errors cannot be read back.  The first call on a
    device looks up the array's address and should come before any stream
    capture.
    """
    _check(q, "q", torch.bfloat16, 3)
    _check(k_cache, "k_cache", torch.bfloat16, 4)
    _check(v_cache, "v_cache", torch.bfloat16, 4)
    _check(block_tables, "block_tables", torch.int32, 2)
    _check(seq_lens, "seq_lens", torch.int32, 1)
    _check(query_start_loc, "query_start_loc", torch.int32, 1)
    _check(out, "out", torch.bfloat16, 3)
    t, hq, d = q.shape
    nb, bs, hkv, d_c = k_cache.shape
    if hkv != num_kv_heads or d_c != d or v_cache.shape != k_cache.shape or out.shape != q.shape:
        raise ValueError("inconsistent shapes")
    s = seq_lens.shape[0]
    if query_start_loc.shape[0] != s + 1 or block_tables.shape[0] != s:
        raise ValueError("seq_lens, query_start_loc and block_tables disagree on num_seqs")
    mb = block_tables.shape[1]
    mql = t if max_query_len is None else int(max_query_len)
    msl = mb * bs if max_seq_len is None else int(max_seq_len)
    dev = q.device
    _same_device(dev, k_cache=k_cache, v_cache=v_cache, block_tables=block_tables,
                 seq_lens=seq_lens, query_start_loc=query_start_loc, out=out)
    with torch.cuda.device(dev):
        st = load().pa_attention_varlen_static(
            q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_tables.data_ptr(), mb,
            seq_lens.data_ptr(), query_start_loc.data_ptr(), s, t, hq, hkv, d, bs, nb, mql, msl,
            float(scale), int(bool(causal)), out.data_ptr(), _stream(stream, dev))
    _raise(st, "pa_attention_varlen_static")
    return out


def attention_smallseq(q, k, v, cu_seqlens_kv, scale, out, max_seqlen_kv=16, workspace=None,
                       stream=None, weights=None):
    """s_q = 1 attention over <= 16 contiguous keys per entry; writes out [B, Hq, D]
    (bf16 or fp16, like q) and, if given, the attention weights [B, Hq, W]."""
    dt = _element_dtype(q, "q")
    _check(q, "q", dt, 3)
    _check(k, "k", dt, 3)
    _check(v, "v", dt, 3)
    _check(cu_seqlens_kv, "cu_seqlens_kv", torch.int32, 1)
    _check(out, "out", dt, 3)
    b, hq, d = q.shape
    _, hkv, d_k = k.shape
    if d_k != d or v.shape != k.shape or out.shape != q.shape or cu_seqlens_kv.shape[0] != b + 1:
        raise ValueError("inconsistent small-seq shapes")
    wp, wlen = None, 0
    if weights is not None:
        _check(weights, "weights", dt, 3)
        if weights.shape[:2] != (b, hq):
            raise ValueError("weights must be [batch, num_q_heads, W]")
        wp, wlen = weights.data_ptr(), weights.shape[2]
    dev = q.device
    _same_device(dev, k=k, v=v, cu_seqlens_kv=cu_seqlens_kv, out=out, weights=weights,
                 workspace=workspace)
    ws = workspace.data_ptr() if workspace is not None else None
    with torch.cuda.device(dev):
        st = load().pa_attention_smallseq_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                             cu_seqlens_kv.data_ptr(), b, hq, hkv, d,
                                             int(max_seqlen_kv), float(scale), _DTYPES[dt],
                                             out.data_ptr(), wp, wlen, ws, _stream(stream, dev))
    _raise(st, "pa_attention_smallseq_ex")
    return out


def attention_smallseq_bwd(q, k, v, dout, weights, cu_seqlens_kv, scale, dq, dk, dv,
                           max_seqlen_kv=16, workspace=None, stream=None):
    """Gradients (dq, dk, dv) of attention_smallseq from its saved weights."""
    dt = _element_dtype(q, "q")
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (dout, "dout"), (weights, "weights"),
                    (dq, "dq"), (dk, "dk"), (dv, "dv")):
        _check(t, name, dt, 3)
    _check(cu_seqlens_kv, "cu_seqlens_kv", torch.int32, 1)
    b, hq, d = q.shape
    _, hkv, d_k = k.shape
    if (d_k != d or v.shape != k.shape or dk.shape != k.shape or dv.shape != k.shape
            or dout.shape != q.shape or dq.shape != q.shape or weights.shape[:2] != (b, hq)
            or cu_seqlens_kv.shape[0] != b + 1):
        raise ValueError("inconsistent small-seq backward shapes")
    dev = q.device
    _same_device(dev, k=k, v=v, dout=dout, weights=weights, cu_seqlens_kv=cu_seqlens_kv, dq=dq,
                 dk=dk, dv=dv, workspace=workspace)
    ws = workspace.data_ptr() if workspace is not None else None
    with torch.cuda.device(dev):
        st = load().pa_attention_smallseq_bwd(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(), weights.data_ptr(),
            weights.shape[2], cu_seqlens_kv.data_ptr(), b, hq, hkv, d, int(max_seqlen_kv),
            float(scale), _DTYPES[dt], dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws,
            _stream(stream, dev))
    _raise(st, "pa_attention_smallseq_bwd")
    return dq, dk, dv


def get_error(workspace, stream=None):
    """Synchronise, read and clear the workspace's device error word: (status, bits)."""
    bits = ctypes.c_uint32(0)
    with torch.cuda.device(workspace.device):
        st = load().pa_get_error(workspace.data_ptr(), _stream(stream, workspace.device),
                                 ctypes.byref(bits))
    return int(st), int(bits.value)
