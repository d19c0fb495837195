"""Reference oracle (fp64 CPU) for paged KV attention — test infrastructure.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of
``bench.py`` may import this package.  The product path never calls it.

The arithmetic lives in ``oracle.c`` (plain C, double precision); this module
only compiles it with gcc and marshals numpy arrays into it.  Inputs are
bfloat16 bit patterns held in ``uint16`` arrays; outputs are ``float64``.

Definitions followed (see the header of ``oracle.c`` for each passage):

* cache write — vllm-spyre PR #853 "Pytorch Native Attention on Spyre",
  description, step 1 (slot_mapping scatter);
* masked softmax attention with GQA — same description, steps 4-6 and the
  repeat_interleave paragraph; bottom-right causal alignment — vllm-omni
  PR #9244, kernel-semantics review; empty rows give zeros — TensorRT-LLM
  "CSA2 Vanilla sparse attention", description;
* small-seq cross attention — ROCm/TransformerEngine PR #461, description.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        p = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_num_threads.restype = i32
        lib.oracle_write_kv.restype = i64
        lib.oracle_write_kv.argtypes = [p, p, p, i64, i32, i32, p, p, i64, i32]
        lib.oracle_attention_varlen.restype = i32
        lib.oracle_attention_varlen.argtypes = [
            p, p, p, p, p, p, i32, i32, i32, i32, f64, i32, p, i64, p]
        lib.oracle_attention_varlen_spans.restype = i32
        lib.oracle_attention_varlen_spans.argtypes = [
            p, p, p, p, p, p, i32, i32, i32, i32, f64, p, p, p, i64, p]
        lib.oracle_attention_varlen_paged.restype = i32
        lib.oracle_attention_varlen_paged.argtypes = [
            p, p, p, p, i32, p, p, i32, i32, i32, i32, i32, i64, f64, i32, p, i64, p]
        lib.oracle_attention_weights.restype = i64
        lib.oracle_attention_weights.argtypes = [
            p, p, p, p, p, p, i32, i32, i32, i32, f64, i32, i64, i32, p]
        lib.oracle_attention_varlen_dtype.restype = i32
        lib.oracle_attention_varlen_dtype.argtypes = [
            p, p, p, p, p, p, i32, i32, i32, i32, f64, i32, i32, p, i64, p]
        lib.oracle_attention_varlen_mods.restype = i32
        lib.oracle_attention_varlen_mods.argtypes = [
            p, p, p, p, p, p, i32, i32, i32, i32, f64, i32, i32, f64, p, p, i64, i64, p, p, p,
            i64, p]
        lib.oracle_attention_smallseq_dtype.restype = i32
        lib.oracle_attention_smallseq_dtype.argtypes = [p, p, p, p, i32, i32, i32, i32, f64, i32, p]
        lib.oracle_smallseq_weights.restype = i32
        lib.oracle_smallseq_weights.argtypes = [p, p, p, i32, i32, i32, i32, f64, i32, i32, p]
        lib.oracle_smallseq_backward.restype = i32
        lib.oracle_smallseq_backward.argtypes = [p, p, p, p, p, i32, i32, i32, i32, f64, i32,
                                                 p, i32, p, p, p]
        lib.oracle_widen.restype = f64
        lib.oracle_widen.argtypes = [ctypes.c_uint16, i32]
        lib.oracle_attention_smallseq.restype = i32
        lib.oracle_attention_smallseq.argtypes = [p, p, p, p, i32, i32, i32, i32, f64, p]
        _lib = lib
    return _lib


def _arr(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return a


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def write_kv(k, v, slot_mapping, k_cache, v_cache, block_size):
    """Literal slot-by-slot write, in place on the uint16 cache arrays.

    k, v: [T, Hkv, D] uint16; slot_mapping: [T] int64;
    caches: [NB, BS, Hkv, D] uint16.  Returns the count of out-of-pool slots.
    """
    k, v = _arr(k, np.uint16), _arr(v, np.uint16)
    sm = _arr(slot_mapping, np.int64)
    if not (k_cache.flags.c_contiguous and v_cache.flags.c_contiguous):
        raise ValueError("caches must be contiguous")
    t, hkv, d = k.shape
    nb = k_cache.shape[0]
    return int(_load().oracle_write_kv(_ptr(k), _ptr(v), _ptr(sm), t, hkv, d,
                                       _ptr(k_cache), _ptr(v_cache), nb, block_size))


def attention_varlen(q, k_seq, v_seq, kv_offsets, seq_lens, query_start_loc,
                     num_kv_heads, scale, causal, rows=None):
    """Logical-form attention; returns float64 [T, Hq, D] (rows not asked for are 0)."""
    q = _arr(q, np.uint16)
    k_seq, v_seq = _arr(k_seq, np.uint16), _arr(v_seq, np.uint16)
    kv_offsets = _arr(kv_offsets, np.int64)
    seq_lens = _arr(seq_lens, np.int32)
    qsl = _arr(query_start_loc, np.int32)
    t, hq, d = q.shape
    out = np.zeros((t, hq, d), dtype=np.float64)
    rows_a = None if rows is None else _arr(rows, np.int64)
    rc = _load().oracle_attention_varlen(
        _ptr(q), _ptr(k_seq), _ptr(v_seq), _ptr(kv_offsets), _ptr(seq_lens), _ptr(qsl),
        len(seq_lens), hq, num_kv_heads, d, float(scale), int(bool(causal)),
        _ptr(rows_a), 0 if rows_a is None else len(rows_a), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_attention_varlen failed ({rc})")
    return out


def attention_varlen_dtype(q, k_seq, v_seq, kv_offsets, seq_lens, query_start_loc,
                           num_kv_heads, scale, causal, dtype, rows=None):
    """attention_varlen for dtype 0 (bf16 bits) or 1 (fp16 bits)."""
    q = _arr(q, np.uint16)
    k_seq, v_seq = _arr(k_seq, np.uint16), _arr(v_seq, np.uint16)
    kv_offsets = _arr(kv_offsets, np.int64)
    seq_lens = _arr(seq_lens, np.int32)
    qsl = _arr(query_start_loc, np.int32)
    t, hq, d = q.shape
    out = np.zeros((t, hq, d), dtype=np.float64)
    rows_a = None if rows is None else _arr(rows, np.int64)
    rc = _load().oracle_attention_varlen_dtype(
        _ptr(q), _ptr(k_seq), _ptr(v_seq), _ptr(kv_offsets), _ptr(seq_lens), _ptr(qsl),
        len(seq_lens), hq, num_kv_heads, d, float(scale), int(bool(causal)), int(dtype),
        _ptr(rows_a), 0 if rows_a is None else len(rows_a), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_attention_varlen_dtype failed ({rc})")
    return out


def attention_varlen_mods(q, k_seq, v_seq, kv_offsets, seq_lens, query_start_loc,
                          num_kv_heads, scale, causal, dtype=0, softcap=0.0, alibi_slopes=None,
                          mask=None, mask_head_stride=0, mask_token_stride=0, rows=None,
                          span_offsets=None, spans=None):
    """attention_varlen with score modifiers: soft-cap (0 = off), ALiBi slopes
    [Hq] float32 or None, an additive float32 mask (flat array addressed as
    h * mask_head_stride + t * mask_token_stride + j) or None."""
    q = _arr(q, np.uint16)
    k_seq, v_seq = _arr(k_seq, np.uint16), _arr(v_seq, np.uint16)
    kv_offsets = _arr(kv_offsets, np.int64)
    seq_lens = _arr(seq_lens, np.int32)
    qsl = _arr(query_start_loc, np.int32)
    slopes = None if alibi_slopes is None else _arr(alibi_slopes, np.float32)
    mk = None if mask is None else _arr(mask, np.float32)
    t, hq, d = q.shape
    if slopes is not None and slopes.shape != (hq,):
        raise ValueError("alibi_slopes must be [num_q_heads]")
    out = np.zeros((t, hq, d), dtype=np.float64)
    rows_a = None if rows is None else _arr(rows, np.int64)
    so = sp = None
    if span_offsets is not None:
        so = _arr(span_offsets, np.int32)
        sp = np.asarray(spans).reshape(-1, 2)
        sp = _arr(sp if sp.size else np.zeros((1, 2), np.int32), np.int32)
    rc = _load().oracle_attention_varlen_mods(
        _ptr(q), _ptr(k_seq), _ptr(v_seq), _ptr(kv_offsets), _ptr(seq_lens), _ptr(qsl),
        len(seq_lens), hq, num_kv_heads, d, float(scale), int(bool(causal)), int(dtype),
        float(softcap), _ptr(slopes), _ptr(mk), int(mask_head_stride), int(mask_token_stride),
        _ptr(so), _ptr(sp), _ptr(rows_a), 0 if rows_a is None else len(rows_a), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_attention_varlen_mods failed ({rc})")
    return out


def smallseq_dtype(q, k, v, cu_seqlens_kv, num_kv_heads, scale, dtype):
    """attention_smallseq for dtype 0 (bf16 bits) or 1 (fp16 bits)."""
    q, k, v = _arr(q, np.uint16), _arr(k, np.uint16), _arr(v, np.uint16)
    cu = _arr(cu_seqlens_kv, np.int32)
    b, hq, d = q.shape
    out = np.zeros((b, hq, d), dtype=np.float64)
    rc = _load().oracle_attention_smallseq_dtype(_ptr(q), _ptr(k), _ptr(v), _ptr(cu), b, hq,
                                                 num_kv_heads, d, float(scale), int(dtype),
                                                 _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_attention_smallseq_dtype failed ({rc})")
    return out


def smallseq_weights(q, k, cu_seqlens_kv, num_kv_heads, scale, wlen, dtype=0):
    """Softmax weights [B, Hq, wlen] (float64; zeros past each entry's keys)."""
    q, k = _arr(q, np.uint16), _arr(k, np.uint16)
    cu = _arr(cu_seqlens_kv, np.int32)
    b, hq, d = q.shape
    w = np.zeros((b, hq, wlen), dtype=np.float64)
    rc = _load().oracle_smallseq_weights(_ptr(q), _ptr(k), _ptr(cu), b, hq, num_kv_heads, d,
                                         float(scale), int(dtype), int(wlen), _ptr(w))
    if rc != 0:
        raise ValueError(f"oracle_smallseq_weights failed ({rc})")
    return w


def smallseq_backward(q, k, v, dout, cu_seqlens_kv, num_kv_heads, scale, dtype=0, weights=None):
    """(dq [B, Hq, D], dk [N, Hkv, D], dv [N, Hkv, D]) in float64.  With
    ``weights`` ([B, Hq, W] float64) the softmax weights are taken as given
    (the forward's saved weights) instead of recomputed from q and k."""
    q, k, v, dout = (_arr(x, np.uint16) for x in (q, k, v, dout))
    cu = _arr(cu_seqlens_kv, np.int32)
    b, hq, d = q.shape
    n = k.shape[0]
    dq = np.zeros((b, hq, d), dtype=np.float64)
    dk = np.zeros((max(n, 1), num_kv_heads, d), dtype=np.float64)
    dv = np.zeros((max(n, 1), num_kv_heads, d), dtype=np.float64)
    wp, wlen = None, 0
    if weights is not None:
        weights = _arr(weights, np.float64)
        if weights.shape[:2] != (b, hq):
            raise ValueError("weights must be [batch, num_q_heads, W]")
        wp, wlen = _ptr(weights), weights.shape[2]
    rc = _load().oracle_smallseq_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(cu), b, hq,
                                          num_kv_heads, d, float(scale), int(dtype), wp, wlen,
                                          _ptr(dq), _ptr(dk), _ptr(dv))
    if rc != 0:
        raise ValueError(f"oracle_smallseq_backward failed ({rc})")
    return dq, dk[:n], dv[:n]


def widen(bits: int, dtype: int) -> float:
    """One 16-bit pattern widened to float (0 = bf16, 1 = fp16)."""
    return _load().oracle_widen(int(bits), int(dtype))


def attention_varlen_spans(q, k_seq, v_seq, kv_offsets, seq_lens, query_start_loc,
                           num_kv_heads, scale, span_offsets, spans, rows=None):
    """Piecewise block-causal attention (full segments + causal rest), logical
    form; span_offsets [S+1] int32, spans [N, 2] int32 (start, end) key
    positions.  Returns float64 [T, Hq, D]."""
    q = _arr(q, np.uint16)
    k_seq, v_seq = _arr(k_seq, np.uint16), _arr(v_seq, np.uint16)
    kv_offsets = _arr(kv_offsets, np.int64)
    seq_lens = _arr(seq_lens, np.int32)
    qsl = _arr(query_start_loc, np.int32)
    so = _arr(span_offsets, np.int32)
    sp = _arr(np.asarray(spans).reshape(-1, 2) if np.asarray(spans).size else
              np.zeros((1, 2), np.int32), np.int32)
    t, hq, d = q.shape
    out = np.zeros((t, hq, d), dtype=np.float64)
    rows_a = None if rows is None else _arr(rows, np.int64)
    rc = _load().oracle_attention_varlen_spans(
        _ptr(q), _ptr(k_seq), _ptr(v_seq), _ptr(kv_offsets), _ptr(seq_lens), _ptr(qsl),
        len(seq_lens), hq, num_kv_heads, d, float(scale), _ptr(so), _ptr(sp),
        _ptr(rows_a), 0 if rows_a is None else len(rows_a), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_attention_varlen_spans failed ({rc})")
    return out


def attention_varlen_paged(q, k_cache, v_cache, block_tables, seq_lens, query_start_loc,
                           num_kv_heads, scale, causal, rows=None):
    """Paged-form attention through the block table; returns float64 [T, Hq, D]."""
    q = _arr(q, np.uint16)
    k_cache, v_cache = _arr(k_cache, np.uint16), _arr(v_cache, np.uint16)
    bt = _arr(block_tables, np.int32)
    seq_lens = _arr(seq_lens, np.int32)
    qsl = _arr(query_start_loc, np.int32)
    t, hq, d = q.shape
    nb, bs = k_cache.shape[0], k_cache.shape[1]
    out = np.zeros((t, hq, d), dtype=np.float64)
    rows_a = None if rows is None else _arr(rows, np.int64)
    rc = _load().oracle_attention_varlen_paged(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(bt), bt.shape[1], _ptr(seq_lens),
        _ptr(qsl), len(seq_lens), hq, num_kv_heads, d, bs, nb, float(scale),
        int(bool(causal)), _ptr(rows_a), 0 if rows_a is None else len(rows_a), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_attention_varlen_paged failed ({rc})")
    return out


def attention_weights(q, k_seq, v_seq, kv_offsets, seq_lens, query_start_loc,
                      num_kv_heads, scale, causal, token, head):
    """Softmax weights of one (token, head) row over its sequence's keys."""
    q = _arr(q, np.uint16)
    k_seq, v_seq = _arr(k_seq, np.uint16), _arr(v_seq, np.uint16)
    kv_offsets = _arr(kv_offsets, np.int64)
    seq_lens = _arr(seq_lens, np.int32)
    qsl = _arr(query_start_loc, np.int32)
    t, hq, d = q.shape
    s = int(np.searchsorted(qsl, token, side="right") - 1)
    w = np.zeros(max(int(seq_lens[s]), 1), dtype=np.float64)
    n = _load().oracle_attention_weights(
        _ptr(q), _ptr(k_seq), _ptr(v_seq), _ptr(kv_offsets), _ptr(seq_lens), _ptr(qsl),
        len(seq_lens), hq, num_kv_heads, d, float(scale), int(bool(causal)),
        int(token), int(head), _ptr(w))
    if n < 0:
        raise ValueError("oracle_attention_weights failed")
    return w[: int(seq_lens[s])], int(n)


def attention_smallseq(q, k, v, cu_seqlens_kv, num_kv_heads, scale):
    """s_q = 1 cross attention over contiguous THD keys; returns float64 [B, Hq, D]."""
    q = _arr(q, np.uint16)
    k, v = _arr(k, np.uint16), _arr(v, np.uint16)
    cu = _arr(cu_seqlens_kv, np.int32)
    b, hq, d = q.shape
    out = np.zeros((b, hq, d), dtype=np.float64)
    rc = _load().oracle_attention_smallseq(_ptr(q), _ptr(k), _ptr(v), _ptr(cu), b, hq,
                                           num_kv_heads, d, float(scale), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_attention_smallseq failed")
    return out
