"""The no-allocation variant of paged varlen attention.

pa_attention_varlen_static serves callers that cannot allocate device memory
(a host that owns all device memory through its own allocator, or a path
where cudaMalloc would synchronise the device): it keeps its scratch in a
fixed device array inside the library instead of a caller workspace.  Here it
is called through the C ABI and through the Python wrapper, and must agree
with pa_attention_varlen (which takes a workspace) on calls in a row, among
them a pure-decode batch with split-KV merges that plans for itself (so no
plan kernel zeroes the arrival counters first), and must reject sizes whose
scratch would not fit.  This file sorts last so that a run stopping at the
first failure has already run every other test.
"""
import ctypes

import pytest
import torch

import paged_kv_gqa_reshape_b200 as pa
import workloads
from tests.gpu_helpers import MAX_ABS, MEAN_ABS, case_to

pytestmark = pytest.mark.gpu


def _static_call(lib, c, out):
    return lib.pa_attention_varlen_static(
        c.q.data_ptr(), c.k_cache.data_ptr(), c.v_cache.data_ptr(), c.block_tables.data_ptr(),
        c.block_tables.shape[1], c.seq_lens.data_ptr(), c.query_start_loc.data_ptr(),
        c.num_seqs, c.num_q_tokens, c.num_q_heads, c.num_kv_heads, c.head_dim, c.block_size,
        c.num_blocks, c.max_query_len, c.max_seq_len, ctypes.c_float(c.scale), int(c.causal),
        out.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _with_workspace(c):
    out = torch.empty_like(c.q)
    pa.attention_varlen(c.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens,
                        c.query_start_loc, c.num_kv_heads, c.scale, c.causal, out,
                        max_query_len=c.max_query_len, max_seq_len=c.max_seq_len)
    return out


def _close(out, ref, what):
    err = (out.double() - ref).abs()
    assert torch.isfinite(out.float()).all(), what
    assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, what


def _mixed_case():
    # prefill chunks and split-KV decodes in one batch, so every part of the
    # scratch (plan lists, partials, arrival counters) is used
    cpu = workloads.build_varlen_case("static", [700, 40, 300, 1, 2000, 17, 5, 129],
                                      [64, 1, 300, 1, 1, 17, 1, 100], 16, 2, 128, True, 21)
    c = case_to(cpu, "cuda")
    pa.write_kv(c.k_new, c.v_new, c.slot_mapping, c.k_cache, c.v_cache)
    return c


def _decode_case():
    # a pure decode batch (one query per sequence) long enough that sequences
    # are split across CTAs and merged; it plans for itself, no plan kernel
    cpu = workloads.build_varlen_case("static_dec", [5000, 3000, 17, 4096, 9000, 1, 2500],
                                      [1] * 7, 32, 8, 128, True, 22)
    c = case_to(cpu, "cuda")
    pa.write_kv(c.k_new, c.v_new, c.slot_mapping, c.k_cache, c.v_cache)
    return c


def test_static_scratch_entry_point_matches_workspace_entry_point():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lib = pa.load()
    mixed, dec = _mixed_case(), _decode_case()
    ref_mixed = _with_workspace(mixed).double()
    ref_dec = _with_workspace(dec).double()
    # the mixed batch twice, then the decode batch twice (its counters sit
    # where the mixed batch's plan kernel left them), then the mixed batch again
    for call, (c, ref) in enumerate([(mixed, ref_mixed), (mixed, ref_mixed), (dec, ref_dec),
                                     (dec, ref_dec), (mixed, ref_mixed)]):
        out = torch.full_like(c.q, float("nan"))
        assert _static_call(lib, c, out) == 0
        torch.cuda.synchronize()
        _close(out, ref, f"C ABI call {call}")


def test_static_scratch_python_wrapper():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    for c in (_decode_case(), _mixed_case()):
        ref = _with_workspace(c).double()
        for call in range(2):
            out = torch.full_like(c.q, float("nan"))
            pa.attention_varlen_static(c.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens,
                                       c.query_start_loc, c.num_kv_heads, c.scale, c.causal,
                                       out, max_query_len=c.max_query_len,
                                       max_seq_len=c.max_seq_len)
            torch.cuda.synchronize()
            _close(out, ref, f"wrapper call {call}, {c.num_seqs} sequences")


def test_static_scratch_rejects_sizes_beyond_its_limit():
    lib = pa.load()
    # 2^25 query tokens need more tile-list scratch than the fixed array holds
    need = pa.varlen_workspace_size(4096, 1 << 25, 64, 8, 128)
    assert need > pa.STATIC_SCRATCH_BYTES
    st = lib.pa_attention_varlen_static(16, 16, 16, 16, 1, 16, 16, 4096, 1 << 25, 64, 8, 128, 16,
                                        1, 1, 16, ctypes.c_float(0.1), 1, 16, None)
    assert st == pa.PA_ERR_UNSUPPORTED  # before anything is launched
    # a bad argument is reported as the workspace entry point reports it, even
    # when the size is also too large (too many query tokens for int32 rows)
    st = lib.pa_attention_varlen_static(16, 16, 16, 16, 1, 16, 16, 4096, 1 << 33, 64, 8, 128, 16,
                                        1, 1, 16, ctypes.c_float(0.1), 1, 16, None)
    assert st == pa.PA_ERR_INVALID_ARG
    st = lib.pa_attention_varlen_static(16, 16, 16, 16, 1, 16, 16, 4, 64, 64, 8, 128, 16,
                                        1, 1, 16, ctypes.c_float(-1.0), 1, 16, None)
    assert st == pa.PA_ERR_INVALID_ARG


def test_static_scratch_wrapper_raises_beyond_its_limit():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    # 1024 decode sequences of 64 query heads need more split-KV partial
    # scratch than the fixed array holds; the call is rejected before any
    # launch, so the tensors' contents do not matter
    s, hq, hkv, d = 1024, 64, 8, 128
    assert pa.varlen_workspace_size(s, s, hq, hkv, d) > pa.STATIC_SCRATCH_BYTES
    q = torch.zeros(s, hq, d, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(4, 16, hkv, d, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(s, 1, dtype=torch.int32, device="cuda")
    sl = torch.ones(s, dtype=torch.int32, device="cuda")
    qsl = torch.arange(s + 1, dtype=torch.int32, device="cuda")
    out = torch.zeros_like(q)
    with pytest.raises(pa.PaError) as e:
        pa.attention_varlen_static(q, kc, kc, bt, sl, qsl, hkv, 0.1, True, out)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED
