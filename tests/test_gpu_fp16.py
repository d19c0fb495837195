"""fp16 inputs (q, k, v, caches, out): the same kernels instantiated for
binary16, against the fp64 oracle reading the same fp16 bit patterns."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_gqa_reshape_b200 as pa
import workloads
from tests.gpu_helpers import assert_attention_close, case_to, run_varlen

pytestmark = pytest.mark.gpu
F16 = torch.float16


def oracle_f16(case, rows=None):
    return oracle.attention_varlen_dtype(
        workloads.bf16_bits(case.q), workloads.bf16_bits(case.k_logical),
        workloads.bf16_bits(case.v_logical), case.kv_offsets.cpu().numpy(),
        case.seq_lens.cpu().numpy(), case.query_start_loc.cpu().numpy(), case.num_kv_heads,
        case.scale, case.causal, 1, rows=rows)


def test_write_kv_fp16_bit_exact():
    cpu = workloads.build_varlen_case("w16", [100, 33, 1], [40, 33, 1], 8, 4, 128, True,
                                      seed=31, dtype=F16)
    dev = case_to(cpu, "cuda")
    _, kc, vc, ws = run_varlen(dev)
    ek, ev = workloads.bf16_bits(cpu.k_cache).copy(), workloads.bf16_bits(cpu.v_cache).copy()
    oracle.write_kv(workloads.bf16_bits(cpu.k_new), workloads.bf16_bits(cpu.v_new),
                    cpu.slot_mapping.numpy(), ek, ev, cpu.block_size)
    assert np.array_equal(workloads.bf16_bits(kc), ek)
    assert np.array_equal(workloads.bf16_bits(vc), ev)


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("g,hkv", [(4, 2), (16, 1), (1, 4)])
def test_varlen_fp16(d, g, hkv):
    # prefill, chunked prefill and decode sequences in one batch
    lens = [700, 40, 300, 1, 2000, 17, 129, 513]
    qlens = [64, 1, 300, 1, 1, 17, 100, 513]
    cpu = workloads.build_varlen_case("v16", lens, qlens, g * hkv, hkv, d, True, seed=32 + d + g,
                                      dtype=F16)
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert out.dtype == F16
    assert_attention_close(out, oracle_f16(cpu), what=f"fp16 d={d} g={g}")
    assert pa.get_error(ws) == (0, 0)


def test_varlen_fp16_non_causal_and_combined_cache():
    lens, qlens = [300, 129, 40], [300, 129, 1]
    cpu = workloads.build_varlen_case("n16", lens, qlens, 8, 2, 128, False, seed=36, dtype=F16)
    dev = case_to(cpu, "cuda")
    kv = torch.stack([dev.k_cache, dev.v_cache], dim=1).contiguous()
    ws = pa.varlen_workspace(dev.num_seqs, dev.num_q_tokens, dev.num_q_heads, dev.num_kv_heads,
                             dev.head_dim)
    pa.write_kv(dev.k_new, dev.v_new, dev.slot_mapping, kv[:, 0], kv[:, 1], workspace=ws)
    out = torch.full_like(dev.q, float("nan"))
    pa.attention_varlen(dev.q, kv[:, 0], kv[:, 1], dev.block_tables, dev.seq_lens,
                        dev.query_start_loc, dev.num_kv_heads, dev.scale, False, out,
                        max_query_len=dev.max_query_len, max_seq_len=dev.max_seq_len, workspace=ws)
    torch.cuda.synchronize()
    assert_attention_close(out, oracle_f16(cpu), what="fp16 non-causal combined cache")
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("d,hq,hkv", [(128, 16, 16), (64, 8, 4)])
def test_smallseq_fp16(d, hq, hkv):
    rng = np.random.default_rng(d + hq + 7)
    lens = rng.integers(0, 17, size=500).tolist()
    cpu = workloads.build_smallseq_case("s16", lens, hq, hkv, d, seed=d + hq, dtype=F16)
    dev = case_to(cpu, "cuda")
    out = torch.full_like(dev.q, float("nan"))
    ws = pa.error_workspace()
    pa.attention_smallseq(dev.q, dev.k, dev.v, dev.cu_seqlens_kv, dev.scale, out, workspace=ws)
    torch.cuda.synchronize()
    ref = oracle.smallseq_dtype(workloads.bf16_bits(cpu.q), workloads.bf16_bits(cpu.k),
                                workloads.bf16_bits(cpu.v), cpu.cu_seqlens_kv.numpy(),
                                hkv, cpu.scale, 1)
    assert_attention_close(out, ref, what="smallseq fp16")
    assert pa.get_error(ws) == (0, 0)


def test_fp16_prefill_and_decode_configs_full_size():
    # the benchmark's fp16 legs: varlen_prefill on sampled rows, decode_batch
    # on every row
    pre = workloads.varlen_prefill(dtype=F16)
    out, _, _, ws = run_varlen(case_to(pre, "cuda"))
    assert pa.get_error(ws) == (0, 0)
    qsl = pre.query_start_loc.tolist()
    rows = sorted({qsl[s] + i for s in range(pre.num_seqs) for i in (0, 127, 128, 2047)
                   if qsl[s] + i < qsl[s + 1]} | {qsl[s + 1] - 1 for s in range(pre.num_seqs)})
    rows = np.array(rows, dtype=np.int64)
    assert_attention_close(out, oracle_f16(pre, rows=rows), rows=rows,
                           what="fp16 prefill full (sampled)")
    dec = workloads.decode_batch(dtype=F16)
    out, _, _, ws = run_varlen(case_to(dec, "cuda"))
    assert pa.get_error(ws) == (0, 0)
    assert_attention_close(out, oracle_f16(dec), what="fp16 decode full")
