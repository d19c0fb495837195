"""GPU parity of piecewise block-causal attention (full-attention spans inside
causal sequences) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_gqa_reshape_b200 as pa
import workloads
from tests.gpu_helpers import assert_attention_close, case_to

pytestmark = pytest.mark.gpu


def run_spans(case, span_offsets, spans, out=None):
    kc, vc = case.k_cache.clone(), case.v_cache.clone()
    ws = pa.varlen_workspace(case.num_seqs, case.num_q_tokens, case.num_q_heads,
                             case.num_kv_heads, case.head_dim)
    if case.k_new.shape[0]:
        pa.write_kv(case.k_new, case.v_new, case.slot_mapping, kc, vc, workspace=ws)
    if out is None:
        out = torch.full_like(case.q, float("nan"))
    so = torch.as_tensor(np.asarray(span_offsets, np.int32), device="cuda")
    sp = torch.as_tensor(np.asarray(spans, np.int32).reshape(-1, 2), device="cuda")
    pa.attention_varlen_spans(case.q, kc, vc, case.block_tables, case.seq_lens,
                              case.query_start_loc, case.num_kv_heads, case.scale, so, sp, out,
                              max_query_len=case.max_query_len, max_seq_len=case.max_seq_len,
                              workspace=ws)
    torch.cuda.synchronize()
    return out, ws


def oracle_spans(case, span_offsets, spans, rows=None):
    return oracle.attention_varlen_spans(
        workloads.bf16_bits(case.q), workloads.bf16_bits(case.k_logical),
        workloads.bf16_bits(case.v_logical), case.kv_offsets.cpu().numpy(),
        case.seq_lens.cpu().numpy(), case.query_start_loc.cpu().numpy(), case.num_kv_heads,
        case.scale, np.asarray(span_offsets, np.int32),
        np.asarray(spans, np.int32).reshape(-1, 2), rows=rows)


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("g,hkv", [(4, 2), (1, 4)])
def test_spans_small(d, g, hkv):
    # prefill, chunked prefill (prior context) and decode sequences in one batch;
    # spans cross 128-row query tiles, 256-row work items and 128-key KV tiles
    lens = [700, 300, 129, 1000, 40]
    qlens = [700, 300, 129, 400, 1]
    spans_per_seq = [[(0, 100), (100, 300), (517, 700)],
                     [(128, 256)],
                     [],
                     [(610, 900), (900, 901), (950, 1000)],
                     [(0, 40)]]
    cpu = workloads.build_varlen_case("spans", lens, qlens, g * hkv, hkv, d, True, seed=d + g)
    offs = np.cumsum([0] + [len(x) for x in spans_per_seq])
    flat = [p for x in spans_per_seq for p in x]
    out, ws = run_spans(case_to(cpu, "cuda"), offs, flat)
    assert_attention_close(out, oracle_spans(cpu, offs, flat), what=f"spans d={d} g={g}")
    assert pa.get_error(ws) == (0, 0)


def test_no_spans_matches_causal_bit_for_bit():
    lens, qlens = [600, 333, 129], [600, 100, 129]
    dev = case_to(workloads.build_varlen_case("c", lens, qlens, 8, 2, 128, True, seed=3), "cuda")
    out_s, _ = run_spans(dev, [0, 0, 0, 0], np.zeros((0, 2), np.int32))
    from tests.gpu_helpers import run_varlen
    out_c, _, _, _ = run_varlen(dev)
    assert torch.equal(out_s, out_c)


def test_malformed_spans_are_ignored_and_reported():
    lens = [400, 300]
    cpu = workloads.build_varlen_case("bad", lens, lens, 4, 4, 128, True, seed=4)
    spans = [(50, 150), (120, 200), (350, 500), (10, 10)]  # 2nd overlaps, 3rd past Lkv; 4th empty
    offs = [0, 3, 4]
    out, ws = run_spans(case_to(cpu, "cuda"), offs, spans)
    assert_attention_close(out, oracle_spans(cpu, offs, spans), what="malformed spans")
    st, bits = pa.get_error(ws)
    assert bits == pa.DEVERR_SPANS


def test_spans_config_full_size_sampled_rows():
    cpu, so, sp = workloads.spans_prefill()
    dev = case_to(cpu, "cuda")
    out, ws = run_spans(dev, so.numpy(), sp.numpy())
    assert pa.get_error(ws) == (0, 0)
    qsl = cpu.query_start_loc.tolist()
    rows = set()
    for s in range(cpu.num_seqs):
        for i in (0, 1, 511, 512, 513, 1000, 2047, 2048, 2049, 3000, 4095):
            rows.add(qsl[s] + i)
    rows = np.array(sorted(rows), dtype=np.int64)
    ref = oracle_spans(cpu, so.numpy(), sp.numpy(), rows=rows)
    assert_attention_close(out, ref, rows=rows, what="spans full (sampled)")
