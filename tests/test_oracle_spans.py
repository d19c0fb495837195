"""Pins for the piecewise block-causal oracle (full segments within a causal sequence).

vllm-omni PR #9244 "Support piecewise block-causal attention for
full_attn_spans" states the result three ways, each used here against the
oracle with an independent library routine (torch scaled_dot_product_attention
in float64 on CPU, expanded KV heads):

* the dense reference of its tests: a key is visible if it is at or before the
  query, or in the same full block as the query;
* the per-segment plan: a causal segment [s, e) is attn(Q[s:e], K[:e],
  causal=True) with bottom-right alignment, a full segment is plain
  bidirectional attention over the truncated prefix K[:e];
* no spans means plain causal attention.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads


def spans_case(lens, qlens, hq, hkv, d, seed):
    return workloads.build_varlen_case("spans", lens, qlens, hq, hkv, d, True, seed)


def run_spans(case, span_offsets, spans, rows=None):
    return oracle.attention_varlen_spans(
        workloads.bf16_bits(case.q), workloads.bf16_bits(case.k_logical),
        workloads.bf16_bits(case.v_logical), case.kv_offsets.numpy(), case.seq_lens.numpy(),
        case.query_start_loc.numpy(), case.num_kv_heads, case.scale,
        np.asarray(span_offsets, np.int32), np.asarray(spans, np.int32).reshape(-1, 2), rows=rows)


def seq_tensors(case, s):
    g = case.num_q_heads // case.num_kv_heads
    qsl = case.query_start_loc.tolist()
    lkv = int(case.seq_lens[s])
    o0 = int(case.kv_offsets[s])
    q = case.q[qsl[s]:qsl[s + 1]].double().transpose(0, 1)
    k = case.k_logical[o0:o0 + lkv].double().repeat_interleave(g, dim=1).transpose(0, 1)
    v = case.v_logical[o0:o0 + lkv].double().repeat_interleave(g, dim=1).transpose(0, 1)
    return q, k, v


def sdpa(q, k, v, mask, scale):
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)


def test_dense_block_causal_reference():
    # queries = keys (a prefill from position 0): visible iff j <= i or same full block
    lens = [300, 129]
    spans_per_seq = [[(10, 70), (70, 71), (128, 257)], [(0, 64)]]
    case = spans_case(lens, lens, 8, 2, 64, seed=5)
    offs = np.cumsum([0] + [len(x) for x in spans_per_seq])
    got = run_spans(case, offs, [p for x in spans_per_seq for p in x])
    qsl = case.query_start_loc.tolist()
    for s, L in enumerate(lens):
        block = np.full(L, -1)
        for b, (a, e) in enumerate(spans_per_seq[s]):
            block[a:e] = b
        i = np.arange(L)[:, None]
        j = np.arange(L)[None, :]
        mask = (j <= i) | ((block[:, None] == block[None, :]) & (block[:, None] >= 0))
        q, k, v = seq_tensors(case, s)
        ref = sdpa(q, k, v, torch.from_numpy(mask), case.scale).transpose(0, 1).numpy()
        assert np.max(np.abs(got[qsl[s]:qsl[s + 1]] - ref)) < 1e-10


def test_segment_plan_with_prior_context():
    # chunked prefill: 100 prior keys, then 220 queries; full segments at key
    # positions [120, 200) and [250, 320)
    case = spans_case([320], [220], 4, 4, 64, seed=6)
    spans = [(120, 200), (250, 320)]
    got = run_spans(case, [0, 2], spans)
    q, k, v = seq_tensors(case, 0)
    off = 320 - 220
    seg_of = {}
    for a, e in spans:
        for pos in range(a, e):
            seg_of[pos] = e
    for i in range(220):
        pos = off + i
        if pos in seg_of:           # full segment: bidirectional over K[:end]
            e = seg_of[pos]
            ref = sdpa(q[:, i:i + 1], k[:, :e], v[:, :e], None, case.scale)
        else:                       # causal segment: keys up to the query's own position
            ref = sdpa(q[:, i:i + 1], k[:, :pos + 1], v[:, :pos + 1], None, case.scale)
        assert np.max(np.abs(got[i] - ref[:, 0].numpy())) < 1e-10, i


def test_no_spans_is_causal_attention():
    lens, qlens = [150, 40, 513], [150, 17, 200]
    case = spans_case(lens, qlens, 8, 4, 128, seed=7)
    got = run_spans(case, [0, 0, 0, 0], np.zeros((0, 2), np.int32))
    qsl = case.query_start_loc.tolist()
    for s in range(3):
        q, k, v = seq_tensors(case, s)
        lq, lkv = qsl[s + 1] - qsl[s], lens[s]
        i = torch.arange(lq)[:, None]
        j = torch.arange(lkv)[None, :]
        ref = sdpa(q, k, v, j <= (lkv - lq) + i, case.scale).transpose(0, 1).numpy()
        assert np.max(np.abs(got[qsl[s]:qsl[s + 1]] - ref)) < 1e-10


def test_one_span_over_everything_is_full_attention():
    case = spans_case([257], [257], 4, 2, 64, seed=8)
    got = run_spans(case, [0, 1], [(0, 257)])
    q, k, v = seq_tensors(case, 0)
    ref = sdpa(q, k, v, None, case.scale).transpose(0, 1).numpy()
    assert np.max(np.abs(got - ref)) < 1e-10


@pytest.mark.parametrize("spans,used", [
    ([(5, 5)], []),                        # empty
    ([(-1, 10)], []),                      # negative start
    ([(10, 400)], []),                     # past the last key
    ([(20, 30), (25, 40)], [(20, 30)]),    # second starts before the first ends
    ([(20, 30), (30, 40)], [(20, 30), (30, 40)]),
])
def test_invalid_spans_are_ignored(spans, used):
    case = spans_case([300], [300], 4, 4, 64, seed=9)
    got = run_spans(case, [0, len(spans)], spans)
    want = run_spans(case, [0, len(used)], used if used else np.zeros((0, 2), np.int32))
    assert np.array_equal(got, want)
