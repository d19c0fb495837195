"""Pins for the fp64 oracle, checked against things other than the oracle itself.

Hand-derived worked examples (tests/golden/, each citing the passage it
follows), closed forms, invariants of the definition, brute force on tiny
inputs and an independent library routine (torch scaled_dot_product_attention
in float64 on CPU, with an explicit boolean mask and repeat_interleave'd KV
heads — the CPU path vllm-spyre PR #853 tests its kernel against).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.conftest import load_golden


def bits(x):
    """float list/array -> bf16 bit patterns (values chosen exactly representable)."""
    t = torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.tensor(np.asarray(x, dtype=np.float32))), "not exact in bf16"
    return t.view(torch.int16).numpy().view(np.uint16)


def logical_inputs(case):
    return (workloads.bf16_bits(case.q), workloads.bf16_bits(case.k_logical),
            workloads.bf16_bits(case.v_logical), case.kv_offsets.numpy(),
            case.seq_lens.numpy(), case.query_start_loc.numpy())


def run_logical(case, causal=None, rows=None):
    q, k, v, off, sl, qsl = logical_inputs(case)
    return oracle.attention_varlen(q, k, v, off, sl, qsl, case.num_kv_heads, case.scale,
                                   case.causal if causal is None else causal, rows=rows)


def sdpa_reference(case, causal=None):
    """Independent: torch SDPA in float64, explicit bool mask, expanded KV heads."""
    causal = case.causal if causal is None else causal
    g = case.num_q_heads // case.num_kv_heads
    out = torch.zeros(case.q.shape, dtype=torch.float64)
    qsl = case.query_start_loc.tolist()
    for s in range(case.num_seqs):
        lq = qsl[s + 1] - qsl[s]
        lkv = int(case.seq_lens[s])
        if lq == 0:
            continue
        q = case.q[qsl[s]:qsl[s + 1]].double().transpose(0, 1)              # [Hq, Lq, D]
        o0 = int(case.kv_offsets[s])
        k = case.k_logical[o0:o0 + lkv].double().repeat_interleave(g, dim=1).transpose(0, 1)
        v = case.v_logical[o0:o0 + lkv].double().repeat_interleave(g, dim=1).transpose(0, 1)
        i = torch.arange(lq)[:, None]
        j = torch.arange(lkv)[None, :]
        mask = (j <= (lkv - lq) + i) if causal else torch.ones(lq, lkv, dtype=torch.bool)
        if lkv == 0:
            continue
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask,
                                                             scale=case.scale)
        empty = ~mask.any(dim=1)
        o[:, empty, :] = 0.0
        out[qsl[s]:qsl[s + 1]] = o.transpose(0, 1)
    return out.numpy()


# ---------------------------------------------------------------------------
# golden worked examples
# ---------------------------------------------------------------------------

def test_golden_write_kv():
    g = load_golden("write_kv_tiny")
    nb, bs, h, d = g["num_blocks"], g["block_size"], g["num_kv_heads"], g["head_dim"]
    kc = np.full((nb, bs, h, d), bits([g["fill"]])[0], dtype=np.uint16)
    vc = kc.copy()
    bad = oracle.write_kv(bits(g["k"]), bits(g["v"]), np.array(g["slot_mapping"], np.int64),
                          kc, vc, bs)
    assert bad == 0
    expect_k = np.full((nb, bs, h, d), bits([g["fill"]])[0], dtype=np.uint16)
    expect_v = expect_k.copy()
    kk, vv = bits(g["k"]), bits(g["v"])
    for blk, off, tok in g["expected_written"]:
        expect_k[blk, off] = kk[tok]
        expect_v[blk, off] = vv[tok]
    assert np.array_equal(kc, expect_k) and np.array_equal(vc, expect_v)


def test_golden_two_keys_closed_form():
    g = load_golden("attention_two_keys")
    e = math.e
    closed = np.array([(1 + 3 * e) / (1 + e), (-1 + 5 * e) / (1 + e)])
    assert np.allclose(np.array(g["expected"]).reshape(2), closed, rtol=0, atol=1e-15)
    out = oracle.attention_varlen(bits(g["q"]), bits(g["k"]), bits(g["v"]),
                                  np.array([0], np.int64), np.array([2], np.int32),
                                  np.array([0, 1], np.int32), 1, g["scale"], g["causal"])
    assert np.allclose(out.reshape(2), closed, rtol=0, atol=1e-14)


def test_golden_scale_is_applied():
    """Same example with scale 1 instead of 0.5: scores (0, 2) -> weights (1, e^2)/(1+e^2)."""
    g = load_golden("attention_two_keys")
    e2 = math.exp(2.0)
    closed = np.array([(1 + 3 * e2) / (1 + e2), (-1 + 5 * e2) / (1 + e2)])
    out = oracle.attention_varlen(bits(g["q"]), bits(g["k"]), bits(g["v"]),
                                  np.array([0], np.int64), np.array([2], np.int32),
                                  np.array([0, 1], np.int32), 1, 1.0, False)
    assert np.allclose(out.reshape(2), closed, rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal", [True, False])
def test_golden_causal_bottom_right(causal):
    g = load_golden("causal_bottom_right")
    out = oracle.attention_varlen(bits(g["q"]), bits(g["k"]), bits(g["v"]),
                                  np.array([0], np.int64), np.array(g["seq_lens"], np.int32),
                                  np.array(g["query_start_loc"], np.int32), 1, g["scale"],
                                  causal)
    expect = g["expected_causal"] if causal else g["expected_full"]
    assert np.array_equal(out, np.array(expect, dtype=np.float64))


def test_golden_gqa_head_mapping():
    g = load_golden("gqa_head_mapping")
    out = oracle.attention_varlen(bits(g["q"]), bits(g["k"]), bits(g["v"]),
                                  np.array([0], np.int64), np.array([1], np.int32),
                                  np.array([0, 1], np.int32), g["num_kv_heads"], g["scale"],
                                  True)
    assert np.array_equal(out, np.array(g["expected"], dtype=np.float64))


def test_golden_empty_rows():
    g = load_golden("empty_rows")
    out = oracle.attention_varlen(bits(g["q"]), bits(g["k"]), bits(g["v"]),
                                  np.array([0], np.int64), np.array(g["seq_lens"], np.int32),
                                  np.array(g["query_start_loc"], np.int32), 1, g["scale"], True)
    assert np.array_equal(out, np.array(g["expected"], dtype=np.float64))


def test_golden_smallseq_segments():
    g = load_golden("smallseq_segments")
    out = oracle.attention_smallseq(bits(g["q"]), bits(g["k"]), bits(g["v"]),
                                    np.array(g["cu_seqlens_kv"], np.int32), 1, g["scale"])
    assert np.allclose(out, np.array(g["expected"], dtype=np.float64), rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# cache write: literal loop vs numpy fancy indexing
# ---------------------------------------------------------------------------

def test_write_kv_matches_fancy_indexing_and_leaves_rest():
    rng = np.random.default_rng(5)
    nb, bs, h, d, t = 9, 16, 2, 8, 40
    slots = rng.permutation(nb * bs)[:t].astype(np.int64)
    slots[3] = -1
    slots[11] = -5
    k = rng.integers(0, 2**16, size=(t, h, d), dtype=np.uint16)
    v = rng.integers(0, 2**16, size=(t, h, d), dtype=np.uint16)
    kc = rng.integers(0, 2**16, size=(nb, bs, h, d), dtype=np.uint16)
    vc = rng.integers(0, 2**16, size=(nb, bs, h, d), dtype=np.uint16)
    ek, ev = kc.copy(), vc.copy()
    keep = slots >= 0
    ek.reshape(-1, h, d)[slots[keep]] = k[keep]
    ev.reshape(-1, h, d)[slots[keep]] = v[keep]
    assert oracle.write_kv(k, v, slots, kc, vc, bs) == 0
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev)


def test_write_kv_counts_out_of_pool_slots():
    nb, bs, h, d = 2, 4, 1, 2
    kc = np.zeros((nb, bs, h, d), np.uint16)
    vc = kc.copy()
    k = np.ones((3, h, d), np.uint16)
    bad = oracle.write_kv(k, k, np.array([0, 8, 100], np.int64), kc, vc, bs)
    assert bad == 2
    assert kc.reshape(-1, h, d)[0].tolist() == [[1, 1]]
    assert kc.sum() == 2


# ---------------------------------------------------------------------------
# closed forms and invariants
# ---------------------------------------------------------------------------

def small_case(seq_lens, query_lens, hq=4, hkv=2, d=16, causal=True, seed=7, **kw):
    return workloads.build_varlen_case("pin", seq_lens, query_lens, hq, hkv, d, causal, seed,
                                       **kw)


def test_identical_keys_give_mean_of_visible_values():
    case = small_case([9, 6], [4, 6])
    case.k_logical[:] = case.k_logical[0:1]          # every key the same vector
    out = run_logical(case)
    qsl = case.query_start_loc.tolist()
    g = case.num_q_heads // case.num_kv_heads
    for s in range(case.num_seqs):
        lq, lkv = qsl[s + 1] - qsl[s], int(case.seq_lens[s])
        o0 = int(case.kv_offsets[s])
        for i in range(lq):
            n = (lkv - lq) + i + 1
            for h in range(case.num_q_heads):
                mean = case.v_logical[o0:o0 + n, h // g].double().mean(0).numpy()
                assert np.allclose(out[qsl[s] + i, h], mean, rtol=0, atol=1e-12)


def test_single_visible_key_returns_its_value_row():
    case = small_case([5], [5])
    out = run_logical(case)
    g = case.num_q_heads // case.num_kv_heads
    for h in range(case.num_q_heads):   # causal row 0 sees key 0 only
        assert np.array_equal(out[0, h], case.v_logical[0, h // g].double().numpy())


def test_fully_masked_rows_are_zero():
    case = small_case([0, 2], [3, 4])   # L_kv = 0, and L_q > L_kv
    out = run_logical(case)
    assert np.all(out[0:3] == 0.0)
    assert np.all(out[3:5] == 0.0)      # rows 0, 1 of seq 1: (2 - 4) + i + 1 <= 0
    assert np.all(np.abs(out[5:7]).sum(-1) > 0)


def test_causal_equals_brute_force_prefix_attention():
    case = small_case([23, 11], [7, 11], d=8)
    out = run_logical(case)
    qsl = case.query_start_loc.tolist()
    for s in range(case.num_seqs):
        lq, lkv = qsl[s + 1] - qsl[s], int(case.seq_lens[s])
        o0 = int(case.kv_offsets[s])
        for i in range(lq):
            n = (lkv - lq) + i + 1          # non-causal attention over the prefix
            t = qsl[s] + i
            single = oracle.attention_varlen(
                workloads.bf16_bits(case.q[t:t + 1]),
                workloads.bf16_bits(case.k_logical[o0:o0 + n]),
                workloads.bf16_bits(case.v_logical[o0:o0 + n]),
                np.array([0], np.int64), np.array([n], np.int32), np.array([0, 1], np.int32),
                case.num_kv_heads, case.scale, False)
            assert np.array_equal(out[t], single[0])


def test_paged_form_equals_logical_form():
    case = small_case([37, 1, 16, 17], [5, 1, 16, 2], hq=6, hkv=3, d=32, pool_blocks=12)
    kc, vc = workloads.bf16_bits(case.k_cache), workloads.bf16_bits(case.v_cache)
    kc, vc = kc.copy(), vc.copy()
    oracle.write_kv(workloads.bf16_bits(case.k_new), workloads.bf16_bits(case.v_new),
                    case.slot_mapping.numpy(), kc, vc, case.block_size)
    paged = oracle.attention_varlen_paged(workloads.bf16_bits(case.q), kc, vc,
                                          case.block_tables.numpy(), case.seq_lens.numpy(),
                                          case.query_start_loc.numpy(), case.num_kv_heads,
                                          case.scale, True)
    assert np.array_equal(paged, run_logical(case))


def test_block_table_permutation_leaves_output_unchanged():
    lens, qlens = [40, 20], [40, 20]
    a = small_case(lens, qlens, seed=11, pool_blocks=7)
    b = small_case(lens, qlens, seed=11, pool_blocks=7)
    # same data, different physical placement: re-place b's pages under a new permutation
    perm = torch.tensor([3, 6, 0, 5, 1, 4, 2], dtype=torch.int32)
    new_table = b.block_tables.clone()
    valid = new_table < 7
    new_table[valid] = perm[new_table[valid].long()]
    kc = torch.empty_like(b.k_cache)
    vc = torch.empty_like(b.v_cache)
    kc[perm.long()] = b.k_cache
    vc[perm.long()] = b.v_cache
    outs = []
    for table, k_c, v_c in ((a.block_tables, a.k_cache, a.v_cache), (new_table, kc, vc)):
        kk, vv = workloads.bf16_bits(k_c).copy(), workloads.bf16_bits(v_c).copy()
        sm = a.slot_mapping if table is a.block_tables else None
        if sm is None:   # slots follow the permuted table
            sm = (perm[(a.slot_mapping // 16).long()].long() * 16 + a.slot_mapping % 16)
        oracle.write_kv(workloads.bf16_bits(a.k_new), workloads.bf16_bits(a.v_new),
                        sm.numpy(), kk, vv, 16)
        outs.append(oracle.attention_varlen_paged(
            workloads.bf16_bits(a.q), kk, vv, table.numpy(), a.seq_lens.numpy(),
            a.query_start_loc.numpy(), a.num_kv_heads, a.scale, True))
    assert np.array_equal(outs[0], outs[1])


def test_gqa_equals_repeat_interleave_mha():
    case = small_case([19, 8], [19, 3], hq=8, hkv=2, d=16)
    out = run_logical(case)
    q, k, v, off, sl, qsl = logical_inputs(case)
    k_rep = workloads.bf16_bits(case.k_logical.repeat_interleave(4, dim=1))
    v_rep = workloads.bf16_bits(case.v_logical.repeat_interleave(4, dim=1))
    mha = oracle.attention_varlen(q, k_rep, v_rep, off, sl, qsl, 8, case.scale, True)
    assert np.array_equal(out, mha)


def test_linearity_in_values():
    case = small_case([13], [6], d=8)
    rng = np.random.default_rng(3)
    v1 = rng.integers(-60, 60, size=case.v_logical.shape).astype(np.float32)
    v2 = rng.integers(-60, 60, size=case.v_logical.shape).astype(np.float32)
    q, k, _, off, sl, qsl = logical_inputs(case)
    o1 = oracle.attention_varlen(q, k, bits(v1), off, sl, qsl, 2, case.scale, True)
    o2 = oracle.attention_varlen(q, k, bits(v2), off, sl, qsl, 2, case.scale, True)
    o12 = oracle.attention_varlen(q, k, bits(v1 + v2), off, sl, qsl, 2, case.scale, True)
    assert np.allclose(o12, o1 + o2, rtol=0, atol=1e-10)


def test_weights_sum_to_one_and_vanish_when_masked():
    case = small_case([12, 5], [4, 5])
    q, k, v, off, sl, qsl = logical_inputs(case)
    for t in range(case.num_q_tokens):
        for h in range(case.num_q_heads):
            w, n = oracle.attention_weights(q, k, v, off, sl, qsl, 2, case.scale, True, t, h)
            assert abs(w.sum() - 1.0) < 1e-12
            assert np.all(w[n:] == 0.0) and np.all(w[:n] > 0.0)


def test_chunked_prefill_rows_equal_full_prefill_rows():
    full = small_case([30], [30], seed=21)
    chunk = small_case([30], [30], seed=21)
    out_full = run_logical(full)
    # same sequence, but only its last 9 tokens are queries (prior context 21)
    q_last = workloads.bf16_bits(full.q[21:])
    out_chunk = oracle.attention_varlen(q_last, workloads.bf16_bits(chunk.k_logical),
                                        workloads.bf16_bits(chunk.v_logical),
                                        np.array([0], np.int64), np.array([30], np.int32),
                                        np.array([0, 9], np.int32), 2, full.scale, True)
    assert np.array_equal(out_chunk, out_full[21:])


def test_decode_equals_last_row_of_full_prefill():
    full = small_case([17], [17], seed=4)
    out_full = run_logical(full)
    dec = oracle.attention_varlen(workloads.bf16_bits(full.q[16:]),
                                  workloads.bf16_bits(full.k_logical),
                                  workloads.bf16_bits(full.v_logical), np.array([0], np.int64),
                                  np.array([17], np.int32), np.array([0, 1], np.int32), 2,
                                  full.scale, True)
    assert np.array_equal(dec[0], out_full[16])


# ---------------------------------------------------------------------------
# independent library routine: torch SDPA (float64, CPU)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [True, False])
def test_tiny_config_matches_torch_sdpa(causal):
    case = workloads.tiny_prefill()
    assert np.allclose(run_logical(case, causal=causal), sdpa_reference(case, causal=causal),
                       rtol=0, atol=1e-12)


@pytest.mark.parametrize("lens,qlens,hq,hkv,d", [
    ([1, 16, 17, 33], [1, 16, 5, 33], 8, 2, 64),
    ([50, 3, 128], [1, 1, 40], 16, 2, 128),
    ([300], [130], 4, 4, 32),
])
def test_random_cases_match_torch_sdpa(lens, qlens, hq, hkv, d):
    case = small_case(lens, qlens, hq=hq, hkv=hkv, d=d, seed=sum(lens))
    assert np.allclose(run_logical(case), sdpa_reference(case), rtol=0, atol=1e-12)


def test_row_subset_matches_full_run():
    case = small_case([40, 9], [12, 9])
    full = run_logical(case)
    rows = np.array([0, 5, 11, 12, 20], np.int64)
    part = run_logical(case, rows=rows)
    assert np.array_equal(part[rows], full[rows])
    others = np.setdiff1d(np.arange(case.num_q_tokens), rows)
    assert np.all(part[others] == 0.0)


def test_smallseq_equals_varlen_with_one_query():
    case = workloads.build_smallseq_case("pin", [2, 0, 16, 5, 12], 8, 4, 64, seed=9)
    out = oracle.attention_smallseq(workloads.bf16_bits(case.q), workloads.bf16_bits(case.k),
                                    workloads.bf16_bits(case.v), case.cu_seqlens_kv.numpy(),
                                    4, case.scale)
    cu = case.cu_seqlens_kv.numpy()
    lens = np.diff(cu).astype(np.int32)
    ref = oracle.attention_varlen(workloads.bf16_bits(case.q), workloads.bf16_bits(case.k),
                                  workloads.bf16_bits(case.v), cu[:-1].astype(np.int64), lens,
                                  np.arange(len(lens) + 1, dtype=np.int32), 4, case.scale,
                                  False)
    assert np.array_equal(out, ref)
    assert np.all(out[1] == 0.0)
    # and against SDPA per entry
    for b in range(case.batch):
        n = int(lens[b])
        if n == 0:
            continue
        q = case.q[b:b + 1].double().transpose(0, 1)
        k = case.k[cu[b]:cu[b] + n].double().repeat_interleave(2, dim=1).transpose(0, 1)
        v = case.v[cu[b]:cu[b] + n].double().repeat_interleave(2, dim=1).transpose(0, 1)
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=case.scale)
        assert np.allclose(out[b], o.transpose(0, 1)[0].numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_scale_zero_gives_mean_of_visible_values(causal):
    """Closed form (pin i with every score equal): at scale 0 each visible key
    has weight 1/|V_i|, so the output is the plain mean of the visible V rows.
    Visible set of query i of a sequence with Lq queries over Lkv keys: all
    Lkv keys, or with causality the first Lkv - Lq + i + 1 (vllm-omni PR
    #9244, kernel-semantics review)."""
    case = workloads.build_varlen_case("pin", [9, 30, 1, 17], [9, 4, 1, 17], 6, 3, 64, causal,
                                       seed=31, scale=0.0)
    out = run_logical(case)
    qsl = case.query_start_loc.tolist()
    g = case.num_q_heads // case.num_kv_heads
    for s in range(case.num_seqs):
        lkv = int(case.seq_lens[s])
        lq = qsl[s + 1] - qsl[s]
        vals = case.v_logical[int(case.kv_offsets[s]):int(case.kv_offsets[s]) + lkv].double()
        for i in range(lq):
            n = (lkv - lq + i + 1) if causal else lkv
            mean = vals[:n].mean(dim=0).repeat_interleave(g, dim=0).numpy()   # [Hq, D]
            assert np.allclose(out[qsl[s] + i], mean, rtol=0, atol=1e-12)


def test_smallseq_scale_zero_gives_mean_of_values():
    case = workloads.build_smallseq_case("pin", [3, 0, 16, 1], 4, 2, 64, seed=12, scale=0.0)
    out = oracle.attention_smallseq(workloads.bf16_bits(case.q), workloads.bf16_bits(case.k),
                                    workloads.bf16_bits(case.v), case.cu_seqlens_kv.numpy(),
                                    2, 0.0)
    cu = case.cu_seqlens_kv.tolist()
    for b in range(case.batch):
        if cu[b + 1] == cu[b]:
            assert np.all(out[b] == 0.0)
            continue
        mean = case.v[cu[b]:cu[b + 1]].double().mean(dim=0).repeat_interleave(2, dim=0)
        assert np.allclose(out[b], mean.numpy(), rtol=0, atol=1e-12)
