"""GPU parity: the sm_100a kernels (through the C ABI) against the fp64 oracle
on the same seeded inputs.  Cache writes must be bit-exact over the whole
pool; attention within max |err| <= 2e-2 and mean |err| <= 2e-3."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import paged_kv_gqa_reshape_b200 as pa
import workloads
from tests.gpu_helpers import (assert_attention_close, case_to, oracle_varlen, run_varlen,
                               sub_case)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def build(lens, qlens, hq, hkv, d, causal=True, seed=0, **kw):
    return workloads.build_varlen_case("t", lens, qlens, hq, hkv, d, causal, seed, **kw)


# ---------------------------------------------------------------------------
# KV scatter: bit-exact over the whole pool
# ---------------------------------------------------------------------------

def oracle_written_pool(case_cpu):
    kc = workloads.bf16_bits(case_cpu.k_cache).copy()
    vc = workloads.bf16_bits(case_cpu.v_cache).copy()
    bad = oracle.write_kv(workloads.bf16_bits(case_cpu.k_new), workloads.bf16_bits(case_cpu.v_new),
                          case_cpu.slot_mapping.numpy(), kc, vc, case_cpu.block_size)
    return kc, vc, bad


@pytest.mark.parametrize("name,lens,qlens,hkv,d", [
    ("tiny", [7, 13], [7, 13], 2, 64),
    ("ragged", [1, 15, 16, 17, 100, 300], [1, 15, 16, 5, 100, 1], 8, 128),
    ("one_head", [40, 9], [40, 9], 1, 64),
])
def test_write_kv_bit_exact_whole_pool(name, lens, qlens, hkv, d):
    cpu = build(lens, qlens, 2 * hkv, hkv, d, seed=len(name), pool_blocks=sum(
        (l + 15) // 16 for l in lens) + 3)
    dev = case_to(cpu, "cuda")
    kc, vc = dev.k_cache.clone(), dev.v_cache.clone()
    ws = pa.error_workspace()
    pa.write_kv(dev.k_new, dev.v_new, dev.slot_mapping, kc, vc, workspace=ws)
    ek, ev, bad = oracle_written_pool(cpu)
    assert bad == 0
    assert np.array_equal(workloads.bf16_bits(kc), ek)
    assert np.array_equal(workloads.bf16_bits(vc), ev)
    assert pa.get_error(ws) == (0, 0)


def test_write_kv_padding_and_out_of_pool_slots():
    cpu = build([20, 10], [20, 10], 4, 2, 64, seed=3, pool_blocks=4)
    cpu.slot_mapping[2] = -1
    cpu.slot_mapping[5] = 4 * 16 + 3          # beyond the pool
    dev = case_to(cpu, "cuda")
    kc, vc = dev.k_cache.clone(), dev.v_cache.clone()
    ws = pa.error_workspace()
    pa.write_kv(dev.k_new, dev.v_new, dev.slot_mapping, kc, vc, workspace=ws)
    ek, ev, bad = oracle_written_pool(cpu)
    assert bad == 1
    assert np.array_equal(workloads.bf16_bits(kc), ek)
    assert np.array_equal(workloads.bf16_bits(vc), ev)
    st, bits = pa.get_error(ws)
    assert st == 4 and bits == pa.DEVERR_SLOT
    assert pa.get_error(ws) == (0, 0)         # cleared by the read


def test_write_kv_varlen_config_full_size():
    cpu = workloads.varlen_prefill()
    dev = case_to(cpu, "cuda")
    kc, vc = dev.k_cache.clone(), dev.v_cache.clone()
    pa.write_kv(dev.k_new, dev.v_new, dev.slot_mapping, kc, vc)
    ek, ev, _ = oracle_written_pool(cpu)
    assert np.array_equal(workloads.bf16_bits(kc), ek)
    assert np.array_equal(workloads.bf16_bits(vc), ev)


# ---------------------------------------------------------------------------
# small-seq
# ---------------------------------------------------------------------------

def run_smallseq(case, max_seqlen_kv=16):
    out = torch.full_like(case.q, float("nan"))
    ws = pa.error_workspace()
    pa.attention_smallseq(case.q, case.k, case.v, case.cu_seqlens_kv, case.scale, out,
                          max_seqlen_kv=max_seqlen_kv, workspace=ws)
    torch.cuda.synchronize()
    return out, ws


def oracle_smallseq(case):
    return oracle.attention_smallseq(workloads.bf16_bits(case.q), workloads.bf16_bits(case.k),
                                     workloads.bf16_bits(case.v), case.cu_seqlens_kv.cpu().numpy(),
                                     case.num_kv_heads, case.scale)


@pytest.mark.parametrize("d,hq,hkv", [(128, 16, 16), (64, 8, 4), (128, 8, 2)])
def test_smallseq_small(d, hq, hkv):
    rng = np.random.default_rng(d + hq)
    lens = rng.integers(0, 17, size=700).tolist()
    lens[:4] = [0, 1, 16, 2]
    cpu = workloads.build_smallseq_case("s", lens, hq, hkv, d, seed=d + hq)
    out, ws = run_smallseq(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_smallseq(cpu), what="smallseq")
    assert torch.all(out[0] == 0)
    assert pa.get_error(ws) == (0, 0)


def test_smallseq_full_config():
    cpu = workloads.smallseq_batch()
    out, ws = run_smallseq(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_smallseq(cpu), what="smallseq full")
    assert pa.get_error(ws) == (0, 0)


def test_smallseq_length_beyond_hint_is_reported():
    cpu = workloads.build_smallseq_case("s", [4, 9, 2], 4, 4, 64, seed=2)
    _, ws = run_smallseq(case_to(cpu, "cuda"), max_seqlen_kv=8)
    st, bits = pa.get_error(ws)
    assert bits == pa.DEVERR_HINT


# ---------------------------------------------------------------------------
# decode (split-KV)
# ---------------------------------------------------------------------------

DECODE_LENS = [0, 1, 2, 15, 16, 17, 63, 64, 65, 255, 256, 257, 511, 512, 700, 1023, 1025, 2049,
               3000]


@pytest.mark.parametrize("g,hkv,d", [(4, 8, 128), (8, 2, 128), (1, 4, 128), (16, 1, 128),
                                     (4, 2, 64), (2, 3, 64)])
def test_decode_small(g, hkv, d):
    lens = DECODE_LENS
    cpu = build(lens, [1 if l > 0 else 0 for l in lens], g * hkv, hkv, d, seed=g * 10 + hkv)
    dev = case_to(cpu, "cuda")
    out, _, _, ws = run_varlen(dev)
    ref = oracle_varlen(cpu)
    assert_attention_close(out, ref, what=f"decode g={g} d={d}")
    assert pa.get_error(ws) == (0, 0)


def test_decode_full_config():
    cpu = workloads.decode_batch()
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what="decode full")
    assert pa.get_error(ws) == (0, 0)


def test_decode_zero_length_sequence_gives_zeros():
    cpu = build([0, 5], [1, 1], 4, 2, 64, seed=1)     # one query over zero keys
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert torch.all(out[0] == 0)
    assert_attention_close(out, oracle_varlen(cpu), what="decode with empty sequence")
    st, bits = pa.get_error(ws)
    assert bits == pa.DEVERR_QLEN


# ---------------------------------------------------------------------------
# prefill (tcgen05) and chunked prefill
# ---------------------------------------------------------------------------

def test_tiny_config():
    cpu = workloads.tiny_prefill()
    out, kc, vc, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what="tiny")
    ek, ev, _ = oracle_written_pool(cpu)
    assert np.array_equal(workloads.bf16_bits(kc), ek)
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("g,hkv", [(4, 2), (1, 3), (8, 1), (16, 1)])
def test_prefill_small(d, causal, g, hkv):
    lens = [2, 15, 16, 17, 127, 128, 129, 300, 513]
    cpu = build(lens, lens, g * hkv, hkv, d, causal=causal, seed=d + g + causal)
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what=f"prefill d={d} causal={causal} g={g}")
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("d", [128, 64])
def test_prefill_exact_tile_multiples(d):
    # query counts on 128-row tile / 256-row work-item boundaries, key counts on
    # 128-key KV-tile boundaries, and one work item whose second tile is empty
    seq_lens = [256, 384, 1024, 128, 512, 640]
    qlens = [256, 384, 128, 128, 256, 128]
    cpu = build(seq_lens, qlens, 8, 2, d, causal=True, seed=40 + d)
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what=f"tile multiples d={d}")
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("d", [128, 64])
def test_chunked_prefill_small(d):
    seq_lens = [600, 333, 129, 64, 1000, 17]
    qlens = [100, 333, 2, 37, 130, 16]           # prior context = seq_len - qlen
    cpu = build(seq_lens, qlens, 16, 2, d, causal=True, seed=d)
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what="chunked")
    assert pa.get_error(ws) == (0, 0)


def test_varlen_config_full_size_sampled_rows():
    cpu = workloads.varlen_prefill()
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    qsl = cpu.query_start_loc.tolist()
    rows = set()
    for s in range(cpu.num_seqs):
        for i in (0, 1, 127, 128, 129, 1000, 2047):
            if qsl[s] + i < qsl[s + 1]:
                rows.add(qsl[s] + i)
        rows.add(qsl[s + 1] - 1)
        rows.add(qsl[s + 1] - 2)
    rows = np.array(sorted(rows), dtype=np.int64)
    ref = oracle_varlen(cpu, rows=rows)
    assert_attention_close(out, ref, rows=rows, what="varlen full (sampled)")
    assert pa.get_error(ws) == (0, 0)


def test_mixed_small():
    lens = [700, 40, 300, 1, 2000, 17, 5, 129]
    qlens = [64, 1, 300, 1, 1, 17, 1, 100]
    cpu = build(lens, qlens, 16, 2, 128, causal=True, seed=11)
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what="mixed small")
    assert pa.get_error(ws) == (0, 0)


def test_mixed_config_full_size():
    """The full mixed chunked-prefill + decode step: every decode row, and every
    prefill chunk at its tile-edge rows (0, 1, 127-129, 255, 256, the last)
    plus every 37th row, each against the oracle.  The sequences are handed to
    the oracle a few at a time so that the host holds a slice of the 17 GB of
    logical K/V, not all of it."""
    dev = workloads.mixed_step(device="cuda")
    out, _, _, ws = run_varlen(dev)
    assert pa.get_error(ws) == (0, 0)
    qsl_full = dev.query_start_loc.cpu().tolist()
    n_seq = dev.num_seqs
    edges = (0, 1, 127, 128, 129, 255, 256, 383, 384, 511)
    got_all, ref_all = [], []
    batch = 32
    for first in range(0, n_seq, batch):
        picks = list(range(first, min(n_seq, first + batch)))
        sub = sub_case(dev, picks)
        sq = sub.query_start_loc.tolist()
        sub_rows, full_rows = [], []
        for k, s in enumerate(picks):
            n = qsl_full[s + 1] - qsl_full[s]
            take = range(n) if n <= 1 else sorted(
                {i for i in edges if i < n} | set(range(0, n, 37)) | {n - 1})
            for i in take:
                sub_rows.append(sq[k] + i)
                full_rows.append(qsl_full[s] + i)
        sub_rows = np.array(sub_rows, np.int64)
        ref_all.append(oracle_varlen(sub, rows=sub_rows)[sub_rows])
        got_all.append(out[torch.tensor(full_rows, device=out.device)].cpu())
        del sub
    got = torch.cat(got_all)
    ref = np.concatenate(ref_all)
    assert got.shape[0] == 248 + sum(
        len({i for i in edges if i < 512} | set(range(0, 512, 37)) | {511}) for _ in range(8))
    assert_attention_close(got, ref, what="mixed full (every decode, chunk edges)")


# ---------------------------------------------------------------------------
# invariants and error reporting on the GPU path
# ---------------------------------------------------------------------------

def test_decode_row_equals_last_prefill_row():
    full = build([777], [777], 8, 2, 128, seed=5)
    dec = dataclasses.replace(full, q=full.q[776:].clone(),
                              query_start_loc=torch.tensor([0, 1], dtype=torch.int32),
                              query_lens=torch.tensor([1], dtype=torch.int32),
                              k_new=full.k_new[:0], v_new=full.v_new[:0],
                              slot_mapping=full.slot_mapping[:0])
    dev_full = case_to(full, "cuda")
    out_full, kc, vc, _ = run_varlen(dev_full)
    dev_dec = case_to(dec, "cuda")
    dev_dec = dataclasses.replace(dev_dec, k_cache=kc, v_cache=vc)
    out_dec, _, _, _ = run_varlen(dev_dec, scatter=False)
    a, b = out_full[776].double(), out_dec[0].double()
    assert (a - b).abs().max().item() <= 2e-2


def test_block_table_permutation_gives_identical_output():
    cpu = build([300, 45, 1000], [300, 1, 64], 8, 2, 128, seed=8)
    dev = case_to(cpu, "cuda")
    out_a, kc, vc, _ = run_varlen(dev)
    nb = cpu.num_blocks
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(1)).cuda()
    kc2, vc2 = torch.empty_like(kc), torch.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    table = dev.block_tables.clone()
    valid = table < nb
    table[valid] = perm[table[valid].long()].int()
    dev2 = dataclasses.replace(dev, k_cache=kc2, v_cache=vc2, block_tables=table)
    out_b, _, _, _ = run_varlen(dev2, scatter=False)
    assert torch.equal(out_a, out_b)


def test_repeated_calls_are_bit_identical():
    cpu = build([900, 1, 3000, 128], [900, 1, 1, 64], 16, 2, 128, seed=9)
    dev = case_to(cpu, "cuda")
    a = run_varlen(dev)[0]
    b = run_varlen(dev)[0]
    assert torch.equal(a, b)


def test_query_longer_than_keys_flags_and_zero_rows():
    # sequence 0: 5 queries over 3 keys, causal; rows 0 and 1 see no key
    cpu = build([3, 20], [3, 20], 4, 2, 64, seed=4)
    q = workloads._randn_bf16((25, 4, 64), torch.Generator().manual_seed(6), "cpu")
    cpu = dataclasses.replace(cpu, q=q, query_start_loc=torch.tensor([0, 5, 25], dtype=torch.int32),
                              query_lens=torch.tensor([5, 20], dtype=torch.int32))
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert torch.all(out[0:2] == 0)
    assert_attention_close(out, oracle_varlen(cpu), what="queries beyond keys")
    st, bits = pa.get_error(ws)
    assert bits == pa.DEVERR_QLEN


def test_bad_block_id_is_reported_not_faulted():
    cpu = build([100, 40], [1, 40], 8, 2, 128, seed=10)
    cpu.block_tables[0, 2] = cpu.num_blocks + 1000
    cpu.block_tables[1, 0] = -5
    dev = case_to(cpu, "cuda")
    out, _, _, ws = run_varlen(dev, scatter=False)
    assert torch.isfinite(out.float()).all()
    st, bits = pa.get_error(ws)
    assert st == 4 and bits & pa.DEVERR_BLOCK


def test_prefill_with_decode_hint_is_reported():
    cpu = build([50, 60], [1, 10], 4, 2, 64, seed=12)
    dev = case_to(cpu, "cuda")
    _, _, _, ws = run_varlen(dev, max_query_len=1)
    st, bits = pa.get_error(ws)
    assert bits & pa.DEVERR_HINT


def test_decode_many_sequences_uses_plan_kernel_lists():
    # more sequences than the decode CTAs plan for themselves
    rng = np.random.default_rng(77)
    lens = rng.integers(0, 300, size=1100).tolist()
    cpu = build(lens, [1 if l > 0 else 0 for l in lens], 8, 2, 128, seed=77)
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what="decode, 1100 sequences")
    assert pa.get_error(ws) == (0, 0)


def test_decode_repeated_calls_reuse_counters():
    # split-KV arrival counters return to zero after every call
    cpu = build([5000, 3000, 17, 4096], [1, 1, 1, 1], 32, 8, 128, seed=13)
    dev = case_to(cpu, "cuda")
    ref = oracle_varlen(cpu)
    ws = pa.varlen_workspace(dev.num_seqs, dev.num_q_tokens, dev.num_q_heads, dev.num_kv_heads,
                             dev.head_dim)
    outs = [run_varlen(dev, workspace=ws)[0] for _ in range(3)]
    for o in outs:
        assert_attention_close(o, ref, what="repeated decode")
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])


def test_workspace_reused_across_batch_shapes():
    # One workspace, sized for the largest call, reused by calls of different
    # shapes in a row: a few long split-KV decodes (their partials fill the
    # workspace's scratch), then a larger pure-decode batch that plans for
    # itself, then a mixed batch, then the larger decode batch again.  The
    # arrival counters must read zero at the start of every call.
    a = build([5000, 4000, 3000, 6000, 2500, 4500, 3500, 5500], [1] * 8, 32, 8, 128, seed=21)
    rng = np.random.default_rng(22)
    lens_b = rng.integers(1, 3000, size=200).tolist()
    b = build(lens_b, [1] * 200, 32, 8, 128, seed=22)
    c = build([700, 40, 300, 1, 2000, 17, 5, 129], [64, 1, 300, 1, 1, 17, 1, 100], 32, 8, 128,
              seed=23)
    ws = pa.varlen_workspace(256, 1024, 32, 8, 128)
    for case in (a, b, c, b):
        out, _, _, _ = run_varlen(case_to(case, "cuda"), workspace=ws)
        assert_attention_close(out, oracle_varlen(case), what=f"reused workspace S={case.num_seqs}")
    assert pa.get_error(ws) == (0, 0)
