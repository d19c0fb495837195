"""GPU parity for cache blocks larger than 16 slots.

The block size is a parameter of the paged cache (vllm-spyre PR #853, the
get_kv_cache_shape change: (num_blocks, 2, block_size, num_kv_heads,
head_size)); serving stacks commonly use 16, 32 or 64.  The kernels fetch keys
in 16-slot pages, so a block of 16k slots holds k pages, and page p of a
sequence is slots [16 (p mod k), +16) of block block_tables[s][p / k].  Each
case scatters through slot_mapping and attends, against the fp64 oracle;
the cache write must be bit-exact over the whole pool."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_gqa_reshape_b200 as pa
import workloads
from tests.gpu_helpers import assert_attention_close, case_to, oracle_varlen, run_varlen

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def build(lens, qlens, hq, hkv, d, bs, causal=True, seed=0, dtype=torch.bfloat16):
    return workloads.build_varlen_case("bs", lens, qlens, hq, hkv, d, causal, seed,
                                       block_size=bs, dtype=dtype)


def oracle_pool(cpu):
    kc = workloads.bf16_bits(cpu.k_cache).copy()
    vc = workloads.bf16_bits(cpu.v_cache).copy()
    oracle.write_kv(workloads.bf16_bits(cpu.k_new), workloads.bf16_bits(cpu.v_new),
                    cpu.slot_mapping.numpy(), kc, vc, cpu.block_size)
    return kc, vc


@pytest.mark.parametrize("bs", [32, 64, 128])
@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("causal", [True, False])
def test_prefill_block_sizes(bs, d, causal):
    lens = [2, 17, 31, 33, 129, 300, 513]
    cpu = build(lens, lens, 8, 2, d, bs, causal, seed=bs + d)
    out, kc, vc, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what=f"prefill bs={bs} d={d}")
    ek, ev = oracle_pool(cpu)
    assert np.array_equal(workloads.bf16_bits(kc), ek)
    assert np.array_equal(workloads.bf16_bits(vc), ev)
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("bs", [32, 64, 256])
@pytest.mark.parametrize("g,hkv", [(4, 8), (8, 2), (16, 1)])
def test_decode_block_sizes(bs, g, hkv):
    lens = [1, 15, 16, 17, 31, 32, 33, 63, 64, 65, 255, 257, 700, 2049, 5000]
    cpu = build(lens, [1] * len(lens), g * hkv, hkv, 128, bs, seed=bs + g)
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what=f"decode bs={bs} g={g}")
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("bs", [32, 64])
def test_mixed_and_chunked_block_sizes(bs):
    lens = [700, 40, 300, 1, 2000, 17, 5, 129, 600, 1000]
    qlens = [64, 1, 300, 1, 1, 17, 1, 100, 100, 130]
    cpu = build(lens, qlens, 16, 2, 128, bs, seed=bs)
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what=f"mixed bs={bs}")
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("bs", [32, 64])
def test_fp16_block_sizes(bs):
    lens = [300, 1, 1000, 129]
    qlens = [300, 1, 1, 64]
    cpu = build(lens, qlens, 16, 4, 128, bs, seed=3 + bs, dtype=torch.float16)
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    ref = oracle.attention_varlen_dtype(
        workloads.bf16_bits(cpu.q), workloads.bf16_bits(cpu.k_logical),
        workloads.bf16_bits(cpu.v_logical), cpu.kv_offsets.numpy(), cpu.seq_lens.numpy(),
        cpu.query_start_loc.numpy(), cpu.num_kv_heads, cpu.scale, cpu.causal, 1)
    assert_attention_close(out, ref, what=f"fp16 bs={bs}")
    assert pa.get_error(ws) == (0, 0)


def hnd_cache(c):
    """The same cache contents stored head-major [NB, Hkv, BS, D], as an
    [NB, BS, Hkv, D]-indexed view."""
    return c.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)


@pytest.mark.parametrize("bs", [32, 64])
def test_head_major_cache_block_sizes_bit_identical(bs):
    # the same contents stored head-major give bit-identical results
    lens = [300, 1, 2000, 129, 45]
    qlens = [300, 1, 1, 64, 1]
    cpu = build(lens, qlens, 8, 2, 128, bs, seed=9 + bs)
    dev = case_to(cpu, "cuda")
    ref_out, ref_kc, ref_vc, _ = run_varlen(dev)
    kc, vc = hnd_cache(dev.k_cache), hnd_cache(dev.v_cache)
    ws = pa.varlen_workspace(dev.num_seqs, dev.num_q_tokens, 8, 2, 128)
    pa.write_kv(dev.k_new, dev.v_new, dev.slot_mapping, kc, vc, workspace=ws)
    assert torch.equal(kc, ref_kc) and torch.equal(vc, ref_vc)
    out = torch.full_like(dev.q, float("nan"))
    pa.attention_varlen(dev.q, kc, vc, dev.block_tables, dev.seq_lens, dev.query_start_loc, 2,
                        dev.scale, True, out, max_query_len=dev.max_query_len,
                        max_seq_len=dev.max_seq_len, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out)
    assert_attention_close(out, oracle_varlen(cpu), what=f"head-major bs={bs}")
    assert pa.get_error(ws) == (0, 0)


def test_bad_block_id_with_large_blocks_is_reported_not_faulted():
    cpu = build([100, 40], [1, 40], 8, 2, 128, 32, seed=10)
    cpu.block_tables[0, 2] = cpu.num_blocks + 1000
    cpu.block_tables[1, 0] = -5
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"), scatter=False)
    assert torch.isfinite(out.float()).all()
    st, bits = pa.get_error(ws)
    assert st == pa.PA_ERR_DEVICE_INDEX and bits & pa.DEVERR_BLOCK


# ---------------------------------------------------------------------------
# GQA groups above 16 (MQA included): the decode kernel cuts a group into
# 16-head slices served by warps that share the KV head's pages
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("g,hkv,d", [(32, 2, 128), (64, 1, 128), (128, 1, 128), (20, 2, 128),
                                     (48, 1, 64), (24, 4, 64)])
def test_decode_large_groups(g, hkv, d):
    lens = [0, 1, 15, 16, 17, 255, 700, 2049, 5000]
    cpu = build(lens, [1 if l > 0 else 0 for l in lens], g * hkv, hkv, d, 16, seed=g + hkv)
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what=f"decode g={g} hkv={hkv} d={d}")
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("g,hkv,bs", [(32, 2, 32), (64, 1, 16)])
def test_mixed_large_groups(g, hkv, bs):
    lens = [700, 40, 300, 1, 2000, 17, 5, 129]
    qlens = [64, 1, 300, 1, 1, 17, 1, 100]
    cpu = build(lens, qlens, g * hkv, hkv, 128, bs, seed=g)
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what=f"mixed g={g} bs={bs}")
    assert pa.get_error(ws) == (0, 0)


def test_large_group_equals_repeat_interleaved_heads():
    # GQA as the explicit repeat_interleave of the KV heads (vllm-spyre PR
    # #853, description): g = 64 over 1 KV head against the same cache with
    # the head repeated 64 times and g = 1 (the split points of the two runs
    # differ, so they agree to rounding, not bit for bit)
    import dataclasses
    lens = [3000, 1, 777, 64]
    cpu = build(lens, [1] * 4, 64, 1, 128, 16, seed=5)
    dev = case_to(cpu, "cuda")
    out_g, kc, vc, _ = run_varlen(dev)
    mha_dev = dataclasses.replace(dev, num_kv_heads=64,
                                  k_cache=kc.repeat_interleave(64, dim=2).contiguous(),
                                  v_cache=vc.repeat_interleave(64, dim=2).contiguous())
    out_m, _, _, _ = run_varlen(mha_dev, scatter=False)
    assert_attention_close(out_g, oracle_varlen(cpu), what="g=64")
    assert (out_g.float() - out_m.float()).abs().max().item() <= 2e-2


@pytest.mark.parametrize("per_head", [True, False])
def test_large_group_with_modifiers(per_head):
    # per_head False: one mask row per token shared by every head (head stride 0)
    lens = [300, 1, 2000, 129]
    qlens = [300, 1, 1, 64]
    hq, hkv = 64, 2
    cpu = build(lens, qlens, hq, hkv, 128, 32, seed=77)
    dev = case_to(cpu, "cuda")
    slopes = torch.tensor([2.0 ** (-8.0 * (h + 1) / hq) for h in range(hq)], dtype=torch.float32)
    t, ld = cpu.num_q_tokens, 2048  # mask rows longer than every sequence
    g = torch.Generator().manual_seed(8)
    shape = (hq, t, ld) if per_head else (t, ld)
    mask = torch.randn(shape, generator=g)
    mask[torch.rand(shape, generator=g) < 0.05] = float("-inf")
    kc, vc = dev.k_cache.clone(), dev.v_cache.clone()
    ws = pa.varlen_workspace(dev.num_seqs, t, hq, hkv, 128)
    pa.write_kv(dev.k_new, dev.v_new, dev.slot_mapping, kc, vc, workspace=ws)
    out = torch.full_like(dev.q, float("nan"))
    pa.attention_varlen(dev.q, kc, vc, dev.block_tables, dev.seq_lens, dev.query_start_loc, hkv,
                        dev.scale, True, out, max_query_len=dev.max_query_len,
                        max_seq_len=dev.max_seq_len, workspace=ws, softcap=30.0,
                        alibi_slopes=slopes.cuda(), mask=mask.cuda())
    torch.cuda.synchronize()
    ref = oracle.attention_varlen_mods(
        workloads.bf16_bits(cpu.q), workloads.bf16_bits(cpu.k_logical),
        workloads.bf16_bits(cpu.v_logical), cpu.kv_offsets.numpy(), cpu.seq_lens.numpy(),
        cpu.query_start_loc.numpy(), hkv, cpu.scale, True, 0, softcap=30.0,
        alibi_slopes=slopes.numpy(), mask=mask.contiguous().numpy().reshape(-1),
        mask_head_stride=t * ld if per_head else 0, mask_token_stride=ld)
    assert_attention_close(out, ref, what=f"g=32 with modifiers, per-head mask {per_head}")
    assert pa.get_error(ws) == (0, 0)


# ---------------------------------------------------------------------------
# large blocks with the other features: full-attention spans and an additive
# mask (prefill, chunked prefill and decode rows in one batch)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bs", [32, 128])
def test_spans_with_large_blocks(bs):
    from tests.test_gpu_spans import oracle_spans, run_spans
    lens = [700, 300, 129, 1000, 40]
    qlens = [700, 300, 129, 400, 1]
    spans_per_seq = [[(0, 100), (100, 300), (517, 700)], [(128, 256)], [],
                     [(610, 900), (900, 901), (950, 1000)], [(0, 40)]]
    cpu = build(lens, qlens, 8, 2, 128, bs, seed=60 + bs)
    offs = np.cumsum([0] + [len(x) for x in spans_per_seq])
    flat = [p for x in spans_per_seq for p in x]
    out, ws = run_spans(case_to(cpu, "cuda"), offs, flat)
    assert_attention_close(out, oracle_spans(cpu, offs, flat), what=f"spans bs={bs}")
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("bs", [32, 64])
def test_additive_mask_with_large_blocks(bs):
    lens, qlens = [400, 33, 129, 1000], [400, 1, 64, 1]
    cpu = build(lens, qlens, 8, 2, 64, bs, seed=70 + bs)
    dev = case_to(cpu, "cuda")
    t, ld = cpu.num_q_tokens, 1024
    g = torch.Generator().manual_seed(71)
    mask = torch.randn((8, t, ld), generator=g) * 2
    mask[torch.rand((8, t, ld), generator=g) < 0.05] = float("-inf")
    kc, vc = dev.k_cache.clone(), dev.v_cache.clone()
    ws = pa.varlen_workspace(dev.num_seqs, t, 8, 2, 64)
    pa.write_kv(dev.k_new, dev.v_new, dev.slot_mapping, kc, vc, workspace=ws)
    out = torch.full_like(dev.q, float("nan"))
    pa.attention_varlen(dev.q, kc, vc, dev.block_tables, dev.seq_lens, dev.query_start_loc, 2,
                        dev.scale, True, out, max_query_len=dev.max_query_len,
                        max_seq_len=dev.max_seq_len, workspace=ws, mask=mask.cuda())
    torch.cuda.synchronize()
    ref = oracle.attention_varlen_mods(
        workloads.bf16_bits(cpu.q), workloads.bf16_bits(cpu.k_logical),
        workloads.bf16_bits(cpu.v_logical), cpu.kv_offsets.numpy(), cpu.seq_lens.numpy(),
        cpu.query_start_loc.numpy(), 2, cpu.scale, True, 0,
        mask=mask.contiguous().numpy().reshape(-1), mask_head_stride=t * ld,
        mask_token_stride=ld)
    assert_attention_close(out, ref, what=f"mask bs={bs}")
    assert pa.get_error(ws) == (0, 0)
