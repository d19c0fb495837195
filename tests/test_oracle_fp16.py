"""Pins for the oracle's fp16 inputs (ROCm/TransformerEngine PR #461 adds FP16 to
the small-seq path; vllm-spyre PR #853 runs in fp16): exact widening of every
binary16 pattern, and attention on fp16 inputs against torch SDPA in float64."""
import numpy as np
import torch

import oracle
import workloads


def test_every_fp16_pattern_widens_exactly():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.widen(int(b), 1) for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])


def test_bf16_patterns_widen_exactly():
    bits = np.arange(0, 1 << 16, 97, dtype=np.uint32).astype(np.uint16)
    ref = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    got = np.array([oracle.widen(int(b), 0) for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])


def test_fp16_varlen_matches_torch_sdpa():
    lens, qlens = [130, 40, 1, 257], [130, 17, 1, 100]
    case = workloads.build_varlen_case("f16", lens, qlens, 8, 2, 64, True, seed=12,
                                       dtype=torch.float16)
    got = oracle.attention_varlen_dtype(
        workloads.bf16_bits(case.q), workloads.bf16_bits(case.k_logical),
        workloads.bf16_bits(case.v_logical), case.kv_offsets.numpy(), case.seq_lens.numpy(),
        case.query_start_loc.numpy(), case.num_kv_heads, case.scale, True, 1)
    qsl = case.query_start_loc.tolist()
    for s in range(4):
        lq, lkv = qsl[s + 1] - qsl[s], lens[s]
        o0 = int(case.kv_offsets[s])
        q = case.q[qsl[s]:qsl[s + 1]].double().transpose(0, 1)
        k = case.k_logical[o0:o0 + lkv].double().repeat_interleave(4, dim=1).transpose(0, 1)
        v = case.v_logical[o0:o0 + lkv].double().repeat_interleave(4, dim=1).transpose(0, 1)
        i = torch.arange(lq)[:, None]
        j = torch.arange(lkv)[None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, k, v, attn_mask=j <= (lkv - lq) + i, scale=case.scale).transpose(0, 1).numpy()
        assert np.max(np.abs(got[qsl[s]:qsl[s + 1]] - ref)) < 1e-10


def test_fp16_smallseq_matches_torch_sdpa():
    lens = [0, 1, 5, 16, 2, 9]
    case = workloads.build_smallseq_case("f16s", lens, 4, 2, 128, seed=13, dtype=torch.float16)
    got = oracle.smallseq_dtype(workloads.bf16_bits(case.q), workloads.bf16_bits(case.k),
                                workloads.bf16_bits(case.v), case.cu_seqlens_kv.numpy(),
                                case.num_kv_heads, case.scale, 1)
    cu = case.cu_seqlens_kv.tolist()
    for b, n in enumerate(lens):
        if n == 0:
            assert not got[b].any()
            continue
        q = case.q[b:b + 1].double().transpose(0, 1)
        k = case.k[cu[b]:cu[b + 1]].double().repeat_interleave(2, dim=1).transpose(0, 1)
        v = case.v[cu[b]:cu[b + 1]].double().repeat_interleave(2, dim=1).transpose(0, 1)
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=case.scale)
        assert np.max(np.abs(got[b] - ref.transpose(0, 1)[0].numpy())) < 1e-10
