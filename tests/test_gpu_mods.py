"""Score modifiers (soft-cap, ALiBi, additive mask) and HND / NHD layouts of
the paged varlen attention on the GPU (auto_round_kernel PR "Migrate CPU SDPA
backend": additive masks and HND/NHD layouts in the public sdpa(); ALiBi
slopes and the TANH30 soft-cap among the library's extensions).

The modifiers are compared with the fp64 oracle given the same fp32 slopes
and mask values, to the attention tolerance.  A layout changes only where
the bytes sit, so a head-major run must give the token-major run's output
bit for bit (and the oracle's, to the tolerance)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_gqa_reshape_b200 as pa
import workloads
from tests.gpu_helpers import assert_attention_close, case_to, oracle_varlen, run_varlen

pytestmark = pytest.mark.gpu
DT = {torch.bfloat16: 0, torch.float16: 1}


def make(lens, qlens, hq, hkv, d, causal, seed, dtype=torch.bfloat16, scale=None):
    return workloads.build_varlen_case("mods", lens, qlens, hq, hkv, d, causal, seed,
                                       scale=scale, dtype=dtype)


def slopes_for(hq):
    return torch.tensor([2.0 ** (-8.0 * (h + 1) / hq) for h in range(hq)], dtype=torch.float32)


def oracle_mods(cpu, dtype=torch.bfloat16, softcap=0.0, slopes=None, mask=None):
    mk, hs, ts = None, 0, 0
    if mask is not None:
        mk = mask.contiguous().numpy().reshape(-1)
        ts = mask.shape[-1]
        hs = mask.shape[-2] * mask.shape[-1] if mask.dim() == 3 else 0
    return oracle.attention_varlen_mods(
        workloads.bf16_bits(cpu.q), workloads.bf16_bits(cpu.k_logical),
        workloads.bf16_bits(cpu.v_logical), cpu.kv_offsets.numpy(), cpu.seq_lens.numpy(),
        cpu.query_start_loc.numpy(), cpu.num_kv_heads, cpu.scale, cpu.causal, DT[dtype],
        softcap=softcap, alibi_slopes=None if slopes is None else slopes.numpy(), mask=mk,
        mask_head_stride=hs, mask_token_stride=ts)


def run_mods(dev, **kw):
    kc, vc = dev.k_cache.clone(), dev.v_cache.clone()
    ws = pa.varlen_workspace(dev.num_seqs, dev.num_q_tokens, dev.num_q_heads, dev.num_kv_heads,
                             dev.head_dim)
    pa.write_kv(dev.k_new, dev.v_new, dev.slot_mapping, kc, vc, workspace=ws)
    out = torch.full_like(dev.q, float("nan"))
    pa.attention_varlen(dev.q, kc, vc, dev.block_tables, dev.seq_lens, dev.query_start_loc,
                        dev.num_kv_heads, dev.scale, dev.causal, out,
                        max_query_len=dev.max_query_len, max_seq_len=dev.max_seq_len,
                        workspace=ws, **kw)
    torch.cuda.synchronize()
    return out, ws


# prefill, chunked prefill (prior context) and decode sequences in one batch
LENS = [700, 40, 300, 1, 2000, 17, 129, 513]
QLENS = [64, 1, 300, 1, 1, 17, 100, 513]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("d,g,hkv", [(128, 4, 2), (64, 16, 1), (128, 1, 4)])
def test_alibi(d, g, hkv, dtype):
    cpu = make(LENS, QLENS, g * hkv, hkv, d, True, seed=40 + d + g, dtype=dtype)
    sl = slopes_for(g * hkv)
    out, ws = run_mods(case_to(cpu, "cuda"), alibi_slopes=sl.cuda())
    assert_attention_close(out, oracle_mods(cpu, dtype, slopes=sl), what="alibi")
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("cap", [30.0, 2.0, 0.5])
def test_softcap(cap, dtype):
    # scale * s ~ N(0, 1) at the usual 1/sqrt(D) scale: cap 30 (TANH30) barely
    # bends it, caps 2 and 0.5 bend it strongly.  (A larger scale makes the
    # softmax nearly one-hot, where P's rounding to 16 bits for P.V dominates
    # the error with or without a cap.)
    cpu = make(LENS, QLENS, 8, 2, 128, True, seed=41, dtype=dtype)
    out, ws = run_mods(case_to(cpu, "cuda"), softcap=cap)
    assert_attention_close(out, oracle_mods(cpu, dtype, softcap=cap), what=f"softcap {cap}")
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("per_head", [False, True])
@pytest.mark.parametrize("causal", [True, False])
def test_additive_mask(per_head, causal):
    lens, qlens = [400, 33, 129, 1000], [400, 1, 64, 1]
    cpu = make(lens, qlens, 8, 2, 64, causal, seed=42)
    t, ld = cpu.num_q_tokens, 1024  # rows longer than every sequence, padded to 16 bytes
    g = torch.Generator().manual_seed(7)
    shape = (8, t, ld) if per_head else (t, ld)
    mask = torch.randn(shape, generator=g) * 2
    mask[torch.rand(shape, generator=g) < 0.05] = float("-inf")
    out, ws = run_mods(case_to(cpu, "cuda"), mask=mask.cuda())
    assert_attention_close(out, oracle_mods(cpu, mask=mask), what="mask")
    assert pa.get_error(ws) == (0, 0)


def test_all_modifiers_together_and_fully_masked_rows():
    lens, qlens = [300, 80, 1, 257], [300, 1, 1, 129]
    cpu = make(lens, qlens, 16, 4, 128, True, seed=43)
    t, ld = cpu.num_q_tokens, 304
    g = torch.Generator().manual_seed(8)
    mask = torch.randn(16, t, ld, generator=g)
    mask[3, 5, :] = float("-inf")            # token 5, head 3: nothing visible
    mask[:, 300, :] = float("-inf")          # the decode token of sequence 1: all heads
    sl = slopes_for(16)
    out, ws = run_mods(case_to(cpu, "cuda"), softcap=30.0, alibi_slopes=sl.cuda(),
                       mask=mask.cuda())
    ref = oracle_mods(cpu, softcap=30.0, slopes=sl, mask=mask)
    assert not ref[5, 3].any() and not ref[300].any()
    assert_attention_close(out, ref, what="all modifiers")
    assert not out[5, 3].any() and not out[300].any()
    assert pa.get_error(ws) == (0, 0)


def test_mask_shorter_than_a_sequence_is_reported():
    cpu = make([200, 40], [200, 1], 4, 2, 64, True, seed=44)
    mask = torch.zeros(cpu.num_q_tokens, 128)   # sequence 0 has 200 keys
    out, ws = run_mods(case_to(cpu, "cuda"), mask=mask.cuda())
    st, bits = pa.get_error(ws)
    assert bits & pa.DEVERR_HINT
    # keys past the mask row get no mask value: with a zero mask the output is plain attention
    assert_attention_close(out, oracle_varlen(cpu), what="short mask")


def test_zero_slopes_match_plain_attention():
    cpu = make(LENS, QLENS, 8, 2, 128, True, seed=45)
    dev = case_to(cpu, "cuda")
    plain, _, _, _ = run_varlen(dev)
    zero_slopes, _ = run_mods(dev, alibi_slopes=torch.zeros(8, device="cuda"))
    # the modifier path rounds scale * s before the log2 scaling, so compare to the tolerance
    assert_attention_close(zero_slopes, oracle_varlen(cpu), what="zero slopes")
    assert_attention_close(plain, oracle_varlen(cpu), what="plain")


# ---------------------------------------------------------------------------
# layouts
# ---------------------------------------------------------------------------

def hnd_cache(c):
    """The same cache contents stored head-major [NB, Hkv, BS, D], as an
    [NB, BS, Hkv, D]-indexed view."""
    return c.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)


def hnd_rows(x):
    """[T, H, D] stored head-major [H, T, D], as a [T, H, D]-indexed view."""
    return x.transpose(0, 1).contiguous().transpose(0, 1)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("d,hq,hkv", [(128, 8, 2), (64, 16, 16)])
def test_hnd_layouts_bit_identical(d, hq, hkv, dtype):
    cpu = make(LENS, QLENS, hq, hkv, d, True, seed=46 + d, dtype=dtype)
    dev = case_to(cpu, "cuda")
    ref_out, ref_kc, ref_vc, _ = run_varlen(dev)
    # the scatter into head-major caches, then attention reading them and
    # head-major q / out
    kc, vc = hnd_cache(dev.k_cache), hnd_cache(dev.v_cache)
    ws = pa.varlen_workspace(dev.num_seqs, dev.num_q_tokens, hq, hkv, d)
    pa.write_kv(dev.k_new, dev.v_new, dev.slot_mapping, kc, vc, workspace=ws)
    assert torch.equal(kc, ref_kc) and torch.equal(vc, ref_vc)
    assert kc.stride(1) == d and kc.stride(2) == kc.shape[1] * d     # really head-major
    q = hnd_rows(dev.q)
    out = hnd_rows(torch.full_like(dev.q, float("nan")))
    pa.attention_varlen(q, kc, vc, dev.block_tables, dev.seq_lens, dev.query_start_loc, hkv,
                        dev.scale, True, out, max_query_len=dev.max_query_len,
                        max_seq_len=dev.max_seq_len, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out)
    assert pa.get_error(ws) == (0, 0)
    # mixed: token-major q / out over a head-major cache
    out2 = torch.full_like(dev.q, float("nan"))
    pa.attention_varlen(dev.q, kc, vc, dev.block_tables, dev.seq_lens, dev.query_start_loc, hkv,
                        dev.scale, True, out2, max_query_len=dev.max_query_len,
                        max_seq_len=dev.max_seq_len, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(out2, ref_out)


def test_hnd_with_modifiers_and_padded_rows():
    cpu = make(LENS, QLENS, 8, 2, 128, True, seed=48)
    dev = case_to(cpu, "cuda")
    # head-major cache with 8 elements of padding after every head row block
    nb, bs, hkv, d = dev.k_cache.shape
    big_k = torch.zeros(nb, hkv, bs * d + 64, dtype=dev.k_cache.dtype, device="cuda")
    big_v = torch.zeros_like(big_k)
    kc = big_k[:, :, :bs * d].view(nb, hkv, bs, d).permute(0, 2, 1, 3)
    vc = big_v[:, :, :bs * d].view(nb, hkv, bs, d).permute(0, 2, 1, 3)
    kc.copy_(dev.k_cache)
    vc.copy_(dev.v_cache)
    ws = pa.varlen_workspace(dev.num_seqs, dev.num_q_tokens, 8, hkv, d)
    pa.write_kv(dev.k_new, dev.v_new, dev.slot_mapping, kc, vc, workspace=ws)
    sl = slopes_for(8)
    out = torch.full_like(dev.q, float("nan"))
    pa.attention_varlen(dev.q, kc, vc, dev.block_tables, dev.seq_lens, dev.query_start_loc, hkv,
                        dev.scale, True, out, max_query_len=dev.max_query_len,
                        max_seq_len=dev.max_seq_len, workspace=ws, softcap=20.0,
                        alibi_slopes=sl.cuda())
    torch.cuda.synchronize()
    assert_attention_close(out, oracle_mods(cpu, softcap=20.0, slopes=sl), what="hnd + mods")
    assert pa.get_error(ws) == (0, 0)


def test_layout_rejections():
    cpu = make([64], [64], 4, 2, 64, True, seed=49)
    dev = case_to(cpu, "cuda")
    out = torch.zeros_like(dev.q)
    ws = pa.varlen_workspace(1, 64, 4, 2, 64)
    # overlapping head rows (head stride 32 < D 64, slot stride 96): unsupported
    bad = torch.zeros(dev.k_cache.shape[0], 16, 96, dtype=torch.bfloat16, device="cuda")
    kc = bad.as_strided(dev.k_cache.shape, (16 * 96, 96, 32, 1))
    with pytest.raises(pa.PaError):
        pa.attention_varlen(dev.q, kc, kc, dev.block_tables, dev.seq_lens, dev.query_start_loc,
                            2, dev.scale, True, out, workspace=ws)
    # a mask row stride that is not a multiple of 4 floats
    mask = torch.zeros(64, 66, device="cuda")[:, :65]
    with pytest.raises(pa.PaError):
        pa.attention_varlen(dev.q, dev.k_cache, dev.v_cache, dev.block_tables, dev.seq_lens,
                            dev.query_start_loc, 2, dev.scale, True, out, workspace=ws,
                            mask=mask)
    assert torch.count_nonzero(out) == 0


def test_spans_with_modifiers():
    # full-attention spans (visibility) with ALiBi and a per-head additive mask (scores)
    lens, qlens = [600, 300], [600, 200]
    cpu = make(lens, qlens, 8, 2, 128, True, seed=50)
    so = torch.tensor([0, 2, 3], dtype=torch.int32)
    sp = torch.tensor([[40, 170], [300, 420], [150, 260]], dtype=torch.int32)
    t, ld = cpu.num_q_tokens, 608
    mask = torch.randn(8, t, ld, generator=torch.Generator().manual_seed(10))
    sl = slopes_for(8)
    dev = case_to(cpu, "cuda")
    kc, vc = dev.k_cache.clone(), dev.v_cache.clone()
    ws = pa.varlen_workspace(dev.num_seqs, dev.num_q_tokens, 8, 2, 128)
    pa.write_kv(dev.k_new, dev.v_new, dev.slot_mapping, kc, vc, workspace=ws)
    out = torch.full_like(dev.q, float("nan"))
    pa.attention_varlen_spans(dev.q, kc, vc, dev.block_tables, dev.seq_lens, dev.query_start_loc,
                              2, dev.scale, so.cuda(), sp.cuda(), out,
                              max_query_len=dev.max_query_len, max_seq_len=dev.max_seq_len,
                              workspace=ws, alibi_slopes=sl.cuda(), mask=mask.cuda())
    torch.cuda.synchronize()
    ref = oracle.attention_varlen_mods(
        workloads.bf16_bits(cpu.q), workloads.bf16_bits(cpu.k_logical),
        workloads.bf16_bits(cpu.v_logical), cpu.kv_offsets.numpy(), cpu.seq_lens.numpy(),
        cpu.query_start_loc.numpy(), 2, cpu.scale, True, alibi_slopes=sl.numpy(),
        mask=mask.numpy().reshape(-1), mask_head_stride=t * ld, mask_token_stride=ld,
        span_offsets=so.numpy(), spans=sp.numpy())
    assert_attention_close(out, ref, what="spans + modifiers")
    assert pa.get_error(ws) == (0, 0)


# ---------------------------------------------------------------------------
# the modifier workloads the benchmark times, at full size, on sampled rows
# ---------------------------------------------------------------------------

def sampled_rows(case):
    """Tile edges, the middle and the last two rows of every sequence."""
    qsl = case.query_start_loc.tolist()
    rows = set()
    for s in range(case.num_seqs):
        for i in (0, 1, 127, 128, 129, 1000, 2047):
            if qsl[s] + i < qsl[s + 1]:
                rows.add(qsl[s] + i)
        rows.update((qsl[s + 1] - 1, qsl[s + 1] - 2))
    return np.array(sorted(rows), dtype=np.int64)


def test_alibi_softcap_prefill_config_full_size_sampled_rows():
    # varlen_prefill (4 causal sequences up to 8192 tokens, Hq 32 / Hkv 8,
    # D 128) with the geometric slopes and the TANH30 soft-cap
    cpu = workloads.varlen_prefill()
    sl = slopes_for(cpu.num_q_heads)
    out, ws = run_mods(case_to(cpu, "cuda"), softcap=30.0, alibi_slopes=sl.cuda())
    assert pa.get_error(ws) == (0, 0)
    rows = sampled_rows(cpu)
    ref = oracle.attention_varlen_mods(
        workloads.bf16_bits(cpu.q), workloads.bf16_bits(cpu.k_logical),
        workloads.bf16_bits(cpu.v_logical), cpu.kv_offsets.numpy(), cpu.seq_lens.numpy(),
        cpu.query_start_loc.numpy(), cpu.num_kv_heads, cpu.scale, cpu.causal, 0,
        softcap=30.0, alibi_slopes=sl.numpy(), rows=rows)
    assert_attention_close(out, ref, rows=rows, what="prefill + ALiBi + TANH30 full (sampled)")


def test_hnd_mask_decode_config_full_size():
    # decode_batch (64 sequences, context 256-4096) over head-major caches
    # with one additive mask shared by all heads, every row checked
    cpu = workloads.decode_batch()
    dev = case_to(cpu, "cuda")
    import dataclasses
    hnd = dataclasses.replace(dev, k_cache=hnd_cache(dev.k_cache), v_cache=hnd_cache(dev.v_cache))
    mlen = (cpu.max_seq_len + 3) // 4 * 4
    mask = torch.randn(cpu.num_q_tokens, mlen, generator=workloads._gen(1008, "cpu"))
    out, ws = run_mods(hnd, mask=mask.cuda())
    assert pa.get_error(ws) == (0, 0)
    assert_attention_close(out, oracle_mods(cpu, mask=mask), what="decode HND + mask full")
