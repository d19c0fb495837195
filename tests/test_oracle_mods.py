"""Pins for the oracle's score modifiers (auto_round_kernel PR "Migrate CPU
SDPA backend", description: additive masks in the public sdpa(), ALiBi slopes
and the TANH30 soft-cap among the library's extensions).

Each is checked against an independent evaluation in float64 with torch:

* ALiBi and additive masks against torch.nn.functional.scaled_dot_product_attention
  given the bias as its float attn_mask (what SDPA itself defines: softmax of
  scale * Q K^T + attn_mask);
* the soft-cap against an explicit torch evaluation, softmax of
  c * tanh(scale * Q K^T / c) + bias;
* special cases that reduce to plain attention (cap -> infinity, zero slopes,
  a row-constant mask), and a fully masked row giving zeros.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads


def make(lens, qlens, hq, hkv, d, causal, seed):
    return workloads.build_varlen_case("mods", lens, qlens, hq, hkv, d, causal, seed)


def run(case, **kw):
    return oracle.attention_varlen_mods(
        workloads.bf16_bits(case.q), workloads.bf16_bits(case.k_logical),
        workloads.bf16_bits(case.v_logical), case.kv_offsets.numpy(), case.seq_lens.numpy(),
        case.query_start_loc.numpy(), case.num_kv_heads, case.scale, case.causal, **kw)


def plain(case):
    return oracle.attention_varlen(
        workloads.bf16_bits(case.q), workloads.bf16_bits(case.k_logical),
        workloads.bf16_bits(case.v_logical), case.kv_offsets.numpy(), case.seq_lens.numpy(),
        case.query_start_loc.numpy(), case.num_kv_heads, case.scale, case.causal)


def seq_parts(case, s):
    """q [Hq, Lq, D], k, v [Hq, Lkv, D] (KV heads expanded), float64."""
    g = case.num_q_heads // case.num_kv_heads
    qsl = case.query_start_loc.tolist()
    lkv, o0 = int(case.seq_lens[s]), int(case.kv_offsets[s])
    q = case.q[qsl[s]:qsl[s + 1]].double().transpose(0, 1)
    k = case.k_logical[o0:o0 + lkv].double().repeat_interleave(g, dim=1).transpose(0, 1)
    v = case.v_logical[o0:o0 + lkv].double().repeat_interleave(g, dim=1).transpose(0, 1)
    return q, k, v


def visible(case, s):
    """[Lq, Lkv] bool: causal (bottom-right) or all."""
    qsl = case.query_start_loc.tolist()
    lq, lkv = qsl[s + 1] - qsl[s], int(case.seq_lens[s])
    i = torch.arange(lq)[:, None]
    j = torch.arange(lkv)[None, :]
    return (j <= (lkv - lq) + i) if case.causal else torch.ones(lq, lkv, dtype=torch.bool)


def alibi_bias(case, s, slopes):
    qsl = case.query_start_loc.tolist()
    lq, lkv = qsl[s + 1] - qsl[s], int(case.seq_lens[s])
    pos = (lkv - lq) + torch.arange(lq, dtype=torch.float64)[:, None]
    j = torch.arange(lkv, dtype=torch.float64)[None, :]
    return torch.from_numpy(slopes.astype(np.float64))[:, None, None] * (j - pos)[None]


def mask_block(mask, case, s, head_stride, token_stride):
    """The [Hq, Lq, Lkv] float64 block of a flat mask for sequence s."""
    qsl = case.query_start_loc.tolist()
    lkv = int(case.seq_lens[s])
    out = np.zeros((case.num_q_heads, qsl[s + 1] - qsl[s], lkv))
    for h in range(case.num_q_heads):
        for i, t in enumerate(range(qsl[s], qsl[s + 1])):
            a = h * head_stride + t * token_stride
            out[h, i] = mask[a:a + lkv]
    return torch.from_numpy(out)


def check_seq(got, case, s, bias, softcap=0.0):
    q, k, v = seq_parts(case, s)
    vis = visible(case, s)
    if softcap == 0.0:
        b = bias.masked_fill(~vis, float("-inf"))
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=b,
                                                               scale=case.scale)
    else:
        sc = case.scale * q @ k.transpose(1, 2)
        sc = softcap * torch.tanh(sc / softcap) + bias
        sc = sc.masked_fill(~vis, float("-inf"))
        ref = torch.softmax(sc, dim=-1) @ v
    qsl = case.query_start_loc.tolist()
    err = np.max(np.abs(got[qsl[s]:qsl[s + 1]] - ref.transpose(0, 1).numpy()))
    assert err < 1e-10, (s, err)


def slopes_for(hq):
    # the geometric ALiBi slopes 2^(-8 h / H), h = 1..H
    return np.array([2.0 ** (-8.0 * (h + 1) / hq) for h in range(hq)], np.float32)


@pytest.mark.parametrize("causal", [True, False])
def test_alibi_matches_sdpa_with_bias(causal):
    lens, qlens = [200, 37, 129], [60, 1, 129]
    case = make(lens, qlens, 8, 2, 64, causal, seed=11)
    sl = slopes_for(8)
    got = run(case, alibi_slopes=sl)
    for s in range(len(lens)):
        check_seq(got, case, s, alibi_bias(case, s, sl))


@pytest.mark.parametrize("head_stride_mode", ["per_head", "shared"])
def test_additive_mask_matches_sdpa(head_stride_mode):
    lens, qlens = [150, 64, 9], [150, 20, 1]
    case = make(lens, qlens, 4, 4, 64, True, seed=12)
    t, hq, ld = case.num_q_tokens, case.num_q_heads, 160
    rng = np.random.default_rng(3)
    nh = hq if head_stride_mode == "per_head" else 1
    mask = rng.standard_normal(nh * t * ld).astype(np.float32) * 2
    mask[rng.random(mask.size) < 0.05] = -np.inf                # some keys masked out
    hs = t * ld if nh > 1 else 0
    got = run(case, mask=mask, mask_head_stride=hs, mask_token_stride=ld)
    for s in range(len(lens)):
        check_seq(got, case, s, mask_block(mask, case, s, hs, ld))


@pytest.mark.parametrize("cap", [30.0, 2.0])
def test_softcap_with_alibi_and_mask_matches_explicit_torch(cap):
    lens, qlens = [100, 33], [100, 5]
    case = make(lens, qlens, 8, 4, 128, True, seed=13)
    t, ld = case.num_q_tokens, 104
    rng = np.random.default_rng(4)
    mask = (rng.standard_normal(t * ld) * 0.5).astype(np.float32)
    sl = slopes_for(8)
    got = run(case, softcap=cap, alibi_slopes=sl, mask=mask, mask_head_stride=0,
              mask_token_stride=ld)
    for s in range(len(lens)):
        bias = alibi_bias(case, s, sl) + mask_block(mask, case, s, 0, ld)
        check_seq(got, case, s, bias, softcap=cap)


def test_special_cases_reduce_to_plain_attention():
    case = make([300, 17], [300, 1], 8, 2, 64, True, seed=14)
    ref = plain(case)
    # a cap far above every score: tanh(x / c) * c = x to well below 1e-10
    assert np.max(np.abs(run(case, softcap=1e7) - ref)) < 1e-10
    # zero slopes
    assert np.max(np.abs(run(case, alibi_slopes=np.zeros(8, np.float32)) - ref)) < 1e-12
    # a mask constant along each row shifts every score of the row equally
    t, ld = case.num_q_tokens, 300
    row_const = np.repeat(np.random.default_rng(5).standard_normal(t).astype(np.float32), ld)
    got = run(case, mask=row_const, mask_head_stride=0, mask_token_stride=ld)
    assert np.max(np.abs(got - ref)) < 1e-10


def test_fully_masked_row_is_zero_and_partial_mask_drops_keys():
    case = make([64], [64], 2, 1, 64, False, seed=15)
    ld = 64
    mask = np.zeros(64 * ld, np.float32)
    mask[5 * ld:6 * ld] = -np.inf          # row 5: every key masked out
    mask[9 * ld + 40:10 * ld] = -np.inf    # row 9: keys 40.. masked out
    got = run(case, mask=mask, mask_head_stride=0, mask_token_stride=ld)
    assert not got[5].any()
    q, k, v = seq_parts(case, 0)
    ref9 = torch.nn.functional.scaled_dot_product_attention(
        q[:, 9:10], k[:, :40], v[:, :40], scale=case.scale)
    assert np.max(np.abs(got[9] - ref9[:, 0].numpy())) < 1e-10


def test_modifiers_with_spans_match_sdpa():
    # full-attention spans decide visibility; ALiBi and the mask add to the scores
    lens = [200]
    case = make(lens, lens, 4, 2, 64, True, seed=16)
    spans = [(20, 60), (100, 180)]
    sl = slopes_for(4)
    ld = 200
    mask = (np.random.default_rng(9).standard_normal(200 * ld) * 0.5).astype(np.float32)
    got = run(case, alibi_slopes=sl, mask=mask, mask_head_stride=0, mask_token_stride=ld,
              span_offsets=np.array([0, 2], np.int32), spans=np.array(spans, np.int32))
    q, k, v = seq_parts(case, 0)
    block = np.full(200, -1)
    for b, (a, e) in enumerate(spans):
        block[a:e] = b
    i = np.arange(200)[:, None]
    j = np.arange(200)[None, :]
    vis = torch.from_numpy((j <= i) | ((block[:, None] == block[None, :]) & (block[:, None] >= 0)))
    bias = alibi_bias(case, 0, sl) + mask_block(mask, case, 0, 0, ld)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, k, v, attn_mask=bias.masked_fill(~vis, float("-inf")), scale=case.scale)
    assert np.max(np.abs(got - ref.transpose(0, 1).numpy())) < 1e-10


def test_golden_softcap_saturation():
    """Hand-derived worked example (tests/golden/softcap_saturation.json): scores
    of +-1000 under a cap of 2 saturate to exactly +-2, so the output is the
    closed form (1/(1+e^-4), e^-4/(1+e^-4), 0, 0); without the cap, or with the
    cap placed after the softmax, the second weight would be 0."""
    from tests.conftest import load_golden
    g = load_golden("softcap_saturation")

    def bits(x):
        t = torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
        assert torch.equal(t.float(), torch.tensor(np.asarray(x, dtype=np.float32)))
        return t.view(torch.int16).numpy().view(np.uint16)
    out = oracle.attention_varlen_mods(
        bits(g["q"]), bits(g["k"]), bits(g["v"]), np.array([0], np.int64),
        np.array([2], np.int32), np.array([0, 1], np.int32), 1, g["scale"], g["causal"],
        softcap=g["softcap"])
    assert np.allclose(out, np.array(g["expected"]), rtol=0, atol=1e-15)
    uncapped = oracle.attention_varlen_mods(
        bits(g["q"]), bits(g["k"]), bits(g["v"]), np.array([0], np.int64),
        np.array([2], np.int32), np.array([0, 1], np.int32), 1, g["scale"], g["causal"])
    assert np.array_equal(uncapped[0, 0], np.array([1.0, 0.0, 0.0, 0.0]))
