"""A seeded randomized sweep over the feature combinations of paged varlen
attention, each case against the fp64 oracle.

The other GPU tests each vary one feature; here every case draws all of them
at once from a fixed seed: the batch mix (prefill, chunked prefill, decode,
empty and one-token sequences), GQA group (1 to 64), head dim (64, 128), cache
block size (16 to 128), element type (bf16, fp16), cache layout (token-major or
head-major), causality, the scale, and score modifiers (soft-cap, ALiBi).  The
cache write is checked bit for bit against the oracle's literal write; the
attention output within max |err| <= 2e-2 and mean |err| <= 2e-3."""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_gqa_reshape_b200 as pa
import workloads
from tests.gpu_helpers import assert_attention_close, case_to

pytestmark = pytest.mark.gpu

DTYPES = {torch.bfloat16: 0, torch.float16: 1}


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def draw(seed):
    rng = np.random.default_rng(seed)
    g = int(rng.choice([1, 2, 4, 8, 16, 32, 64]))
    hkv = int(rng.choice([1, 2, 4])) if g <= 16 else int(rng.choice([1, 2]))
    d = int(rng.choice([64, 128]))
    bs = int(rng.choice([16, 32, 64, 128]))
    dtype = torch.float16 if rng.random() < 0.3 else torch.bfloat16
    causal = bool(rng.random() < 0.8)
    n = int(rng.integers(1, 9))
    lens, qlens = [], []
    for _ in range(n):
        kind = rng.choice(["prefill", "chunk", "decode", "empty", "one"])
        if kind == "prefill":
            L = int(rng.integers(2, 700))
            lens.append(L)
            qlens.append(L)
        elif kind == "chunk":
            L = int(rng.integers(2, 1500))
            lens.append(L)
            qlens.append(int(rng.integers(2, L + 1)))
        elif kind == "decode":
            lens.append(int(rng.integers(1, 3000)))
            qlens.append(1)
        elif kind == "empty":
            lens.append(0)
            qlens.append(0)
        else:
            lens.append(1)
            qlens.append(1)
    u = rng.random()
    scale = 1.0 / math.sqrt(d) if u < 0.7 else (0.5 / math.sqrt(d) if u < 0.85 else 0.0)
    mods = {}
    if scale > 0 and rng.random() < 0.4:
        if rng.random() < 0.5:
            mods["softcap"] = float(rng.choice([5.0, 30.0]))
        if rng.random() < 0.6:
            mods["alibi"] = True
    hnd = bool(rng.random() < 0.3)
    return dict(g=g, hkv=hkv, d=d, bs=bs, dtype=dtype, causal=causal, lens=lens, qlens=qlens,
                scale=scale, mods=mods, hnd=hnd)


def hnd_cache(c):
    """The same cache contents stored head-major [NB, Hkv, BS, D], as an
    [NB, BS, Hkv, D]-indexed view."""
    return c.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)


@pytest.mark.parametrize("seed", range(32))
def test_random_feature_combinations(seed):
    c = draw(7000 + seed)
    hq = c["g"] * c["hkv"]
    cpu = workloads.build_varlen_case("fuzz", c["lens"], c["qlens"], hq, c["hkv"], c["d"],
                                      c["causal"], 7000 + seed, block_size=c["bs"],
                                      scale=c["scale"], dtype=c["dtype"])
    if cpu.num_q_tokens == 0:
        pytest.skip("no query tokens drawn")
    dev = case_to(cpu, "cuda")
    kc, vc = dev.k_cache.clone(), dev.v_cache.clone()
    if c["hnd"]:
        kc, vc = hnd_cache(kc), hnd_cache(vc)
    ws = pa.varlen_workspace(dev.num_seqs, dev.num_q_tokens, hq, c["hkv"], c["d"])
    pa.write_kv(dev.k_new, dev.v_new, dev.slot_mapping, kc, vc, workspace=ws)
    slopes = None
    if c["mods"].get("alibi"):
        slopes = torch.tensor([2.0 ** (-8.0 * (h + 1) / hq) for h in range(hq)],
                              dtype=torch.float32)
    out = torch.full_like(dev.q, float("nan"))
    pa.attention_varlen(dev.q, kc, vc, dev.block_tables, dev.seq_lens, dev.query_start_loc,
                        c["hkv"], c["scale"], c["causal"], out, max_query_len=dev.max_query_len,
                        max_seq_len=dev.max_seq_len, workspace=ws,
                        softcap=c["mods"].get("softcap", 0.0),
                        alibi_slopes=None if slopes is None else slopes.cuda())
    torch.cuda.synchronize()
    # the cache write, bit for bit
    ek = workloads.bf16_bits(cpu.k_cache).copy()
    ev = workloads.bf16_bits(cpu.v_cache).copy()
    oracle.write_kv(workloads.bf16_bits(cpu.k_new), workloads.bf16_bits(cpu.v_new),
                    cpu.slot_mapping.numpy(), ek, ev, cpu.block_size)
    assert np.array_equal(workloads.bf16_bits(kc.contiguous()), ek)
    assert np.array_equal(workloads.bf16_bits(vc.contiguous()), ev)
    # the attention output
    ref = oracle.attention_varlen_mods(
        workloads.bf16_bits(cpu.q), workloads.bf16_bits(cpu.k_logical),
        workloads.bf16_bits(cpu.v_logical), cpu.kv_offsets.numpy(), cpu.seq_lens.numpy(),
        cpu.query_start_loc.numpy(), c["hkv"], c["scale"], c["causal"], DTYPES[c["dtype"]],
        softcap=c["mods"].get("softcap", 0.0),
        alibi_slopes=None if slopes is None else slopes.numpy())
    assert_attention_close(out, ref, what=f"seed {seed}: {c}")
    assert pa.get_error(ws) == (0, 0)
