"""Seeded synthetic inputs for paged KV attention, shared by tests and bench.

This module draws inputs and lays them out; it holds none of the attention
arithmetic (no scores, softmax, masking or output).  Both the CUDA path and
the oracle consume exactly the bfloat16 bits drawn here.

Recipe (every draw from a ``torch.Generator`` seeded per case):

* Q, K, V ~ N(0, 1) in fp32, rounded to bf16.
* Lengths are uniform integers over the stated inclusive ranges.
* Physical blocks are a random permutation of the pool, handed to the
  sequences in order; block-table entries past a sequence's last block hold
  an id outside the pool, so any read of them is an error.
* Each sequence's keys/values are drawn as one logical array
  ``[seq_len, Hkv, D]``.  The last ``query_len`` rows are this step's new
  tokens (``k_new``/``v_new``, written by the scatter under test through
  ``slot_mapping``); the rows before them are prior context and are placed
  into the cache here.  Slot of position p of sequence s:
  ``block_tables[s, p // BS] * BS + p % BS`` — the vLLM v1 slot_mapping
  convention of vllm-spyre PR #853 "Pytorch Native Attention on Spyre".
* Every cache slot holding no prior-context row (unused tail slots, slots of
  this step's new tokens, spare blocks) holds a large finite sentinel
  (K = +64, V = +1024) so that reading a slot that should be masked, or one
  the scatter failed to write, shows up as an O(1) error.

The five named configurations are the workload table of the paged attention
hot path: a tiny paged prefill, a decode batch, a varlen causal prefill, a
small-seq cross-attention batch and a mixed chunked-prefill + decode step.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

K_SENTINEL = 64.0
V_SENTINEL = 1024.0
BLOCK_SIZE = 16


@dataclass
class VarlenCase:
    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    scale: float
    causal: bool
    seq_lens: torch.Tensor          # int32 [S]  keys per sequence (prior + new)
    query_lens: torch.Tensor        # int32 [S]  new/query tokens per sequence
    query_start_loc: torch.Tensor   # int32 [S+1]
    block_tables: torch.Tensor      # int32 [S, max_blocks]
    num_blocks: int
    q: torch.Tensor                 # bf16 [T, Hq, D]
    k_new: torch.Tensor             # bf16 [T, Hkv, D]
    v_new: torch.Tensor             # bf16 [T, Hkv, D]
    slot_mapping: torch.Tensor      # int64 [T]
    k_cache: torch.Tensor           # bf16 [NB, BS, Hkv, D]
    v_cache: torch.Tensor           # bf16 [NB, BS, Hkv, D]
    kv_offsets: torch.Tensor        # int64 [S]  first logical row of each sequence
    k_logical: Optional[torch.Tensor] = None   # bf16 [sum(seq_lens), Hkv, D]
    v_logical: Optional[torch.Tensor] = None
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.seq_lens.numel())

    @property
    def num_q_tokens(self) -> int:
        return int(self.q.shape[0])

    @property
    def max_query_len(self) -> int:
        return int(self.query_lens.max().item()) if self.num_seqs else 0

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max().item()) if self.num_seqs else 0


@dataclass
class SmallSeqCase:
    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    scale: float
    cu_seqlens_kv: torch.Tensor     # int32 [B+1]
    q: torch.Tensor                 # bf16 [B, Hq, D]
    k: torch.Tensor                 # bf16 [sum, Hkv, D]
    v: torch.Tensor                 # bf16 [sum, Hkv, D]
    max_seqlen_kv: int
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return int(self.q.shape[0])


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn_bf16(shape, gen, device, chunk_rows: int = 1 << 20,
                dtype=torch.bfloat16) -> torch.Tensor:
    """N(0,1) fp32 rounded to `dtype` (bf16 or fp16), drawn in row chunks to
    bound fp32 temporaries."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(shape[0], -1) if len(shape) > 1 else out.view(-1, 1)
    for r0 in range(0, flat.shape[0], chunk_rows):
        r1 = min(flat.shape[0], r0 + chunk_rows)
        flat[r0:r1] = torch.randn((r1 - r0, flat.shape[1]), generator=gen,
                                  device=device, dtype=torch.float32).to(dtype)
    return out


def build_varlen_case(name: str, seq_lens, query_lens, num_q_heads: int, num_kv_heads: int,
                      head_dim: int, causal: bool, seed: int, device="cpu",
                      block_size: int = BLOCK_SIZE, pool_blocks: Optional[int] = None,
                      scale: Optional[float] = None, keep_logical: bool = True,
                      spare_table_cols: int = 1, dtype=torch.bfloat16) -> VarlenCase:
    """Lay out one paged varlen batch.

    seq_lens[s] keys per sequence, of which the last query_lens[s] are this
    step's tokens.  pool_blocks defaults to exactly the blocks needed.
    """
    device = torch.device(device)
    seq_lens = [int(x) for x in seq_lens]
    query_lens = [int(x) for x in query_lens]
    assert len(seq_lens) == len(query_lens)
    S = len(seq_lens)
    nblk = [math.ceil(L / block_size) for L in seq_lens]
    need = sum(nblk)
    pool = need if pool_blocks is None else int(pool_blocks)
    assert pool >= need, "pool too small"
    max_blocks = max([1] + nblk) + spare_table_cols
    g_cpu = _gen(seed, "cpu")
    perm = torch.randperm(pool, generator=g_cpu).to(torch.int32)
    table = torch.full((S, max_blocks), pool + 7, dtype=torch.int32)  # outside the pool
    cur = 0
    for s in range(S):
        table[s, : nblk[s]] = perm[cur: cur + nblk[s]]
        cur += nblk[s]

    qsl = [0]
    for ql in query_lens:
        qsl.append(qsl[-1] + ql)
    T = qsl[-1]
    kv_offsets = [0]
    for L in seq_lens:
        kv_offsets.append(kv_offsets[-1] + L)
    total_kv = kv_offsets[-1]

    gen = _gen(seed + 7919, device)
    k_log = _randn_bf16((max(total_kv, 1), num_kv_heads, head_dim), gen, device,
                        dtype=dtype)[:total_kv]
    v_log = _randn_bf16((max(total_kv, 1), num_kv_heads, head_dim), gen, device,
                        dtype=dtype)[:total_kv]
    q = _randn_bf16((max(T, 1), num_q_heads, head_dim), gen, device, dtype=dtype)[:T]

    # logical row of every key, its slot, and whether it is this step's token
    table_dev = table.to(device)
    seq_of_row = torch.repeat_interleave(torch.arange(S, device=device),
                                         torch.tensor(seq_lens, device=device))
    pos_of_row = (torch.arange(total_kv, device=device)
                  - torch.tensor(kv_offsets[:-1], device=device, dtype=torch.int64)[seq_of_row])
    slot_of_row = (table_dev[seq_of_row, pos_of_row // block_size].to(torch.int64) * block_size
                   + pos_of_row % block_size)
    new_from = (torch.tensor(seq_lens, device=device) - torch.tensor(query_lens, device=device))
    is_new = pos_of_row >= new_from[seq_of_row]

    k_cache = torch.full((pool, block_size, num_kv_heads, head_dim), K_SENTINEL,
                         dtype=dtype, device=device)
    v_cache = torch.full((pool, block_size, num_kv_heads, head_dim), V_SENTINEL,
                         dtype=dtype, device=device)
    prior = ~is_new
    k_cache.view(-1, num_kv_heads, head_dim)[slot_of_row[prior]] = k_log[prior]
    v_cache.view(-1, num_kv_heads, head_dim)[slot_of_row[prior]] = v_log[prior]

    k_new = k_log[is_new].contiguous()
    v_new = v_log[is_new].contiguous()
    slot_mapping = slot_of_row[is_new].contiguous()
    # one new K/V row per query token, except in the degenerate (invalid)
    # case query_len > seq_len, where only seq_len rows exist
    assert k_new.shape[0] == sum(min(a, b) for a, b in zip(query_lens, seq_lens))

    case = VarlenCase(
        name=name, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
        block_size=block_size,
        scale=float(scale if scale is not None else 1.0 / math.sqrt(head_dim)),
        causal=bool(causal),
        seq_lens=torch.tensor(seq_lens, dtype=torch.int32, device=device),
        query_lens=torch.tensor(query_lens, dtype=torch.int32, device=device),
        query_start_loc=torch.tensor(qsl, dtype=torch.int32, device=device),
        block_tables=table_dev, num_blocks=pool,
        q=q.contiguous(), k_new=k_new, v_new=v_new, slot_mapping=slot_mapping,
        k_cache=k_cache, v_cache=v_cache,
        kv_offsets=torch.tensor(kv_offsets[:-1], dtype=torch.int64, device=device),
        k_logical=k_log if keep_logical else None,
        v_logical=v_log if keep_logical else None,
        meta={"seed": seed},
    )
    if not keep_logical:
        del k_log, v_log
    return case


def build_smallseq_case(name: str, kv_lens, num_q_heads: int, num_kv_heads: int,
                        head_dim: int, seed: int, device="cpu",
                        scale: Optional[float] = None, dtype=torch.bfloat16) -> SmallSeqCase:
    device = torch.device(device)
    kv_lens = [int(x) for x in kv_lens]
    cu = [0]
    for L in kv_lens:
        cu.append(cu[-1] + L)
    B = len(kv_lens)
    gen = _gen(seed + 7919, device)
    q = _randn_bf16((max(B, 1), num_q_heads, head_dim), gen, device, dtype=dtype)[:B]
    k = _randn_bf16((max(cu[-1], 1), num_kv_heads, head_dim), gen, device, dtype=dtype)[: cu[-1]]
    v = _randn_bf16((max(cu[-1], 1), num_kv_heads, head_dim), gen, device, dtype=dtype)[: cu[-1]]
    return SmallSeqCase(
        name=name, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
        scale=float(scale if scale is not None else 1.0 / math.sqrt(head_dim)),
        cu_seqlens_kv=torch.tensor(cu, dtype=torch.int32, device=device),
        q=q.contiguous(), k=k.contiguous(), v=v.contiguous(),
        max_seqlen_kv=max(kv_lens) if kv_lens else 0, meta={"seed": seed})


# ---------------------------------------------------------------------------
# The named workloads
# ---------------------------------------------------------------------------

def _uniform_ints(lo: int, hi: int, n: int, seed: int):
    g = _gen(seed, "cpu")
    return torch.randint(lo, hi + 1, (n,), generator=g).tolist()


def tiny_prefill(device="cpu", seed=1001) -> VarlenCase:
    """2 sequences (7 and 13 tokens), causal prefill, Hq 4 / Hkv 2, D 64,
    block 16, randomly permuted table over an 8-block pool, scale 1/8; every
    token is new and goes through the scatter first."""
    return build_varlen_case("tiny_prefill", [7, 13], [7, 13], 4, 2, 64, True, seed,
                             device=device, pool_blocks=8, scale=1.0 / 8.0)


def decode_batch(device="cpu", seed=1002, num_seqs=64, lo=256, hi=4096,
                 num_q_heads=32, num_kv_heads=8, head_dim=128, keep_logical=True,
                 dtype=torch.bfloat16) -> VarlenCase:
    """64 sequences with one query each, context uniform in [256, 4096],
    Hq 32 / Hkv 8, D 128; the new token is scattered before attention."""
    lens = _uniform_ints(lo, hi, num_seqs, seed)
    return build_varlen_case("decode_batch", lens, [1] * num_seqs, num_q_heads, num_kv_heads,
                             head_dim, True, seed, device=device, keep_logical=keep_logical,
                             dtype=dtype)


def varlen_prefill(device="cpu", seed=1003, lens=(2048, 3000, 4096, 8192),
                   num_q_heads=32, num_kv_heads=8, head_dim=128, causal=True,
                   keep_logical=True, dtype=torch.bfloat16) -> VarlenCase:
    """4 packed sequences of 2048, 3000, 4096 and 8192 tokens, causal,
    Hq 32 / Hkv 8, D 128, shuffled table."""
    return build_varlen_case("varlen_prefill", list(lens), list(lens), num_q_heads,
                             num_kv_heads, head_dim, causal, seed, device=device,
                             keep_logical=keep_logical, dtype=dtype)


def spans_prefill(device="cpu", seed=1006, num_seqs=4, text=512, cond=1536, target=2048,
                  num_q_heads=32, num_kv_heads=8, head_dim=128, keep_logical=True):
    """Piecewise block-causal prefill: each sequence is a causal text run
    followed by two image blocks with full attention (condition, target),
    4 x (512 + 1536 + 2048) = 16 384 tokens, Hq 32 / Hkv 8, D 128.
    Returns (case, span_offsets int32 [S+1], spans int32 [2S, 2])."""
    n = text + cond + target
    case = build_varlen_case("spans_prefill", [n] * num_seqs, [n] * num_seqs, num_q_heads,
                             num_kv_heads, head_dim, True, seed, device=device,
                             keep_logical=keep_logical)
    spans = []
    for _ in range(num_seqs):
        spans += [(text, text + cond), (text + cond, n)]
    span_offsets = torch.arange(0, 2 * num_seqs + 1, 2, dtype=torch.int32, device=device)
    return case, span_offsets, torch.tensor(spans, dtype=torch.int32, device=device)


def spans_visible_pairs(seq_lens, query_lens, span_offsets, spans) -> int:
    """Visible (query, key) pairs under the span rule (per head)."""
    total = 0
    so = [int(x) for x in span_offsets]
    sp = [(int(a), int(b)) for a, b in spans]
    for s, (lkv, lq) in enumerate(zip(seq_lens, query_lens)):
        lkv, lq = int(lkv), int(lq)
        if lq <= 1:
            total += lkv * lq
            continue
        ends = {}
        prev = 0
        for a, b in sp[so[s]:so[s + 1]]:
            if 0 <= a < b <= lkv and a >= prev:
                for pos in range(a, b):
                    ends[pos] = b
            prev = b
        off = lkv - lq
        for i in range(lq):
            pos = off + i
            total += max(0, min(lkv, ends.get(pos, pos + 1)))
    return total


def smallseq_batch(device="cpu", seed=1004, batch=30720, heads=16, head_dim=128,
                   choices=(2, 4, 6, 8, 12, 16)) -> SmallSeqCase:
    """batch 30720, s_q = 1, s_kv uniform over {2,4,6,8,12,16}, 16 heads,
    D 128, contiguous THD keys with cu_seqlens_kv, no causal mask."""
    g = _gen(seed, "cpu")
    idx = torch.randint(0, len(choices), (batch,), generator=g).tolist()
    lens = [choices[i] for i in idx]
    return build_smallseq_case("smallseq_batch", lens, heads, heads, head_dim, seed,
                               device=device)


def mixed_step(device="cpu", seed=1005, num_chunks=8, chunk=512, prior_hi=16384,
               num_decodes=248, dec_lo=128, dec_hi=32768, num_q_heads=64, num_kv_heads=8,
               head_dim=128, keep_logical=True) -> VarlenCase:
    """8 prefill chunks of 512 query tokens with prior context uniform in
    [0, 16384] (causal within the chunk, full over the prior context), then
    248 decodes with context uniform in [128, 32768]; Hq 64 / Hkv 8, D 128;
    all new tokens scattered in the same step."""
    prior = _uniform_ints(0, prior_hi, num_chunks, seed)
    dec = _uniform_ints(dec_lo, dec_hi, num_decodes, seed + 1)
    seq_lens = [p + chunk for p in prior] + dec
    query_lens = [chunk] * num_chunks + [1] * num_decodes
    return build_varlen_case("mixed_step", seq_lens, query_lens, num_q_heads, num_kv_heads,
                             head_dim, True, seed, device=device, keep_logical=keep_logical)


NAMED = {
    "tiny_prefill": tiny_prefill,
    "decode_batch": decode_batch,
    "varlen_prefill": varlen_prefill,
    "smallseq_batch": smallseq_batch,
    "mixed_step": mixed_step,
}


def bf16_bits(t: torch.Tensor):
    """A 16-bit (bf16 or fp16) tensor's bit patterns as a host numpy uint16 array."""
    import numpy as np
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
