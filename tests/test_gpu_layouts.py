"""The combined (num_blocks, 2, block_size, Hkv, D) cache layout: the K and V
halves of one tensor, passed as strided views, give exactly the results of
separate caches (scatter bit for bit; attention bit for bit, same kernels)."""
import numpy as np
import pytest
import torch

import paged_kv_gqa_reshape_b200 as pa
import workloads
from tests.gpu_helpers import assert_attention_close, case_to, oracle_varlen, run_varlen

pytestmark = pytest.mark.gpu


def combined_from(case):
    """A [NB, 2, BS, Hkv, D] cache holding the case's K and V, plus its two views."""
    kv = torch.stack([case.k_cache, case.v_cache], dim=1).contiguous()
    return kv, kv[:, 0], kv[:, 1]


def attend(case, kc, vc, ws):
    out = torch.full_like(case.q, float("nan"))
    pa.attention_varlen(case.q, kc, vc, case.block_tables, case.seq_lens, case.query_start_loc,
                        case.num_kv_heads, case.scale, case.causal, out,
                        max_query_len=case.max_query_len, max_seq_len=case.max_seq_len,
                        workspace=ws)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("d,hq,hkv", [(128, 16, 4), (64, 8, 8)])
def test_combined_cache_scatter_and_attention(d, hq, hkv):
    lens = [700, 40, 300, 1, 2000, 17, 5, 129]
    qlens = [64, 1, 300, 1, 1, 17, 1, 100]
    cpu = workloads.build_varlen_case("layout", lens, qlens, hq, hkv, d, True, seed=21 + d)
    dev = case_to(cpu, "cuda")
    # separate caches: the reference run
    out_sep, kc_sep, vc_sep, _ = run_varlen(dev)
    # combined cache: scatter into the views, then attend through them
    kv, kview, vview = combined_from(dev)
    ws = pa.varlen_workspace(dev.num_seqs, dev.num_q_tokens, dev.num_q_heads, dev.num_kv_heads,
                             dev.head_dim)
    pa.write_kv(dev.k_new, dev.v_new, dev.slot_mapping, kview, vview, workspace=ws)
    assert torch.equal(kv[:, 0], kc_sep) and torch.equal(kv[:, 1], vc_sep)
    out_comb = attend(dev, kview, vview, ws)
    assert torch.equal(out_comb, out_sep)
    assert_attention_close(out_comb, oracle_varlen(cpu), what="combined layout")
    assert pa.get_error(ws) == (0, 0)


def test_cache_views_must_share_strides_and_rows():
    kv = torch.zeros(8, 2, 16, 2, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(2, 2, 64, dtype=torch.bfloat16, device="cuda")
    slots = torch.zeros(2, dtype=torch.int64, device="cuda")
    sep_v = torch.zeros(8, 16, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        pa.write_kv(k, k, slots, kv[:, 0], sep_v)            # strides differ
    with pytest.raises(ValueError):
        pa.write_kv(k, k, slots, kv[:, 0].transpose(1, 2), kv[:, 1].transpose(1, 2))  # rows not contiguous
