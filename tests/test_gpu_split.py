"""The plan kernel's split of the SMs between the prefill and decode kernels of
a mixed call, read back from the workspace after the call.

The plan kernel writes, at byte 256 of the workspace, five int32 counts: the
entries of the prefill work list (256 query rows of one sequence each; the
prefill kernel takes one work item per entry and query head), the 16-key
decode pages, the work counter, and the SMs the prefill and the decode kernel
may each use.  The split minimises the later of
two finish times: the prefill's KV-tile visits (1.15 SM-us each at head_dim
128, over P SMs) against the decode's bytes (56 GB/s per SM on the other SMs,
7.2 TB/s at most in all).  Here that model is evaluated on the host from the
call's lengths in float32, in the kernel's order of operations, and the
kernel's choice must be its minimiser (within one SM, for rounding)."""
import math

import numpy as np
import pytest
import torch

import paged_kv_gqa_reshape_b200 as pa
import workloads

pytestmark = pytest.mark.gpu

HEADER = 256  # byte offset of the plan header in the workspace


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def plan_header(ws):
    h = ws[HEADER:HEADER + 20].cpu().view(torch.int32).tolist()
    return dict(items=h[0], pages=h[1], next=h[2], prefill_sms=h[3], decode_sms=h[4])


def host_counts(seq_lens, query_lens):
    """Prefill work items, per-head KV-tile visits of their 128-row tiles
    (causal, bottom-right aligned) and decode pages, from the lengths."""
    items = visits = pages = 0
    for L, q in zip(seq_lens, query_lens):
        if q == 1:
            pages += math.ceil(L / 16)
        elif q > 1:
            for r in range(0, q, 256):
                items += 1
                for r0 in (r, r + 128):
                    rows = min(128, q - r0)
                    if rows <= 0:
                        continue
                    vis = max(0, min(L, L - q + r0 + rows))
                    visits += math.ceil(vis / 128)
    return items, visits, pages


def model_times(visits, pages, sms, hq, hkv, d):
    """Finish time of each split P = 1 .. sms-1 under the cost model, float32."""
    f = np.float32
    wp = f(f(f(f(visits) * f(hq)) * f(1.15)) * f(d)) / f(128.0)
    nbytes = f(f(f(f(pages) * f(16)) * f(hkv)) * f(d)) * f(4.0)
    t_hbm = nbytes / f(7.2e6)
    p = np.arange(1, sms, dtype=np.int64)
    t_pre = wp / p.astype(np.float32)
    t_dec = nbytes / ((sms - p).astype(np.float32) * f(56.0e3))
    return p, np.maximum(t_pre, np.maximum(t_dec, t_hbm))


def run_call(case):
    ws = pa.varlen_workspace(case.num_seqs, case.num_q_tokens, case.num_q_heads,
                             case.num_kv_heads, case.head_dim)
    out = torch.empty_like(case.q)
    pa.attention_varlen(case.q, case.k_cache, case.v_cache, case.block_tables, case.seq_lens,
                        case.query_start_loc, case.num_kv_heads, case.scale, case.causal, out,
                        max_query_len=case.max_query_len, max_seq_len=case.max_seq_len,
                        workspace=ws)
    torch.cuda.synchronize()
    assert pa.get_error(ws) == (0, 0)
    return plan_header(ws)


@pytest.mark.parametrize("num_chunks,num_decodes,dec_hi", [(8, 248, 32768), (2, 64, 4096),
                                                          (8, 16, 2048), (1, 512, 8192)])
def test_mixed_split_minimises_the_cost_model(num_chunks, num_decodes, dec_hi):
    case = workloads.mixed_step(device="cuda", keep_logical=False, num_chunks=num_chunks,
                                num_decodes=num_decodes, dec_hi=dec_hi)
    seq_lens = case.seq_lens.tolist()
    qsl = case.query_start_loc.tolist()
    qlens = [qsl[i + 1] - qsl[i] for i in range(case.num_seqs)]
    h = run_call(case)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    items, visits, pages = host_counts(seq_lens, qlens)
    assert h["items"] == items
    assert h["pages"] == pages
    assert 1 <= h["prefill_sms"] < sms
    assert h["prefill_sms"] + h["decode_sms"] == sms
    p, t = model_times(visits, pages, sms, case.num_q_heads, case.num_kv_heads, case.head_dim)
    best = int(p[np.argmin(t)])
    assert abs(h["prefill_sms"] - best) <= 1, (h, best)
    # a neighbour of the host's choice only where the two times tie to rounding
    assert t[h["prefill_sms"] - 1] <= t.min() * (1 + 1e-4), (h, best)


def test_pure_prefill_takes_every_sm():
    # no decode pages: both kernels may use the whole machine (the decode
    # kernel's CTAs find nothing to do)
    case = workloads.build_varlen_case("split", [700, 300, 129], [700, 300, 129], 8, 2, 128,
                                       True, 91, device="cuda", keep_logical=False)
    h = run_call(case)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert h["pages"] == 0
    assert h["items"] == host_counts([700, 300, 129], [700, 300, 129])[0]
    assert h["prefill_sms"] == sms and h["decode_sms"] == sms
