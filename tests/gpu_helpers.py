"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and compare."""
import numpy as np
import torch

import oracle
import paged_kv_gqa_reshape_b200 as pa
import workloads

MAX_ABS = 2e-2   # attention tolerance: max |gpu - oracle|
MEAN_ABS = 2e-3  # attention tolerance: mean |gpu - oracle|


def case_to(case, device):
    """Copy every tensor of a VarlenCase/SmallSeqCase to `device`."""
    import dataclasses
    kw = {}
    for f in dataclasses.fields(case):
        v = getattr(case, f.name)
        kw[f.name] = v.to(device) if isinstance(v, torch.Tensor) else v
    return type(case)(**kw)


def run_varlen(case, scatter=True, max_query_len=None, max_seq_len=None, workspace=None,
               out=None):
    """Scatter this step's K/V (optional) then attend; returns (out, k_cache, v_cache, ws)."""
    kc, vc = case.k_cache.clone(), case.v_cache.clone()
    ws = workspace if workspace is not None else pa.varlen_workspace(
        case.num_seqs, case.num_q_tokens, case.num_q_heads, case.num_kv_heads, case.head_dim)
    if scatter and case.k_new.shape[0]:
        pa.write_kv(case.k_new, case.v_new, case.slot_mapping, kc, vc, workspace=ws)
    if out is None:
        out = torch.full_like(case.q, float("nan"))
    pa.attention_varlen(case.q, kc, vc, case.block_tables, case.seq_lens, case.query_start_loc,
                        case.num_kv_heads, case.scale, case.causal, out,
                        max_query_len=case.max_query_len if max_query_len is None else max_query_len,
                        max_seq_len=case.max_seq_len if max_seq_len is None else max_seq_len,
                        workspace=ws)
    torch.cuda.synchronize()
    return out, kc, vc, ws


def oracle_varlen(case, rows=None):
    """Oracle (logical form) on a CPU copy of the case."""
    return oracle.attention_varlen(
        workloads.bf16_bits(case.q), workloads.bf16_bits(case.k_logical),
        workloads.bf16_bits(case.v_logical), case.kv_offsets.cpu().numpy(),
        case.seq_lens.cpu().numpy(), case.query_start_loc.cpu().numpy(), case.num_kv_heads,
        case.scale, case.causal, rows=rows)


def errors(gpu_out, ref, rows=None):
    g = gpu_out.detach().double().cpu().numpy()
    if rows is not None:
        g, ref = g[rows], ref[rows]
    assert np.isfinite(g).all(), "non-finite output"
    e = np.abs(g - ref)
    return float(e.max()), float(e.mean())


def assert_attention_close(gpu_out, ref, rows=None, what=""):
    mx, mean = errors(gpu_out, ref, rows)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean


def sub_case(case, seqs, device="cpu"):
    """The sub-batch of `seqs` of a (possibly device-resident, full-size) case,
    with its logical keys/values, as a CPU case the oracle can take."""
    qsl = case.query_start_loc.cpu().tolist()
    sl = case.seq_lens.cpu().tolist()
    off = case.kv_offsets.cpu().tolist()
    qs, ks, vs, new_qsl, new_off, lens = [], [], [], [0], [], []
    cur = 0
    for s in seqs:
        qs.append(case.q[qsl[s]:qsl[s + 1]].cpu())
        ks.append(case.k_logical[off[s]:off[s] + sl[s]].cpu())
        vs.append(case.v_logical[off[s]:off[s] + sl[s]].cpu())
        new_qsl.append(new_qsl[-1] + qsl[s + 1] - qsl[s])
        new_off.append(cur)
        cur += sl[s]
        lens.append(sl[s])
    import dataclasses
    return dataclasses.replace(
        case, q=torch.cat(qs), k_logical=torch.cat(ks), v_logical=torch.cat(vs),
        query_start_loc=torch.tensor(new_qsl, dtype=torch.int32),
        kv_offsets=torch.tensor(new_off, dtype=torch.int64),
        seq_lens=torch.tensor(lens, dtype=torch.int32),
        query_lens=torch.tensor(np.diff(new_qsl), dtype=torch.int32))
