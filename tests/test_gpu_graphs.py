"""The library's calls inside CUDA graphs, as a serving loop captures them:
no call synchronises or allocates, so write_kv + attention capture into one
graph (the decode launch keeps its programmatic dependency on the scatter),
and replays give the eager calls' results bit for bit, including after the
step's inputs are rewritten in place between replays."""
import pytest
import torch

import paged_kv_gqa_reshape_b200 as pa
import workloads
from tests.gpu_helpers import assert_attention_close, case_to, oracle_varlen

pytestmark = pytest.mark.gpu


def capture(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


@pytest.mark.parametrize("name,lens,qlens", [
    ("decode", [300, 1000, 17, 4096, 64], [1, 1, 1, 1, 1]),
    ("mixed", [700, 40, 300, 1, 2000, 17], [64, 1, 300, 1, 1, 17]),
])
def test_graph_replay_equals_eager(name, lens, qlens):
    cpu = workloads.build_varlen_case(name, lens, qlens, 16, 4, 128, True, seed=70)
    dev = case_to(cpu, "cuda")
    mql, msl = dev.max_query_len, dev.max_seq_len
    ws = pa.varlen_workspace(dev.num_seqs, dev.num_q_tokens, 16, 4, 128)
    kc, vc = dev.k_cache.clone(), dev.v_cache.clone()
    out = torch.full_like(dev.q, float("nan"))

    def step():
        pa.write_kv(dev.k_new, dev.v_new, dev.slot_mapping, kc, vc, workspace=ws)
        pa.attention_varlen(dev.q, kc, vc, dev.block_tables, dev.seq_lens, dev.query_start_loc,
                            4, dev.scale, True, out, max_query_len=mql, max_seq_len=msl,
                            workspace=ws)

    step()
    torch.cuda.synchronize()
    eager = out.clone()
    assert_attention_close(eager, oracle_varlen(cpu), what=f"{name} eager")
    g = capture(step)
    out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
    assert pa.get_error(ws) == (0, 0)

    # new queries written in place: the replay reads them
    q2 = workloads._randn_bf16(tuple(cpu.q.shape), workloads._gen(71, "cpu"), "cpu")
    dev.q.copy_(q2.cuda())
    g.replay()
    torch.cuda.synchronize()
    import dataclasses
    assert_attention_close(out, oracle_varlen(dataclasses.replace(cpu, q=q2)),
                           what=f"{name} replay, new q")
    for _ in range(5):
        g.replay()
    torch.cuda.synchronize()
    assert pa.get_error(ws) == (0, 0)
    del g


def test_smallseq_forward_and_backward_in_one_graph():
    cpu = workloads.build_smallseq_case("g", [3, 16, 0, 8, 12], 8, 2, 128, seed=72)
    ss = case_to(cpu, "cuda")
    out = torch.empty_like(ss.q)
    w = torch.empty(ss.batch, 8, 16, dtype=torch.bfloat16, device="cuda")
    dout = torch.randn_like(ss.q)
    dq, dk, dv = torch.empty_like(ss.q), torch.empty_like(ss.k), torch.empty_like(ss.v)

    def step():
        pa.attention_smallseq(ss.q, ss.k, ss.v, ss.cu_seqlens_kv, ss.scale, out, weights=w)
        pa.attention_smallseq_bwd(ss.q, ss.k, ss.v, dout, w, ss.cu_seqlens_kv, ss.scale, dq, dk,
                                  dv)

    step()
    torch.cuda.synchronize()
    ref = [t.clone() for t in (out, w, dq, dk, dv)]
    g = capture(step)
    for t in (out, w, dq, dk, dv):
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    for got, want in zip((out, w, dq, dk, dv), ref):
        assert torch.equal(got, want)
    del g
