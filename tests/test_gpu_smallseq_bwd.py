"""Small-seq attention weights (forward output) and backward (dQ, dK, dV) on
the GPU against the fp64 oracle, ROCm/TransformerEngine PR #461 (the forward
saves the softmax weights [batch, Hq, 1, s_kv] in the q/k/v dtype; the
backward reads them and computes grad_V, grad_attn, the softmax backward and
grad_Q / grad_K).

Tolerances, derived from the arithmetic:

* weights: the kernel computes each weight in fp32 (relative error ~1e-6) and
  rounds it once to the element type, so |w - w_ref| <= u |w_ref| + 1e-5 with
  u the unit roundoff (2^-8 bf16, 2^-11 fp16, a little slack for fp32 error
  that moves a value across a rounding midpoint);
* backward from given weights: the oracle takes the same weights (rounded to
  the element type by torch, widened exactly), so the only differences are
  fp32 sums (|dP| ~ sqrt(D), absolute error ~1e-5 after scaling) and the one
  rounding of each output: |g - g_ref| <= u |g_ref| + 5e-4;
* the forward -> backward chain against the exact-softmax oracle adds the
  weights' own rounding, |w - p| <= u p.  It moves dV_j by at most
  u sum_h p_hj |dO_h| and dS_hj by at most u p_hj (|dP_hj| + 2 sum_k p_hk |dP_hk|)
  =: u T_hj, hence dQ_h by u scale sum_j T_hj |k_j| and dK_j by
  u scale sum_h T_hj |q_h|; each output is held to that (x1.05) plus its own
  rounding u |g_ref| and 5e-4 for the fp32 sums (chain_bounds below).  A flat
  absolute bound does not fit: dV sums g heads' contributions, so |dV| reaches
  ~2g and one rounding of it alone is u |dV|.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_gqa_reshape_b200 as pa
import workloads

pytestmark = pytest.mark.gpu
BF16, F16 = torch.bfloat16, torch.float16
UNIT = {BF16: 2.0 ** -8, F16: 2.0 ** -11}  # unit roundoff 2^-p, p = 8 / 11 bits
DT = {BF16: 0, F16: 1}


def bits(t):
    return workloads.bf16_bits(t.cpu())


def to_dev(c):
    import dataclasses
    return dataclasses.replace(c, q=c.q.cuda(), k=c.k.cuda(), v=c.v.cuda(),
                               cu_seqlens_kv=c.cu_seqlens_kv.cuda())


def make_case(lens, hq, hkv, d, seed, dtype):
    return workloads.build_smallseq_case("bwd", lens, hq, hkv, d, seed=seed, dtype=dtype)


def upstream(c, seed, dtype):
    return workloads._randn_bf16((c.batch, c.num_q_heads, c.head_dim),
                                 workloads._gen(seed, "cpu"), "cpu", dtype=dtype)


def gpu_forward(dev, wlen, max_seqlen_kv=16):
    out = torch.full_like(dev.q, float("nan"))
    w = torch.full((dev.batch, dev.num_q_heads, wlen), float("nan"), dtype=dev.q.dtype,
                   device="cuda")
    ws = pa.error_workspace()
    pa.attention_smallseq(dev.q, dev.k, dev.v, dev.cu_seqlens_kv, dev.scale, out,
                          max_seqlen_kv=max_seqlen_kv, workspace=ws, weights=w)
    torch.cuda.synchronize()
    return out, w, ws


def gpu_backward(dev, dout, w, max_seqlen_kv=16):
    dq = torch.full_like(dev.q, float("nan"))
    dk = torch.full_like(dev.k, float("nan"))
    dv = torch.full_like(dev.v, float("nan"))
    ws = pa.error_workspace()
    pa.attention_smallseq_bwd(dev.q, dev.k, dev.v, dout, w, dev.cu_seqlens_kv, dev.scale, dq, dk,
                              dv, max_seqlen_kv=max_seqlen_kv, workspace=ws)
    torch.cuda.synchronize()
    return dq, dk, dv, ws


def assert_rel_close(got, ref, u, atol, what):
    got = got.double().cpu().numpy()
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bound = 1.01 * u * np.abs(ref) + atol
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements out of bound, worst "
                           f"{float(np.max(err - bound)):.3e} over")


def chain_bounds(q, k, v, dout, cu, hkv, scale, u):
    """Per-element error bounds of the chain (module docstring), float64."""
    q, k, v, dout = (torch.as_tensor(x).double() for x in (q, k, v, dout))
    b_, hq, d = q.shape
    g = hq // hkv
    bq = torch.zeros(b_, hq, d, dtype=torch.float64)
    bk = torch.zeros(k.shape, dtype=torch.float64)
    bv = torch.zeros(v.shape, dtype=torch.float64)
    for b in range(b_):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        if s1 == s0:
            continue
        kb = k[s0:s1].repeat_interleave(g, dim=1)              # [n, Hq, D]
        vb = v[s0:s1].repeat_interleave(g, dim=1)
        p = torch.softmax(scale * torch.einsum("hd,nhd->hn", q[b], kb), dim=1)
        adp = torch.einsum("hd,nhd->hn", dout[b], vb).abs()
        t = p * (adp + 2 * (p * adp).sum(1, keepdim=True))
        bq[b] = scale * torch.einsum("hn,nhd->hd", t, kb.abs())
        n = s1 - s0
        bk[s0:s1] = (scale * torch.einsum("hn,hd->nhd", t, q[b].abs())).reshape(n, hkv, g, d).sum(2)
        bv[s0:s1] = torch.einsum("hn,hd->nhd", p, dout[b].abs()).reshape(n, hkv, g, d).sum(2)
    return (1.05 * u * x.numpy() for x in (bq, bk, bv))


def assert_chain_close(got, ref, extra, u, what):
    got = got.double().cpu().numpy()
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bound = 1.01 * u * np.abs(ref) + extra + 5e-4
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements out of bound, worst "
                           f"{float(np.max(err - bound)):.3e} over")
    return float(np.max(err)), float(np.mean(err))


SHAPES = [(128, 16, 16), (128, 8, 2), (64, 8, 4), (64, 16, 1)]


@pytest.mark.parametrize("dtype", [BF16, F16])
@pytest.mark.parametrize("d,hq,hkv", SHAPES)
def test_weights_output(d, hq, hkv, dtype):
    rng = np.random.default_rng(d + hq + hkv)
    lens = rng.integers(0, 17, size=400).tolist()
    cpu = make_case(lens, hq, hkv, d, seed=60 + d, dtype=dtype)
    out, w, ws = gpu_forward(to_dev(cpu), 16)
    ref = oracle.smallseq_weights(bits(cpu.q), bits(cpu.k), cpu.cu_seqlens_kv.numpy(), hkv,
                                  cpu.scale, 16, dtype=DT[dtype])
    assert_rel_close(w, ref, UNIT[dtype], 1e-5, "weights")
    # zeros past each entry's keys, exactly
    wn = w.double().cpu().numpy()
    for b, n in enumerate(lens):
        assert not wn[b, :, n:].any()
    # the output of the same call is unchanged by asking for the weights
    ref_out = oracle.smallseq_dtype(bits(cpu.q), bits(cpu.k), bits(cpu.v),
                                    cpu.cu_seqlens_kv.numpy(), hkv, cpu.scale, DT[dtype])
    err = np.abs(out.double().cpu().numpy() - ref_out)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3
    assert pa.get_error(ws) == (0, 0)


def test_weights_width_equal_to_longest_entry_and_hint():
    lens = [3, 12, 0, 7, 12, 1]
    cpu = make_case(lens, 8, 2, 128, seed=61, dtype=BF16)
    dev = to_dev(cpu)
    _, w, ws = gpu_forward(dev, 12)
    ref = oracle.smallseq_weights(bits(cpu.q), bits(cpu.k), cpu.cu_seqlens_kv.numpy(), 2,
                                  cpu.scale, 12)
    assert_rel_close(w, ref, UNIT[BF16], 1e-5, "weights W=12")
    assert pa.get_error(ws) == (0, 0)
    # a row narrower than an entry: the first weights_len weights, and the hint bit
    _, w8, ws8 = gpu_forward(dev, 8)
    full = oracle.smallseq_weights(bits(cpu.q), bits(cpu.k), cpu.cu_seqlens_kv.numpy(), 2,
                                   cpu.scale, 12)
    assert_rel_close(w8, full[:, :, :8], UNIT[BF16], 1e-5, "weights W=8")
    status, bits_ = pa.get_error(ws8)
    assert status != 0 and bits_ == pa.DEVERR_HINT


@pytest.mark.parametrize("dtype", [BF16, F16])
@pytest.mark.parametrize("d,hq,hkv", SHAPES)
def test_backward_from_given_weights(d, hq, hkv, dtype):
    rng = np.random.default_rng(d * hq + hkv)
    lens = rng.integers(0, 17, size=300).tolist()
    lens[:4] = [0, 16, 1, 2]
    cpu = make_case(lens, hq, hkv, d, seed=70 + d, dtype=dtype)
    dout = upstream(cpu, 71 + d, dtype)
    exact = oracle.smallseq_weights(bits(cpu.q), bits(cpu.k), cpu.cu_seqlens_kv.numpy(), hkv,
                                    cpu.scale, 16, dtype=DT[dtype])
    w = torch.from_numpy(exact).to(dtype)                 # what a 16-bit forward saves
    dq, dk, dv, ws = gpu_backward(to_dev(cpu), dout.cuda(), w.cuda())
    rq, rk, rv = oracle.smallseq_backward(bits(cpu.q), bits(cpu.k), bits(cpu.v), bits(dout),
                                          cpu.cu_seqlens_kv.numpy(), hkv, cpu.scale,
                                          dtype=DT[dtype], weights=w.double().numpy())
    u = UNIT[dtype]
    assert_rel_close(dq, rq, u, 5e-4, "dq")
    assert_rel_close(dk, rk, u, 5e-4, "dk")
    assert_rel_close(dv, rv, u, 5e-4, "dv")
    assert not dq[0].any()                                # empty entry: zero dQ
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("dtype", [BF16, F16])
@pytest.mark.parametrize("d,hq,hkv", [(128, 16, 16), (64, 8, 2)])
def test_forward_then_backward_chain(d, hq, hkv, dtype):
    rng = np.random.default_rng(d + 5 * hq)
    lens = rng.choice([2, 4, 6, 8, 12, 16], size=300).tolist()
    cpu = make_case(lens, hq, hkv, d, seed=80 + d, dtype=dtype)
    dev = to_dev(cpu)
    dout = upstream(cpu, 81 + d, dtype)
    _, w, _ = gpu_forward(dev, 16)
    dq, dk, dv, ws = gpu_backward(dev, dout.cuda(), w)
    rq, rk, rv = oracle.smallseq_backward(bits(cpu.q), bits(cpu.k), bits(cpu.v), bits(dout),
                                          cpu.cu_seqlens_kv.numpy(), hkv, cpu.scale,
                                          dtype=DT[dtype])
    eq, ek, ev = chain_bounds(cpu.q, cpu.k, cpu.v, dout, cpu.cu_seqlens_kv.tolist(), hkv,
                              cpu.scale, UNIT[dtype])
    for got, ref, extra, name in ((dq, rq, eq, "dq"), (dk, rk, ek, "dk"), (dv, rv, ev, "dv")):
        assert_chain_close(got, ref, extra, UNIT[dtype], name)
    assert pa.get_error(ws) == (0, 0)


def test_backward_rejects_before_launch():
    cpu = make_case([3, 4], 8, 2, 128, seed=90, dtype=BF16)
    dev = to_dev(cpu)
    dout = torch.zeros_like(dev.q)
    w = torch.zeros(2, 8, 16, dtype=BF16, device="cuda")
    dq, dk, dv = torch.zeros_like(dev.q), torch.zeros_like(dev.k), torch.zeros_like(dev.v)
    with pytest.raises(pa.PaError):       # s_kv hint above 16
        pa.attention_smallseq_bwd(dev.q, dev.k, dev.v, dout, w, dev.cu_seqlens_kv, dev.scale,
                                  dq, dk, dv, max_seqlen_kv=17)
    with pytest.raises(TypeError):        # weights of another dtype
        pa.attention_smallseq_bwd(dev.q, dev.k, dev.v, dout, w.half(), dev.cu_seqlens_kv,
                                  dev.scale, dq, dk, dv)
    q32 = make_case([3, 4], 32, 1, 128, seed=91, dtype=BF16)   # group 32 > 16
    d32 = to_dev(q32)
    with pytest.raises(pa.PaError):
        pa.attention_smallseq_bwd(d32.q, d32.k, d32.v, torch.zeros_like(d32.q),
                                  torch.zeros(2, 32, 16, dtype=BF16, device="cuda"),
                                  d32.cu_seqlens_kv, d32.scale, torch.zeros_like(d32.q),
                                  torch.zeros_like(d32.k), torch.zeros_like(d32.v))
    assert torch.count_nonzero(dq) == 0


def test_backward_full_size_sampled():
    # the bench workload (batch 30720, s_kv over {2,..,16}, 16 heads, D 128):
    # forward with weights, then backward, checked on sampled entries, which
    # are independent of each other, so a sub-batch oracle computes them exactly
    ss = workloads.smallseq_batch(device="cuda")
    torch.manual_seed(0)
    dout = workloads._randn_bf16(tuple(ss.q.shape), workloads._gen(92, "cuda"), "cuda")
    w = torch.empty(ss.batch, ss.num_q_heads, 16, dtype=BF16, device="cuda")
    out = torch.empty_like(ss.q)
    pa.attention_smallseq(ss.q, ss.k, ss.v, ss.cu_seqlens_kv, ss.scale, out, weights=w)
    dq, dk, dv, ws = gpu_backward(ss, dout, w)
    assert pa.get_error(ws) == (0, 0)
    cu = ss.cu_seqlens_kv.cpu().tolist()
    rng = np.random.default_rng(93)
    pick = sorted(set(rng.integers(0, ss.batch, size=200).tolist()) | {0, ss.batch - 1})
    kk = torch.cat([ss.k[cu[b]:cu[b + 1]] for b in pick]).cpu()
    vv = torch.cat([ss.v[cu[b]:cu[b + 1]] for b in pick]).cpu()
    lens = [cu[b + 1] - cu[b] for b in pick]
    sub_cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    rq, rk, rv = oracle.smallseq_backward(bits(ss.q[pick]), bits(kk), bits(vv),
                                          bits(dout[pick]), sub_cu, ss.num_kv_heads, ss.scale)
    gk = torch.cat([dk[cu[b]:cu[b + 1]] for b in pick])
    gv = torch.cat([dv[cu[b]:cu[b + 1]] for b in pick])
    eq, ek, ev = chain_bounds(ss.q[pick].cpu(), kk, vv, dout[pick].cpu(), sub_cu.tolist(),
                              ss.num_kv_heads, ss.scale, UNIT[BF16])
    for got, ref, extra, name in ((dq[pick], rq, eq, "dq"), (gk, rk, ek, "dk"),
                                  (gv, rv, ev, "dv")):
        assert_chain_close(got, ref, extra, UNIT[BF16], name)


def test_weights_full_size_sampled():
    # the benchmark's forward with the weights output (batch 30720, width 16):
    # sampled entries against the oracle on their sub-batch, and zeros past
    # every entry's keys over the whole output
    ss = workloads.smallseq_batch(device="cuda")
    out, w, ws = gpu_forward(ss, 16)
    assert pa.get_error(ws) == (0, 0)
    cu = ss.cu_seqlens_kv.cpu()
    lens = (cu[1:] - cu[:-1]).to("cuda")
    past = torch.arange(16, device="cuda")[None, None, :] >= lens[:, None, None]
    assert torch.count_nonzero(w.masked_select(past)) == 0
    cu = cu.tolist()
    rng = np.random.default_rng(94)
    pick = sorted(set(rng.integers(0, ss.batch, size=300).tolist()) | {0, ss.batch - 1})
    kk = torch.cat([ss.k[cu[b]:cu[b + 1]] for b in pick]).cpu()
    sub_cu = np.concatenate([[0], np.cumsum([cu[b + 1] - cu[b] for b in pick])]).astype(np.int32)
    ref = oracle.smallseq_weights(bits(ss.q[pick]), bits(kk), sub_cu, ss.num_kv_heads, ss.scale,
                                  16, dtype=0)
    assert_rel_close(w[pick], ref, UNIT[BF16], 1e-5, "weights full (sampled)")
