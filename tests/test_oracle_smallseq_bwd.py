"""Pins for the small-seq attention weights and backward of the oracle
(ROCm/TransformerEngine PR #461: the forward returns the attention weights;
the backward gives grad_Q, grad_K, grad_V): torch autograd in float64 on the
same inputs, and central finite differences of the oracle's own forward."""
import numpy as np
import torch

import oracle
import workloads


def case(lens, hq, hkv, d, seed, dtype=torch.bfloat16):
    return workloads.build_smallseq_case("b", lens, hq, hkv, d, seed=seed, dtype=dtype)


def bits(t):
    return workloads.bf16_bits(t)


def torch_grads(c, dout):
    """Autograd through softmax attention per entry, float64, expanded KV heads."""
    g = c.num_q_heads // c.num_kv_heads
    q = c.q.double().requires_grad_(True)
    k = c.k.double().requires_grad_(True)
    v = c.v.double().requires_grad_(True)
    cu = c.cu_seqlens_kv.tolist()
    outs, weights = [], []
    for b in range(c.batch):
        if cu[b + 1] == cu[b]:
            outs.append(torch.zeros(c.num_q_heads, c.head_dim, dtype=torch.float64))
            weights.append(None)
            continue
        kb = k[cu[b]:cu[b + 1]].repeat_interleave(g, dim=1)       # [n, Hq, D]
        vb = v[cu[b]:cu[b + 1]].repeat_interleave(g, dim=1)
        s = torch.einsum("hd,nhd->hn", q[b], kb) * c.scale
        p = torch.softmax(s, dim=1)
        outs.append(torch.einsum("hn,nhd->hd", p, vb))
        weights.append(p.detach())
    out = torch.stack(outs)
    out.backward(dout.double())
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy(), weights


def test_weights_and_backward_match_autograd():
    lens = [3, 16, 1, 0, 7, 12]
    c = case(lens, 8, 2, 64, seed=41)
    dout = workloads._randn_bf16((c.batch, c.num_q_heads, c.head_dim), workloads._gen(5, "cpu"),
                                 "cpu")
    dq, dk, dv = oracle.smallseq_backward(bits(c.q), bits(c.k), bits(c.v), bits(dout),
                                          c.cu_seqlens_kv.numpy(), c.num_kv_heads, c.scale)
    tq, tk, tv, tw = torch_grads(c, dout)
    assert np.max(np.abs(dq - tq)) < 1e-10
    assert np.max(np.abs(dk - tk)) < 1e-10
    assert np.max(np.abs(dv - tv)) < 1e-10
    w = oracle.smallseq_weights(bits(c.q), bits(c.k), c.cu_seqlens_kv.numpy(), c.num_kv_heads,
                                c.scale, 16)
    for b, n in enumerate(lens):
        if n == 0:
            assert not w[b].any()
            continue
        assert np.max(np.abs(w[b, :, :n] - tw[b].numpy())) < 1e-12
        assert not w[b, :, n:].any()
        assert np.allclose(w[b, :, :n].sum(axis=1), 1.0, atol=1e-12)


def test_backward_matches_finite_differences_of_the_forward():
    # L(q, k, v) = sum(dout * out): dL/dx by central differences on a few coordinates
    lens = [5, 2]
    c = case(lens, 2, 1, 64, seed=42)
    rng = np.random.default_rng(3)
    dout = rng.standard_normal((c.batch, c.num_q_heads, c.head_dim))
    dout_bits = bits(torch.from_numpy(dout).to(torch.bfloat16))
    dout = torch.from_numpy(dout).to(torch.bfloat16).double().numpy()

    def loss(qd, kd, vd):
        # the oracle's forward in float64 on arbitrary real inputs: evaluate the
        # definition directly (the oracle itself takes 16-bit patterns)
        cu = c.cu_seqlens_kv.tolist()
        total = 0.0
        for b in range(c.batch):
            kb, vb = kd[cu[b]:cu[b + 1], 0], vd[cu[b]:cu[b + 1], 0]
            for h in range(c.num_q_heads):
                s = c.scale * kb @ qd[b, h]
                p = np.exp(s - s.max())
                p /= p.sum()
                total += float(dout[b, h] @ (p @ vb))
        return total

    qd, kd, vd = (t.double().numpy() for t in (c.q, c.k, c.v))
    dq, dk, dv = oracle.smallseq_backward(bits(c.q), bits(c.k), bits(c.v), dout_bits,
                                          c.cu_seqlens_kv.numpy(), c.num_kv_heads, c.scale)
    eps = 1e-6
    for arr, grad, idx in ((qd, dq, (0, 1, 3)), (kd, dk, (4, 0, 10)), (vd, dv, (6, 0, 63)),
                           (kd, dk, (0, 0, 0)), (qd, dq, (1, 0, 17))):
        plus, minus = arr.copy(), arr.copy()
        plus[idx] += eps
        minus[idx] -= eps
        args_p = [qd, kd, vd]
        args_m = [qd, kd, vd]
        which = 0 if arr is qd else (1 if arr is kd else 2)
        args_p[which], args_m[which] = plus, minus
        fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        assert abs(fd - grad[idx]) < 1e-6, (idx, fd, grad[idx])


def test_backward_from_given_weights_matches_torch_softmax_backward():
    # The backward reads the forward's saved weights.  With arbitrary weights W
    # (here the exact softmax rounded to bf16, as a 16-bit forward saves it,
    # so W is no longer an exact softmax), the gradients are still
    #   dV_j = sum_h W_hj dO_h,  dS = softmax_backward(dP, W),
    #   dQ = scale dS K,  dK_j = scale sum_h dS_hj q_h,
    # checked here with torch's own softmax backward on the output W.
    lens = [4, 16, 0, 9]
    c = case(lens, 4, 2, 64, seed=43)
    g = c.num_q_heads // c.num_kv_heads
    dout = workloads._randn_bf16((c.batch, c.num_q_heads, c.head_dim), workloads._gen(6, "cpu"),
                                 "cpu")
    exact = oracle.smallseq_weights(bits(c.q), bits(c.k), c.cu_seqlens_kv.numpy(), c.num_kv_heads,
                                    c.scale, 16)
    w = torch.from_numpy(exact).to(torch.bfloat16).double().numpy()
    dq, dk, dv = oracle.smallseq_backward(bits(c.q), bits(c.k), bits(c.v), bits(dout),
                                          c.cu_seqlens_kv.numpy(), c.num_kv_heads, c.scale,
                                          weights=w)
    cu = c.cu_seqlens_kv.tolist()
    qd, kd, vd, gd = (t.double() for t in (c.q, c.k, c.v, dout))
    for b, n in enumerate(lens):
        if n == 0:
            assert not dq[b].any()
            continue
        kb = kd[cu[b]:cu[b + 1]].repeat_interleave(g, dim=1)      # [n, Hq, D]
        vb = vd[cu[b]:cu[b + 1]].repeat_interleave(g, dim=1)
        wb = torch.from_numpy(w[b, :, :n])                        # [Hq, n]
        dp = torch.einsum("hd,nhd->hn", gd[b], vb)
        ds = torch._softmax_backward_data(dp, wb, 1, torch.float64)
        ref_dq = c.scale * torch.einsum("hn,nhd->hd", ds, kb)
        ref_dk = c.scale * torch.einsum("hn,hd->nhd", ds, qd[b]).reshape(
            n, c.num_kv_heads, g, c.head_dim).sum(2)
        ref_dv = torch.einsum("hn,hd->nhd", wb, gd[b]).reshape(
            n, c.num_kv_heads, g, c.head_dim).sum(2)
        assert np.max(np.abs(dq[b] - ref_dq.numpy())) < 1e-10
        assert np.max(np.abs(dk[cu[b]:cu[b + 1]] - ref_dk.numpy())) < 1e-10
        assert np.max(np.abs(dv[cu[b]:cu[b + 1]] - ref_dv.numpy())) < 1e-10
    # the rounded weights move the gradients, by about their own relative error
    dq0, _, dv0 = oracle.smallseq_backward(bits(c.q), bits(c.k), bits(c.v), bits(dout),
                                           c.cu_seqlens_kv.numpy(), c.num_kv_heads, c.scale)
    assert 0 < np.max(np.abs(dv - dv0)) < 2 ** -8 * np.max(np.abs(dv0)) * 4
