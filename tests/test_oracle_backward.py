"""Pins for the backward oracle (oracle/backward.py), independent of its code:

* torch autograd through a float64 forward written another way (softmax over
  the visible logits plus one virtual key of logit s_h and value 0, then the
  virtual column dropped): dq, dk, dv and dsink agree to 1e-10, with and
  without a sink, several windows, GQA groups and packed sequences;
* central finite differences of the C oracle's forward (fp64 sink and scale
  arguments) in the sink and in the softmax scale: dsink, and the identity
  dL/dscale = sum_i q_i.dq_i / scale = sum_j k_j.dk_j / scale;
* a closed form: with q = 0 every visible weight is 1 / (n_i + e^s), so
  dv_j = sum over the rows i that see j of dO_i / (n_i + e^s);
* the sampled-place entry (o and lse computed for the rows it needs, or
  taken from a whole forward) and dsink from a forward's o / lse equal the
  full backward;
* the sums of dk and dv over each sequence's keys, from the forward's o and
  lse alone (sum_j dA_ij = Delta_i p_sink,i), equal the full backward's.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob
from sliding_window_attention_sink_b200 import workloads as wl

from test_oracle import torch_sink_attention


def autograd_grads(c, dout, W, sink):
    """Gradients of sum(dout * o) by torch autograd through the augmented
    softmax forward, sequence by sequence (float64)."""
    Hq, Hkv, D = c["Hq"], c["Hkv"], c["D"]
    q = c["q"].double().requires_grad_(True)
    k = c["k"].double().requires_grad_(True)
    v = c["v"].double().requires_grad_(True)
    s = None if sink is None else sink.double().clone().requires_grad_(True)
    cu = c["cu_seqlens"].tolist()
    loss = 0.0
    for a, b in zip(cu[:-1], cu[1:]):
        if b == a:
            continue
        o, _, _ = torch_sink_attention(q[a:b], k[a:b], v[a:b], W, s, D ** -0.5)
        loss = loss + (o * dout[a:b]).sum()
    loss.backward()
    ds = np.zeros(Hq) if s is None else s.grad.numpy()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy(), ds


CASES = [  # (seqlens, Hq, Hkv, D, W, sink)
    ([9], 2, 1, 8, 4, "normal"),
    ([20, 3, 0, 11], 4, 2, 8, 5, "normal"),
    ([16], 4, 1, 16, 0, "uniform2"),
    ([13], 6, 2, 4, 1, "normal"),
    ([12, 7], 2, 2, 8, 3, None),
    ([25], 8, 1, 8, 64, "normal"),
]


@pytest.mark.parametrize("seqlens,Hq,Hkv,D,W,sink", CASES)
def test_backward_equals_autograd(seqlens, Hq, Hkv, D, W, sink):
    c = wl.prefill_case(seqlens, Hq, Hkv, D, W, sigma=0.8, sink=sink, seed=sum(seqlens) + D)
    g = torch.Generator().manual_seed(7)
    dout = torch.randn(c["q"].shape, generator=g, dtype=torch.float64)
    dq, dk, dv, ds = ob.prefill_backward(c["q"], c["k"], c["v"], dout.numpy(), c["cu_seqlens"],
                                         Hq, Hkv, D, W, sink=c["sink"])
    rq, rk, rv, rs = autograd_grads(c, dout, W, c["sink"])
    for got, ref in ((dq, rq), (dk, rk), (dv, rv), (ds, rs)):
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-10)


def _loss(c, dout, W, sink, scale):
    o, _, _ = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], c["Hq"], c["Hkv"], c["D"],
                             W, sink=sink, scale=scale)
    return float((o * dout).sum())


@pytest.mark.parametrize("W", [6, 0])
def test_backward_finite_differences_of_the_c_oracle(W):
    c = wl.prefill_case([30, 17], 4, 2, 16, W, sigma=0.8, sink="normal", seed=5)
    dout = np.random.default_rng(1).standard_normal(c["q"].shape)
    sc = 0.25
    dq, dk, dv, ds = ob.prefill_backward(c["q"], c["k"], c["v"], dout, c["cu_seqlens"], 4, 2, 16,
                                         W, sink=c["sink"], scale=sc)
    sink = c["sink"].double().numpy()
    eps = 1e-6
    for h in range(4):
        sp, sm = sink.copy(), sink.copy()
        sp[h] += eps
        sm[h] -= eps
        fd = (_loss(c, dout, W, sp, sc) - _loss(c, dout, W, sm, sc)) / (2 * eps)
        assert abs(fd - ds[h]) <= 1e-6 * max(1.0, abs(fd)), (h, fd, ds[h])
    fd = (_loss(c, dout, W, sink, sc + eps) - _loss(c, dout, W, sink, sc - eps)) / (2 * eps)
    q = c["q"].double().numpy()
    k = c["k"].double().numpy()
    via_q = (q * dq).sum() / sc
    via_k = (k * dk).sum() / sc
    assert abs(fd - via_q) <= 1e-6 * max(1.0, abs(fd)), (fd, via_q)
    assert abs(via_q - via_k) <= 1e-9 * max(1.0, abs(via_q))


def test_backward_zero_query_closed_form():
    L, Hq, Hkv, D, W = 19, 2, 1, 8, 5
    c = wl.prefill_case([L], Hq, Hkv, D, W, sigma=1.0, sink="normal", seed=8)
    c["q"] = torch.zeros_like(c["q"])
    dout = np.random.default_rng(2).standard_normal(c["q"].shape)
    _, _, dv, _ = ob.prefill_backward(c["q"], c["k"], c["v"], dout, c["cu_seqlens"], Hq, Hkv, D,
                                      W, sink=c["sink"])
    s = c["sink"].double().numpy()
    want = np.zeros((L, D))
    for i in range(L):
        n = min(i + 1, W)
        for j in range(i - n + 1, i + 1):
            for h in range(Hq):
                want[j] += dout[i, h] / (n + math.exp(s[h]))
    np.testing.assert_allclose(dv[:, 0], want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("W", [7, 0])
def test_sampled_entry_and_dsink_from_forward(W):
    c = wl.prefill_case([40, 1, 23], 8, 2, 16, W, sigma=0.7, sink="normal", seed=9)
    dout = torch.randn(c["q"].shape, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    dq, dk, dv, ds = ob.prefill_backward(c["q"], c["k"], c["v"], dout, c["cu_seqlens"], 8, 2, 16,
                                         W, sink=c["sink"])
    rng = np.random.default_rng(4)
    rt = rng.integers(0, 64, 20)
    rh = rng.integers(0, 8, 20)
    kt = np.concatenate([rng.integers(0, 64, 10), [0, 39, 40, 41, 63]])
    kh = rng.integers(0, 2, len(kt))
    sq, sk, sv = ob.prefill_backward_rows(c["q"], c["k"], c["v"], dout, c["cu_seqlens"], 8, 2, 16,
                                          W, rt, rh, kt, kh, sink=c["sink"])
    np.testing.assert_allclose(sq, dq[rt, rh], rtol=0, atol=1e-12)
    np.testing.assert_allclose(sk, dk[kt, kh], rtol=0, atol=1e-12)
    np.testing.assert_allclose(sv, dv[kt, kh], rtol=0, atol=1e-12)
    o, lse, _ = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], 8, 2, 16, W,
                               sink=c["sink"])
    # the same places with o and lse taken from the whole layer's forward
    fq, fk, fv = ob.prefill_backward_rows(c["q"], c["k"], c["v"], dout, c["cu_seqlens"], 8, 2,
                                          16, W, rt, rh, kt, kh, sink=c["sink"],
                                          forward=(o, lse))
    np.testing.assert_allclose(fq, dq[rt, rh], rtol=0, atol=1e-12)
    np.testing.assert_allclose(fk, dk[kt, kh], rtol=0, atol=1e-12)
    np.testing.assert_allclose(fv, dv[kt, kh], rtol=0, atol=1e-12)
    np.testing.assert_allclose(ob.dsink_from_forward(o, lse, dout, c["sink"]), ds, rtol=0,
                               atol=1e-12)


@pytest.mark.parametrize("W,sink", [(7, "normal"), (0, "uniform2"), (3, None)])
def test_key_sums_from_forward_equal_the_full_backward(W, sink):
    """The sums of dk and dv over each sequence's keys, from the forward's o
    and lse alone, equal the full backward's; a sequence of length 1 and an
    empty one included."""
    seqlens = [40, 1, 0, 23]
    c = wl.prefill_case(seqlens, 8, 2, 16, W, sigma=0.7, sink=sink, seed=10)
    dout = torch.randn(c["q"].shape, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    s = c["sink"] if sink else None
    _, dk, dv, _ = ob.prefill_backward(c["q"], c["k"], c["v"], dout, c["cu_seqlens"], 8, 2, 16,
                                       W, sink=s)
    o, lse, _ = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], 8, 2, 16, W, sink=s)
    sk, sv = ob.key_sums_from_forward(c["q"], o, lse, dout, c["cu_seqlens"], 8, 2, sink=s)
    cu = c["cu_seqlens"].tolist()
    for b in range(len(seqlens)):
        np.testing.assert_allclose(sk[b], dk[cu[b]:cu[b + 1]].sum(axis=0), rtol=0, atol=1e-11)
        np.testing.assert_allclose(sv[b], dv[cu[b]:cu[b + 1]].sum(axis=0), rtol=0, atol=1e-11)
    if sink is None:
        assert np.abs(sk).max() == 0.0
    else:  # the identity is not trivially zero: the sink term carries it
        assert np.abs(sk).max() > 1e-3
