"""GPU parity of swa_sink_attn_bwd (through the C ABI) against the backward
oracle (oracle/backward.py, fp64 gradients of the exact function) on the same
seeded inputs: whole layers on small shapes (sliding windows, global layers,
packed sequences with empty and length-1 ones, GQA groups 1..8, head dims 64
and 128, no sink, extreme sinks), and the bench's full SWA and global layers:
sampled rows and keys, dsink, and the sums of dk and dv over every key.

Tolerance, from the arithmetic: the kernels take the forward's bf16 o (in
Delta), round P and dS to bf16 for the tensor cores and round dq, dk, dv to
bf16. Each rounding is at most 2^-9 relative (bf16 has 8 significant bits);
the last one alone puts up to 2^-9 of max|ref| on the largest element, and
the two earlier ones reach a gradient through sums whose terms have both
signs, so their share of an element's error is of the same order but can be
a few times larger where the sum cancels (dP - Delta for a window of 1). The
tcgen05 kernels measured, over the cases below (the full layers included):
largest error up to 5.2e-3 of max|ref| (2.7 x 2^-9; global layer, D = 64,
dq) and mean error up to 2.3e-3 of mean|ref|, 4.0e-3 for the window of 1.
The bounds are at most twice the largest of these: max error <= 1e-2
max|ref|, mean error <= 6e-3 mean|ref| (1.5x). dsink = -sum_i p_sink,i
Delta_i cancels too: its error scales with S_h = sum_i p_sink,i
sum_d |dout_id o_id| (each product of Delta off by about 2^-9 of itself
through the bf16 o, with both signs); measured at most 1.7e-4 S_h, bounded
by 3.4e-4 S_h.

The key sums. Summed over a sequence's keys, dk and dv are fixed by the
forward (sum_j dA_ij = Delta_i p_sink,i), so the full layers are checked on
every key that way. The error of a sum over N keys is rounding noise that
adds up, measured against g = sqrt(sum_j g_jd^2) of the elements summed: bf16
rounding of the outputs alone gives about 2^-9 / sqrt(3) of g per sum, and
Delta from the bf16 o adds errors that are shared by all the keys a row sees,
so they add up coherently over those keys. Measured on the bench's layers: at
most 1.04e-2 g (SWA layer, dk; global layer 7.6e-3); the bound is 2e-2 g.
One 128-key tile of a 32K-key layer lost or doubled moves each column's sum
by about sqrt(128 / 32768) g = 0.06 g (the square root of its share of the
summed squares), its largest of 128 columns by nearly three times that.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob
from sliding_window_attention_sink_b200 import binding as B
from sliding_window_attention_sink_b200 import workloads as wl

from _parity import to_cuda

pytestmark = pytest.mark.gpu

MAX_REL = 1e-2      # largest error / largest reference magnitude
MEAN_REL = 6e-3     # mean error / mean reference magnitude
DSINK_REL = 3.4e-4  # dsink error / S_h
KEYSUM_REL = 2e-2   # key-sum error / sqrt(sum over the keys of the element squared)


def run_bwd(c, dout, sink="case"):
    d = to_cuda(c)
    s = d["sink"] if sink == "case" else sink
    o, lse = B.attn_fwd(d["q"], d["k"], d["v"], d["cu_seqlens"], c["window"], sink=s,
                        max_seqlen=c["max_seqlen"])
    dq, dk, dv, ds = B.attn_bwd(d["q"], d["k"], d["v"], o, lse, dout.cuda(), d["cu_seqlens"],
                                c["window"], sink=s, max_seqlen=c["max_seqlen"])
    torch.cuda.synchronize()
    assert B.swa_sink_device_error() == 0
    return dq, dk, dv, ds


def check_grad(got, ref, what):
    g = got.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(g).all(), what
    err = np.abs(g - ref)
    scale_max = max(np.abs(ref).max(), 1e-30)
    scale_mean = max(np.abs(ref).mean(), 1e-30)
    stats = (float(err.max() / scale_max), float(err.mean() / scale_mean))
    print("%s: max err / max|ref| %.3g, mean err / mean|ref| %.3g" % (what, *stats))
    assert stats[0] <= MAX_REL and stats[1] <= MEAN_REL, (what, stats)
    return stats


def dsink_scale(c, dout, sink):
    """S_h = sum_i p_sink,i sum_d |dout_id o_id| from the C oracle's forward."""
    o, lse, _ = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], c["Hq"], c["Hkv"],
                               c["D"], c["window"], sink=sink)
    return dsink_scale_from(o, lse, dout, sink)


def dsink_scale_from(o, lse, dout, sink):
    if sink is None:
        return np.zeros(o.shape[1])
    s = sink.double().numpy()
    dO = dout.float().numpy().astype(np.float64)
    absdot = np.einsum("thd,thd->ht", np.abs(dO), np.abs(o))
    return (np.exp(s[:, None] - lse) * absdot).sum(axis=1)


def check_dsink(got, ref, scale, what):
    g = got.cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    ratio = float((err / np.maximum(scale, 1e-30)).max()) if scale.any() else 0.0
    print("%s: dsink error / S_h max %.3g" % (what, ratio))
    assert np.all(err <= DSINK_REL * scale + 1e-6), (what, ratio)


SMALL = [  # (name, seqlens, Hq, Hkv, D, W, sink)
    ("swa_g8", [300], 64, 8, 128, 128, "normal"),
    ("swa_varlen", [100, 0, 257, 1, 33], 16, 2, 128, 128, "normal"),
    ("global", [400], 16, 2, 128, 0, "normal"),
    ("global_varlen_d64", [129, 300, 5], 8, 1, 64, 0, "uniform2"),
    ("g4_w20", [200], 8, 2, 128, 20, "normal"),
    ("g1_d64", [150], 2, 2, 64, 64, "normal"),
    ("no_sink", [257], 8, 1, 128, 128, None),
    ("w1", [70], 8, 1, 64, 1, "normal"),
]


@pytest.mark.parametrize("name,seqlens,Hq,Hkv,D,W,sink", SMALL, ids=[s[0] for s in SMALL])
def test_backward_matches_oracle(name, seqlens, Hq, Hkv, D, W, sink):
    c = wl.prefill_case(seqlens, Hq, Hkv, D, W, sigma=0.5, sink=sink, seed=21)
    dout = wl.make_dout(c["q"].shape, seed=22)
    dq, dk, dv, ds = run_bwd(c, dout)
    rq, rk, rv, rs = ob.prefill_backward(c["q"], c["k"], c["v"], dout, c["cu_seqlens"], Hq, Hkv,
                                         D, W, sink=c["sink"])
    check_grad(dq, rq, name + " dq")
    check_grad(dk, rk, name + " dk")
    check_grad(dv, rv, name + " dv")
    check_dsink(ds, rs, dsink_scale(c, dout, c["sink"]), name + " dsink")


@pytest.mark.parametrize("sval", [6.0, -6.0])
def test_backward_extreme_sinks(sval):
    c = wl.prefill_case([200], 8, 1, 128, 128, sigma=0.5, sink=None, seed=23)
    c["sink"] = torch.full((8,), sval)
    dout = wl.make_dout(c["q"].shape, seed=24)
    dq, dk, dv, ds = run_bwd(c, dout)
    rq, rk, rv, rs = ob.prefill_backward(c["q"], c["k"], c["v"], dout, c["cu_seqlens"], 8, 1, 128,
                                         128, sink=c["sink"])
    for got, ref, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        check_grad(got, ref, "sink=%g %s" % (sval, n))
    check_dsink(ds, rs, dsink_scale(c, dout, c["sink"]), "sink=%g dsink" % sval)


def check_key_sums(got, ref, sampled, n_first, n_keys, what):
    """got: the kernel's dk or dv of one sequence [n_keys, Hkv, D]; ref: the
    oracle's sums over its keys [Hkv, D]; sampled: the oracle's dk or dv at the
    sampled keys, the first n_first of the sequence and then keys drawn
    uniformly from the rest. Each sum's error is measured against
    sqrt(sum_j g_jd^2), the size of the rounding noise that adds up in it,
    estimated from the samples (the first keys exactly, the rest scaled by
    their share of the sequence)."""
    g = got.double().sum(dim=0).cpu().numpy()
    e2 = (sampled[:n_first] ** 2).sum() + (sampled[n_first:] ** 2).sum() * (
        (n_keys - n_first) / max(len(sampled) - n_first, 1))
    noise = np.sqrt(e2 / sampled.shape[1])
    ratio = float(np.abs(g - ref).max() / noise)
    print("%s: key-sum error / sqrt(sum_j g_j^2) max %.3g" % (what, ratio))
    assert ratio <= KEYSUM_REL, (what, ratio)


@pytest.mark.parametrize("wname", ["swa_backward_32k", "global_backward_8k"])
def test_backward_full_layers(wname):
    """The bench's two backward workloads at full size, in its launch
    configuration, against the C oracle's forward over every row (o, lse):
    dq at whole query groups of sampled tokens; dk / dv at the first 16 keys
    (a global layer's largest: every later row sees them) and at keys drawn
    across the sequence; dsink; and the sums of dk and dv over every key of
    each kv head, which the forward fixes (sum_j dA_ij = Delta_i p_sink,i), so
    that a tile computed twice, dropped or written to the wrong keys anywhere
    in the launch moves a sum."""
    c = wl.make_prefill(wl.WORKLOADS[wname])
    dout = c["dout"]
    dq, dk, dv, ds = run_bwd(c, dout)
    T, Hq, Hkv, D, W = c["total"], c["Hq"], c["Hkv"], c["D"], c["window"]
    assert len(c["seqlens"]) == 1
    G = Hq // Hkv
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all().item()
    o, lse, _ = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], Hq, Hkv, D, W,
                               sink=c["sink"])
    rng = np.random.default_rng(5)
    toks = np.unique(np.concatenate([rng.integers(0, T, 24), [0, 1, 127, T - 1]]))
    gq = rng.integers(0, Hkv, len(toks))
    rt = np.repeat(toks, G)
    rh = (np.repeat(gq * G, G) + np.tile(np.arange(G), len(toks))).astype(np.int32)
    n_first = 16
    kt = np.concatenate([np.arange(n_first), rng.choice(np.arange(n_first, T), 24,
                                                        replace=False)])
    kh = rng.integers(0, Hkv, len(kt))
    sq, sk, sv = ob.prefill_backward_rows(c["q"], c["k"], c["v"], dout, c["cu_seqlens"], Hq, Hkv,
                                          D, W, rt, rh, kt, kh, sink=c["sink"],
                                          forward=(o, lse))
    ti, hi = torch.from_numpy(rt).cuda(), torch.from_numpy(rh.astype(np.int64)).cuda()
    check_grad(dq[ti, hi], sq, wname + " dq")
    ki, khi = torch.from_numpy(kt).cuda(), torch.from_numpy(kh.astype(np.int64)).cuda()
    check_grad(dk[ki, khi], sk, wname + " dk")
    check_grad(dv[ki, khi], sv, wname + " dv")
    check_dsink(ds, ob.dsink_from_forward(o, lse, dout, c["sink"]),
                dsink_scale_from(o, lse, dout, c["sink"]), wname + " dsink")
    rk, rv = ob.key_sums_from_forward(c["q"], o, lse, dout, c["cu_seqlens"], Hq, Hkv,
                                      sink=c["sink"])
    check_key_sums(dk, rk[0], sk, n_first, T, wname + " dk")
    check_key_sums(dv, rv[0], sv, n_first, T, wname + " dv")
