"""Pins for the fp64 oracle against facts fixed by the pages and by
mathematics, independent of the oracle's own code:

* with no sink it is textbook masked softmax attention (torch SDPA, float64);
* with a sink it is softmax over the keys plus one virtual key of logit s_h
  and value 0 (the "virtual sink" of the MiMo-V2-Flash report summary,
  section 2.2.2), computed here with a plain unstabilised formula;
* weights plus the sink weight sum to one, and the sink weight is
  exp(s_h - lse);
* closed forms (zero queries, equal keys, huge / tiny sinks, W = 1) and the
  window length min(i+1, W) read back from the zero-query closed form;
* decode over a ring equals prefill over the rebuilt contiguous sequence, and
  a rotated ring gives the same result;
* packed varlen sequences never see each other.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from sliding_window_attention_sink_b200 import workloads as wl

TOL = 1e-12


def f64(x):
    return x.to(torch.float64)


def _expand_kv(x, G):
    # [L, Hkv, D] -> [Hq, L, D] with query head h reading kv head h // G
    return x.permute(1, 0, 2).repeat_interleave(G, dim=0)


def band_mask(L, W):
    i = torch.arange(L)[:, None]
    j = torch.arange(L)[None, :]
    m = j <= i
    if W > 0:
        m &= j >= i - W + 1
    return m


def torch_sink_attention(q, k, v, W, sink, scale):
    """Augmented-logit reference for one sequence: softmax over the visible
    keys plus one virtual key (logit s_h, value 0), then drop the sink column.
    q [L,Hq,D], k/v [L,Hkv,D] float64; sink [Hq] float64 or None."""
    L, Hq, D = q.shape
    G = Hq // k.shape[1]
    qh = q.permute(1, 0, 2)
    kh, vh = _expand_kv(k, G), _expand_kv(v, G)
    logits = scale * qh @ kh.transpose(1, 2)                   # [Hq, L, L]
    logits = logits.masked_fill(~band_mask(L, W), float("-inf"))
    s = (torch.full((Hq,), float("-inf"), dtype=torch.float64) if sink is None
         else sink)
    aug = torch.cat([logits, s[:, None, None].expand(Hq, L, 1)], dim=2)
    w = torch.softmax(aug, dim=2)
    o = w[:, :, :L] @ vh                                        # [Hq, L, D]
    lse = torch.logsumexp(aug, dim=2)                           # [Hq, L]
    return o.permute(1, 0, 2), lse, w[:, :, L]


SHAPES = [  # (seqlens, Hq, Hkv, D, W)
    ([37], 4, 1, 16, 8),
    ([64], 8, 2, 32, 16),
    ([50, 1, 23, 0, 70], 4, 2, 8, 12),
    ([200], 2, 2, 64, 128),
    ([130], 8, 1, 16, 0),
]


@pytest.mark.parametrize("seqlens,Hq,Hkv,D,W", SHAPES)
def test_no_sink_equals_sdpa(seqlens, Hq, Hkv, D, W):
    c = wl.prefill_case(seqlens, Hq, Hkv, D, W, sigma=1.0, sink=None, seed=11)
    scale = 1.0 / math.sqrt(D)
    o, lse, _ = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], Hq, Hkv,
                               D, W, sink=None, scale=scale)
    cu = c["cu_seqlens"].tolist()
    G = Hq // Hkv
    for s in range(len(seqlens)):
        a, b = cu[s], cu[s + 1]
        if a == b:
            continue
        q, k, v = f64(c["q"][a:b]), f64(c["k"][a:b]), f64(c["v"][a:b])
        ref = torch.nn.functional.scaled_dot_product_attention(
            q.permute(1, 0, 2)[None], _expand_kv(k, G)[None],
            _expand_kv(v, G)[None], attn_mask=band_mask(b - a, W), scale=scale)
        ref = ref[0].permute(1, 0, 2).numpy()
        np.testing.assert_allclose(o[a:b], ref, rtol=0, atol=TOL)
        ref_lse = torch.logsumexp(
            (scale * q.permute(1, 0, 2) @ _expand_kv(k, G).transpose(1, 2))
            .masked_fill(~band_mask(b - a, W), float("-inf")), dim=2).numpy()
        np.testing.assert_allclose(lse[:, a:b], ref_lse, rtol=0, atol=TOL)


@pytest.mark.parametrize("seqlens,Hq,Hkv,D,W", SHAPES)
@pytest.mark.parametrize("sink_kind", ["uniform2", "normal"])
def test_sink_equals_augmented_softmax(seqlens, Hq, Hkv, D, W, sink_kind):
    c = wl.prefill_case(seqlens, Hq, Hkv, D, W, sigma=1.0, sink=sink_kind, seed=5)
    scale = 1.0 / math.sqrt(D)
    o, lse, ws = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], Hq,
                                Hkv, D, W, sink=c["sink"], scale=scale,
                                want_wsink=True)
    cu = c["cu_seqlens"].tolist()
    for s in range(len(seqlens)):
        a, b = cu[s], cu[s + 1]
        if a == b:
            continue
        ro, rl, rw = torch_sink_attention(f64(c["q"][a:b]), f64(c["k"][a:b]),
                                          f64(c["v"][a:b]), W, f64(c["sink"]), scale)
        np.testing.assert_allclose(o[a:b], ro.numpy(), rtol=0, atol=TOL)
        np.testing.assert_allclose(lse[:, a:b], rl.numpy(), rtol=0, atol=TOL)
        np.testing.assert_allclose(ws[:, a:b], rw.numpy(), rtol=0, atol=TOL)


def test_full_window_equals_global():
    """W >= L is full causal attention with the sink, and equals W <= 0."""
    c = wl.prefill_case([96, 40], 4, 2, 16, 0, sigma=1.0, sink="normal", seed=3)
    args = (c["q"], c["k"], c["v"], c["cu_seqlens"], 4, 2, 16)
    o0, l0, _ = oracle.prefill(*args, 0, sink=c["sink"])
    o1, l1, _ = oracle.prefill(*args, 96, sink=c["sink"])
    o2, l2, _ = oracle.prefill(*args, 10 ** 6, sink=c["sink"])
    assert np.array_equal(o0, o1) and np.array_equal(o0, o2)
    assert np.array_equal(l0, l1) and np.array_equal(l0, l2)


def _naive_row(qr, keys, vals, s, scale):
    """Unstabilised textbook formula with the sink as an extra denominator
    term, in pure Python floats."""
    ex = [math.exp(scale * sum(a * b for a, b in zip(qr, kr))) for kr in keys]
    den = sum(ex) + (0.0 if s is None else math.exp(s))
    D = len(qr)
    o = [sum(e * vr[d] for e, vr in zip(ex, vals)) / den for d in range(D)]
    return o, math.log(den)


@pytest.mark.parametrize("L,G,Hkv,D,W,sinkval", [
    (9, 1, 1, 4, 1, 0.3), (12, 2, 1, 8, 3, -1.5), (16, 4, 1, 4, 5, 2.5),
    (11, 2, 2, 8, 0, None), (16, 1, 3, 2, 16, -3.0), (7, 3, 1, 8, 2, 0.0)])
def test_brute_force_tiny(L, G, Hkv, D, W, sinkval):
    Hq = G * Hkv
    c = wl.prefill_case([L], Hq, Hkv, D, W, sigma=0.7, sink=None, seed=L * 7 + D)
    sink = None if sinkval is None else torch.full((Hq,), sinkval) + \
        torch.arange(Hq, dtype=torch.float32) * 0.25
    o, lse, _ = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], Hq, Hkv,
                               D, W, sink=sink)
    q = c["q"].float().tolist()
    k = c["k"].float().tolist()
    v = c["v"].float().tolist()
    scale = 1.0 / math.sqrt(D)
    for i in range(L):
        for h in range(Hq):
            g = h // G
            js = [j for j in range(L) if j <= i and (W <= 0 or j >= i - W + 1)]
            assert len(js) == (i + 1 if W <= 0 else min(i + 1, W))
            s = None if sink is None else float(sink[h])
            ro, rl = _naive_row(q[i][h], [k[j][g] for j in js],
                                [v[j][g] for j in js], s, scale)
            np.testing.assert_allclose(o[i, h], ro, rtol=0, atol=TOL)
            assert abs(lse[h, i] - rl) <= TOL * max(1.0, abs(rl))


@pytest.mark.parametrize("W", [1, 4, 9, 0])
def test_one_hot_values_expose_weights(W):
    """v_j = e_j makes o_i[j] the weight of key j: every (i, j) pair is
    enumerated, invisible keys get exactly 0, and the row weights plus the
    sink weight sum to 1."""
    L, Hq, Hkv, D = 24, 2, 1, 32
    c = wl.prefill_case([L], Hq, Hkv, D, W, sigma=1.0, sink="normal", seed=9)
    v = torch.zeros((L, Hkv, D), dtype=torch.bfloat16)
    for j in range(L):
        v[j, :, j] = 1.0
    o, lse, ws = oracle.prefill(c["q"], c["k"], v, c["cu_seqlens"], Hq, Hkv, D,
                                W, sink=c["sink"], want_wsink=True)
    for i in range(L):
        for h in range(Hq):
            vis = [(j <= i and (W <= 0 or j >= i - W + 1)) for j in range(D)]
            for j in range(D):
                if vis[j]:
                    assert o[i, h, j] > 0.0
                else:
                    assert o[i, h, j] == 0.0
            assert abs(o[i, h].sum() + ws[h, i] - 1.0) <= TOL
            assert abs(math.exp(float(c["sink"][h]) - lse[h, i]) - ws[h, i]) <= TOL


@pytest.mark.parametrize("W", [1, 5, 128])
def test_zero_query_closed_form(W):
    """q = 0: every logit is 0, so lse_i = ln(n_i + e^s) and
    o_i = sum_{j in window} v_j / (n_i + e^s) with n_i = min(i+1, W)."""
    L, Hq, Hkv, D = 300, 2, 1, 8
    c = wl.prefill_case([L], Hq, Hkv, D, W, sigma=1.0, sink="uniform2", seed=2)
    q = torch.zeros_like(c["q"])
    o, lse, _ = oracle.prefill(q, c["k"], c["v"], c["cu_seqlens"], Hq, Hkv, D, W,
                               sink=c["sink"])
    v = f64(c["v"]).numpy()
    for h in range(Hq):
        es = math.exp(float(c["sink"][h]))
        for i in range(L):
            n = min(i + 1, W)
            assert abs(lse[h, i] - math.log(n + es)) <= TOL
            # the window length read back from the closed form
            assert round(math.exp(lse[h, i]) - es) == n
            ref = v[i - n + 1:i + 1, 0].sum(axis=0) / (n + es)
            np.testing.assert_allclose(o[i, h], ref, rtol=0, atol=TOL)


def test_equal_keys_closed_form():
    """All keys equal to c: each row's logits are equal to a = scale q_i.c,
    so o_i = e^a sum v_j / (n e^a + e^s) and lse_i = ln(n e^a + e^s)."""
    L, Hq, Hkv, D, W = 40, 4, 2, 16, 7
    c = wl.prefill_case([L], Hq, Hkv, D, W, sigma=0.5, sink="normal", seed=4)
    k = c["k"][:1].expand(L, Hkv, D).contiguous()
    o, lse, _ = oracle.prefill(c["q"], k, c["v"], c["cu_seqlens"], Hq, Hkv, D, W,
                               sink=c["sink"])
    q, kk, v = f64(c["q"]).numpy(), f64(k).numpy(), f64(c["v"]).numpy()
    scale = 1.0 / math.sqrt(D)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        es = math.exp(float(c["sink"][h]))
        for i in range(L):
            n = min(i + 1, W)
            a = scale * float(q[i, h] @ kk[0, g])
            den = n * math.exp(a) + es
            assert abs(lse[h, i] - math.log(den)) <= TOL
            ref = math.exp(a) * v[i - n + 1:i + 1, g].sum(axis=0) / den
            np.testing.assert_allclose(o[i, h], ref, rtol=0, atol=TOL)


def test_extreme_sinks():
    L, Hq, Hkv, D, W = 50, 2, 1, 16, 8
    c = wl.prefill_case([L], Hq, Hkv, D, W, sigma=1.0, sink=None, seed=6)
    args = (c["q"], c["k"], c["v"], c["cu_seqlens"], Hq, Hkv, D, W)
    # a huge sink takes all the weight: o -> 0, lse -> s
    o, lse, ws = oracle.prefill(*args, sink=torch.full((Hq,), 1000.0),
                                want_wsink=True)
    assert np.abs(o).max() < 1e-300
    assert np.all(lse == 1000.0) and np.all(ws == 1.0)
    # a very negative sink is the textbook softmax
    o1, l1, _ = oracle.prefill(*args, sink=torch.full((Hq,), -1e4))
    o0, l0, _ = oracle.prefill(*args, sink=None)
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(l1, l0, rtol=0, atol=1e-15)


def test_window_one_closed_form():
    """W = 1: each row sees itself only: o_i = v_i e^a/(e^a + e^s)."""
    L, Hq, Hkv, D = 20, 2, 2, 8
    c = wl.prefill_case([L], Hq, Hkv, D, 1, sigma=1.0, sink="normal", seed=8)
    o, lse, _ = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], Hq, Hkv,
                               D, 1, sink=c["sink"])
    q, k, v = f64(c["q"]).numpy(), f64(c["k"]).numpy(), f64(c["v"]).numpy()
    for i in range(L):
        for h in range(Hq):
            a = float(q[i, h] @ k[i, h]) / math.sqrt(D)
            s = float(c["sink"][h])
            w = 1.0 / (1.0 + math.exp(s - a))
            np.testing.assert_allclose(o[i, h], w * v[i, h], rtol=0, atol=TOL)
            assert abs(lse[h, i] - (a + math.log1p(math.exp(s - a)))) <= 1e-11


def test_varlen_sequences_are_independent():
    seqlens = [33, 0, 70, 1, 45]
    Hq, Hkv, D, W = 4, 2, 16, 16
    c = wl.prefill_case(seqlens, Hq, Hkv, D, W, sigma=1.0, sink="normal", seed=12)
    o, lse, _ = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], Hq, Hkv,
                               D, W, sink=c["sink"])
    cu = c["cu_seqlens"].tolist()
    for s in range(len(seqlens)):
        a, b = cu[s], cu[s + 1]
        if a == b:
            continue
        one = torch.tensor([0, b - a], dtype=torch.int32)
        os_, ls_, _ = oracle.prefill(c["q"][a:b], c["k"][a:b], c["v"][a:b], one,
                                     Hq, Hkv, D, W, sink=c["sink"])
        assert np.array_equal(o[a:b], os_) and np.array_equal(lse[:, a:b], ls_)


def test_rows_variant_matches_full():
    c = wl.prefill_case([90, 60], 8, 2, 32, 24, sigma=1.0, sink="normal", seed=13)
    args = (c["q"], c["k"], c["v"], c["cu_seqlens"], 8, 2, 32, 24)
    o, lse, _ = oracle.prefill(*args, sink=c["sink"])
    rng = np.random.default_rng(0)
    rt = rng.integers(0, 150, 40)
    rh = rng.integers(0, 8, 40)
    orow, lrow, _ = oracle.prefill_rows(*args, rt, rh, sink=c["sink"])
    for u in range(40):
        assert np.array_equal(orow[u], o[rt[u], rh[u]])
        assert lrow[u] == lse[rh[u], rt[u]]


def rebuild_sequences(d):
    """For each decode sequence, the contiguous token sequence ring (in
    position order) + new tokens, as a packed prefill batch. Returns
    (q, k, v, cu_seqlens, index of each decode query row in the batch)."""
    B, n_q, W = d["B"], d["n_q"], d["W"]
    qs, ks, vs, lens, rows = [], [], [], [], []
    off = 0
    for b in range(B):
        P = int(d["pos"][b])
        first = max(0, P - W)
        slots = [p % W for p in range(first, P)]
        kr = d["k_ring"][b, slots]
        vr = d["v_ring"][b, slots]
        nr = len(slots)
        k = torch.cat([kr, d["k_new"][b]], 0)
        v = torch.cat([vr, d["v_new"][b]], 0)
        q = torch.cat([torch.zeros((nr,) + tuple(d["q"].shape[2:]),
                                   dtype=torch.bfloat16), d["q"][b]], 0)
        qs.append(q); ks.append(k); vs.append(v)
        lens.append(nr + n_q)
        rows.append(list(range(off + nr, off + nr + n_q)))
        off += nr + n_q
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    return torch.cat(qs), torch.cat(ks), torch.cat(vs), cu, rows


@pytest.mark.parametrize("n_q", [1, 2, 4])
def test_decode_equals_prefill_bitwise(n_q):
    """Decode over the ring is prefill over the rebuilt sequence (same key
    order, same arithmetic), so the two agree bit for bit."""
    Hq, Hkv, D, W = 4, 2, 16, 16
    d = wl.decode_case(6, n_q, Hq, Hkv, D, W, sigma=1.0, sink="normal", seed=21,
                       pos_lo=0, pos_hi=40)
    d["pos"][0] = 0          # empty ring
    d["pos"][1] = 3          # partly filled ring
    d["pos"][2] = W          # exactly full
    o, lse, _ = oracle.decode(d["q"], d["k_new"], d["v_new"], d["k_ring"],
                              d["v_ring"], d["pos"], d["B"], n_q, Hq, Hkv, D, W,
                              sink=d["sink"])
    q, k, v, cu, rows = rebuild_sequences(d)
    po, pl, _ = oracle.prefill(q, k, v, cu, Hq, Hkv, D, W, sink=d["sink"])
    for b in range(d["B"]):
        for t in range(n_q):
            r = rows[b][t]
            assert np.array_equal(o[b, t], po[r])
            assert np.array_equal(lse[b, t], pl[:, r])


def test_ring_rotation_invariance():
    Hq, Hkv, D, W, n_q = 4, 1, 8, 12, 3
    d = wl.decode_case(3, n_q, Hq, Hkv, D, W, sigma=1.0, sink="normal", seed=22,
                       pos_lo=W, pos_hi=500)
    o, lse, _ = oracle.decode(d["q"], d["k_new"], d["v_new"], d["k_ring"],
                              d["v_ring"], d["pos"], 3, n_q, Hq, Hkv, D, W,
                              sink=d["sink"])
    for r in (1, 5, W - 1, W):
        kr = torch.roll(d["k_ring"], shifts=r, dims=1)
        vr = torch.roll(d["v_ring"], shifts=r, dims=1)
        o2, l2, _ = oracle.decode(d["q"], d["k_new"], d["v_new"], kr, vr,
                                  d["pos"] + r, 3, n_q, Hq, Hkv, D, W,
                                  sink=d["sink"])
        assert np.array_equal(o, o2) and np.array_equal(lse, l2)


def test_commit_then_decode_equals_prefill():
    """Commit n accepted drafts, advance pos, decode the next token: equal
    to prefill over the whole history."""
    Hq, Hkv, D, W, n_q, B = 2, 1, 8, 10, 4, 4
    g = torch.Generator().manual_seed(3)
    hist_len = [3, 25, 9, 40]
    hist = [torch.randn((L, 2, Hkv, D), generator=g).to(torch.bfloat16)
            for L in hist_len]                               # [L, (k,v), Hkv, D]
    k_ring = torch.zeros((B, W, Hkv, D), dtype=torch.bfloat16)
    v_ring = torch.zeros((B, W, Hkv, D), dtype=torch.bfloat16)
    for b, L in enumerate(hist_len):
        for p in range(max(0, L - W), L):
            k_ring[b, p % W] = hist[b][p, 0]
            v_ring[b, p % W] = hist[b][p, 1]
    pos = torch.tensor(hist_len, dtype=torch.int32)
    new = torch.randn((B, n_q, 2, Hkv, D), generator=g).to(torch.bfloat16)
    n_acc = torch.tensor([0, 1, 3, 4], dtype=torch.int32)
    kr, vr = oracle.kv_commit(k_ring, v_ring, new[:, :, 0], new[:, :, 1], pos,
                              n_acc, B, n_q, Hkv, D, W)
    # n_accept = 0 leaves that ring untouched
    assert np.array_equal(kr[0], k_ring[0].view(torch.int16).numpy().view(np.uint16))
    kr_t = torch.from_numpy(kr.view(np.int16)).view(torch.bfloat16)
    vr_t = torch.from_numpy(vr.view(np.int16)).view(torch.bfloat16)
    pos2 = pos + n_acc
    nxt = torch.randn((B, 1, 2, Hkv, D), generator=g).to(torch.bfloat16)
    qn = torch.randn((B, 1, Hq, D), generator=g).to(torch.bfloat16)
    sink = torch.randn((Hq,), generator=g)
    o, lse, _ = oracle.decode(qn, nxt[:, :, 0], nxt[:, :, 1], kr_t, vr_t, pos2, B,
                              1, Hq, Hkv, D, W, sink=sink)
    for b in range(B):
        a = int(n_acc[b])
        ks = torch.cat([hist[b][:, 0], new[b, :a, 0], nxt[b, :, 0]], 0)
        vs = torch.cat([hist[b][:, 1], new[b, :a, 1], nxt[b, :, 1]], 0)
        L = ks.shape[0]
        qs = torch.zeros((L, Hq, D), dtype=torch.bfloat16)
        qs[-1] = qn[b, 0]
        po, pl, _ = oracle.prefill(qs, ks, vs, torch.tensor([0, L], dtype=torch.int32),
                                   Hq, Hkv, D, W, sink=sink)
        assert np.array_equal(o[b, 0], po[-1])
        assert np.array_equal(lse[b, 0], pl[:, -1])


def test_oracle_rejects_bad_arguments():
    c = wl.prefill_case([8], 4, 2, 8, 4, sink=None)
    with pytest.raises(ValueError):
        oracle.prefill(c["q"], c["k"], c["v"], torch.tensor([0, 9, 8], dtype=torch.int32),
                       4, 2, 8, 4)
    with pytest.raises(ValueError):
        oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], 4, 3, 8, 4)
