"""Gradients of the sliding-window / global attention with a per-head sink:
the backward pass, in plain numpy (fp64).

TEST INFRASTRUCTURE: see the package docstring.

Source. The pages give the forward only (MiMo-V2-Flash report summary,
mlpod.com, section 2.2.2: the sink joins the softmax denominator and the max;
the ICML talk write-up, hzrcw.cc, Q&A: the sink must be trained with care at
scale, its initialisation and gradient updates keep the architecture from
collapsing). The gradients below are the calculus of that forward (the
reading of the oracle's prefill: a_ij = scale q_i.k_j over the visible keys,
p_ij = exp(a_ij - lse_i), p_sink,i = exp(s_h - lse_i), o_i = sum_j p_ij v_j,
the sink has no value). For a loss L with dL/do_i = dO_i:

    Delta_i  = dO_i . o_i
    dV_j    += sum_i p_ij dO_i
    dA_ij    = p_ij (dO_i . v_j - Delta_i)          (softmax with the sink)
    dQ_i     = scale sum_j dA_ij k_j
    dK_j    += scale sum_i dA_ij q_i
    dsink_h  = - sum_i p_sink,i Delta_i              (over the rows of head h)

(d/ds of o_i is -p_sink,i o_i: the sink takes weight from every key and gives
back no value.) K and V gradients of a kv head sum over its G query heads.
Everything is recomputed in fp64 from q, k, v: the gradient of the exact
function at the given inputs, not of a rounded forward.
"""
import numpy as np

from . import oracle as _core
from .rope import bits_to_f64


def _f64(x):
    return bits_to_f64(_core._bits(x))


def prefill_backward(q, k, v, dout, cu_seqlens, Hq, Hkv, D, window, sink=None, scale=None):
    """q [total,Hq,D], k/v [total,Hkv,D] bf16; dout [total,Hq,D] (bf16 or
    float). Returns (dq [total,Hq,D], dk [total,Hkv,D], dv [total,Hkv,D],
    dsink [Hq]) in fp64 (dsink is zero without a sink)."""
    Q, K, V = _f64(q), _f64(k), _f64(v)
    dO = _f64(dout) if not (hasattr(dout, "dtype") and dout.dtype == np.float64) else dout
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    sc = (1.0 / np.sqrt(D)) if (scale is None or scale <= 0) else float(scale)
    G = Hq // Hkv
    s_all = (np.full(Hq, -np.inf) if sink is None
             else np.asarray(sink.detach().cpu().numpy() if hasattr(sink, "detach") else sink,
                             dtype=np.float64))
    dq = np.zeros_like(Q)
    dk = np.zeros_like(K)
    dv = np.zeros_like(V)
    dsink = np.zeros(Hq)
    for si in range(len(cu) - 1):
        lo, hi = int(cu[si]), int(cu[si + 1])
        L = hi - lo
        if L == 0:
            continue
        i = np.arange(L)[:, None]
        j = np.arange(L)[None, :]
        vis = j <= i
        if window > 0:
            vis &= j >= i - window + 1
        for h in range(Hq):
            g = h // G
            q_, k_, v_, do_ = Q[lo:hi, h], K[lo:hi, g], V[lo:hi, g], dO[lo:hi, h]
            s = s_all[h]
            a = np.where(vis, sc * (q_ @ k_.T), -np.inf)
            m = np.maximum(a.max(axis=1), s)
            e = np.where(vis, np.exp(a - m[:, None]), 0.0)
            es = np.exp(s - m)
            den = e.sum(axis=1) + es
            p = e / den[:, None]
            psink = es / den
            o = p @ v_
            delta = (do_ * o).sum(axis=1)
            dv[lo:hi, g] += p.T @ do_
            da = p * (do_ @ v_.T - delta[:, None])
            dq[lo:hi, h] = sc * (da @ k_)
            dk[lo:hi, g] += sc * (da.T @ q_)
            dsink[h] += -(psink * delta).sum()
    return dq, dk, dv, dsink


def prefill_backward_rows(q, k, v, dout, cu_seqlens, Hq, Hkv, D, window, row_tok, row_head,
                          key_tok, key_head, sink=None, scale=None, nthreads=None, forward=None):
    """The same gradients at sampled places only, for layers too large to do
    whole: dq at the (token, head) rows row_tok/row_head and dk, dv at the
    (token, kv head) keys key_tok/key_head. A row needs the keys it sees; a
    key needs the rows that see it (W tokens x G heads for a sliding window,
    the rest of the sequence for a global layer), with their o and lse: from
    `forward` = (o [total,Hq,D], lse [Hq,total]), the C oracle's prefill of
    the whole layer, when it is given, else from the C oracle's prefill on
    those rows. Returns (dq [n,D], dk [m,D], dv [m,D])."""
    Q, K, V = _f64(q), _f64(k), _f64(v)
    dO = _f64(dout)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    sc = (1.0 / np.sqrt(D)) if (scale is None or scale <= 0) else float(scale)
    G = Hq // Hkv
    total = int(cu[-1])
    seq_of = np.searchsorted(cu, np.arange(total), side="right") - 1

    def first_key(t):
        lo = int(cu[seq_of[t]])
        return lo if window <= 0 else max(lo, t - window + 1)

    def last_row(j):  # the last token that sees key j
        hi = int(cu[seq_of[j] + 1])
        return hi - 1 if window <= 0 else min(hi - 1, j + window - 1)

    # every (token, head) row whose o and lse are needed
    need = set((int(t), int(h)) for t, h in zip(row_tok, row_head))
    for j, g in zip(key_tok, key_head):
        for t in range(int(j), last_row(int(j)) + 1):
            for h in range(int(g) * G, (int(g) + 1) * G):
                need.add((t, h))
    need = sorted(need)
    rt = np.array([t for t, _ in need], np.int64)
    rh = np.array([h for _, h in need], np.int32)
    if forward is None:
        o, lse, _ = _core.prefill_rows(q, k, v, cu_seqlens, Hq, Hkv, D, window, rt, rh,
                                       sink=sink, scale=scale, nthreads=nthreads)
    else:
        o, lse = forward[0][rt, rh], forward[1][rh, rt]
    where = {key: n for n, key in enumerate(need)}
    delta = np.einsum("nd,nd->n", dO[rt, rh], o)

    dq = np.zeros((len(row_tok), D))
    for n, (t, h) in enumerate(zip(row_tok, row_head)):
        t, h = int(t), int(h)
        g = h // G
        ks = np.arange(first_key(t), t + 1)
        r = where[(t, h)]
        p = np.exp(sc * (K[ks, g] @ Q[t, h]) - lse[r])
        da = p * (V[ks, g] @ dO[t, h] - delta[r])
        dq[n] = sc * (da @ K[ks, g])
    dk = np.zeros((len(key_tok), D))
    dv = np.zeros((len(key_tok), D))
    for n, (j, g) in enumerate(zip(key_tok, key_head)):
        j, g = int(j), int(g)
        rows = [(t, h) for t in range(j, last_row(j) + 1) for h in range(g * G, (g + 1) * G)]
        idx = np.array([where[x] for x in rows])
        ts = np.array([t for t, _ in rows])
        hs = np.array([h for _, h in rows])
        qr, dr = Q[ts, hs], dO[ts, hs]
        p = np.exp(sc * (qr @ K[j, g]) - lse[idx])
        dv[n] = p @ dr
        dk[n] = sc * ((p * (dr @ V[j, g] - delta[idx])) @ qr)
    return dq, dk, dv


def dsink_from_forward(o, lse, dout, sink):
    """dsink_h = -sum_i exp(s_h - lse_hi) (dO_hi . o_hi) from a forward's o
    [total,Hq,D] and lse [Hq,total] (fp64)."""
    dO = _f64(dout)
    s = np.asarray(sink.detach().cpu().numpy() if hasattr(sink, "detach") else sink, np.float64)
    delta = np.einsum("thd,thd->ht", dO, o)
    return -(np.exp(s[:, None] - lse) * delta).sum(axis=1)


def key_sums_from_forward(q, o, lse, dout, cu_seqlens, Hq, Hkv, sink=None, scale=None):
    """The sums of dK and dV over the keys of each sequence and kv head,
    from a forward's o [total,Hq,D] and lse [Hq,total] (fp64) alone.

    Summed over the keys row i sees, dA_ij gives
        sum_j p_ij (dO_i . v_j) - Delta_i sum_j p_ij = Delta_i - Delta_i (1 - p_sink,i)
                                                     = Delta_i p_sink,i,
    because sum_j p_ij v_j = o_i and the visible weights add up to 1 - p_sink,i.
    Every key of a sequence is seen only by rows of that sequence, so over the
    keys of sequence b and kv head g:
        sum_j dK_j = scale sum_{h in g} sum_{i in b} Delta_ih p_sink,ih q_ih
        sum_j dV_j = sum_{h in g} sum_{i in b} (1 - p_sink,ih) dO_ih.
    Without a sink p_sink = 0: the dK sum is zero and the dV sum is that of dO.
    Returns (sum_dk, sum_dv), each [num_seqs, Hkv, D]."""
    Q = _f64(q)
    dO = _f64(dout) if not (hasattr(dout, "dtype") and dout.dtype == np.float64) else dout
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    total, _, D = Q.shape
    sc = (1.0 / np.sqrt(D)) if (scale is None or scale <= 0) else float(scale)
    G = Hq // Hkv
    if sink is None:
        ps = np.zeros((total, Hq))
    else:
        s = np.asarray(sink.detach().cpu().numpy() if hasattr(sink, "detach") else sink,
                       np.float64)
        ps = np.exp(s[None, :] - lse.T)                      # p_sink [total, Hq]
    delta = np.einsum("thd,thd->th", dO, o)
    wk = (sc * delta * ps)[:, :, None] * Q                   # [total, Hq, D]
    wv = (1.0 - ps)[:, :, None] * dO
    n = len(cu) - 1
    sum_dk = np.zeros((n, Hkv, D))
    sum_dv = np.zeros((n, Hkv, D))
    for b in range(n):
        lo, hi = int(cu[b]), int(cu[b + 1])
        sum_dk[b] = wk[lo:hi].sum(axis=0).reshape(Hkv, G, D).sum(axis=1)
        sum_dv[b] = wv[lo:hi].sum(axis=0).reshape(Hkv, G, D).sum(axis=1)
    return sum_dk, sum_dv
