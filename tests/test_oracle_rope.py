"""Pins for the RoPE part of the oracle (oracle/rope.py), independent of its
code:

* bf16 rounding straight from the double: equal to torch's float32 -> bf16
  cast wherever the value is a float32 (one rounding either way), ties to
  even, subnormals, overflow, and the case where rounding through float32
  first would give a different answer;
* the rotation equals multiplying each pair, read as a complex number, by
  exp(i p theta_c) (the complex form of the rotary embedding), with theta_c
  computed through exp/log rather than a power;
* closed forms: position 0 is the identity, theta_0 = 1 for every base,
  theta_{D/4} = base^(-1/2), a quarter turn moves a unit vector onto its
  partner;
* invariants: every pair keeps its norm; q.k after rotating both depends only
  on the difference of their positions; attention over rotated inputs does
  not change when every position moves by the same amount (fp64, no rounding);
* the ring the prefill writes, read back by the decode oracle for the tokens
  that follow, gives bit for bit the prefill over the longer sequence.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import rope
from sliding_window_attention_sink_b200 import workloads as wl


def torch_bf16_bits(x32):
    t = torch.from_numpy(np.ascontiguousarray(x32, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_bf16_round_matches_torch_on_float32_values():
    g = np.random.default_rng(5)
    xs = np.concatenate([g.standard_normal(50000) * s for s in (1e-3, 0.3, 1.0, 1e4)])
    x32 = xs.astype(np.float32)
    # every tie between two bf16 neighbours, and subnormals
    u = g.integers(0, 1 << 31, 20000, dtype=np.uint64).astype(np.uint32)
    ties = ((u & 0xFFFF0000) | 0x8000).view(np.float32)
    sub = (g.integers(1, 1 << 23, 5000).astype(np.uint32)).view(np.float32)
    x32 = np.concatenate([x32, ties[np.isfinite(ties)], sub, -sub])
    got = rope.bf16_round_bits(x32.astype(np.float64))
    assert np.array_equal(got, torch_bf16_bits(x32))


def test_bf16_round_closed_forms():
    f = lambda v: int(rope.bf16_round_bits(np.array([v]))[0])  # noqa: E731
    assert f(1.0) == 0x3F80 and f(-2.0) == 0xC000 and f(0.0) == 0x0000
    assert f(1.0 + 2.0 ** -8) == 0x3F80            # tie -> even (1.0)
    assert f(1.0 + 3 * 2.0 ** -8) == 0x3F82        # tie -> even (1 + 2^-6)
    # just above a tie: rounds up. Rounding to float32 first would land on the
    # tie and then go down to 1.0.
    assert f(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81
    assert f(2.0 ** -133) == 0x0001                # smallest subnormal
    assert f(2.0 ** -134) == 0x0000                # half of it: tie -> even (0)
    assert f(3.3895313892515355e38) == 0x7F7F      # largest finite
    assert f(3.4e38) == 0x7F80                     # beyond: +inf
    assert np.array_equal(rope.bits_to_f64(np.array([0x3F81], np.uint16)), [1.0078125])


@pytest.mark.parametrize("interleaved", [False, True])
@pytest.mark.parametrize("D,base", [(8, 10000.0), (64, 640000.0), (128, 5e6), (128, 1e4)])
def test_rotation_is_complex_multiplication(D, base, interleaved):
    g = np.random.default_rng(D)
    n, H = 37, 3
    x = g.standard_normal((n, H, D))
    pos = g.integers(0, 300000, n)
    got = rope.rope_rotate(x, pos, base, interleaved)
    half = D // 2
    theta = np.exp(-(2.0 * np.arange(half) / D) * math.log(base))
    if interleaved:
        z = x[..., 0::2] + 1j * x[..., 1::2]
    else:
        z = x[..., :half] + 1j * x[..., half:]
    zr = z * np.exp(1j * pos[:, None, None] * theta[None, None, :])
    want = np.empty_like(x)
    if interleaved:
        want[..., 0::2], want[..., 1::2] = zr.real, zr.imag
    else:
        want[..., :half], want[..., half:] = zr.real, zr.imag
    # angles reach 3e5 rad; both sides reduce them in double
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-9)


def test_rotation_closed_forms():
    D = 8
    x = np.random.default_rng(1).standard_normal((5, 2, D))
    assert np.array_equal(rope.rope_rotate(x, np.zeros(5, np.int64), 1e4), x)
    for base in (10.0, 1e4, 6.4e5, 5e6):
        th = rope.rope_freqs(D, base)
        assert th[0] == 1.0
        assert abs(th[D // 4] - base ** -0.5) <= 1e-15 * base ** -0.5
    # theta_0 = 1: position p turns pair 0 by p radians
    e0 = np.zeros((1, 1, D))
    e0[0, 0, 0] = 1.0
    r = rope.rope_rotate(e0, np.array([3]), 1e4)
    np.testing.assert_allclose(r[0, 0], [math.cos(3), 0, 0, 0, math.sin(3), 0, 0, 0], atol=1e-15)
    # theta_2 = 1e4^(-1/2) = 0.01 for D = 8: position 50*pi is a quarter turn,
    # unit vector e_2 -> e_6 (rotate half) and e_4 -> e_5 (interleaved)
    p = np.array([50 * math.pi])
    e2 = np.zeros((1, 1, D))
    e2[0, 0, 2] = 1.0
    np.testing.assert_allclose(rope.rope_rotate(e2, p, 1e4)[0, 0], np.eye(D)[6], atol=1e-12)
    e4 = np.zeros((1, 1, D))
    e4[0, 0, 4] = 1.0
    np.testing.assert_allclose(rope.rope_rotate(e4, p, 1e4, True)[0, 0], np.eye(D)[5], atol=1e-12)


@pytest.mark.parametrize("interleaved", [False, True])
def test_rotation_invariants(interleaved):
    D = 64
    g = np.random.default_rng(2)
    q = g.standard_normal((50, 1, D))
    k = g.standard_normal((50, 1, D))
    p = g.integers(0, 200000, 50)
    p2 = g.integers(0, 200000, 50)
    a, b = rope.rope_pairs(D, interleaved)
    qr = rope.rope_rotate(q, p, 1e4, interleaved)
    np.testing.assert_allclose(qr[..., a] ** 2 + qr[..., b] ** 2, q[..., a] ** 2 + q[..., b] ** 2,
                               rtol=1e-12)
    kr = rope.rope_rotate(k, p2, 1e4, interleaved)
    dot = np.sum(qr * kr, axis=-1)
    for delta in (1, 77, 4096):
        qs = rope.rope_rotate(q, p + delta, 1e4, interleaved)
        ks = rope.rope_rotate(k, p2 + delta, 1e4, interleaved)
        np.testing.assert_allclose(np.sum(qs * ks, axis=-1), dot, rtol=0, atol=1e-9)
    # same position on both sides: the dot product is unchanged
    kq = rope.rope_rotate(k, p, 1e4, interleaved)
    np.testing.assert_allclose(np.sum(qr * kq, axis=-1), np.sum(q * k, axis=-1), atol=1e-11)


def _attend_f64(q, k, v, W, sink, scale):
    """Brute-force sink attention of one sequence in fp64: explicit key lists,
    unstabilised exponentials (small inputs)."""
    L, Hq, D = q.shape
    G = Hq // k.shape[1]
    o = np.zeros((L, Hq, D))
    for i in range(L):
        js = [j for j in range(i + 1) if W <= 0 or j >= i - W + 1]
        for h in range(Hq):
            e = np.array([math.exp(scale * float(q[i, h] @ k[j, h // G])) for j in js])
            den = e.sum() + math.exp(sink[h])
            o[i, h] = (e[:, None] * v[js, h // G]).sum(0) / den
    return o


def test_attention_is_shift_invariant_in_fp64():
    L, Hq, Hkv, D, W = 24, 4, 2, 16, 7
    c = wl.prefill_case([L], Hq, Hkv, D, W, sigma=0.7, sink="normal", seed=9)
    q, k, v = (c[n].to(torch.float64).numpy() for n in ("q", "k", "v"))
    sink = c["sink"].double().numpy()
    pos = np.arange(L)
    ref = _attend_f64(rope.rope_rotate(q, pos, 1e4), rope.rope_rotate(k, pos, 1e4), v, W,
                      sink, D ** -0.5)
    for p0 in (1, 1000, 262000):
        got = _attend_f64(rope.rope_rotate(q, pos + p0, 1e4),
                          rope.rope_rotate(k, pos + p0, 1e4), v, W, sink, D ** -0.5)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-9)
    # and it is not the identity: rotated attention differs from plain
    plain = _attend_f64(q, k, v, W, sink, D ** -0.5)
    assert np.abs(plain - ref).max() > 1e-3


def test_positions_of_packed_sequences():
    cu = np.array([0, 3, 3, 7])
    assert rope.token_positions(cu).tolist() == [0, 1, 2, 0, 1, 2, 3]
    assert rope.token_positions(cu, [10, 5, 100]).tolist() == [10, 11, 12, 100, 101, 102, 103]


@pytest.mark.parametrize("interleaved", [False, True])
def test_emitted_ring_then_decode_equals_longer_prefill(interleaved):
    """Prefill (with RoPE) writes the ring; the decode oracle over that ring
    for the next n_q tokens (rotated at their positions) gives bit for bit the
    rows of a prefill over the whole, longer sequences."""
    Hq, Hkv, D, W, n_q, base = 4, 2, 16, 12, 3, 1e4
    lens = [5, 12, 30, 1]
    pos0 = [0, 0, 77, 0]
    B = len(lens)
    full = wl.prefill_case([L + n_q for L in lens], Hq, Hkv, D, W, sigma=0.8, sink="normal",
                           seed=31)
    cu_f = full["cu_seqlens"].numpy()
    # split every sequence into its first L tokens (prefill) and n_q more (decode)
    pre_idx = np.concatenate([np.arange(cu_f[s], cu_f[s] + lens[s]) for s in range(B)])
    new_idx = np.concatenate([np.arange(cu_f[s] + lens[s], cu_f[s + 1]) for s in range(B)])
    cu_p = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    q, k, v = full["q"], full["k"], full["v"]
    o_p, l_p, qr, kr = rope.prefill_rope(q[pre_idx], k[pre_idx], v[pre_idx], cu_p, Hq, Hkv, D,
                                         W, base, pos0=pos0, sink=full["sink"],
                                         interleaved=interleaved)
    ring0 = np.full((B, W, Hkv, D), 0x7FC0, np.uint16)  # NaN: never read
    k_ring, v_ring = rope.emit_ring(kr, v[pre_idx], cu_p, ring0, ring0, W, pos0=pos0)
    # slots of positions the prefill covered are written, the rest untouched
    for s in range(B):
        written = {(pos0[s] + i) % W for i in range(max(0, lens[s] - W), lens[s])}
        for slot in range(W):
            assert np.all(k_ring[s, slot] != 0x7FC0) == (slot in written)
    P = np.array([pos0[s] + lens[s] for s in range(B)], np.int32)
    new_pos = (P[:, None] + np.arange(n_q)[None, :]).reshape(-1)
    qn = rope.rope_bf16(q[new_idx], new_pos, base, interleaved).reshape(B, n_q, Hq, D)
    kn = rope.rope_bf16(k[new_idx], new_pos, base, interleaved).reshape(B, n_q, Hkv, D)
    vn = v[new_idx].reshape(B, n_q, Hkv, D)
    # sequences with pos0 > 0 start at a nonzero position but have no earlier
    # tokens: only those with lens >= W or pos0 = 0 have a complete ring
    o_d, l_d, _ = oracle.decode(qn, kn, vn, k_ring, v_ring, P, B, n_q, Hq, Hkv, D, W,
                                sink=full["sink"])
    o_f, l_f, _, _ = rope.prefill_rope(q, k, v, full["cu_seqlens"], Hq, Hkv, D, W, base,
                                       pos0=pos0, sink=full["sink"], interleaved=interleaved)
    for s in range(B):
        if pos0[s] > 0 and lens[s] < W:
            continue
        for t in range(n_q):
            r = cu_f[s] + lens[s] + t
            assert np.array_equal(o_d[s, t], o_f[r])
            assert np.array_equal(l_d[s, t], l_f[:, r])
    # the prefill part of the longer call equals the shorter call
    for s in range(B):
        rows = np.arange(cu_f[s], cu_f[s] + lens[s])
        assert np.array_equal(o_f[rows], o_p[cu_p[s].item():cu_p[s + 1].item()])


def test_global_cache_is_position_indexed():
    """W at least the context: every token lands at slot = position."""
    Hq, Hkv, D = 2, 1, 8
    c = wl.prefill_case([6, 9], Hq, Hkv, D, 0, seed=4)
    pos0 = [3, 0]
    Wc = 16
    _, _, _, kr = rope.prefill_rope(c["q"], c["k"], c["v"], c["cu_seqlens"], Hq, Hkv, D, 0, 1e4,
                                    pos0=pos0)
    ring0 = np.zeros((2, Wc, Hkv, D), np.uint16)
    k_c, v_c = rope.emit_ring(kr, c["v"], c["cu_seqlens"], ring0, ring0, Wc, pos0=pos0)
    vb = c["v"].view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(k_c[0, 3:9], kr[0:6]) and np.array_equal(v_c[1, 0:9], vb[6:15])
    assert not k_c[0, :3].any() and not k_c[0, 9:].any()


@pytest.mark.parametrize("W", [9, 0])
def test_sampled_rows_equal_whole_prefill(W):
    c = wl.prefill_case([40, 3, 25], 8, 2, 16, W, sigma=0.7, sink="normal", seed=12)
    pos0 = [17, 0, 300]
    o, lse, _, _ = rope.prefill_rope(c["q"], c["k"], c["v"], c["cu_seqlens"], 8, 2, 16, W, 1e4,
                                     pos0=pos0, sink=c["sink"], interleaved=True)
    rng = np.random.default_rng(6)
    rt = np.concatenate([rng.integers(0, 68, 30), [0, 39, 40, 42, 43, 67]])
    rh = rng.integers(0, 8, len(rt)).astype(np.int32)
    so, sl = rope.prefill_rope_rows(c["q"], c["k"], c["v"], c["cu_seqlens"], 8, 2, 16, W, 1e4,
                                    rt, rh, pos0=pos0, sink=c["sink"], interleaved=True)
    assert np.array_equal(so, o[rt, rh]) and np.array_equal(sl, lse[rh, rt])
