"""Rotary position embedding (RoPE) applied before the attention, and the
prefill that also writes the decode ring, in plain numpy (fp64).

TEST INFRASTRUCTURE: see the package docstring.

Sources. The MiMo-V2-Flash report summary (mlpod.com), section 3.1 "Data
Scheduler", gives the RoPE base of each layer type: 10,000 for the SWA layers
and 640,000 for the global layers in the first stage, the global base raised to
5,000,000 for the 256K extension. The ICML talk write-up (hzrcw.cc), in its
Q&A on position encoding, says the SWA base stays fixed through training and
that the position index keeps increasing as the window slides (no reset).
No page prints the rotation itself. The reading taken here is the standard
rotary embedding over the whole head dimension:

    theta_c = base ** (-2c / D)                       c = 0 .. D/2 - 1
    (x_a, x_b) -> (x_a cos(p theta_c) - x_b sin(p theta_c),
                   x_b cos(p theta_c) + x_a sin(p theta_c))

at absolute position p, where the pair (a, b) is (c, c + D/2) ("rotate
half", the default) or (2c, 2c + 1) (``interleaved``). Positions of a packed
sequence s are pos0[s] + i for its i-th token (pos0 = 0 when not given).

The rotated q and k are rounded to bf16 (round to nearest even) before the
attention: they are bf16 activations in the unfused pipeline (rotate, store,
attend), and the decode ring stores the rotated K in bf16. The attention is
then the C oracle's prefill on those bf16 values, so the fused call must equal
"rotate -> bf16 -> attend" of the same inputs.

Ring emission: after the prefill of sequence s (positions pos0[s] ..
pos0[s] + L - 1), slot p mod W of its ring holds the rotated K and the V of
position p for the last min(L, W) positions; the other slots keep their
contents. With W >= pos0[s] + L the ring is a plain position-indexed cache
(the global layers' convention).
"""
import numpy as np

from . import oracle as _core


def rope_freqs(D: int, base: float) -> np.ndarray:
    """theta_c = base ** (-2c / D), c = 0 .. D/2 - 1, float64."""
    c = np.arange(D // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * c / D)


def rope_pairs(D: int, interleaved: bool):
    """Indices (a, b) of the rotated pairs."""
    c = np.arange(D // 2)
    if interleaved:
        return 2 * c, 2 * c + 1
    return c, c + D // 2


def rope_rotate(x, positions, base: float, interleaved: bool = False) -> np.ndarray:
    """x: float array [n, H, D] (token-major); positions: int [n]. Returns the
    rotated float64 array (no rounding)."""
    x = np.asarray(x, dtype=np.float64)
    n, _, D = x.shape
    ang = np.asarray(positions, dtype=np.float64)[:, None] * rope_freqs(D, base)[None, :]
    cs, sn = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]  # [n, 1, D/2]
    a, b = rope_pairs(D, interleaved)
    out = np.empty_like(x)
    out[..., a] = x[..., a] * cs - x[..., b] * sn
    out[..., b] = x[..., b] * cs + x[..., a] * sn
    return out


def bf16_round_bits(x) -> np.ndarray:
    """float64 -> bf16 bit patterns (uint16), round to nearest even, directly
    from the double (no intermediate float32 rounding); finite inputs only,
    magnitudes at or above the bf16 overflow threshold become +-inf."""
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("bf16_round_bits: finite inputs only")
    ax = np.abs(x)
    # quantum of the bf16 grid at |x|: 2^(e - 7) for |x| in [2^e, 2^(e+1)),
    # 2^-133 below the smallest normal 2^-126
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    # log2 may be off by one next to a power of two: settle e exactly
    e = np.where(np.ldexp(1.0, e.astype(np.int64)) > ax, e - 1, e)
    e = np.where(np.ldexp(1.0, (e + 1).astype(np.int64)) <= ax, e + 1, e)
    e = np.maximum(e, -126.0)
    qexp = (e - 7).astype(np.int64)
    r = np.ldexp(np.rint(np.ldexp(ax, -qexp)), qexp)  # rint: ties to even
    r = np.where(ax == 0, 0.0, r)
    r = np.where(r >= 2.0 ** 128, np.inf, r)
    r = np.copysign(r, x)
    return (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def bits_to_f64(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def token_positions(cu_seqlens, pos0=None) -> np.ndarray:
    """Absolute position of every packed token: pos0[s] + i."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    S = len(cu) - 1
    p0 = np.zeros(S, np.int64) if pos0 is None else np.asarray(pos0, np.int64)
    out = np.empty(int(cu[-1]), np.int64)
    for s in range(S):
        out[cu[s]:cu[s + 1]] = p0[s] + np.arange(cu[s + 1] - cu[s])
    return out


def _f64_of(x):
    """bf16 tensor or uint16 bit array -> float64 numpy."""
    return bits_to_f64(_core._bits(x))


def rope_bf16(x, positions, base: float, interleaved: bool = False) -> np.ndarray:
    """bf16 input -> rotated, rounded bf16 bit patterns [n, H, D]."""
    return bf16_round_bits(rope_rotate(_f64_of(x), positions, base, interleaved))


def prefill_rope(q, k, v, cu_seqlens, Hq, Hkv, D, window, base, pos0=None,
                 sink=None, scale=None, interleaved=False, nthreads=None):
    """Rotate q and k at their absolute positions, round to bf16, attend.
    Returns (o [total,Hq,D], lse [Hq,total], q_rot bits, k_rot bits)."""
    pos = token_positions(cu_seqlens, pos0)
    qr = rope_bf16(q, pos, base, interleaved)
    kr = rope_bf16(k, pos, base, interleaved)
    o, lse, _ = _core.prefill(qr, kr, v, cu_seqlens, Hq, Hkv, D, window, sink=sink,
                              scale=scale, nthreads=nthreads)
    return o, lse, qr, kr


def prefill_rope_rows(q, k, v, cu_seqlens, Hq, Hkv, D, window, base, row_tok, row_head,
                      pos0=None, sink=None, scale=None, interleaved=False, nthreads=None):
    """prefill_rope on a sample of (token, head) rows: (o [n,D], lse [n]).
    Only the sampled tokens' query rows are rotated (no other query row is
    read); every key row is."""
    pos = token_positions(cu_seqlens, pos0)
    qb = _core._bits(q).copy()
    toks = np.unique(np.asarray(row_tok, dtype=np.int64))
    qb[toks] = rope_bf16(qb[toks], pos[toks], base, interleaved)
    kr = rope_bf16(k, pos, base, interleaved)
    o, lse, _ = _core.prefill_rows(qb, kr, v, cu_seqlens, Hq, Hkv, D, window, row_tok,
                                   row_head, sink=sink, scale=scale, nthreads=nthreads)
    return o, lse


def emit_ring(k_rot_bits, v, cu_seqlens, k_ring, v_ring, W, pos0=None):
    """The ring after the prefill: returns new (k_ring, v_ring) uint16 arrays
    [num_seqs, W, Hkv, D]; the inputs are untouched."""
    kr = _core._bits(k_ring).copy()
    vr = _core._bits(v_ring).copy()
    kb = np.asarray(k_rot_bits, dtype=np.uint16)
    vb = _core._bits(v)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    pos = token_positions(cu_seqlens, pos0)
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        for t in range(max(lo, hi - W), hi):
            slot = int(pos[t]) % W
            kr[s, slot] = kb[t]
            vr[s, slot] = vb[t]
    return kr, vr
