"""GPU parity of swa_sink_attn_fwd_rope (through the C ABI) against the oracle
(oracle/rope.py: fp64 rotation, bf16 rounding, then the fp64 attention), on the
same seeded inputs: the fused ring kernel (G = 8, 4, 2; D = 128 and 64) and
the workspace path (global layers, wide windows, G = 1), both pairings,
sequence start positions (pos0) up to the 2^24 limit, ragged and empty
sequences; the ring it writes (rotated K equal to the oracle's bf16 values but
for rare elements next to a rounding boundary, V bit exact, other slots
untouched); and the full SWA and global layers on every row."""
import numpy as np
import pytest
import torch

from oracle import rope
from sliding_window_attention_sink_b200 import binding as B
from sliding_window_attention_sink_b200 import workloads as wl

from _parity import check, check_every_row, to_cuda

pytestmark = pytest.mark.gpu

POISON = 0x7FC1  # a NaN bit pattern: ring slots the call must not touch


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def run(c, base, pos0=None, interleaved=False, ring_W=0, window=None, fused=False):
    d = to_cuda(c)
    w = c["window"] if window is None else window
    S = len(c["seqlens"])
    p0 = None if pos0 is None else torch.tensor(pos0, dtype=torch.int32).cuda()
    kr = vr = None
    if ring_W:
        kr = torch.full((S, ring_W, c["Hkv"], c["D"]), POISON, dtype=torch.int16).view(
            torch.bfloat16).cuda()
        vr = kr.clone()
    o = torch.full_like(d["q"], float("nan"))
    o, lse = B.attn_fwd_rope(d["q"], d["k"], d["v"], d["cu_seqlens"], w, base, sink=d["sink"],
                             pos0=p0, interleaved=interleaved, k_ring=kr, v_ring=vr, out=o,
                             max_seqlen=c["max_seqlen"], fused=fused)
    torch.cuda.synchronize()
    assert B.swa_sink_device_error() == 0
    return o, lse, kr, vr


def check_ring(c, kr_gpu, vr_gpu, k_rot_ref, W, pos0, interleaved):
    ring0 = np.full((len(c["seqlens"]), W, c["Hkv"], c["D"]), POISON, np.uint16)
    kr_ref, vr_ref = rope.emit_ring(k_rot_ref, c["v"], c["cu_seqlens"], ring0, ring0, W,
                                    pos0=pos0)
    # the unrotated keys in ring order, for the error bound
    k_in = rope.emit_ring(c["k"].view(torch.int16).numpy().view(np.uint16), c["v"],
                          c["cu_seqlens"], ring0, ring0, W, pos0=pos0)[0]
    kg, vg = bits(kr_gpu), bits(vr_gpu)
    assert np.array_equal(vg, vr_ref)
    # untouched slots keep the poison
    written = kr_ref != POISON
    assert np.array_equal(kg == POISON, ~written)
    check_rotated(kg[written], kr_ref[written], pair_norm(k_in, interleaved)[written])


def pair_norm(k_bits, interleaved):
    """|(x_a, x_b)| of the pair each element belongs to (rotation keeps it)."""
    x = rope.bits_to_f64(k_bits)
    a, b = rope.rope_pairs(x.shape[-1], interleaved)
    n = np.sqrt(x[..., a] ** 2 + x[..., b] ** 2)
    out = np.empty_like(x)
    out[..., a] = n
    out[..., b] = n
    return out


# Error of the kernel's fp32 rotation before its bf16 rounding, as a fraction
# of the pair's norm N (positions below 2^24):
#   angle: theta/(2 pi) as hi + lo floats (off by <= 2^-48 of itself, times
#   p < 2^24: 2^-24 rad); fma(p, lo, te) rounded (|value| <= 2^-23 p hi <=
#   0.32 turn: <= 2^-26 turn); t = fr + that rounded (|t| < 1: <= 2^-25
#   turn); in all dphi <= 2^-24 + 2 pi (2^-26 + 2^-25) < 3.4e-7 rad. To first
#   order an angle error moves output a by dphi * |r_b| <= dphi * N.
#   sincospif: <= 1 ulp each (CUDA's documented bound), so |x dc| + |y ds|
#   <= 2^-23 (|x c| + |y s|) <= 2^-23 N (Cauchy-Schwarz).
#   the product y s rounded (2^-24 N) and the FMA's one rounding (2^-24 N).
# e32 <= (3.4e-7 + 2^-23 + 2^-23) N < 5.8e-7 N.
# Then both sides round to bf16 (unit roundoff 2^-8): the kernel's fp32 value
# r' (|r' - r| <= e32) and the oracle's exact r. So
#   |bf16(r') - bf16(r)| <= 2^-8 |r'| + e32 + 2^-8 |r|
#                        <= 2^-7 (1 + 2^-7) |bf16(r)| + (1 + 2^-8) e32,
# using |r| <= |bf16(r)| / (1 - 2^-8). With |r| above about 2^8 e32 the two
# roundings are equal or neighbours (one bf16 ulp, which the first term
# covers); below it (cancellation next to zero) the e32 term takes over.
ROT_REL = 2.0 ** -7 * (1.0 + 2.0 ** -7)
ROT_NORM = 5.9e-7


def check_rotated(got_bits, ref_bits, norm):
    """A rotated element is the oracle's correctly rounded bf16 value except
    where the kernel's fp32 error lands it on the other side of a rounding
    boundary; the bound above covers that, and such elements are rare."""
    g, r = rope.bits_to_f64(got_bits), rope.bits_to_f64(ref_bits)
    bound = np.abs(r) * ROT_REL + ROT_NORM * norm
    assert np.all(np.abs(g - r) <= bound), (np.abs(g - r) - bound).max()
    assert (got_bits != ref_bits).mean() < 1e-3, (got_bits != ref_bits).mean()


CASES = [  # (name, seqlens, Hq, Hkv, D, W, pos0, interleaved, ring_W)
    ("ring_g8", [300], 64, 8, 128, 128, None, False, 128),
    ("ring_g8_varlen", [100, 0, 257, 1, 33], 16, 2, 128, 128, [5, 0, 262000, 9, 0], False, 128),
    ("ring_g8_interleaved", [400], 16, 2, 128, 128, [1000], True, 128),
    ("ring_g4", [333], 8, 2, 128, 128, [77], False, 64),
    ("ring_g2_d64", [290, 40], 4, 2, 64, 128, [3, 16776000], False, 128),
    ("ring_small_window", [200], 16, 2, 128, 20, [1], True, 32),
    ("global_ws", [700], 16, 2, 128, 0, [0], False, 1024),
    ("global_ws_varlen", [129, 300, 5], 8, 1, 64, 0, [10, 0, 500], True, 512),
    ("wide_window_ws", [600], 8, 1, 64, 300, None, False, 300),
    ("g1_ws", [300], 2, 2, 64, 128, [12345], False, 128),
    ("g3_ws", [300], 12, 4, 128, 128, [17], True, 128),
]


@pytest.mark.parametrize("name,seqlens,Hq,Hkv,D,W,pos0,inter,ring_W", CASES,
                         ids=[c[0] for c in CASES])
def test_rope_prefill_matches_oracle(name, seqlens, Hq, Hkv, D, W, pos0, inter, ring_W):
    """Both routes: with the workspace (rotation pass, plain prefill) and, for
    the ring kernel's shapes, without (rotation in its shared memory)."""
    base = 1e4 if W > 0 else 640000.0
    c = wl.prefill_case(seqlens, Hq, Hkv, D, W, sigma=0.5, sink="normal", seed=13)
    assert B.swa_sink_attn_fwd_rope_workspace(c["total"], Hq, Hkv, D, W) > 0
    ro, rl, _, k_rot = rope.prefill_rope(c["q"], c["k"], c["v"], c["cu_seqlens"], Hq, Hkv, D,
                                         W, base, pos0=pos0, sink=c["sink"],
                                         interleaved=inter)
    for fused in ((False, True) if name.startswith("ring") else (False,)):
        o, lse, kr, vr = run(c, base, pos0=pos0, interleaved=inter, ring_W=ring_W, fused=fused)
        check(o, lse, ro, rl, "%s fused=%s" % (name, fused))
        check_ring(c, kr, vr, k_rot, ring_W, pos0, inter)


def test_rope_equals_plain_prefill_on_rotated_inputs():
    """Fused rotation = rotate (oracle, bf16) then the plain prefill kernel,
    within the parity tolerance (rare 1-ulp rotations differ)."""
    c = wl.prefill_case([1000, 24], 64, 8, 128, 128, sigma=0.5, sink="normal", seed=14)
    o, lse, _, _ = run(c, 1e4, pos0=[40000, 7])
    pos = rope.token_positions(c["cu_seqlens"], [40000, 7])
    qr = torch.from_numpy(rope.rope_bf16(c["q"], pos, 1e4).view(np.int16)).view(torch.bfloat16)
    kr = torch.from_numpy(rope.rope_bf16(c["k"], pos, 1e4).view(np.int16)).view(torch.bfloat16)
    d = to_cuda(c)
    o2, l2 = B.attn_fwd(qr.cuda(), kr.cuda(), d["v"], d["cu_seqlens"], 128, sink=d["sink"])
    torch.cuda.synchronize()
    err = (o.float() - o2.float()).abs()
    assert err.max().item() <= 1e-2 and err.mean().item() <= 1e-4
    assert (lse - l2).abs().max().item() <= 1e-3


def test_rope_ring_then_decode_matches_longer_prefill():
    """The ring written by the prefill feeds swa_sink_attn_decode for the next
    tokens (rotated at their positions): equal to the oracle's prefill over
    the longer sequences."""
    Hq, Hkv, D, W, n_q = 64, 8, 128, 128, 4
    lens = [300, 128, 50]
    full = wl.prefill_case([L + n_q for L in lens], Hq, Hkv, D, W, sigma=0.5, sink="normal",
                           seed=15)
    cu_f = full["cu_seqlens"].numpy()
    pre = np.concatenate([np.arange(cu_f[s], cu_f[s] + lens[s]) for s in range(3)])
    new = np.concatenate([np.arange(cu_f[s] + lens[s], cu_f[s + 1]) for s in range(3)])
    pc = dict(full)
    pc.update(q=full["q"][pre], k=full["k"][pre], v=full["v"][pre], seqlens=lens,
              cu_seqlens=torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32),
              total=sum(lens), max_seqlen=max(lens))
    _, _, kr, vr = run(pc, 1e4, ring_W=W)
    # rings of sequences shorter than W hold poison beyond their tokens: the
    # decode must not read them (positions < 0 are invisible)
    P = torch.tensor(lens, dtype=torch.int32)
    new_pos = (P[:, None] + torch.arange(n_q)[None, :]).reshape(-1).numpy()
    qn = torch.from_numpy(rope.rope_bf16(full["q"][new], new_pos, 1e4).view(np.int16)).view(
        torch.bfloat16).reshape(3, n_q, Hq, D)
    kn = torch.from_numpy(rope.rope_bf16(full["k"][new], new_pos, 1e4).view(np.int16)).view(
        torch.bfloat16).reshape(3, n_q, Hkv, D)
    vn = full["v"][new].reshape(3, n_q, Hkv, D)
    od, ld = B.attn_decode(qn.cuda(), kn.cuda(), vn.cuda(), kr, vr, P.cuda(),
                           sink=full["sink"].cuda())
    torch.cuda.synchronize()
    ro, rl, _, _ = rope.prefill_rope(full["q"], full["k"], full["v"], full["cu_seqlens"], Hq,
                                     Hkv, D, W, 1e4, sink=full["sink"])
    rows = np.array([cu_f[s] + lens[s] + t for s in range(3) for t in range(n_q)])
    check(od.reshape(-1, Hq, D), ld.reshape(-1, Hq).T, ro[rows], rl[:, rows], "ring->decode")


def rotated_bits(x, pos, base, chunk=2048):
    """The oracle's rotated bf16 bits of a whole [total, H, D] tensor, rotated
    a chunk of tokens at a time (fp64 temporaries stay small)."""
    out = np.empty(tuple(x.shape), np.uint16)
    for t0 in range(0, x.shape[0], chunk):
        t1 = min(x.shape[0], t0 + chunk)
        out[t0:t1] = rope.rope_bf16(x[t0:t1], pos[t0:t1], base)
    return out


@pytest.mark.parametrize("fused", [False, True], ids=["two_pass", "fused"])
def test_rope_full_swa_layer_every_row(fused):
    """The benchmark's SWA layer (T=32768) with RoPE (base 1e4) and ring
    emission, on both routes (the benchmark's is the two-pass one, with the
    workspace); every row vs the oracle (rotated at bf16, then attended in
    fp64)."""
    c = wl.make_prefill(wl.WORKLOADS["swa_prefill_32k_rope"])
    assert c["rope_base"] == 1e4 and c["ring_W"] == 128
    o, lse, kr, vr = run(c, 1e4, ring_W=128, fused=fused)
    T = c["total"]
    pos = np.arange(T)
    q_rot, k_rot = rotated_bits(c["q"], pos, 1e4), rotated_bits(c["k"], pos, 1e4)
    check_every_row(o, lse, q_rot, k_rot, c["v"], c["cu_seqlens"], c["Hq"], c["Hkv"], c["D"],
                    c["window"], c["sink"], "swa_prefill_32k rope fused=%s" % fused)
    # the ring holds the last 128 tokens
    tail = np.arange(T - 128, T)
    kg = bits(kr)[0][tail % 128]
    assert np.array_equal(bits(vr)[0][tail % 128], bits(c["v"][T - 128:]))
    check_rotated(kg, k_rot[T - 128:], pair_norm(bits(c["k"][T - 128:]), False))


def test_rope_full_global_layer_every_row():
    """The benchmark's global layer (T=8192, full causal) with RoPE (base
    640000) through the workspace path, writing a position-indexed cache of
    8192 slots; every row vs the oracle, the cache holds every token."""
    c = wl.make_prefill(wl.WORKLOADS["global_prefill_8k_rope"])
    base, W = c["rope_base"], c["ring_W"]
    assert B.swa_sink_attn_fwd_rope_workspace(c["total"], 64, 8, 128, 0) > 0
    o, lse, kr, vr = run(c, base, ring_W=W)
    T = c["total"]
    pos = np.arange(T)
    q_rot, k_rot = rotated_bits(c["q"], pos, base), rotated_bits(c["k"], pos, base)
    check_every_row(o, lse, q_rot, k_rot, c["v"], c["cu_seqlens"], c["Hq"], c["Hkv"], c["D"],
                    0, c["sink"], "global_prefill_8k rope")
    assert np.array_equal(bits(vr)[0], bits(c["v"]))
    check_rotated(bits(kr)[0], k_rot, pair_norm(bits(c["k"]), False))
