"""GPU parity of swa_sink_attn_fwd_rope (through the C ABI) against the oracle
(oracle/rope.py: fp64 rotation, bf16 rounding, then the fp64 attention), on the
same seeded inputs: the fused ring kernel (G = 8, 4, 2; D = 128 and 64) and
the workspace path (global layers, wide windows, G = 1), both pairings,
sequence start positions (pos0) up to the 2^24 limit, ragged and empty
sequences; the ring it writes (rotated K equal to the oracle's bf16 values but
for rare elements next to a rounding boundary, V bit exact, other slots
untouched); and the full SWA layer on sampled rows."""
import numpy as np
import pytest
import torch

from oracle import rope
from sliding_window_attention_sink_b200 import binding as B
from sliding_window_attention_sink_b200 import workloads as wl

from _parity import check, to_cuda

pytestmark = pytest.mark.gpu

POISON = 0x7FC1  # a NaN bit pattern: ring slots the call must not touch


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def run(c, base, pos0=None, interleaved=False, ring_W=0, window=None):
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
                             max_seqlen=c["max_seqlen"])
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


def check_rotated(got_bits, ref_bits, norm):
    """A rotated element is the oracle's correctly rounded bf16 value except
    where fp32 arithmetic (angle error a few 1e-8 rad, products and sums a few
    float ulps, all relative to the pair's norm) lands on the other side of a
    rounding boundary: then it is within one bf16 ulp of the value plus
    2e-6 of the pair's norm. Such elements are rare."""
    g, r = rope.bits_to_f64(got_bits), rope.bits_to_f64(ref_bits)
    bound = np.abs(r) * 2.0 ** -7 + 2e-6 * norm
    assert np.all(np.abs(g - r) <= bound), np.abs(g - r).max()
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
]


@pytest.mark.parametrize("name,seqlens,Hq,Hkv,D,W,pos0,inter,ring_W", CASES,
                         ids=[c[0] for c in CASES])
def test_rope_prefill_matches_oracle(name, seqlens, Hq, Hkv, D, W, pos0, inter, ring_W):
    base = 1e4 if W > 0 else 640000.0
    c = wl.prefill_case(seqlens, Hq, Hkv, D, W, sigma=0.5, sink="normal", seed=13)
    need = B.swa_sink_attn_fwd_rope_workspace(c["total"], Hq, Hkv, D, W)
    assert (need == 0) == name.startswith("ring"), need
    o, lse, kr, vr = run(c, base, pos0=pos0, interleaved=inter, ring_W=ring_W)
    ro, rl, _, k_rot = rope.prefill_rope(c["q"], c["k"], c["v"], c["cu_seqlens"], Hq, Hkv, D,
                                         W, base, pos0=pos0, sink=c["sink"],
                                         interleaved=inter)
    check(o, lse, ro, rl, name)
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


def test_rope_full_swa_layer_sampled():
    """The benchmark's SWA layer (T=32768) with RoPE (base 1e4) and ring
    emission, in the launch configuration the benchmark times; sampled rows
    (whole query groups) vs the oracle, every row written."""
    c = wl.make_prefill(wl.WORKLOADS["swa_prefill_32k_rope"])
    assert c["rope_base"] == 1e4 and c["ring_W"] == 128
    o, lse, kr, vr = run(c, 1e4, ring_W=128)
    rng = np.random.default_rng(2)
    toks = np.unique(np.concatenate([rng.integers(0, c["total"], 160), [0, 1, 127, 128,
                                                                       c["total"] - 1]]))
    G = c["Hq"] // c["Hkv"]
    heads = rng.integers(0, c["Hkv"], len(toks)) * G
    rt = np.repeat(toks, G)
    rh = (np.repeat(heads, G) + np.tile(np.arange(G), len(toks))).astype(np.int32)
    ro, rl = rope.prefill_rope_rows(c["q"], c["k"], c["v"], c["cu_seqlens"], c["Hq"], c["Hkv"],
                                    c["D"], c["window"], 1e4, rt, rh, sink=c["sink"])
    ti = torch.from_numpy(rt).cuda()
    hi = torch.from_numpy(rh.astype(np.int64)).cuda()
    check(o[ti, hi], lse[hi, ti], ro, rl, "swa_prefill_32k rope")
    assert torch.isfinite(o).all().item() and torch.isfinite(lse).all().item()
    # the ring holds the last 128 tokens
    T = c["total"]
    pos = np.arange(T - 128, T)
    k_ref = rope.rope_bf16(c["k"][T - 128:], pos, 1e4)
    kg = bits(kr)[0][pos % 128]
    assert np.array_equal(bits(vr)[0][pos % 128], bits(c["v"][T - 128:]))
    check_rotated(kg, k_ref, pair_norm(bits(c["k"][T - 128:]), False))


def test_rope_full_global_layer_sampled():
    """The benchmark's global layer (T=8192, full causal) with RoPE (base
    640000) through the workspace path, writing a position-indexed cache of
    8192 slots; sampled rows vs the oracle, the cache holds every token."""
    c = wl.make_prefill(wl.WORKLOADS["global_prefill_8k_rope"])
    base, W = c["rope_base"], c["ring_W"]
    assert B.swa_sink_attn_fwd_rope_workspace(c["total"], 64, 8, 128, 0) > 0
    o, lse, kr, vr = run(c, base, ring_W=W)
    rng = np.random.default_rng(3)
    toks = np.unique(np.concatenate([rng.integers(0, c["total"], 48), [0, 1, c["total"] - 1]]))
    G = c["Hq"] // c["Hkv"]
    heads = rng.integers(0, c["Hkv"], len(toks)) * G
    rt = np.repeat(toks, G)
    rh = (np.repeat(heads, G) + np.tile(np.arange(G), len(toks))).astype(np.int32)
    ro, rl = rope.prefill_rope_rows(c["q"], c["k"], c["v"], c["cu_seqlens"], c["Hq"], c["Hkv"],
                                    c["D"], 0, base, rt, rh, sink=c["sink"])
    ti = torch.from_numpy(rt).cuda()
    hi = torch.from_numpy(rh.astype(np.int64)).cuda()
    check(o[ti, hi], lse[hi, ti], ro, rl, "global_prefill_8k rope")
    assert torch.isfinite(o).all().item() and torch.isfinite(lse).all().item()
    T = c["total"]
    k_ref = rope.rope_bf16(c["k"], np.arange(T), base)
    assert np.array_equal(bits(vr)[0], bits(c["v"]))
    check_rotated(bits(kr)[0], k_ref, pair_norm(bits(c["k"]), False))
