"""Seeded synthetic inputs shaped like the workloads the MiMo pages describe.

This module only draws random numbers and packs them; it holds none of the
attention arithmetic. Both the CUDA path and the CPU oracle are fed from here,
so they see identical bytes. Every tensor is made on the CPU with a
``torch.Generator`` seeded per case; floating inputs are drawn in fp32 and
rounded to bf16 (round to nearest even); the sink stays fp32.

Shapes (the pages give none of these; they are the workload definitions used
throughout this package):

* prefill: q [total, Hq, D], k/v [total, Hkv, D] bf16, packed varlen with
  cu_seqlens [num_seqs + 1] int32 (first entry 0), sink [Hq] fp32.
* decode: q [B, n_q, Hq, D], k_new/v_new [B, n_q, Hkv, D], ring k/v
  [B, W, Hkv, D] bf16, pos [B] int32, sink [Hq] fp32.
* decode over an FP8 ring: the ring k/v are uint8 E4M3 codes [B, W, Hkv, D]
  (drawn through torch's float8_e4m3fn cast) and kv_scale [2 * Hkv] fp32.
"""
from dataclasses import dataclass, field
from typing import List, Optional

import torch


@dataclass
class PrefillCase:
    name: str
    seqlens: List[int]
    Hq: int
    Hkv: int
    D: int
    window: int            # > 0: sliding window incl. self; <= 0: full causal
    sigma: float           # q, k, v ~ N(0, 1) * sigma
    sink: Optional[str]    # "uniform2" (U(-2,2)), "normal" (N(0,1)) or None
    seed: int
    varlen_draw: Optional[tuple] = None  # (num_seqs, lo, hi) drawn from seed
    # > 0: q and k are given before the rotary embedding with this base (token
    # i of a sequence at position i), and the call writes a ring of ring_W
    # slots per sequence
    rope_base: float = 0.0
    ring_W: int = 0
    # the backward of this layer (output gradient dout ~ N(0,1) * sigma, bf16,
    # drawn with seed + 1; o and lse from the forward)
    backward: bool = False


@dataclass
class DecodeCase:
    name: str
    B: int
    n_q: int
    Hq: int
    Hkv: int
    D: int
    W: int
    sigma: float
    sink: Optional[str]
    seed: int
    pos_lo: int = 128
    pos_hi: int = 262144   # inclusive
    # "ring": a W-slot ring (sliding-window layers); "full": a cache of W >=
    # every context (global layers, split-KV decode with max_ctx = pos_hi)
    cache: str = "ring"
    # "bf16": the ring holds bf16 K/V; "fp8": E4M3 codes with one fp32 scale
    # per kv head for K and one for V
    kv: str = "bf16"


# The workloads: a tiny parity case, one SWA layer and one global layer (each
# also with the rotary embedding applied inside the call and the decode ring /
# position-indexed cache written, and each also backward), a packed
# varlen SWA batch, a decode / draft-verification batch of the SWA layers and
# one of a global layer over long contexts.
WORKLOADS = {
    "tiny_swa_prefill": PrefillCase(
        "tiny_swa_prefill T=512 Hq=4 Hkv=1 D=64 W=128", [512], 4, 1, 64, 128,
        1.0, "uniform2", 0),
    "swa_prefill_32k": PrefillCase(
        "swa_prefill T=32768 Hq=64 Hkv=8 D=128 W=128", [32768], 64, 8, 128,
        128, 0.5, "normal", 2),
    "swa_prefill_32k_rope": PrefillCase(
        "swa_prefill_rope T=32768 Hq=64 Hkv=8 D=128 W=128 rope_base=1e4 ring=128", [32768],
        64, 8, 128, 128, 0.5, "normal", 2, rope_base=1e4, ring_W=128),
    "global_prefill_8k": PrefillCase(
        "global_prefill T=8192 Hq=64 Hkv=8 D=128 full-causal", [8192], 64, 8,
        128, 0, 0.5, "normal", 3),
    "global_prefill_8k_rope": PrefillCase(
        "global_prefill_rope T=8192 Hq=64 Hkv=8 D=128 full-causal rope_base=640000 cache=8192",
        [8192], 64, 8, 128, 0, 0.5, "normal", 3, rope_base=640000.0, ring_W=8192),
    "swa_backward_32k": PrefillCase(
        "swa_backward T=32768 Hq=64 Hkv=8 D=128 W=128", [32768], 64, 8, 128, 128, 0.5,
        "normal", 2, backward=True),
    "global_backward_8k": PrefillCase(
        "global_backward T=8192 Hq=64 Hkv=8 D=128 full-causal", [8192], 64, 8, 128, 0, 0.5,
        "normal", 3, backward=True),
    "varlen_swa_prefill": PrefillCase(
        "varlen_swa_prefill 16 seqs L~U[1024,16384] Hq=64 Hkv=8 D=128 W=128",
        [], 64, 8, 128, 128, 0.5, "normal", 4, varlen_draw=(16, 1024, 16384)),
    "swa_decode_mtp": DecodeCase(
        "swa_decode B=256 n_q=4 ring=128 Hq=64 Hkv=8 D=128", 256, 4, 64, 8,
        128, 128, 0.5, "normal", 5),
    "ga_decode_16k": DecodeCase(
        "ga_decode B=16 n_q=4 ctx~U[8192,16380] cache=16384 Hq=64 Hkv=8 D=128", 16, 4,
        64, 8, 128, 16384, 0.5, "normal", 6, pos_lo=8192, pos_hi=16380, cache="full"),
    "swa_decode_mtp_fp8": DecodeCase(
        "swa_decode_fp8 B=256 n_q=4 ring=128 e4m3 Hq=64 Hkv=8 D=128", 256, 4, 64, 8,
        128, 128, 0.5, "normal", 7, kv="fp8"),
}


def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def _sink(kind, Hq, g):
    if kind is None:
        return None
    if kind == "uniform2":
        return torch.rand((Hq,), generator=g, dtype=torch.float32) * 4.0 - 2.0
    if kind == "normal":
        return torch.randn((Hq,), generator=g, dtype=torch.float32)
    raise ValueError(kind)


def _fp8_codes(shape, g):
    """Random E4M3 codes over the format's whole range: N(0, 64^2) draws
    clamped to the largest finite magnitude, cast by torch."""
    x = (torch.randn(shape, generator=g) * 64.0).clamp_(-448.0, 448.0)
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def _fp8_scales(Hkv, sigma, g):
    """fp32 [2 * Hkv] (K scales, then V scales) around sigma / 64, so that the
    dequantized ring values have about the spread of the bf16 draws."""
    return (torch.rand((2 * Hkv,), generator=g, dtype=torch.float32) * 1.5 + 0.5) * (sigma / 64.0)


def make_prefill(case: PrefillCase):
    """Returns a dict of CPU tensors: q, k, v, cu_seqlens, sink, plus sizes."""
    g = torch.Generator().manual_seed(case.seed)
    seqlens = list(case.seqlens)
    if case.varlen_draw is not None:
        n, lo, hi = case.varlen_draw
        seqlens = torch.randint(lo, hi + 1, (n,), generator=g).tolist()
    cu = torch.zeros(len(seqlens) + 1, dtype=torch.int32)
    if seqlens:
        cu[1:] = torch.cumsum(torch.tensor(seqlens, dtype=torch.int64), 0).to(torch.int32)
    total = int(cu[-1])
    q = _bf16(torch.randn((total, case.Hq, case.D), generator=g) * case.sigma)
    k = _bf16(torch.randn((total, case.Hkv, case.D), generator=g) * case.sigma)
    v = _bf16(torch.randn((total, case.Hkv, case.D), generator=g) * case.sigma)
    sink = _sink(case.sink, case.Hq, g)
    return dict(q=q, k=k, v=v, cu_seqlens=cu, sink=sink, seqlens=seqlens,
                total=total, Hq=case.Hq, Hkv=case.Hkv, D=case.D,
                window=case.window, max_seqlen=max(seqlens) if seqlens else 0,
                rope_base=case.rope_base, ring_W=case.ring_W, backward=case.backward,
                dout=(make_dout(q.shape, case.sigma, case.seed + 1) if case.backward else None))


def make_decode(case: DecodeCase):
    """Returns a dict of CPU tensors for one decode / verification step."""
    g = torch.Generator().manual_seed(case.seed)
    pos = torch.randint(case.pos_lo, case.pos_hi + 1, (case.B,), generator=g,
                        dtype=torch.int64).to(torch.int32)
    s = case.sigma
    q = _bf16(torch.randn((case.B, case.n_q, case.Hq, case.D), generator=g) * s)
    k_new = _bf16(torch.randn((case.B, case.n_q, case.Hkv, case.D), generator=g) * s)
    v_new = _bf16(torch.randn((case.B, case.n_q, case.Hkv, case.D), generator=g) * s)
    ring_shape = (case.B, case.W, case.Hkv, case.D)
    if case.kv == "fp8":
        k_ring, v_ring = _fp8_codes(ring_shape, g), _fp8_codes(ring_shape, g)
    else:
        k_ring = _bf16(torch.randn(ring_shape, generator=g) * s)
        v_ring = _bf16(torch.randn(ring_shape, generator=g) * s)
    sink = _sink(case.sink, case.Hq, g)
    out = dict(q=q, k_new=k_new, v_new=v_new, k_ring=k_ring, v_ring=v_ring,
               pos=pos, sink=sink, B=case.B, n_q=case.n_q, Hq=case.Hq,
               Hkv=case.Hkv, D=case.D, W=case.W)
    if case.kv == "fp8":
        out["kv_scale"] = _fp8_scales(case.Hkv, s, g)
    return out


def make_dout(shape, sigma=0.5, seed=0):
    """An output gradient for the backward: N(0,1) * sigma rounded to bf16."""
    g = torch.Generator().manual_seed(seed)
    return _bf16(torch.randn(shape, generator=g) * sigma)


def prefill_case(seqlens, Hq, Hkv, D, window, sigma=0.5, sink="normal", seed=0):
    """An ad-hoc prefill case (tests use it for edge shapes)."""
    return make_prefill(PrefillCase("adhoc", list(seqlens), Hq, Hkv, D, window,
                                    sigma, sink, seed))


def decode_case(B, n_q, Hq, Hkv, D, W, sigma=0.5, sink="normal", seed=0,
                pos_lo=128, pos_hi=262144, kv="bf16"):
    return make_decode(DecodeCase("adhoc", B, n_q, Hq, Hkv, D, W, sigma, sink,
                                  seed, pos_lo, pos_hi, kv=kv))


def shard_units(num_units: int, world_size: int, rank: int):
    """Contiguous block split of independent units (sequences, decode rows)
    over ranks: rank r gets [lo, hi). Sizes differ by at most one."""
    if world_size <= 0 or not (0 <= rank < world_size):
        raise ValueError("bad rank / world size")
    base, extra = divmod(num_units, world_size)
    lo = rank * base + min(rank, extra)
    hi = lo + base + (1 if rank < extra else 0)
    return lo, hi


def slice_sequences(c, lo, hi):
    """The packed sub-batch of sequences [lo, hi) of a prefill input dict:
    contiguous token slices of q, k, v and a rebased cu_seqlens."""
    cu = c["cu_seqlens"]
    a, b = int(cu[lo]), int(cu[hi])
    sub = dict(c)
    sub["q"], sub["k"], sub["v"] = c["q"][a:b], c["k"][a:b], c["v"][a:b]
    sub["cu_seqlens"] = (cu[lo:hi + 1] - a).to(torch.int32)
    sub["seqlens"] = list(c["seqlens"][lo:hi])
    sub["total"] = b - a
    sub["max_seqlen"] = max(sub["seqlens"]) if sub["seqlens"] else 0
    sub["token_range"] = (a, b)
    return sub
