"""GPU parity of swa_sink_attn_decode_splitkv (split-KV decode over a long
cache: the global-attention layers) against the fp64 oracle: caches of a
global layer (W >= the context), a ring that has wrapped (pos > W), D = 64,
n_q = 8, caches whose unwritten slots hold NaN, agreement with
swa_sink_attn_decode on rings both support, the device flag when max_ctx
understates a position, and the bench's global-layer decode at full size on
every row. Also the NaN-slot case for swa_sink_attn_decode."""
import numpy as np
import pytest
import torch

import oracle
from sliding_window_attention_sink_b200 import binding as B
from sliding_window_attention_sink_b200 import workloads as wl

from _parity import check, to_cuda

pytestmark = pytest.mark.gpu


def oracle_decode(d):
    return oracle.decode(d["q"], d["k_new"], d["v_new"], d["k_ring"], d["v_ring"], d["pos"],
                         d["B"], d["n_q"], d["Hq"], d["Hkv"], d["D"], d["W"], sink=d["sink"])


def run_split(d, max_ctx):
    g = to_cuda(d)
    o = torch.full_like(g["q"], float("nan"))
    o, lse = B.attn_decode_splitkv(g["q"], g["k_new"], g["v_new"], g["k_ring"], g["v_ring"],
                                   g["pos"], max_ctx, sink=g["sink"], out=o)
    torch.cuda.synchronize()
    return o, lse


def poison_unwritten(d):
    """Slots holding no committed token (positions < 0 or >= pos) get NaN."""
    W, pos = d["W"], d["pos"]
    kr, vr = d["k_ring"].clone(), d["v_ring"].clone()
    for b in range(d["B"]):
        P = int(pos[b])
        if P < W:  # slots P .. W-1 were never written
            kr[b, P:] = float("nan")
            vr[b, P:] = float("nan")
    d = dict(d)
    d["k_ring"], d["v_ring"] = kr, vr
    return d


CASES = [  # (B, n_q, Hq, Hkv, D, W, pos_lo, pos_hi, sink)
    (3, 4, 64, 8, 128, 4096, 0, 4000, "normal"),     # global layer, short to long contexts
    (2, 1, 16, 2, 128, 8192, 5000, 8000, "normal"),  # one token, many ranges
    (2, 4, 16, 2, 128, 1024, 1500, 6000, "normal"),  # a ring that has wrapped: SWA, W = 1024
    (3, 3, 16, 2, 64, 2048, 10, 2000, "uniform2"),   # D = 64
    (2, 8, 16, 4, 128, 1024, 100, 1000, "normal"),   # 8 new tokens, G = 4
    (2, 2, 8, 1, 128, 64, 64, 500, None),            # smallest W, no sink
]


@pytest.mark.parametrize("Bn,n_q,Hq,Hkv,D,W,lo,hi,sink", CASES)
def test_splitkv_matches_oracle(Bn, n_q, Hq, Hkv, D, W, lo, hi, sink):
    d = wl.decode_case(Bn, n_q, Hq, Hkv, D, W, sigma=0.5, sink=sink, seed=13, pos_lo=lo,
                       pos_hi=hi)
    if W >= hi + n_q:  # a global cache: the slots past pos hold nothing yet
        d = poison_unwritten(d)
    o, lse = run_split(d, max_ctx=hi)
    assert B.swa_sink_device_error() == 0
    ro, rl, _ = oracle_decode(d)
    check(o, lse, ro, rl, "splitkv B=%d n_q=%d W=%d D=%d" % (Bn, n_q, W, D))


def test_splitkv_equals_ring_decode():
    # W = 128: both calls define the same result; both are checked against the oracle
    d = wl.decode_case(16, 4, 64, 8, 128, 128, sigma=0.5, sink="normal", seed=14)
    g = to_cuda(d)
    o1, l1 = B.attn_decode(g["q"], g["k_new"], g["v_new"], g["k_ring"], g["v_ring"], g["pos"],
                           sink=g["sink"])
    o2, l2 = run_split(d, max_ctx=262144)
    assert B.swa_sink_device_error() == 0
    ro, rl, _ = oracle_decode(d)
    check(o1, l1, ro, rl, "ring decode")
    check(o2, l2, ro, rl, "split-KV decode")


def test_ring_decode_ignores_unwritten_slots():
    # fewer committed tokens than ring slots; the never-written slots hold NaN
    d = wl.decode_case(8, 4, 64, 8, 128, 128, sigma=0.5, sink="normal", seed=15, pos_lo=0,
                       pos_hi=120)
    d = poison_unwritten(d)
    g = to_cuda(d)
    o, lse = B.attn_decode(g["q"], g["k_new"], g["v_new"], g["k_ring"], g["v_ring"], g["pos"],
                           sink=g["sink"])
    torch.cuda.synchronize()
    assert B.swa_sink_device_error() == 0
    ro, rl, _ = oracle_decode(d)
    check(o, lse, ro, rl, "ring decode, NaN in unwritten slots")


def test_splitkv_full_workload_all_rows():
    """The bench's global-layer decode (16 sequences, contexts 8K to 16K over a
    16384-slot cache, 4 new tokens, Hq = 64, Hkv = 8) in its launch
    configuration (max_ctx = the largest context it draws), every row; then
    the same call with the never-written slots holding NaN, which no range may
    read."""
    case = wl.WORKLOADS["ga_decode_16k"]
    d = wl.make_decode(case)
    ro, rl, _ = oracle_decode(d)
    o, lse = run_split(d, max_ctx=case.pos_hi)
    assert B.swa_sink_device_error() == 0
    check(o, lse, ro, rl, "ga_decode_16k")
    o, lse = run_split(poison_unwritten(d), max_ctx=case.pos_hi)
    assert B.swa_sink_device_error() == 0
    check(o, lse, ro, rl, "ga_decode_16k, NaN in unwritten slots")


def test_splitkv_flags_pos_beyond_max_ctx():
    d = wl.decode_case(2, 2, 16, 2, 128, 4096, sigma=0.5, sink="normal", seed=16, pos_lo=3000,
                       pos_hi=3500)
    run_split(d, max_ctx=1000)  # understated: the split covers too few positions
    assert B.swa_sink_device_error() & 2
