"""GPU parity of swa_sink_attn_decode and swa_sink_kv_commit (through the C
ABI) against the fp64 oracle: n_q = 1..4 (plain decode and draft
verification), rings that are empty / partly filled / full, G = 4 and 8,
D = 64 and 128, no sink, the full decode workload (every row), decode vs the
prefill kernel on rebuilt sequences, and commit bit-exactness."""
import numpy as np
import pytest
import torch

import oracle
from sliding_window_attention_sink_b200 import binding as B
from sliding_window_attention_sink_b200 import workloads as wl

from _parity import check, to_cuda

pytestmark = pytest.mark.gpu


def run_decode(d, sink="case"):
    g = to_cuda(d)
    s = g["sink"] if sink == "case" else sink
    o = torch.full_like(g["q"], float("nan"))
    o, lse = B.attn_decode(g["q"], g["k_new"], g["v_new"], g["k_ring"], g["v_ring"],
                           g["pos"], sink=s, out=o)
    torch.cuda.synchronize()
    assert B.swa_sink_device_error() == 0
    return o, lse


def oracle_decode(d, sink="case"):
    s = d["sink"] if sink == "case" else sink
    return oracle.decode(d["q"], d["k_new"], d["v_new"], d["k_ring"], d["v_ring"], d["pos"],
                         d["B"], d["n_q"], d["Hq"], d["Hkv"], d["D"], d["W"], sink=s)


CASES = [  # (B, n_q, Hq, Hkv, D, W, sink)
    (16, 1, 64, 8, 128, 128, "normal"),
    (16, 2, 64, 8, 128, 128, "normal"),
    (16, 3, 64, 8, 128, 128, "normal"),
    (16, 4, 64, 8, 128, 128, "normal"),
    (8, 4, 16, 4, 64, 128, "uniform2"),
    (8, 4, 32, 8, 128, 128, None),
    (8, 2, 8, 1, 128, 64, "normal"),
    (8, 3, 16, 2, 64, 40, "normal"),
    # the largest rings
    (6, 2, 16, 2, 128, 256, "normal"),
    (6, 4, 32, 8, 128, 200, "uniform2"),
    # rings that are not a multiple of 8 rows (new rows start at roundup8(W)),
    # a one-slot ring, and 8 new tokens
    (8, 4, 64, 8, 128, 127, "normal"),
    (8, 3, 16, 2, 64, 13, "uniform2"),
    (8, 1, 8, 1, 128, 1, "normal"),
    (8, 8, 16, 4, 128, 100, "normal"),
    # either side of the tcgen05 kernel's limit of 144 padded keys: a ring of
    # 136 slots and 8 new tokens fills it exactly (no padding rows); 137 slots
    # take the mma.sync kernel (160 padded keys)
    (6, 8, 16, 4, 128, 136, "normal"),
    (6, 8, 16, 4, 128, 137, "uniform2"),
    # more units than SMs with few rows per unit
    (400, 1, 8, 8, 64, 128, "normal"),
]


@pytest.mark.parametrize("Bn,n_q,Hq,Hkv,D,W,sink", CASES)
def test_decode_matches_oracle(Bn, n_q, Hq, Hkv, D, W, sink):
    d = wl.decode_case(Bn, n_q, Hq, Hkv, D, W, sigma=0.5, sink=sink, seed=Bn + n_q,
                       pos_lo=0, pos_hi=3 * W)
    d["pos"][0] = 0
    d["pos"][1] = 1
    d["pos"][2] = W - 1
    d["pos"][3] = W
    o, lse = run_decode(d)
    ro, rl, _ = oracle_decode(d)
    check(o, lse, ro, rl, "decode")


def test_decode_full_workload_all_rows():
    d = wl.make_decode(wl.WORKLOADS["swa_decode_mtp"])
    o, lse = run_decode(d)
    ro, rl, _ = oracle_decode(d)
    check(o, lse, ro, rl, "swa_decode_mtp")


def test_decode_equals_prefill_kernel():
    """The decode kernel and the prefill kernel agree on the same tokens: each
    ring (in position order) plus the new tokens rebuilt as a sequence."""
    d = wl.decode_case(6, 4, 64, 8, 128, 128, sigma=0.5, sink="normal", seed=31,
                       pos_lo=0, pos_hi=600)
    d["pos"][0] = 2
    o_dec, l_dec = run_decode(d)
    from test_oracle import rebuild_sequences
    q, k, v, cu, rows = rebuild_sequences(d)
    o_pre, l_pre = B.attn_fwd(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), 128,
                              sink=d["sink"].cuda())
    torch.cuda.synchronize()
    for b in range(d["B"]):
        for t in range(d["n_q"]):
            r = rows[b][t]
            diff = (o_dec[b, t].float() - o_pre[r].float()).abs().max().item()
            assert diff <= 1e-2, (b, t, diff)
            assert (l_dec[b, t] - l_pre[:, r]).abs().max().item() <= 1e-3


def test_kv_commit_bitexact_and_followup_decode():
    Bn, n_q, Hq, Hkv, D, W = 8, 4, 64, 8, 128, 128
    d = wl.decode_case(Bn, n_q, Hq, Hkv, D, W, sigma=0.5, sink="normal", seed=41,
                       pos_lo=0, pos_hi=1000)
    n_acc = torch.tensor([0, 1, 2, 3, 4, 4, 1, 0], dtype=torch.int32)
    g = to_cuda(d)
    kr, vr = g["k_ring"].clone(), g["v_ring"].clone()
    B.kv_commit(kr, vr, g["k_new"], g["v_new"], g["pos"], n_acc.cuda())
    torch.cuda.synchronize()
    assert B.swa_sink_device_error() == 0
    ek, ev = oracle.kv_commit(d["k_ring"], d["v_ring"], d["k_new"], d["v_new"], d["pos"],
                              n_acc, Bn, n_q, Hkv, D, W)
    assert np.array_equal(kr.cpu().view(torch.int16).numpy().view(np.uint16), ek)
    assert np.array_equal(vr.cpu().view(torch.int16).numpy().view(np.uint16), ev)


def test_kv_commit_flags_bad_n_accept():
    Bn, n_q, Hkv, D, W = 2, 2, 2, 64, 16
    d = wl.decode_case(Bn, n_q, 4, Hkv, D, W, seed=3, pos_lo=0, pos_hi=50)
    g = to_cuda(d)
    B.kv_commit(g["k_ring"], g["v_ring"], g["k_new"], g["v_new"], g["pos"],
                torch.tensor([5, 1], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert B.swa_sink_device_error() == 2
    assert B.swa_sink_device_error() == 0


def test_decode_flags_negative_position():
    """A negative position is read as 0 (only the new tokens are visible) and
    flagged; the other sequences are unaffected."""
    d = wl.decode_case(4, 2, 16, 2, 128, 128, sigma=0.5, sink="normal", seed=17, pos_lo=0,
                       pos_hi=300)
    d["pos"][1] = -3
    g = to_cuda(d)
    o = torch.full_like(g["q"], float("nan"))
    o, lse = B.attn_decode(g["q"], g["k_new"], g["v_new"], g["k_ring"], g["v_ring"], g["pos"],
                           sink=g["sink"], out=o)
    torch.cuda.synchronize()
    assert B.swa_sink_device_error() == 2
    assert B.swa_sink_device_error() == 0
    d["pos"][1] = 0
    ro, rl, _ = oracle_decode(d)
    check(o, lse, ro, rl, "negative position read as 0")
