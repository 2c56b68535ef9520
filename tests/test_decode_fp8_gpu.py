"""GPU parity of the FP8 (E4M3) ring calls, swa_sink_attn_decode_fp8kv and
swa_sink_kv_commit_fp8 (through the C ABI), against the fp64 oracle over the
dequantized ring: shapes as for the bf16 ring (n_q 1..8, rings empty / partly
filled / full, odd W, D 64 and 128, no sink), every finite code in the ring,
NaN codes in never-written slots, the full FP8 decode workload (every row),
agreement with the bf16 kernel on exactly representable rings,
and bit-exact commits (saturation, ties, subnormals)."""
import numpy as np
import pytest
import torch

from oracle import fp8
from sliding_window_attention_sink_b200 import binding as B
from sliding_window_attention_sink_b200 import workloads as wl

from _parity import check, to_cuda

pytestmark = pytest.mark.gpu


def _f(x):
    return x.to(torch.float64).numpy()


def run_fp8(d, sink="case"):
    g = to_cuda(d)
    s = g["sink"] if sink == "case" else sink
    o = torch.full_like(g["q"], float("nan"))
    o, lse = B.attn_decode_fp8kv(g["q"], g["k_new"], g["v_new"], g["k_ring"], g["v_ring"],
                                 g["kv_scale"], g["pos"], sink=s, out=o)
    torch.cuda.synchronize()
    assert B.swa_sink_device_error() == 0
    return o, lse


def oracle_fp8(d, sink="case", rows=None):
    s = d["sink"] if sink == "case" else sink
    bs = slice(None) if rows is None else rows
    pos = d["pos"].numpy()[bs]
    return fp8.decode_fp8(_f(d["q"][bs]), _f(d["k_new"][bs]), _f(d["v_new"][bs]),
                          d["k_ring"].numpy()[bs], d["v_ring"].numpy()[bs],
                          d["kv_scale"].numpy(), pos, len(pos), d["n_q"], d["Hq"], d["Hkv"],
                          d["D"], d["W"], sink=None if s is None else s.numpy())


CASES = [  # (B, n_q, Hq, Hkv, D, W, sink)
    (16, 4, 64, 8, 128, 128, "normal"),
    (16, 1, 64, 8, 128, 128, "normal"),
    (8, 4, 16, 4, 64, 128, "uniform2"),
    (8, 4, 32, 8, 128, 128, None),
    (8, 3, 16, 2, 64, 40, "normal"),
    (6, 2, 16, 2, 128, 256, "normal"),     # 8 warps
    (6, 8, 32, 8, 128, 200, "uniform2"),   # 8 warps, 8 new tokens
    (6, 2, 16, 4, 64, 200, "normal"),      # 8 warps of 8 head-dim columns
    (8, 4, 64, 8, 128, 127, "normal"),     # new rows at roundup8(W)
    (8, 3, 16, 2, 64, 13, "uniform2"),
    (8, 1, 8, 1, 128, 1, "normal"),
    (300, 2, 8, 8, 64, 128, "normal"),     # more units than SMs
]


@pytest.mark.parametrize("Bn,n_q,Hq,Hkv,D,W,sink", CASES)
def test_fp8_decode_matches_oracle(Bn, n_q, Hq, Hkv, D, W, sink):
    d = wl.decode_case(Bn, n_q, Hq, Hkv, D, W, sink=sink, seed=Bn + 7 * n_q, pos_lo=0,
                       pos_hi=3 * W, kv="fp8")
    d["pos"][0] = 0
    d["pos"][1] = 1
    d["pos"][2] = W - 1
    d["pos"][3] = W
    o, lse = run_fp8(d)
    ro, rl = oracle_fp8(d)
    check(o, lse, ro, rl, "fp8 decode")


def test_fp8_decode_every_code():
    """The ring holds every finite E4M3 code (subnormals, +-0, +-448), with
    scales far from 1."""
    d = wl.decode_case(8, 4, 32, 4, 128, 128, sink="normal", seed=77, pos_lo=128, pos_hi=900,
                       kv="fp8")
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    n = d["k_ring"].numel()
    d["k_ring"] = torch.from_numpy(np.resize(finite, n).reshape(d["k_ring"].shape))
    d["v_ring"] = torch.from_numpy(np.resize(finite[::-1], n).reshape(d["v_ring"].shape))
    d["kv_scale"] = torch.tensor([1e-3, 2e-3, 3e-3, 4e-3, 3e-4, 1e-3, 7e-4, 5e-4],
                                 dtype=torch.float32)
    o, lse = run_fp8(d)
    ro, rl = oracle_fp8(d)
    check(o, lse, ro, rl, "every code")


def test_fp8_decode_nan_in_unwritten_slots():
    """Slots at or past pos (never written while pos < W) hold NaN codes; the
    result must ignore them."""
    Bn, n_q, Hq, Hkv, D, W = 6, 4, 64, 8, 128, 128
    d = wl.decode_case(Bn, n_q, Hq, Hkv, D, W, sink="normal", seed=5, pos_lo=0, pos_hi=W - 1,
                       kv="fp8")
    d["pos"] = torch.tensor([0, 1, 5, 64, 100, 127], dtype=torch.int32)
    for b in range(Bn):
        p = int(d["pos"][b])
        d["k_ring"][b, p:] = 0x7F
        d["v_ring"][b, p:] = 0xFF
    o, lse = run_fp8(d)
    ro, rl = oracle_fp8(d)
    check(o, lse, ro, rl, "NaN in unwritten slots")


def test_fp8_full_workload_all_rows():
    """The bench's FP8-ring decode (256 sequences, 4 new tokens, ring 128,
    Hq = 64, Hkv = 8) in its launch configuration, every row."""
    d = wl.make_decode(wl.WORKLOADS["swa_decode_mtp_fp8"])
    o, lse = run_fp8(d)
    ro, rl = oracle_fp8(d)
    check(o, lse, ro, rl, "swa_decode_mtp_fp8")


def test_fp8_equals_bf16_kernel_on_exact_rings():
    """Power-of-two scales make every dequantized value a bf16 number: the
    bf16 kernel over those values and the FP8 kernel over the codes agree."""
    d = wl.decode_case(16, 4, 64, 8, 128, 128, sink="normal", seed=12, pos_lo=0, pos_hi=400,
                       kv="fp8")
    d["kv_scale"] = torch.tensor([2.0 ** -(6 + (i % 4)) for i in range(16)],
                                 dtype=torch.float32)
    o8, l8 = run_fp8(d)
    sc = d["kv_scale"].numpy()
    kr = torch.from_numpy(fp8.dequantize(d["k_ring"].numpy(), sc, 8, 0)).to(torch.bfloat16)
    vr = torch.from_numpy(fp8.dequantize(d["v_ring"].numpy(), sc, 8, 1)).to(torch.bfloat16)
    g = to_cuda(d)
    ob, lb = B.attn_decode(g["q"], g["k_new"], g["v_new"], kr.cuda(), vr.cuda(), g["pos"],
                           sink=g["sink"])
    torch.cuda.synchronize()
    # the two kernels round P differently (f16 against bf16): each is within
    # the oracle bounds, so they agree within twice those
    diff = (o8.float() - ob.float()).abs()
    assert diff.max().item() <= 2e-2 and diff.mean().item() <= 2e-3
    assert (l8 - lb).abs().max().item() <= 1e-4


def _commit_case(Bn, n_q, Hkv, D, W, seed, big=1.0):
    d = wl.decode_case(Bn, n_q, 4, Hkv, D, W, seed=seed, pos_lo=0, pos_hi=4 * W, kv="fp8")
    d["k_new"] = (d["k_new"].float() * big).to(torch.bfloat16)
    return d


@pytest.mark.parametrize("big", [1.0, 40.0])
def test_fp8_commit_bitexact(big):
    """big = 40 pushes part of x / scale beyond 448 (saturation); the small
    draws land in the subnormal range."""
    Bn, n_q, Hkv, D, W = 8, 4, 8, 128, 128
    d = _commit_case(Bn, n_q, Hkv, D, W, 41, big)
    n_acc = torch.tensor([0, 1, 2, 3, 4, 4, 1, 0], dtype=torch.int32)
    g = to_cuda(d)
    kr, vr = g["k_ring"].clone(), g["v_ring"].clone()
    B.kv_commit_fp8(kr, vr, g["k_new"], g["v_new"], g["kv_scale"], g["pos"], n_acc.cuda())
    torch.cuda.synchronize()
    assert B.swa_sink_device_error() == 0
    ek, ev = fp8.kv_commit_fp8(d["k_ring"].numpy(), d["v_ring"].numpy(), d["k_new"].float().numpy(),
                               d["v_new"].float().numpy(), d["kv_scale"].numpy(),
                               d["pos"].numpy(), n_acc.numpy(), Bn, n_q, Hkv, D, W)
    assert np.array_equal(kr.cpu().numpy(), ek)
    assert np.array_equal(vr.cpu().numpy(), ev)
    if big > 1.0:
        assert np.any(ek == 0x7E) and np.any(ek == 0xFE)


def test_fp8_commit_ties_to_even():
    """Scale 1 and new values exactly halfway between neighbouring E4M3
    values (bf16 numbers): every one rounds to the even code."""
    Bn, n_q, Hkv, D, W = 2, 2, 1, 128, 8
    v = fp8.e4m3_table()[:0x7F]
    mids = (v[:-1] + v[1:]) / 2
    vals = np.resize(np.concatenate([mids, -mids]), Bn * n_q * Hkv * D).reshape(Bn, n_q, Hkv, D)
    kn = torch.from_numpy(vals).to(torch.bfloat16)
    assert np.array_equal(kn.double().numpy(), vals)
    ring = torch.zeros((Bn, W, Hkv, D), dtype=torch.uint8)
    pos = torch.tensor([3, 7], dtype=torch.int32)
    n_acc = torch.tensor([2, 2], dtype=torch.int32)
    sc = torch.ones(2, dtype=torch.float32)
    kr, vr = ring.cuda(), ring.clone().cuda()
    B.kv_commit_fp8(kr, vr, kn.cuda(), kn.cuda(), sc.cuda(), pos.cuda(), n_acc.cuda())
    torch.cuda.synchronize()
    ek, _ = fp8.kv_commit_fp8(ring.numpy(), ring.numpy(), vals, vals, sc.numpy(), pos.numpy(),
                              n_acc.numpy(), Bn, n_q, Hkv, D, W)
    got = kr.cpu().numpy()
    assert np.array_equal(got, ek)
    written = got[[0, 0, 1, 1], [3, 4, 7, 0]]
    assert np.all(written % 2 == 0)


def test_fp8_commit_then_decode_sees_the_new_tokens():
    """Decode, commit all n_q tokens, then decode the next step with n_q = 1:
    the committed tokens are read back through the ring."""
    Bn, n_q, Hq, Hkv, D, W = 4, 4, 32, 4, 128, 64
    d = wl.decode_case(Bn, n_q, Hq, Hkv, D, W, sink="normal", seed=8, pos_lo=10, pos_hi=300,
                       kv="fp8")
    g = to_cuda(d)
    kr, vr = g["k_ring"].clone(), g["v_ring"].clone()
    n_acc = torch.full((Bn,), n_q, dtype=torch.int32)
    B.kv_commit_fp8(kr, vr, g["k_new"], g["v_new"], g["kv_scale"], g["pos"], n_acc.cuda())
    nxt = wl.decode_case(Bn, 1, Hq, Hkv, D, W, sink="normal", seed=9, kv="fp8")
    d2 = dict(d, q=nxt["q"], k_new=nxt["k_new"], v_new=nxt["v_new"], n_q=1,
              pos=d["pos"] + n_q, k_ring=kr.cpu(), v_ring=vr.cpu())
    o, lse = run_fp8(d2)
    ro, rl = oracle_fp8(d2)
    check(o, lse, ro, rl, "decode after commit")


def test_fp8_flags_bad_scale():
    d = wl.decode_case(2, 1, 8, 2, 64, 16, seed=2, pos_lo=0, pos_hi=40, kv="fp8")
    d["kv_scale"][1] = 0.0
    g = to_cuda(d)
    B.attn_decode_fp8kv(g["q"], g["k_new"], g["v_new"], g["k_ring"], g["v_ring"],
                        g["kv_scale"], g["pos"], sink=g["sink"])
    torch.cuda.synchronize()
    assert B.swa_sink_device_error() == 2
    assert B.swa_sink_device_error() == 0
