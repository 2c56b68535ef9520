"""Pins for the FP8 (E4M3) pieces of the oracle, independent of its code:

* the code table equals torch's float8_e4m3fn decoding for all 256 codes and
  the closed forms of the format (zero, subnormals, one, 448, NaN codes);
* the encoder equals torch's float32 -> float8_e4m3fn cast (round to nearest,
  ties to even) for every value below 464 in magnitude, including every exact
  midpoint between neighbouring codes, and saturates beyond 448;
* the round trip stays within half a unit in the last place;
* the fp64 decode over a float ring equals the C oracle's decode over the
  same bf16 ring, and over an FP8 ring whose dequantized values are exactly
  bf16 (power-of-two scales) it equals the C oracle too;
* the FP8 commit writes the same slots as the bf16 commit, with codes equal
  to torch's cast of the float32 quotient x / scale.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import fp8
from sliding_window_attention_sink_b200 import workloads as wl

TOL = 1e-12


def torch_codes(x32):
    """float32 numpy -> codes through torch's cast."""
    return torch.from_numpy(np.ascontiguousarray(x32, np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_table_matches_torch():
    t = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    ref = t.to(torch.float64).numpy()
    got = fp8.e4m3_table()
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])
    assert np.array_equal(np.signbit(ref[ok]), np.signbit(got[ok]))


def test_table_closed_forms():
    v = fp8.e4m3_table()
    assert v[0x00] == 0.0 and not np.signbit(v[0x00])
    assert v[0x80] == 0.0 and np.signbit(v[0x80])
    assert v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9      # subnormals
    assert v[0x08] == 2.0 ** -6                                     # smallest normal
    assert v[0x38] == 1.0 and v[0xB8] == -1.0
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    pos = v[:0x7F]
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(v[0x80:0xFF], -pos)


def test_encode_matches_torch_random():
    g = np.random.default_rng(11)
    xs = [g.standard_normal(20000) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)]
    xs.append(g.uniform(-448.0, 448.0, 20000))
    x = np.concatenate(xs).astype(np.float32)
    x = x[np.abs(x) < 464.0]  # torch's cast is not saturating: NaN from 464 up
    assert np.array_equal(fp8.e4m3_encode(x), torch_codes(x))


def test_encode_midpoints_ties_to_even():
    v = fp8.e4m3_table()[:0x7F]
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (v[:-1] + v[1:]) / 2)  # exact in fp32
    codes = fp8.e4m3_encode(mids)
    assert np.all(codes % 2 == 0)                  # the even-mantissa neighbour
    assert np.all((codes == np.arange(126)) | (codes == np.arange(1, 127)))
    assert np.array_equal(codes, torch_codes(mids))
    assert np.array_equal(fp8.e4m3_encode(-mids), codes | 0x80)
    # just off the midpoints: the nearer neighbour
    up = np.nextafter(mids, np.float32(np.inf))
    dn = np.nextafter(mids, np.float32(-np.inf))
    assert np.array_equal(fp8.e4m3_encode(up), np.arange(1, 127))
    assert np.array_equal(fp8.e4m3_encode(dn[1:]), np.arange(1, 126))


def test_encode_saturates_and_nan():
    big = np.array([448.0, 449.0, 463.9, 464.0, 500.0, 1e30, np.inf], np.float32)
    assert np.all(fp8.e4m3_encode(big) == 0x7E)
    assert np.all(fp8.e4m3_encode(-big) == 0xFE)
    assert fp8.e4m3_encode(np.array([np.nan], np.float32))[0] & 0x7F == 0x7F
    assert fp8.e4m3_encode(np.array([-0.0], np.float32))[0] == 0x80
    assert fp8.e4m3_encode(np.array([2.0 ** -11], np.float32))[0] == 0x00  # below half of 2^-9
    assert fp8.e4m3_encode(np.array([2.0 ** -10 * 1.01], np.float32))[0] == 0x01


def test_roundtrip_within_half_ulp():
    g = np.random.default_rng(12)
    x = np.concatenate([g.uniform(2.0 ** -6, 448.0, 50000),
                        g.uniform(0, 2.0 ** -6, 5000)]).astype(np.float32)
    back = fp8.e4m3_table()[fp8.e4m3_encode(x)]
    xd = x.astype(np.float64)
    normal = xd >= 2.0 ** -6
    assert np.all(np.abs(back - xd)[normal] <= 2.0 ** -4 * xd[normal])
    assert np.all(np.abs(back - xd)[~normal] <= 2.0 ** -10)


def _c_decode(c, k_ring, v_ring, scale=None):
    o, lse, _ = oracle.decode(c["q"], c["k_new"], c["v_new"], k_ring, v_ring, c["pos"], c["B"],
                              c["n_q"], c["Hq"], c["Hkv"], c["D"], c["W"], sink=c["sink"],
                              scale=scale)
    return o, lse


def _f(x):
    return x.to(torch.float64).numpy()


@pytest.mark.parametrize("B,n_q,Hq,Hkv,D,W,pos_lo,pos_hi,sink", [
    (3, 4, 8, 2, 64, 16, 0, 40, "normal"),
    (2, 1, 4, 1, 64, 128, 100, 300, None),
    (2, 8, 4, 2, 64, 13, 0, 5, "uniform2"),
])
def test_decode_values_equals_c_oracle(B, n_q, Hq, Hkv, D, W, pos_lo, pos_hi, sink):
    c = wl.decode_case(B, n_q, Hq, Hkv, D, W, sink=sink, seed=3, pos_lo=pos_lo, pos_hi=pos_hi)
    o_ref, lse_ref = _c_decode(c, c["k_ring"], c["v_ring"])
    o, lse = fp8.decode_values(_f(c["q"]), _f(c["k_new"]), _f(c["v_new"]), _f(c["k_ring"]),
                               _f(c["v_ring"]), c["pos"].numpy(), B, n_q, Hq, Hkv, D, W,
                               sink=None if c["sink"] is None else c["sink"].numpy())
    assert np.max(np.abs(o - o_ref)) < TOL
    assert np.max(np.abs(lse - lse_ref)) < TOL


@pytest.mark.parametrize("W,pos_lo,pos_hi", [(16, 0, 40), (32, 200, 400)])
def test_decode_fp8_equals_c_oracle_on_exact_rings(W, pos_lo, pos_hi):
    """Power-of-two scales keep every dequantized value a bf16 number, so the
    C oracle on the bf16 ring must give the same result."""
    B, n_q, Hq, Hkv, D = 2, 4, 8, 2, 64
    c = wl.decode_case(B, n_q, Hq, Hkv, D, W, seed=5, pos_lo=pos_lo, pos_hi=pos_hi, kv="fp8")
    kv_scale = np.array([2.0 ** -7, 2.0 ** -5, 2.0 ** -6, 2.0 ** -8], np.float32)
    kr = fp8.dequantize(c["k_ring"].numpy(), kv_scale, Hkv, 0)
    vr = fp8.dequantize(c["v_ring"].numpy(), kv_scale, Hkv, 1)
    kb, vb = torch.from_numpy(kr).to(torch.bfloat16), torch.from_numpy(vr).to(torch.bfloat16)
    assert np.array_equal(_f(kb), kr) and np.array_equal(_f(vb), vr)
    o_ref, lse_ref = _c_decode(c, kb, vb)
    o, lse = fp8.decode_fp8(_f(c["q"]), _f(c["k_new"]), _f(c["v_new"]), c["k_ring"].numpy(),
                            c["v_ring"].numpy(), kv_scale, c["pos"].numpy(), B, n_q, Hq, Hkv,
                            D, W, sink=c["sink"].numpy())
    assert np.max(np.abs(o - o_ref)) < TOL
    assert np.max(np.abs(lse - lse_ref)) < TOL


def test_dequantize_applies_per_head_scales():
    codes = np.full((1, 2, 3, 4), 0x38, np.uint8)  # every value 1.0
    sc = np.array([1, 2, 3, 4, 5, 6], np.float32)
    assert np.array_equal(fp8.dequantize(codes, sc, 3, 0)[0, 0, :, 0], [1, 2, 3])
    assert np.array_equal(fp8.dequantize(codes, sc, 3, 1)[0, 1, :, 3], [4, 5, 6])


def test_kv_commit_fp8_slots_and_codes():
    B, n_q, Hkv, D, W = 3, 4, 2, 64, 8
    c = wl.decode_case(B, n_q, 4, Hkv, D, W, seed=9, pos_lo=0, pos_hi=30, kv="fp8")
    n_acc = np.array([0, 4, 2], np.int32)
    pos = c["pos"].numpy()
    kc, vc = fp8.kv_commit_fp8(c["k_ring"].numpy(), c["v_ring"].numpy(), _f(c["k_new"]),
                               _f(c["v_new"]), c["kv_scale"].numpy(), pos, n_acc, B, n_q, Hkv,
                               D, W)
    # the slots the bf16 commit writes (marker rings: 0 everywhere, new tokens 1.0)
    zero = torch.zeros((B, W, Hkv, D), dtype=torch.bfloat16)
    one = torch.ones((B, n_q, Hkv, D), dtype=torch.bfloat16)
    km, _ = oracle.kv_commit(zero, zero, one, one, c["pos"], torch.from_numpy(n_acc), B, n_q,
                             Hkv, D, W)
    written = km != 0
    old_k, old_v = c["k_ring"].numpy(), c["v_ring"].numpy()
    assert np.array_equal(kc[~written], old_k[~written])
    assert np.array_equal(vc[~written], old_v[~written])
    sc = c["kv_scale"].numpy()
    for b in range(B):
        for u in range(n_acc[b]):
            slot = (pos[b] + u) % W
            for gh in range(Hkv):
                xk = c["k_new"][b, u, gh].float().numpy() / sc[gh]
                xv = c["v_new"][b, u, gh].float().numpy() / sc[Hkv + gh]
                assert np.array_equal(kc[b, slot, gh], torch_codes(xk))
                assert np.array_equal(vc[b, slot, gh], torch_codes(xv))


def test_kv_commit_fp8_exact_values_roundtrip():
    """Scale 1 and new values that are E4M3 numbers: the committed ring
    dequantizes back to the new values exactly."""
    B, n_q, Hkv, D, W = 2, 2, 1, 64, 4
    g = np.random.default_rng(4)
    finite = np.concatenate([np.arange(0, 0x7F), np.arange(0x80, 0xFF)])
    vals = fp8.e4m3_table()[g.choice(finite, (B, n_q, Hkv, D))]
    ring = np.zeros((B, W, Hkv, D), np.uint8)
    pos = np.array([3, 6], np.int32)
    kc, vc = fp8.kv_commit_fp8(ring, ring, vals, -vals, np.ones(2, np.float32), pos,
                               np.array([2, 2], np.int32), B, n_q, Hkv, D, W)
    t = fp8.e4m3_table()
    for b in range(B):
        for u in range(2):
            s = (pos[b] + u) % W
            assert np.array_equal(t[kc[b, s]], vals[b, u])
            assert np.array_equal(t[vc[b, s]], -vals[b, u])


def test_fp8_workload_inputs():
    c = wl.decode_case(2, 2, 4, 2, 64, 16, seed=1, kv="fp8")
    assert c["k_ring"].dtype == torch.uint8 and c["kv_scale"].shape == (4,)
    codes = c["k_ring"].numpy()
    assert not np.any((codes & 0x7F) == 0x7F)   # no NaN codes
    assert len(np.unique(codes)) > 150          # spread over the format
    assert torch.all(c["kv_scale"] > 0)
