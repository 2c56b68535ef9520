"""The seeded input generators (sliding_window_attention_sink_b200/workloads.py),
which feed both the CUDA path and the oracle, pinned to their stated recipe by
drawing it again here step by step: one torch.Generator per case, in the
order varlen lengths, q, k, v (fp32 N(0,1) x sigma rounded to bf16), sink;
decode: pos, q, k_new, v_new, the ring (bf16 draws, or E4M3 codes from
N(0, 64^2) clamped to +-448), sink, then the FP8 scales U(0.5, 2) x sigma / 64.
Plus the ranges and invariants the kernels rely on."""
import pytest
import torch

from sliding_window_attention_sink_b200 import workloads as wl


def bits(t):
    return t.contiguous().view(torch.int16 if t.dtype == torch.bfloat16 else torch.uint8)


def same(a, b):
    assert a.dtype == b.dtype and a.shape == b.shape
    if a.dtype in (torch.bfloat16, torch.uint8):
        assert torch.equal(bits(a), bits(b))
    else:
        assert torch.equal(a, b)


@pytest.mark.parametrize("sink", ["normal", "uniform2", None])
def test_prefill_recipe(sink):
    case = wl.PrefillCase("t", [5, 0, 7], 4, 2, 8, 3, 0.7, sink, 11)
    c = wl.make_prefill(case)
    g = torch.Generator().manual_seed(11)
    q = (torch.randn((12, 4, 8), generator=g) * 0.7).to(torch.bfloat16)
    k = (torch.randn((12, 2, 8), generator=g) * 0.7).to(torch.bfloat16)
    v = (torch.randn((12, 2, 8), generator=g) * 0.7).to(torch.bfloat16)
    same(c["q"], q)
    same(c["k"], k)
    same(c["v"], v)
    if sink is None:
        assert c["sink"] is None
    elif sink == "normal":
        same(c["sink"], torch.randn((4,), generator=g))
    else:
        same(c["sink"], torch.rand((4,), generator=g) * 4.0 - 2.0)
    assert c["cu_seqlens"].dtype == torch.int32
    assert c["cu_seqlens"].tolist() == [0, 5, 5, 12]
    assert (c["total"], c["max_seqlen"], c["dout"]) == (12, 7, None)


def test_varlen_draw_and_dout():
    case = wl.PrefillCase("t", [], 2, 1, 8, 4, 0.5, "normal", 3, varlen_draw=(6, 2, 9),
                          backward=True)
    c = wl.make_prefill(case)
    g = torch.Generator().manual_seed(3)
    lens = torch.randint(2, 10, (6,), generator=g).tolist()
    assert c["seqlens"] == lens and all(2 <= n <= 9 for n in lens)
    cu = c["cu_seqlens"].tolist()
    assert cu[0] == 0 and all(b - a == n for a, b, n in zip(cu, cu[1:], lens))
    # dout: its own generator, seed + 1
    g2 = torch.Generator().manual_seed(4)
    same(c["dout"], (torch.randn(c["q"].shape, generator=g2) * 0.5).to(torch.bfloat16))


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_decode_recipe(kv):
    case = wl.DecodeCase("t", 3, 2, 4, 2, 8, 16, 0.5, "normal", 9, pos_lo=3, pos_hi=40, kv=kv)
    d = wl.make_decode(case)
    g = torch.Generator().manual_seed(9)
    pos = torch.randint(3, 41, (3,), generator=g, dtype=torch.int64).to(torch.int32)
    same(d["pos"], pos)
    same(d["q"], (torch.randn((3, 2, 4, 8), generator=g) * 0.5).to(torch.bfloat16))
    same(d["k_new"], (torch.randn((3, 2, 2, 8), generator=g) * 0.5).to(torch.bfloat16))
    same(d["v_new"], (torch.randn((3, 2, 2, 8), generator=g) * 0.5).to(torch.bfloat16))
    shape = (3, 16, 2, 8)
    for name in ("k_ring", "v_ring"):
        if kv == "fp8":
            x = (torch.randn(shape, generator=g) * 64.0).clamp(-448.0, 448.0)
            same(d[name], x.to(torch.float8_e4m3fn).view(torch.uint8))
        else:
            same(d[name], (torch.randn(shape, generator=g) * 0.5).to(torch.bfloat16))
    same(d["sink"], torch.randn((4,), generator=g))
    if kv == "fp8":
        sc = (torch.rand((4,), generator=g) * 1.5 + 0.5) * (0.5 / 64.0)
        same(d["kv_scale"], sc)


def test_fp8_codes_are_finite_and_cover_the_range():
    d = wl.make_decode(wl.WORKLOADS["swa_decode_mtp_fp8"])
    for name in ("k_ring", "v_ring"):
        codes = d[name]
        assert codes.dtype == torch.uint8
        assert not ((codes & 0x7F) == 0x7F).any()  # the E4M3 NaN codes
        assert int((codes >> 3 & 0xF).unique().numel()) == 16  # every exponent field used
    s = d["kv_scale"] / (0.5 / 64.0)
    assert ((s >= 0.5) & (s <= 2.0)).all()


def test_inputs_are_deterministic():
    a = wl.make_decode(wl.WORKLOADS["swa_decode_mtp"])
    b = wl.make_decode(wl.WORKLOADS["swa_decode_mtp"])
    for key in ("q", "k_new", "v_new", "k_ring", "v_ring", "pos", "sink"):
        same(a[key], b[key])
    assert ((a["pos"] >= 128) & (a["pos"] <= 262144)).all()


def test_named_workloads_match_their_names():
    for key, case in wl.WORKLOADS.items():
        words = dict(w.split("=", 1) for w in case.name.split() if "=" in w)
        for field in ("Hq", "Hkv", "D", "W", "B", "n_q"):
            if field in words and hasattr(case, field if field != "W" else "window"):
                want = getattr(case, field if field != "W" else "window")
                assert str(want) == words[field], (key, field)
        if "T" in words:
            assert sum(case.seqlens) == int(words["T"]), key
    G = {k: c.Hq // c.Hkv for k, c in wl.WORKLOADS.items()}
    assert all(64 % g == 0 for g in G.values())


def test_slice_sequences_rebases():
    c = wl.prefill_case([4, 0, 6, 3], 2, 1, 8, 2, seed=1)
    s = wl.slice_sequences(c, 1, 3)
    assert s["cu_seqlens"].tolist() == [0, 0, 6] and s["total"] == 6
    same(s["q"], c["q"][4:10])
    assert s["token_range"] == (4, 10) and s["max_seqlen"] == 6
