"""GPU parity of swa_sink_attn_fwd (through the C ABI) against the fp64 oracle
on the same seeded inputs: small shapes and the full workloads (the SWA layer,
the global layer and the packed varlen batch) compared element by element on
every row, plus edge cases (ragged tails, empty and length-1 sequences, tiles
straddling sequences, no sink, extreme sinks, W = 1, G = 1 and G = 16,
chunked windows and global layers, and query groups that do not divide 128,
which run the fallback kernel)."""
import math

import numpy as np
import pytest
import torch

import oracle
from sliding_window_attention_sink_b200 import binding as B
from sliding_window_attention_sink_b200 import workloads as wl

from _parity import check, check_every_row, to_cuda

pytestmark = pytest.mark.gpu


def run_gpu(c, window=None, sink="case", poison=True):
    d = to_cuda(c)
    w = c["window"] if window is None else window
    s = d["sink"] if sink == "case" else sink
    o = torch.full_like(d["q"], float("nan")) if poison else None
    o, lse = B.attn_fwd(d["q"], d["k"], d["v"], d["cu_seqlens"], w, sink=s, out=o,
                        max_seqlen=c["max_seqlen"])
    torch.cuda.synchronize()
    assert B.swa_sink_device_error() == 0
    return o, lse


SMALL = [  # (name, seqlens, Hq, Hkv, D, W, sink)
    ("tiny_cfg", [512], 4, 1, 64, 128, "uniform2"),
    ("swa_ragged", [300], 64, 8, 128, 128, "normal"),
    ("varlen_edges", [100, 0, 257, 1, 33], 16, 2, 128, 128, "normal"),
    ("global_chunks", [700], 16, 2, 128, 0, "normal"),
    ("global_varlen", [129, 300, 5], 8, 1, 64, 0, "uniform2"),
    ("wide_window", [600], 8, 1, 64, 300, "normal"),
    ("g1", [300], 2, 2, 64, 128, "normal"),
    ("g16", [200], 32, 2, 128, 64, "normal"),
    ("g2_w8", [90], 4, 2, 128, 8, "normal"),
    ("no_sink", [257], 8, 1, 128, 128, None),
    ("w1", [70], 8, 1, 64, 1, "normal"),
    ("short_seqs", [1, 2, 3, 17], 8, 1, 128, 128, "normal"),
    # G does not divide 128: the fallback kernel (tiles of floor(128/G) tokens)
    ("fallback_g3_swa", [300], 12, 4, 128, 128, "normal"),
    ("fallback_g3_global", [500], 48, 16, 128, 0, "normal"),
    ("fallback_g6_varlen", [100, 0, 257, 1, 33], 6, 1, 128, 128, "normal"),
    ("fallback_g5_d64_global_varlen", [129, 300, 5], 10, 2, 64, 0, "uniform2"),
    ("fallback_g7_w37", [200], 7, 1, 64, 37, "normal"),
    ("fallback_g96_one_token_tiles", [150], 96, 1, 64, 128, "normal"),
    ("fallback_g3_wide_window", [600], 3, 1, 128, 300, "normal"),
    ("fallback_g3_no_sink", [257], 12, 4, 128, 128, None),
]


@pytest.mark.parametrize("name,seqlens,Hq,Hkv,D,W,sink", SMALL, ids=[s[0] for s in SMALL])
def test_prefill_matches_oracle(name, seqlens, Hq, Hkv, D, W, sink):
    seed = 0 if name == "tiny_cfg" else 7
    sigma = 1.0 if name == "tiny_cfg" else 0.5
    c = wl.prefill_case(seqlens, Hq, Hkv, D, W, sigma=sigma, sink=sink, seed=seed)
    o, lse = run_gpu(c)
    ro, rl, _ = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], Hq, Hkv, D, W,
                               sink=c["sink"])
    check(o, lse, ro, rl, name)


@pytest.mark.parametrize("W", [128, 0])
@pytest.mark.parametrize("sval", [30.0, -30.0, 0.0])
def test_prefill_extreme_sinks(sval, W):
    n = 200 if W else 450
    c = wl.prefill_case([n], 8, 1, 128, W, sigma=0.5, sink=None, seed=3)
    sink = torch.full((8,), sval)
    c["sink"] = sink
    o, lse = run_gpu(c)
    ro, rl, _ = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], 8, 1, 128, W,
                               sink=sink)
    check(o, lse, ro, rl, "sink=%g W=%d" % (sval, W))


@pytest.mark.parametrize("W,seqlens", [(0, [900]), (1000, [900]), (0, [300, 700])])
def test_prefill_growing_logits(W, seqlens):
    # key norms grow along each sequence, so a row's running max rises by many
    # log2 units from one 128-key chunk to the next (and falls back at a new
    # sequence): the online-softmax rescale of O runs often
    c = wl.prefill_case(seqlens, 8, 1, 128, W, sigma=0.5, sink="normal", seed=11)
    n = sum(seqlens)
    ramp = torch.cat([torch.linspace(0.2, 40.0, s) for s in seqlens])
    c["k"] = (c["k"].float() * ramp[:, None, None]).to(torch.bfloat16)
    o, lse = run_gpu(c)
    ro, rl, _ = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], 8, 1, 128, W,
                               sink=c["sink"])
    check(o, lse, ro, rl, "growing W=%d n=%d" % (W, n))


def test_prefill_window_ge_len_equals_global():
    c = wl.prefill_case([333], 16, 2, 128, 0, sigma=0.5, sink="normal", seed=4)
    o0, l0 = run_gpu(c, window=0)
    o1, l1 = run_gpu(c, window=4096)
    ro, rl, _ = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], 16, 2, 128, 0,
                               sink=c["sink"])
    check(o0, l0, ro, rl, "W=0")
    check(o1, l1, ro, rl, "W=4096")


def test_prefill_lse_optional_and_scale():
    c = wl.prefill_case([150], 8, 2, 64, 32, sigma=0.5, sink="normal", seed=5)
    d = to_cuda(c)
    o, lse = B.attn_fwd(d["q"], d["k"], d["v"], d["cu_seqlens"], 32, sink=d["sink"],
                        softmax_scale=0.3, want_lse=False)
    torch.cuda.synchronize()
    assert lse is None
    ro, rl, _ = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], 8, 2, 64, 32,
                               sink=c["sink"], scale=float(np.float32(0.3)))
    check(o, None, ro, rl, "scale=0.3")


@pytest.mark.parametrize("wname", ["swa_prefill_32k", "global_prefill_8k",
                                   "varlen_swa_prefill"])
def test_prefill_full_workloads_every_row(wname):
    """The benchmark's launch configuration at full size, every (token, head)
    row against the oracle (the global layer's oracle takes about a minute on
    16 host threads)."""
    case = wl.WORKLOADS[wname]
    c = wl.make_prefill(case)
    o, lse = run_gpu(c)
    check_every_row(o, lse, c["q"], c["k"], c["v"], c["cu_seqlens"], c["Hq"], c["Hkv"],
                    c["D"], c["window"], c["sink"], wname)


def test_prefill_repeated_calls_on_two_streams():
    # 70 rounds of a sliding-window and a global call, alternating between two
    # streams: every output equals the first one bit for bit
    c = wl.prefill_case([700, 300], 16, 2, 128, 128, sigma=0.5, sink="normal", seed=5)
    d = to_cuda(c)
    ref_o, ref_l = B.attn_fwd(d["q"], d["k"], d["v"], d["cu_seqlens"], 128, sink=d["sink"])
    g = wl.prefill_case([2000], 16, 2, 128, 0, sigma=0.5, sink="normal", seed=6)
    dg = to_cuda(g)
    ref_go, ref_gl = B.attn_fwd(dg["q"], dg["k"], dg["v"], dg["cu_seqlens"], 0, sink=dg["sink"])
    torch.cuda.synchronize()
    outs = []
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    for it in range(70):
        with torch.cuda.stream(s1 if it % 2 else s2):
            o, lse = B.attn_fwd(d["q"], d["k"], d["v"], d["cu_seqlens"], 128, sink=d["sink"])
            go, gl = B.attn_fwd(dg["q"], dg["k"], dg["v"], dg["cu_seqlens"], 0, sink=dg["sink"])
        outs.append((o, lse, go, gl))
    torch.cuda.synchronize()
    assert B.swa_sink_device_error() == 0
    for o, lse, go, gl in outs:
        assert torch.equal(o, ref_o) and torch.equal(lse, ref_l)
        assert torch.equal(go, ref_go) and torch.equal(gl, ref_gl)


def test_prefill_many_calls_in_flight_on_several_streams():
    """96 calls queued at once on four streams, each stream held back by a
    timed sleep kernel until all are queued, so that many run on the GPU at
    the same time (most are a few CTAs). The sliding-window kernel keeps no
    state between calls (its load balancing cancels launches of its own grid),
    so every output equals the serial result bit for bit."""
    cases = [
        wl.prefill_case([40], 16, 2, 128, 128, sigma=0.5, sink="normal", seed=31),
        wl.prefill_case([700, 300], 16, 2, 128, 128, sigma=0.5, sink="normal", seed=32),
        wl.prefill_case([257, 3], 8, 1, 64, 128, sigma=0.5, sink="normal", seed=33),
        wl.prefill_case([33], 64, 8, 128, 128, sigma=0.5, sink=None, seed=34),
        wl.prefill_case([500], 16, 2, 128, 0, sigma=0.5, sink="normal", seed=35),
    ]
    devs = [to_cuda(c) for c in cases]

    def call(c, d):
        return B.attn_fwd(d["q"], d["k"], d["v"], d["cu_seqlens"], c["window"], sink=d["sink"],
                          max_seqlen=c["max_seqlen"])

    refs = []
    for c, d in zip(cases, devs):
        refs.append(call(c, d))
        torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in range(4)]
    for st in streams:
        with torch.cuda.stream(st):
            torch.cuda._sleep(40_000_000)  # a bounded spin of about 20 ms
    outs = []
    for it in range(96):
        i = it % len(cases)
        with torch.cuda.stream(streams[(it // len(cases)) % len(streams)]):
            outs.append((i, *call(cases[i], devs[i])))
    torch.cuda.synchronize()
    assert B.swa_sink_device_error() == 0
    for i, o, lse in outs:
        assert torch.equal(o, refs[i][0]) and torch.equal(lse, refs[i][1]), i
