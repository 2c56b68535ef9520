"""The benchmark's work model (the algorithmic FLOPs and bytes every roofline
figure divides by), checked against brute-force enumeration of the visible
(query, key) pairs on small shapes."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def pairs_prefill(seqlens, W):
    n = 0
    for L in seqlens:
        for i in range(L):
            n += sum(1 for j in range(i + 1) if W <= 0 or j >= i - W + 1)
    return n


@pytest.mark.parametrize("seqlens,W", [([1], 128), ([5, 0, 9], 3), ([130], 128), ([300], 0),
                                       ([7, 40, 1], 1), ([64, 65], 64)])
def test_prefill_work(seqlens, W):
    Hq, Hkv, D = 8, 2, 64
    flops, nbytes = bench.prefill_work(seqlens, Hq, Hkv, D, W)
    assert flops == 4 * D * Hq * pairs_prefill(seqlens, W)
    T = sum(seqlens)
    assert nbytes == (T * Hq * D * 4 + T * Hkv * D * 4 + Hq * T * 4 + Hq * 4
                      + (len(seqlens) + 1) * 4)


@pytest.mark.parametrize("seqlens,W", [([33, 2], 8), ([100], 0)])
def test_backward_work(seqlens, W):
    Hq, Hkv, D = 8, 1, 128
    f_fwd, _ = bench.prefill_work(seqlens, Hq, Hkv, D, W)
    flops, nbytes = bench.backward_work(seqlens, Hq, Hkv, D, W)
    assert flops == 10 * D * Hq * pairs_prefill(seqlens, W) == f_fwd * 5 // 2
    T = sum(seqlens)
    # q, o, dO read and dq written; k, v read and dk, dv written; lse read
    assert nbytes == (T * Hq * D * 2 * 4 + T * Hkv * D * 2 * 4 + Hq * T * 4 + Hq * 8
                      + (len(seqlens) + 1) * 4)


@pytest.mark.parametrize("pos,n_q,W", [([0, 3, 128, 500], 4, 128), ([7, 1], 1, 8),
                                       ([0], 2, 1)])
def test_decode_work(pos, n_q, W):
    Hq, Hkv, D = 8, 2, 64
    flops, nbytes = bench.decode_work(pos, n_q, Hq, Hkv, D, W)
    pairs = 0
    cached = 0
    for P in pos:
        ring = [p for p in range(max(0, P - W), P)]  # committed tokens in the ring
        cached += len(ring)
        for t in range(n_q):
            # ring tokens inside the window, and every new token 0..t (the
            # decode's definition: drafts see each other causally)
            pairs += sum(1 for p in ring if p >= P + t - W + 1) + (t + 1)
    assert flops == 4 * D * Hq * pairs
    B = len(pos)
    assert nbytes == (cached * Hkv * D * 2 * 2 + B * n_q * Hkv * D * 2 * 2
                      + B * n_q * Hq * D * 2 * 2 + B * n_q * Hq * 4 + B * 4 + Hq * 4)


def test_percentiles():
    # nearest rank on the sorted values: p10 of 1..20 is the 2nd, p90 the 18th
    got = bench.percentiles(list(range(20, 0, -1)))
    assert got == {"p10": 2, "median": 10.5, "p90": 18}
    one = bench.percentiles([3.0])
    assert one == {"p10": 3.0, "median": 3.0, "p90": 3.0}
    got = bench.percentiles([5.0, 1.0, 4.0, 2.0, 3.0])
    assert got == {"p10": 1.0, "median": 3.0, "p90": 5.0}
