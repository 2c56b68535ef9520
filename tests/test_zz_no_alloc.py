"""GPU check of swa_sink_attn_fwd_noalloc, the entry point for callers that
cannot allocate device memory: its sliding-window kernel draws tile ranges
from counters in a static slot of the library instead of cancelling launches
of its own grid as swa_sink_attn_fwd does. Two calls in a row on the same
slot (the second finds the slot as the first left it) must give exactly what
swa_sink_attn_fwd gives, for the sliding-window ring kernel (the one with a
scheduler) and for a global layer (no scheduler). The file is named to be
collected last, so it also runs after every other GPU test in the same
process."""
import pytest
import torch

from sliding_window_attention_sink_b200 import binding as B
from sliding_window_attention_sink_b200 import workloads as wl

from _parity import to_cuda

pytestmark = pytest.mark.gpu


def fwd(d, c, noalloc_slot=None):
    total, Hq, D = d["q"].shape
    Hkv = d["k"].shape[1]
    o = torch.full_like(d["q"], float("nan"))
    lse = torch.full((Hq, total), float("nan"), device=d["q"].device)
    args = (d["q"], d["k"], d["v"], d["cu_seqlens"], d["cu_seqlens"].numel() - 1,
            c["max_seqlen"], total, Hq, Hkv, D, c["window"], d["sink"], 0.0, o, lse)
    if noalloc_slot is None:
        rc = B.swa_sink_attn_fwd(*args)
    else:
        rc = B.swa_sink_attn_fwd_noalloc(*args, noalloc_slot)
    assert rc == 0, B.status_string(rc)
    return o, lse


@pytest.mark.parametrize("seqlens,Hq,Hkv,D,W", [
    ([3000, 700, 1], 64, 8, 128, 128),   # ring kernel, static share + dynamic ranges
    ([900], 16, 2, 64, 128),             # ring kernel, D = 64
    ([1500, 400], 16, 2, 128, 0),        # global layer: chunked kernel, no scheduler
])
@pytest.mark.parametrize("slot", [0, 7])
def test_noalloc_matches_fwd_twice_in_a_row(seqlens, Hq, Hkv, D, W, slot):
    c = wl.prefill_case(seqlens, Hq, Hkv, D, W, sigma=0.5, sink="normal", seed=21)
    d = to_cuda(c)
    ref_o, ref_l = fwd(d, c)
    o1, l1 = fwd(d, c, noalloc_slot=slot)
    o2, l2 = fwd(d, c, noalloc_slot=slot)
    torch.cuda.synchronize()
    assert B.swa_sink_device_error() == 0
    assert torch.equal(o1, ref_o) and torch.equal(l1, ref_l)
    assert torch.equal(o2, ref_o) and torch.equal(l2, ref_l)
