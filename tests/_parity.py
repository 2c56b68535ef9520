"""Shared helpers for the GPU parity tests: device transfer and the error
bounds stated for bf16 I/O with fp32 accumulation (output error: max
|O - O_ref| <= 1e-2, mean <= 1e-3; max |LSE - LSE_ref| <= 1e-3) against the
fp64 oracle."""
import numpy as np
import torch

MAX_ABS_O = 1e-2
MEAN_ABS_O = 1e-3
MAX_ABS_LSE = 1e-3


def to_cuda(d):
    out = {}
    for k, v in d.items():
        out[k] = v.cuda() if isinstance(v, torch.Tensor) else v
    return out


def check(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    o = o_gpu.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(o).all(), "%s: non-finite output" % what
    err = np.abs(o - o_ref)
    stats = dict(max_o=float(err.max()) if err.size else 0.0,
                 mean_o=float(err.mean()) if err.size else 0.0)
    if lse_gpu is not None:
        l = lse_gpu.cpu().numpy().astype(np.float64)
        assert np.isfinite(l).all(), "%s: non-finite lse" % what
        stats["max_lse"] = float(np.abs(l - lse_ref).max()) if l.size else 0.0
    assert stats["max_o"] <= MAX_ABS_O, (what, stats)
    assert stats["mean_o"] <= MEAN_ABS_O, (what, stats)
    if lse_gpu is not None:
        assert stats["max_lse"] <= MAX_ABS_LSE, (what, stats)
    return stats
