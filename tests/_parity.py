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


def check_every_row(o_gpu, lse_gpu, q, k, v, cu_seqlens, Hq, Hkv, D, window, sink, what,
                    chunk_tokens=2048):
    """Every (token, head) row of a prefill against the oracle, element by
    element, one chunk of tokens at a time (the oracle's output for a whole
    32K-token layer would be 2 GB of float64). The bounds are those of
    check(): the largest error over all rows, and the mean over all rows.
    q, k, v are what the oracle attends over (bf16 tensors or bit arrays)."""
    import oracle
    total = o_gpu.shape[0]
    qb, kb, vb = oracle.oracle._bits(q), oracle.oracle._bits(k), oracle.oracle._bits(v)
    max_o = max_l = 0.0
    sum_o = 0.0
    n_o = 0
    for t0 in range(0, total, chunk_tokens):
        t1 = min(total, t0 + chunk_tokens)
        rt = np.repeat(np.arange(t0, t1, dtype=np.int64), Hq)
        rh = np.tile(np.arange(Hq, dtype=np.int32), t1 - t0)
        ro, rl, _ = oracle.prefill_rows(qb, kb, vb, cu_seqlens, Hq, Hkv, D, window, rt, rh,
                                        sink=sink)
        og = o_gpu[t0:t1].float().cpu().numpy().astype(np.float64).reshape(-1, D)
        assert np.isfinite(og).all(), "%s: non-finite output in tokens [%d, %d)" % (what, t0, t1)
        err = np.abs(og - ro)
        max_o = max(max_o, float(err.max()))
        sum_o += float(err.sum())
        n_o += err.size
        if lse_gpu is not None:
            lg = lse_gpu[:, t0:t1].t().contiguous().cpu().numpy().astype(np.float64).reshape(-1)
            assert np.isfinite(lg).all(), "%s: non-finite lse" % what
            max_l = max(max_l, float(np.abs(lg - rl).max()))
        assert max_o <= MAX_ABS_O and max_l <= MAX_ABS_LSE, (what, t0, max_o, max_l)
    stats = dict(max_o=max_o, mean_o=sum_o / max(n_o, 1), max_lse=max_l, rows=total * Hq)
    print("%s: every row %s" % (what, stats))
    assert stats["mean_o"] <= MEAN_ABS_O, (what, stats)
    return stats
