"""Golden fixtures: the window the pages fix (W = 128, row i sees min(i+1, W)
keys under the reading recorded in the fixture) and a frozen fp64 snapshot of
the oracle on one tiny case."""
import json
import math
import os

import numpy as np
import torch

import oracle
from sliding_window_attention_sink_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_pages_window_counts_via_zero_query_closed_form():
    fx = json.load(open(os.path.join(GOLDEN, "pages_window.json")))
    W = fx["window"]
    rows = {int(k): v for k, v in fx["visible_keys_by_row"].items()}
    L = 300
    c = wl.prefill_case([L], 1, 1, 8, W, sigma=1.0, sink="normal", seed=1)
    q = torch.zeros_like(c["q"])
    sel = [r for r in rows if r < L]
    o, lse, _ = oracle.prefill_rows(q, c["k"], c["v"], c["cu_seqlens"], 1, 1, 8,
                                    W, sel, [0] * len(sel), sink=c["sink"])
    es = math.exp(float(c["sink"][0]))
    for u, r in enumerate(sel):
        # lse = ln(n + e^s) when every logit is 0
        assert round(math.exp(lse[u]) - es) == rows[r]
    for r, n in rows.items():
        assert n == min(r + 1, W)


def test_oracle_snapshot():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "make_golden", os.path.join(GOLDEN, "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    o, lse, _ = mg.compute()
    n = 0
    for line in open(os.path.join(GOLDEN, "oracle_tiny.txt")):
        if line.startswith("#"):
            continue
        f = line.split()
        if f[0] == "lse":
            assert float(f[3]) == lse[int(f[1]), int(f[2])]
        else:
            assert float(f[4]) == o[int(f[1]), int(f[2]), int(f[3])]
        n += 1
    assert n == lse.size + o.size
    assert np.isfinite(o).all()
