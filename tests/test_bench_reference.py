"""The reference arm's CPU sampling (bench.oracle_sample, which
`bench.py --impl reference` and the cpu_baseline leg time) on every workload
kind, each scaled down to a few hundred tokens or a few sequences so the
fp64 oracle finishes at once: same heads, window, RoPE, backward and FP8
settings. Checks the sample runs, reports work in proportion to the rows or
sequences it covered, and describes itself."""
import dataclasses
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from sliding_window_attention_sink_b200 import workloads as wl  # noqa: E402


def small(case):
    if isinstance(case, wl.PrefillCase):
        return dataclasses.replace(case, seqlens=[200, 57], varlen_draw=None, Hq=8, Hkv=2,
                                   ring_W=min(case.ring_W, 64) if case.ring_W else 0)
    return dataclasses.replace(case, B=3, Hq=8, Hkv=2,
                               W=min(case.W, 256), pos_lo=min(case.pos_lo, 100),
                               pos_hi=min(case.pos_hi, 250 if case.cache == "full" else 400))


@pytest.mark.parametrize("name", sorted(wl.WORKLOADS))
def test_oracle_sample_runs(name, monkeypatch):
    monkeypatch.setitem(wl.WORKLOADS, name, small(wl.WORKLOADS[name]))
    bench._INPUTS.clear()
    try:
        f, nbytes, el, desc, threads = bench.oracle_sample(name, wl, 0.05, 2, seed=1)
    finally:
        bench._INPUTS.clear()
    assert f > 0 and nbytes > 0 and el > 0 and threads >= 1
    assert name in desc
    # the work reported is the whole workload's times the fraction sampled
    words = desc.split()  # "<n> of <total> <unit> of <workload>, <threads> threads"
    n, total = int(words[0]), int(words[2])
    case = wl.WORKLOADS[name]
    if isinstance(case, wl.PrefillCase):
        c = bench._cached_inputs(name, wl)
        F, Bt = bench.prefill_work(c["seqlens"], c["Hq"], c["Hkv"], c["D"], c["window"])
        if c["backward"]:
            F, Bt = bench.backward_work(c["seqlens"], c["Hq"], c["Hkv"], c["D"], c["window"])
            F = F * 3 // 5
        bench._INPUTS.clear()
        assert total == sum(c["seqlens"]) * c["Hq"]
        assert f == pytest.approx(F * n / total)
    else:
        assert total == case.B and 1 <= n <= total


@pytest.mark.parametrize("name", ["swa_prefill_32k", "swa_decode_mtp"])
def test_reference_arm_line(name, monkeypatch, capsys):
    """--impl reference prints one JSON line with our arm's config (the same
    dict workload_config gives the GPU arm), the oracle's CPU model and core
    count, and covers the whole (scaled-down) workload each step."""
    import json
    import types
    monkeypatch.setitem(wl.WORKLOADS, name, small(wl.WORKLOADS[name]))
    bench._INPUTS.clear()
    monkeypatch.delenv("RANK", raising=False)
    args = types.SimpleNamespace(workload=name, steps=2, warmup=1, gpus=1)
    try:
        bench.run_reference(args, wl)
        line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
        assert line["impl"] == "reference" and line["steps"] == 2
        assert line["config"] == bench.workload_config(wl.WORKLOADS[name], wl, 1)
        cpu = line["cpu_baseline"]
        assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["cpu_model"]
        words = cpu["sample"].split()
        assert words[0] == words[2]  # "<n> of <total> ...": every row / sequence
        assert line["e2e"]["h2d_bytes_per_step"] == 0
    finally:
        bench._INPUTS.clear()
