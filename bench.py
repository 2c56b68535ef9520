"""Benchmark of the sliding-window / global attention with a per-head sink on
B200, through the C ABI of libswasink.so.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

One JSON line on rank 0. A step is one call of the hot path over the
workload's whole batch (default: one SWA layer, T=32768, Hq=64, Hkv=8, D=128,
W=128). `value` is whole-job throughput from CUDA events with the inputs
resident in HBM; `e2e` adds the host->device copy of the inputs from pinned
memory and the device->host copy of the outputs, per step. With N > 1 (one
process per GPU under torch.distributed.run) every rank runs its own replica
of the workload on its own seeded inputs (independent sequences: no
collective on the data path), timing is the max over ranks, and `value`
counts the work of all ranks (weak scaling).

`--impl reference` times the fp64 CPU oracle instead, on bounded samples of
the same workload (rank 0 only; the other ranks exit at once).
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SWA+sink attention TFLOP/s (prefill), GB/s (decode); % of 1×B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- work model --
def prefill_work(seqlens, Hq, Hkv, D, window):
    """Algorithmic FLOPs and bytes of one prefill call: FLOPs = 4*D*Hq*pairs
    (QK^T and PV over the visible (query, key) pairs; softmax not counted);
    bytes = read q, k, v, sink, cu_seqlens once + write o, lse once."""
    pairs = 0
    for L in seqlens:
        if window > 0 and window < L:
            pairs += window * (window + 1) // 2 + (L - window) * window
        else:
            pairs += L * (L + 1) // 2
    total = sum(seqlens)
    flops = 4 * D * Hq * pairs
    nbytes = (total * Hq * D * 2 * 2          # q read, o write
              + total * Hkv * D * 2 * 2      # k, v read
              + Hq * total * 4               # lse write
              + Hq * 4 + (len(seqlens) + 1) * 4)
    return flops, nbytes


def backward_work(seqlens, Hq, Hkv, D, window):
    """Algorithmic FLOPs and bytes of one backward call: FLOPs = 10*D*Hq*pairs
    (five contractions over the visible pairs: S recomputed, dP = dO V^T,
    dV = P^T dO, dQ = dS K, dK = dS^T Q); bytes = read q, k, v, o, dO, lse,
    sink, cu_seqlens once + write dq, dk, dv, dsink once."""
    f_fwd, _ = prefill_work(seqlens, Hq, Hkv, D, window)
    total = sum(seqlens)
    nbytes = (total * Hq * D * 2 * 4          # q, o, dO read; dq written
              + total * Hkv * D * 2 * 4      # k, v read; dk, dv written
              + Hq * total * 4               # lse read
              + Hq * 4 * 2 + (len(seqlens) + 1) * 4)
    return f_fwd * 5 // 2, nbytes


def decode_work(pos, n_q, Hq, Hkv, D, W, kv_bytes=2, Hkv_scales=0):
    """FLOPs over visible pairs; bytes = the cached K/V rows of committed
    tokens (min(pos, W) per sequence, kv_bytes per element: 2 for bf16, 1 for
    E4M3 codes) + new K/V + q + pos + sink (+ the FP8 scales) read once,
    o + lse written once."""
    pairs = 0
    cached = 0
    for P in pos:
        cached += min(P, W)
        for t in range(n_q):
            pairs += min(P, max(0, W - 1 - t)) + (t + 1)   # ring keys + new keys 0..t
    B = len(pos)
    flops = 4 * D * Hq * pairs
    nbytes = (cached * Hkv * D * kv_bytes * 2 + B * n_q * Hkv * D * 2 * 2
              + B * n_q * Hq * D * 2 * 2 + B * n_q * Hq * 4 + B * 4 + Hq * 4
              + Hkv_scales * 2 * 4)
    return flops, nbytes


def decode_work_of(d, fp8):
    return decode_work(d["pos"].tolist(), d["n_q"], d["Hq"], d["Hkv"], d["D"], d["W"],
                       kv_bytes=1 if fp8 else 2, Hkv_scales=d["Hkv"] if fp8 else 0)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# The device sources (and the launch code in swa_sink.cu) that decide each
# workload's kernel; a recorded DRAM traffic figure holds only while they are
# unchanged.
KERNEL_SOURCES = {
    "ring": ["prefill_swa_ring_sm100.cuh", "prefill_sm100.cuh", "ptx_sm100.cuh", "swa_sink.cu"],
    "ring_rope": ["prefill_swa_ring_sm100.cuh", "rope_sm100.cuh", "prefill_sm100.cuh",
                  "ptx_sm100.cuh", "swa_sink.cu"],
    "chunked": ["prefill_chunked_sm100.cuh", "prefill_sm100.cuh", "ptx_sm100.cuh", "swa_sink.cu"],
    "chunked_rope": ["prefill_chunked_sm100.cuh", "rope_sm100.cuh", "prefill_sm100.cuh",
                     "ptx_sm100.cuh", "swa_sink.cu"],
    "backward": ["backward_sm100.cuh", "prefill_sm100.cuh", "ptx_sm100.cuh", "swa_sink.cu"],
    "decode": ["decode_tc_sm100.cuh", "decode_sm100.cuh", "ptx_sm100.cuh", "swa_sink.cu"],
    "decode_fp8": ["decode_fp8_sm100.cuh", "decode_sm100.cuh", "ptx_sm100.cuh", "swa_sink.cu"],
    "splitkv": ["decode_splitkv_tc_sm100.cuh", "decode_splitkv_sm100.cuh", "decode_tc_sm100.cuh",
                "decode_sm100.cuh", "ptx_sm100.cuh", "swa_sink.cu"],
}
WORKLOAD_KERNEL = {"tiny_swa_prefill": "ring", "swa_prefill_32k": "ring",
                   "swa_prefill_32k_rope": "ring_rope", "global_prefill_8k_rope": "chunked_rope",
                   "swa_backward_32k": "backward", "global_backward_8k": "backward",
                   "varlen_swa_prefill": "ring", "global_prefill_8k": "chunked",
                   "swa_decode_mtp": "decode", "ga_decode_16k": "splitkv",
                   "swa_decode_mtp_fp8": "decode_fp8"}


def kernel_source_hash(workload):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sliding_window_attention_sink_b200", "csrc")
    for fn in KERNEL_SOURCES[WORKLOAD_KERNEL[workload]]:
        h.update(open(os.path.join(csrc, fn), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current sources of the workload's kernel; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path)).get(workload)
    except Exception:
        return None
    if not rec or rec.get("source_hash") != kernel_source_hash(workload):
        return None
    return rec.get("dram_bytes_per_launch")


# -------------------------------------------------------------------- clocks --
class ClockSampler:
    """nvidia-smi samples (50 ms) of this process's GPU during the timed region."""

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + q,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ workloads --
def describe_prefill(c):
    out = {"Hq": c["Hq"], "Hkv": c["Hkv"], "head_dim": c["D"], "window": c["window"],
           "num_seqs": len(c["seqlens"]), "tokens": c["total"]}
    if c["rope_base"] > 0:
        out.update(rope_base=c["rope_base"], ring=c["ring_W"])
    if c["backward"]:
        out["pass"] = "backward"
    return out


def describe_decode(d, full, fp8):
    out = {"batch": d["B"], "n_q": d["n_q"], "Hq": d["Hq"], "Hkv": d["Hkv"],
           "head_dim": d["D"], ("cache" if full else "ring"): d["W"]}
    if fp8:
        out["kv_cache"] = "e4m3, one fp32 scale per kv head for K and for V"
    return out


def decode_sets(full):
    """Input sets the decode timing rotates over (the SWA batch is near L2)."""
    return 1 if full else 3


def l2_note(nbytes, nsets=1):
    if nsets > 1:
        return ("%d input sets rotated, %.0f MB each, %.0f MB together (> L2): a step's inputs "
                "are not L2-resident" % (nsets, nbytes / 1e6, nsets * nbytes / 1e6))
    return "inputs larger than L2 (%.0f MB per step)" % (nbytes / 1e6)


def workload_config(case, wl, world, c=None):
    """The bench line's config for a workload (both arms print the same)."""
    c = c if c is not None else _cached_inputs_of(case, wl)
    if isinstance(case, wl.PrefillCase):
        if c["backward"]:
            _, nbytes = backward_work(c["seqlens"], c["Hq"], c["Hkv"], c["D"], c["window"])
        else:
            _, nbytes = prefill_work(c["seqlens"], c["Hq"], c["Hkv"], c["D"], c["window"])
            if c["rope_base"] > 0:
                nbytes += sum(min(L, c["ring_W"]) for L in c["seqlens"]) * c["Hkv"] * c["D"] * 4
        desc, note = describe_prefill(c), l2_note(nbytes)
    else:
        full, fp8 = case.cache == "full", case.kv == "fp8"
        _, nbytes = decode_work_of(c, fp8)
        desc, note = describe_decode(c, full, fp8), l2_note(nbytes, decode_sets(full))
    return dict({"workload": case.name, "parallelism": "replicas" if world == 1 else
                 "dp%d" % world, "l2": note}, **desc)


def percentiles(values):
    """p10, median and p90 of per-call durations (p10 and p90 by nearest rank
    on the sorted values)."""
    v = sorted(values)
    n = len(v)

    def rank(p):
        return v[min(n - 1, max(0, int(math.ceil(p * n)) - 1))]
    return {"p10": rank(0.10), "median": statistics.median(v), "p90": rank(0.90)}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


class PrefillRunner:
    def __init__(self, case, rank, torch, B, wl):
        self.torch, self.B = torch, B
        case = wl.PrefillCase(**{**case.__dict__, "seed": case.seed + 1000 * rank})
        c = wl.make_prefill(case)
        self.c = c
        self.flops, self.bytes = prefill_work(c["seqlens"], c["Hq"], c["Hkv"], c["D"],
                                              c["window"])
        self.rope = c["rope_base"] > 0
        self.backward = c["backward"]
        if self.backward:
            self.flops, self.bytes = backward_work(c["seqlens"], c["Hq"], c["Hkv"], c["D"],
                                                   c["window"])
        dev = torch.device("cuda")
        self.k_ring = self.v_ring = self.ws = None
        if self.rope:
            # the ring the call writes: rotated K and V of each sequence's last
            # ring_W tokens
            S, W = len(c["seqlens"]), c["ring_W"]
            self.k_ring = torch.empty((S, W, c["Hkv"], c["D"]), dtype=torch.bfloat16, device=dev)
            self.v_ring = torch.empty_like(self.k_ring)
            self.bytes += sum(min(L, W) for L in c["seqlens"]) * c["Hkv"] * c["D"] * 2 * 2
            need = B.swa_sink_attn_fwd_rope_workspace(c["total"], c["Hq"], c["Hkv"], c["D"],
                                                      c["window"])
            self.ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
            self.rope_pass = need > 0  # a rotation pass into the workspace, then the prefill
        self.q, self.k, self.v = c["q"].to(dev), c["k"].to(dev), c["v"].to(dev)
        self.cu = c["cu_seqlens"].to(dev)
        self.sink = c["sink"].to(dev) if c["sink"] is not None else None
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((c["Hq"], c["total"]), dtype=torch.float32, device=dev)
        # pinned host copies for the end-to-end leg
        self.h_in = [c["q"].pin_memory(), c["k"].pin_memory(), c["v"].pin_memory(),
                     c["cu_seqlens"].pin_memory()]
        self.d_in = [self.q, self.k, self.v, self.cu]
        if c["sink"] is not None:
            self.h_in.append(c["sink"].pin_memory())
            self.d_in.append(self.sink)
        self.h_out = [torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory(),
                      torch.empty(self.lse.shape, dtype=self.lse.dtype).pin_memory()]
        self.d_out = [self.o, self.lse]
        if self.backward:
            # the forward's o and lse (outside the timed region), then the
            # backward's inputs and outputs
            B.attn_fwd(self.q, self.k, self.v, self.cu, c["window"], sink=self.sink,
                       max_seqlen=c["max_seqlen"], out=self.o, lse=self.lse)
            torch.cuda.synchronize()
            self.dout = c["dout"].to(dev)
            self.dq, self.dk, self.dv = (torch.empty_like(self.q), torch.empty_like(self.k),
                                         torch.empty_like(self.v))
            self.dsink = torch.empty((c["Hq"],), dtype=torch.float32, device=dev)
            need = B.swa_sink_attn_bwd_workspace(c["total"], c["Hq"])
            self.bws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
            self.h_in += [self.o.cpu().pin_memory(), self.lse.cpu().pin_memory(),
                          c["dout"].pin_memory()]
            self.d_in += [self.o, self.lse, self.dout]
            self.h_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory()
                          for t in (self.dq, self.dk, self.dv, self.dsink)]
            self.d_out = [self.dq, self.dk, self.dv, self.dsink]
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in)
        self.d2h = sum(t.numel() * t.element_size() for t in self.h_out)
        self.units = c["total"]
        self.rope_fused = False  # RoPE: rotate inside the ring kernel, no workspace
        self.launches_per_call = 2 if getattr(self, "rope_pass", False) else 1
        if self.backward:
            self.launches_per_call = 2  # dq (with Delta and dsink), dk and dv

    def call(self, stream):
        c = self.c
        if self.backward:
            rc = self.B.swa_sink_attn_bwd(
                self.q, self.k, self.v, self.o, self.dout, self.lse, self.cu, len(c["seqlens"]),
                c["max_seqlen"], c["total"], c["Hq"], c["Hkv"], c["D"], c["window"], self.sink,
                0.0, self.dq, self.dk, self.dv, self.dsink, self.bws, self.bws.numel(), stream)
            if rc != 0:
                raise RuntimeError("swa_sink_attn_bwd: %s" % self.B.status_string(rc))
            return
        if self.rope:
            ws = None if self.rope_fused else self.ws
            rc = self.B.swa_sink_attn_fwd_rope(
                self.q, self.k, self.v, self.cu, len(c["seqlens"]), c["max_seqlen"], c["total"],
                c["Hq"], c["Hkv"], c["D"], c["window"], self.sink, 0.0, c["rope_base"], 0, None,
                self.k_ring, self.v_ring, c["ring_W"], ws, 0 if ws is None else ws.numel(),
                self.o, self.lse, stream)
            if rc != 0:
                raise RuntimeError("swa_sink_attn_fwd_rope: %s" % self.B.status_string(rc))
            return
        rc = self.B.swa_sink_attn_fwd(self.q, self.k, self.v, self.cu, len(c["seqlens"]),
                                      c["max_seqlen"], c["total"], c["Hq"], c["Hkv"], c["D"],
                                      c["window"], self.sink, 0.0, self.o, self.lse, stream)
        if rc != 0:
            raise RuntimeError("swa_sink_attn_fwd: %s" % self.B.status_string(rc))

    def describe(self):
        return describe_prefill(self.c)


class DecodeRunner:
    """The SWA decode batch reads ~170 MB, close to the 126 MB L2, so the
    timed steps rotate over three independent input sets (> 500 MB together);
    a global-layer batch (cache "full", split-KV call) is far larger than L2."""

    def __init__(self, case, rank, torch, B, wl):
        self.torch, self.B = torch, B
        case = wl.DecodeCase(**{**case.__dict__, "seed": case.seed + 1000 * rank})
        d = wl.make_decode(case)
        self.d = d
        self.fp8 = case.kv == "fp8"
        self.flops, self.bytes = decode_work_of(d, self.fp8)
        dev = torch.device("cuda")
        names = ["q", "k_new", "v_new", "k_ring", "v_ring", "pos", "sink"]
        if self.fp8:
            names.append("kv_scale")
        self.g = {n: d[n].to(dev) for n in names}
        self.full = case.cache == "full"
        self.max_ctx = case.pos_hi
        self.NSETS = decode_sets(self.full)
        self.sets = [self.g] + [{n: (t.clone() if n != "pos" else t) for n, t in self.g.items()}
                                for _ in range(self.NSETS - 1)]
        self.ws = None
        if self.full:
            need = B.swa_sink_decode_splitkv_workspace(d["B"], d["n_q"], d["Hq"], d["Hkv"],
                                                       d["D"], d["W"], self.max_ctx)
            self.ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
            self.rope_pass = need > 0  # a rotation pass into the workspace, then the prefill
        self.turn = 0
        self.o = torch.empty_like(self.g["q"])
        self.lse = torch.empty((d["B"], d["n_q"], d["Hq"]), dtype=torch.float32, device=dev)
        self.h_in = [d[n].pin_memory() for n in names]
        self.d_in = [self.g[n] for n in names]
        self.h_out = [torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory(),
                      torch.empty(self.lse.shape, dtype=self.lse.dtype).pin_memory()]
        self.d_out = [self.o, self.lse]
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in)
        self.d2h = sum(t.numel() * t.element_size() for t in self.h_out)
        self.units = d["B"]
        self.launches_per_call = 2 if getattr(self, "full", False) else 1

    def call(self, stream):
        d, g = self.d, self.sets[self.turn]
        self.turn = (self.turn + 1) % self.NSETS
        if self.full:
            rc = self.B.swa_sink_attn_decode_splitkv(
                g["q"], g["k_new"], g["v_new"], g["k_ring"], g["v_ring"], g["pos"], d["B"],
                d["n_q"], d["Hq"], d["Hkv"], d["D"], d["W"], self.max_ctx, g["sink"], 0.0,
                self.o, self.lse, self.ws, self.ws.numel(), stream)
            if rc != 0:
                raise RuntimeError("swa_sink_attn_decode_splitkv: %s" % self.B.status_string(rc))
            return
        if self.fp8:
            rc = self.B.swa_sink_attn_decode_fp8kv(
                g["q"], g["k_new"], g["v_new"], g["k_ring"], g["v_ring"], g["kv_scale"],
                g["pos"], d["B"], d["n_q"], d["Hq"], d["Hkv"], d["D"], d["W"], g["sink"], 0.0,
                self.o, self.lse, stream)
            if rc != 0:
                raise RuntimeError("swa_sink_attn_decode_fp8kv: %s" % self.B.status_string(rc))
            return
        rc = self.B.swa_sink_attn_decode(g["q"], g["k_new"], g["v_new"], g["k_ring"],
                                         g["v_ring"], g["pos"], d["B"], d["n_q"], d["Hq"],
                                         d["Hkv"], d["D"], d["W"], g["sink"], 0.0, self.o,
                                         self.lse, stream)
        if rc != 0:
            raise RuntimeError("swa_sink_attn_decode: %s" % self.B.status_string(rc))

    def describe(self):
        return describe_decode(self.d, self.full, self.fp8)


# ------------------------------------------------------------ oracle timing --
_INPUTS = {}


def _cached_inputs_of(case, wl):
    key = repr(case)
    if key not in _INPUTS:
        _INPUTS[key] = (wl.make_prefill(case) if isinstance(case, wl.PrefillCase)
                        else wl.make_decode(case))
    return _INPUTS[key]


def _cached_inputs(workload, wl):
    return _cached_inputs_of(wl.WORKLOADS[workload], wl)


def oracle_sample(workload, wl, seconds, threads, seed=0, full_if_within=0.0):
    """Time the fp64 oracle on a bounded sample of the workload (about
    `seconds` of work), or on all of it when a whole pass is estimated to take
    at most `full_if_within` seconds. Returns (flops_done, bytes_equiv,
    elapsed_s, description, threads used)."""
    import numpy as np
    import oracle
    case = wl.WORKLOADS[workload]
    rng = np.random.default_rng(seed)
    if isinstance(case, wl.PrefillCase):
        c = _cached_inputs(workload, wl)
        F, Bt = prefill_work(c["seqlens"], c["Hq"], c["Hkv"], c["D"], c["window"])
        total_rows = c["total"] * c["Hq"]

        if c["backward"]:
            F, Bt = backward_work(c["seqlens"], c["Hq"], c["Hkv"], c["D"], c["window"])
            F, Bt = F * 3 // 5, Bt * 3 // 5  # the dq side the sample runs

        def run(n):
            rt = rng.integers(0, c["total"], n)
            rh = rng.integers(0, c["Hq"], n).astype(np.int32)
            t0 = time.perf_counter()
            if c["backward"]:
                # dq at n rows: three of the backward's five contractions
                # (S, dP, dQ) over those rows' pairs
                from oracle import backward as obw
                obw.prefill_backward_rows(c["q"], c["k"], c["v"], c["dout"], c["cu_seqlens"],
                                          c["Hq"], c["Hkv"], c["D"], c["window"], rt, rh,
                                          np.zeros(0, np.int64), np.zeros(0, np.int64),
                                          sink=c["sink"], nthreads=threads)
            elif c["rope_base"] > 0:
                from oracle import rope as orope
                orope.prefill_rope_rows(c["q"], c["k"], c["v"], c["cu_seqlens"], c["Hq"],
                                        c["Hkv"], c["D"], c["window"], c["rope_base"], rt, rh,
                                        sink=c["sink"], nthreads=threads)
            else:
                oracle.prefill_rows(c["q"], c["k"], c["v"], c["cu_seqlens"], c["Hq"], c["Hkv"],
                                    c["D"], c["window"], rt, rh, sink=c["sink"],
                                    nthreads=threads)
            return time.perf_counter() - t0
        unit = ("random (token, head) rows of dq (3 of the 5 backward contractions)"
                if c["backward"] else "random (token, head) rows")
    else:
        d = _cached_inputs(workload, wl)
        fp8 = case.kv == "fp8"
        F, Bt = decode_work_of(d, fp8)
        total_rows = d["B"]
        if fp8:
            from oracle import fp8 as ofp8
            threads = 1  # numpy, one thread

        def run(n):
            idx = np.sort(rng.choice(d["B"], size=min(n, d["B"]), replace=False))
            sub = {k: (d[k][idx] if k in ("q", "k_new", "v_new", "k_ring", "v_ring", "pos")
                       else d[k]) for k in d}
            t0 = time.perf_counter()
            if fp8:
                f64 = lambda t: t.double().numpy()  # noqa: E731
                ofp8.decode_fp8(f64(sub["q"]), f64(sub["k_new"]), f64(sub["v_new"]),
                                sub["k_ring"].numpy(), sub["v_ring"].numpy(),
                                d["kv_scale"].numpy(), sub["pos"].numpy(), len(idx), d["n_q"],
                                d["Hq"], d["Hkv"], d["D"], d["W"], sink=d["sink"].numpy())
            else:
                oracle.decode(sub["q"], sub["k_new"], sub["v_new"], sub["k_ring"],
                              sub["v_ring"], sub["pos"], len(idx), d["n_q"], d["Hq"], d["Hkv"],
                              d["D"], d["W"], sink=d["sink"], nthreads=threads)
            return time.perf_counter() - t0
        unit = "sequences"
    # calibrate on a small sample, then size the timed sample to `seconds`
    n0 = max(1, min(total_rows, 2000 if unit != "sequences" else 4))
    t_cal = run(n0)
    if t_cal * total_rows / n0 <= full_if_within:
        n = total_rows
    else:
        n = int(min(total_rows, max(n0, n0 * seconds / max(t_cal, 1e-3))))
    elapsed = run(n)
    frac = n / total_rows
    return F * frac, Bt * frac, elapsed, "%d of %d %s of %s, %d threads" % (
        n, total_rows, unit, workload, threads), threads


def run_reference(args, wl):
    """The reference arm: the fp64 CPU oracle as it stands. Each timed step is
    the whole workload when all steps together stay within about four minutes
    (the SWA layer: about 7 s a pass on 16 threads), else a bounded sample of
    it; warm-up steps are short samples."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    if args.steps <= 0:
        args.steps = 3
    import oracle
    threads = oracle.default_threads()
    case = wl.WORKLOADS[args.workload]
    is_prefill = isinstance(case, wl.PrefillCase)
    per_step = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    full_within = 240.0 / max(1, args.steps)
    for _ in range(args.warmup):
        oracle_sample(args.workload, wl, 1.0, threads)
    flops = nb = el = 0.0
    desc = ""
    for s in range(args.steps):
        f, b, e, desc, threads_used = oracle_sample(args.workload, wl, per_step, threads,
                                                    seed=s + 1, full_if_within=full_within)
        flops += f
        nb += b
        el += e
    value = flops / el / 1e12 if is_prefill else nb / el / 1e9
    unit = "TFLOP/s" if is_prefill else "GB/s"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(case, wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": unit, "cores": threads_used, "kind": "oracle",
                         "cpu_model": cpu_model(), "sample": desc + " per step"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------- main --
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=0,
                    help="timed steps (default: about one second of work, at least 20)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="swa_prefill_32k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--rope-fused", action="store_true",
                    help="RoPE workloads of the ring kernel's shapes: pass no workspace, so "
                         "the ring kernel rotates q and k itself (default: the rotation pass "
                         "into the workspace, then the plain prefill)")
    ap.add_argument("--seqlen", type=int, default=0,
                    help="prefill workloads: replace the sequence lengths by one "
                         "sequence of this length (small cases for profiling)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    from sliding_window_attention_sink_b200 import workloads as wl
    if args.impl == "reference":
        run_reference(args, wl)
        return

    import torch
    import torch.distributed as dist
    from sliding_window_attention_sink_b200 import binding as B

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE %d" % (args.gpus, world))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    B.load()

    case = wl.WORKLOADS[args.workload]
    is_prefill = isinstance(case, wl.PrefillCase)
    if args.seqlen > 0 and is_prefill:
        import dataclasses
        case = dataclasses.replace(case, seqlens=[args.seqlen], varlen_draw=None,
                                   name="%s (T=%d)" % (case.name, args.seqlen))
        args.no_cpu_baseline = True
    runner = (PrefillRunner if is_prefill else DecodeRunner)(case, rank, torch, B, wl)
    if args.rope_fused and getattr(runner, "rope", False):
        runner.rope_fused = True
        runner.launches_per_call = 1
    stream = torch.cuda.Stream()
    sptr = stream.cuda_stream
    if args.steps <= 0:
        # about one second of timed work (enough clock samples), >= 20 steps,
        # sized from 20 back-to-back calls (one call alone also times its
        # launch)
        with torch.cuda.stream(stream):
            runner.call(sptr)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(20):
                runner.call(sptr)
            b.record(stream)
        torch.cuda.synchronize()
        per_call = max(a.elapsed_time(b) / 20.0, 1e-3)
        args.steps = int(max(20, min(100000, 1100.0 / per_call)))
        if world > 1:  # every rank must time the same number of steps
            t = torch.tensor([args.steps], device="cuda", dtype=torch.int64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            args.steps = int(t.item())

    # CPU baseline (rank 0, N = 1), before the GPU timing so it does not overlap
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        threads = oracle.default_threads()
        f, b, e, desc, threads = oracle_sample(args.workload, wl, args.cpu_seconds, threads)
        cpu = {"value": (f / e / 1e12) if is_prefill else (b / e / 1e9),
               "unit": "TFLOP/s" if is_prefill else "GB/s", "cores": threads,
               "cpu_model": cpu_model(), "kind": "oracle", "sample": desc + ", %.1f s" % e}
        # the same oracle on one core, a smaller bounded sample
        f, b, e, desc, _ = oracle_sample(args.workload, wl, args.cpu_seconds / 5, 1, seed=7)
        cpu["one_core"] = {"value": (f / e / 1e12) if is_prefill else (b / e / 1e9),
                           "unit": cpu["unit"], "cores": 1, "sample": desc + ", %.1f s" % e}

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # warm-up
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            runner.call(sptr)
    barrier()

    # timed region: K steps, one call each; the kernel's own duration from
    # event pairs around every EVERY-th call (events between all calls would
    # add their own gaps to the step time of short kernels such as the decode)
    every = 1 if args.steps < 160 else 8
    sampled = list(range(0, args.steps, every))
    ev = {s: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for s in sampled}
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        barrier()
        with torch.cuda.stream(stream):
            t_start.record(stream)
            for s in range(args.steps):
                pair = ev.get(s)
                if pair is not None:
                    pair[0].record(stream)
                runner.call(sptr)
                if pair is not None:
                    pair[1].record(stream)
            t_end.record(stream)
        barrier()
        time.sleep(0.3)
    total_ms = t_start.elapsed_time(t_end)
    kern_ms = [a.elapsed_time(b) for a, b in ev.values()]
    if world > 1:
        t = torch.tensor([total_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_per_step = total_ms / args.steps
    kern_avg = sum(kern_ms) / len(kern_ms)

    # end to end: pinned host inputs -> device, the call, outputs -> pinned host
    e2e = None
    if not args.no_e2e:
        e_steps = max(3, min(args.steps, 10))
        with torch.cuda.stream(stream):
            for _ in range(2):
                if hasattr(runner, "turn"):
                    runner.turn = 0
                for h, dd in zip(runner.h_in, runner.d_in):
                    dd.copy_(h, non_blocking=True)
                runner.call(sptr)
                for h, dd in zip(runner.h_out, runner.d_out):
                    h.copy_(dd, non_blocking=True)
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            for _ in range(e_steps):
                if hasattr(runner, "turn"):
                    runner.turn = 0   # the copies below refill input set 0
                for h, dd in zip(runner.h_in, runner.d_in):
                    dd.copy_(h, non_blocking=True)
                runner.call(sptr)
                for h, dd in zip(runner.h_out, runner.d_out):
                    h.copy_(dd, non_blocking=True)
            b.record(stream)
        barrier()
        e_ms = a.elapsed_time(b)
        if world > 1:
            t = torch.tensor([e_ms], device="cuda")
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t.item())
        e_step = e_ms / e_steps
        e_val = (runner.flops * world / (e_step * 1e-3) / 1e12) if is_prefill else (
            runner.bytes * world / (e_step * 1e-3) / 1e9)
        e2e = {"value": e_val, "unit": "TFLOP/s" if is_prefill else "GB/s",
               "ms_per_step": e_step, "h2d_bytes_per_step": runner.h2d * world,
               "d2h_bytes_per_step": runner.d2h * world}

    flag = B.swa_sink_device_error()
    peaks, src = load_peaks()
    if is_prefill:
        value = runner.flops * world / (ms_per_step * 1e-3) / 1e12
        unit = "TFLOP/s"
    else:
        value = runner.bytes * world / (ms_per_step * 1e-3) / 1e9
        unit = "GB/s"
    # roofline of the (only) kernel in the step: the slower of tensor and HBM time.
    # The tensor peak is the burst figure for a short timed region and the
    # sustained one (the power cap's steady state) for one of half a second
    # or more.
    sustained = total_ms >= 500.0 and "bf16_tflops_sustained" in peaks
    tensor_peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    t_tensor = runner.flops / (tensor_peak * 1e12)
    t_hbm = runner.bytes / (peaks["hbm_gbs"] * 1e9)
    if t_hbm >= t_tensor:
        achieved = runner.bytes / (kern_avg * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"]}
    else:
        achieved = runner.flops / (kern_avg * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tensor_peak,
                "unit": "TFLOP/s", "frac": achieved / tensor_peak,
                "peak_kind": "sustained" if sustained else "burst"}
    roof["peak_source"] = src
    roof["algorithmic_bytes"] = runner.bytes
    roof["algorithmic_flops"] = runner.flops
    roof["kernel_ms"] = kern_avg
    roof["kernel_timed_calls"] = len(kern_ms)  # calls with an event pair around them
    roof["kernel_ms_percentiles"] = percentiles(kern_ms)
    # (a record is for the workload's own sizes, not a --seqlen variant)
    roof["traffic"] = recorded_traffic(args.workload) if args.seqlen <= 0 else None

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": dict({"workload": case.name,
                            "parallelism": "replicas" if world == 1 else "dp%d" % world,
                            "l2": l2_note(runner.bytes, getattr(runner, "NSETS", 1))},
                           **runner.describe(),
                           **({"rope_route": "fused"} if getattr(runner, "rope_fused", False)
                              else {})),
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps * runner.launches_per_call, "clocks": clk.summary(), "device_error_flags": flag,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
