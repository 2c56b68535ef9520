"""Planted mistakes: each one, put into a copy of the oracle on the CPU, must
fail at least one pin, so the pins would catch it in the oracle itself.

* C oracle (swa_sink_oracle.c, compiled with the mistake into a temporary
  library): window off by one, the sink left out of the denominator, a wrong
  query-head -> kv-head map, the decode ring's first key off by one, the LSE
  without the max. Pins: torch SDPA without a sink, the augmented softmax with
  one, brute force, decode = prefill.
* Backward oracle (oracle/backward.py, imported as a mutant module): Delta
  dropped from dS, dsink's sign flipped, dq without the scale, dk of a kv head
  overwritten instead of summed over its query heads, the sink left out of
  the denominator, the window off by one; in the key sums from a forward,
  p_sink dropped from dk, dv weighted by 1 instead of 1 - p_sink, query heads
  grouped by stride; in the sampled entry given a whole forward, o taken from
  the wrong head. Pins: torch autograd, finite differences of the C oracle,
  the zero-query closed form, the sampled entry and the key sums against the
  full backward.
* RoPE oracle (oracle/rope.py): the frequency exponent halved, the rotation's
  sign flipped, the rotate-half pairing replaced by the interleaved one. Pins:
  the complex-multiplication form, the closed forms, the invariants.
* FP8 oracle (oracle/fp8.py): the exponent bias, the tie rule, the K / V
  scale index, the encoder's sign, the commit slot. Pins: torch's E4M3
  decoding and cast, the midpoint ties, the C oracle on exactly representable
  rings, the per-head scales, the commit's slots and codes.
The unmutated oracles pass the same pin sets (checked first), so a failure
comes from the planted mistake.
"""
import importlib.util
import os
import subprocess

import pytest

import oracle
import oracle.oracle as core
import test_oracle as TO
import test_oracle_backward as TB
import test_oracle_fp8 as TF
import test_oracle_rope as TR

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_DIR = os.path.join(ROOT, "oracle")


def run_pins(pins):
    failed = []
    for name, fn in pins:
        try:
            fn()
        except Exception:  # an assertion, or anything the mistake breaks
            failed.append(name)
    return failed


# ---------------------------------------------------------------- C oracle --
C_PINS = [
    ("sdpa gqa", lambda: TO.test_no_sink_equals_sdpa([64], 8, 2, 32, 16)),
    ("sdpa global", lambda: TO.test_no_sink_equals_sdpa([130], 8, 1, 16, 0)),
    ("augmented softmax", lambda: TO.test_sink_equals_augmented_softmax(
        [50, 1, 23, 0, 70], 4, 2, 8, 12, "normal")),
    ("brute force", lambda: TO.test_brute_force_tiny(12, 2, 1, 8, 3, -1.5)),
    ("decode = prefill", lambda: TO.test_decode_equals_prefill_bitwise(4)),
]

C_MUTATIONS = {
    "window off by one": [("i - J->window + 1 > lo", "i - J->window > lo"),
                          ("lo = i - J->window + 1;", "lo = i - J->window;")],
    "sink left out of the denominator": [("double den = sink_term;", "double den = 0.0;")],
    "wrong q->kv head map": [("int g = h / G;", "int g = h % J->Hkv;")],
    "decode ring start off by one": [("int64_t first = P + t - J->W + 1;",
                                      "int64_t first = P + t - J->W + 2;")],
    "LSE without the max": [("*lse = m + log(den);", "*lse = log(den);")],
}


def build_c(tmp_path, edits):
    src = open(os.path.join(ORACLE_DIR, "swa_sink_oracle.c")).read()
    for old, new in edits:
        assert old in src, old
        src = src.replace(old, new)
    path = tmp_path / "mutant.c"
    path.write_text(src)
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o",
                           str(lib), str(path), "-lm"])
    return str(lib)


def use_c(monkeypatch, lib):
    monkeypatch.setattr(core, "_lib", None)
    monkeypatch.setattr(core, "build", lambda *a, **k: lib)


def test_c_pins_pass_unmutated(tmp_path, monkeypatch):
    use_c(monkeypatch, build_c(tmp_path, []))
    assert run_pins(C_PINS) == []


@pytest.mark.parametrize("mistake", sorted(C_MUTATIONS))
def test_c_mistake_fails_a_pin(mistake, tmp_path, monkeypatch):
    use_c(monkeypatch, build_c(tmp_path, C_MUTATIONS[mistake]))
    assert run_pins(C_PINS), mistake


# ------------------------------------------------------- Python oracles -----
def load_mutant(module, edits, tmp_path):
    src = open(os.path.join(ORACLE_DIR, module + ".py")).read()
    for old, new in edits:
        assert old in src, old
        src = src.replace(old, new)
    path = tmp_path / (module + "_mutant.py")
    path.write_text(src)
    spec = importlib.util.spec_from_file_location("oracle._mutant_" + module, str(path))
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"  # its relative imports resolve inside the package
    spec.loader.exec_module(mod)
    return mod


BWD_PINS = [
    ("autograd gqa varlen", lambda: TB.test_backward_equals_autograd(*TB.CASES[1])),
    ("autograd global", lambda: TB.test_backward_equals_autograd(*TB.CASES[2])),
    ("autograd window 1", lambda: TB.test_backward_equals_autograd(*TB.CASES[3])),
    ("finite differences", lambda: TB.test_backward_finite_differences_of_the_c_oracle(6)),
    ("zero query", TB.test_backward_zero_query_closed_form),
    ("sampled entry", lambda: TB.test_sampled_entry_and_dsink_from_forward(7)),
    ("key sums", lambda: TB.test_key_sums_from_forward_equal_the_full_backward(7, "normal")),
    ("key sums global", lambda: TB.test_key_sums_from_forward_equal_the_full_backward(
        0, "uniform2")),
]

BWD_MUTATIONS = {
    "Delta dropped from dS": [("da = p * (do_ @ v_.T - delta[:, None])", "da = p * (do_ @ v_.T)")],
    "dsink sign flipped": [("dsink[h] += -(psink * delta).sum()",
                            "dsink[h] += (psink * delta).sum()")],
    "dq without the scale": [("dq[lo:hi, h] = sc * (da @ k_)", "dq[lo:hi, h] = da @ k_")],
    "dk overwritten, not summed over the group": [("dk[lo:hi, g] += sc * (da.T @ q_)",
                                                   "dk[lo:hi, g] = sc * (da.T @ q_)")],
    "sink left out of the denominator": [("den = e.sum(axis=1) + es", "den = e.sum(axis=1)")],
    "window off by one": [("vis &= j >= i - window + 1", "vis &= j >= i - window")],
    "key sums: p_sink dropped from dk": [("wk = (sc * delta * ps)[:, :, None] * Q",
                                          "wk = (sc * delta)[:, :, None] * Q")],
    "key sums: dv weighted by 1, not 1 - p_sink": [("wv = (1.0 - ps)[:, :, None] * dO",
                                                    "wv = dO")],
    "key sums: query heads grouped by stride": [(".reshape(Hkv, G, D).sum(axis=1)",
                                                 ".reshape(G, Hkv, D).sum(axis=0)")],
    "sampled entry: o of the group's first head": [
        ("o, lse = forward[0][rt, rh], forward[1][rh, rt]",
         "o, lse = forward[0][rt, rh // G * G], forward[1][rh, rt]")],
}


def test_backward_pins_pass_unmutated(tmp_path, monkeypatch):
    monkeypatch.setattr(TB, "ob", load_mutant("backward", [], tmp_path))
    assert run_pins(BWD_PINS) == []


@pytest.mark.parametrize("mistake", sorted(BWD_MUTATIONS))
def test_backward_mistake_fails_a_pin(mistake, tmp_path, monkeypatch):
    monkeypatch.setattr(TB, "ob", load_mutant("backward", BWD_MUTATIONS[mistake], tmp_path))
    assert run_pins(BWD_PINS), mistake


ROPE_PINS = [
    ("complex form", lambda: TR.test_rotation_is_complex_multiplication(64, 640000.0, False)),
    ("complex form interleaved",
     lambda: TR.test_rotation_is_complex_multiplication(128, 1e4, True)),
    ("closed forms", TR.test_rotation_closed_forms),
    ("invariants", lambda: TR.test_rotation_invariants(False)),
]

ROPE_MUTATIONS = {
    "frequency exponent halved": [("np.power(float(base), -2.0 * c / D)",
                                   "np.power(float(base), -1.0 * c / D)")],
    "rotation sign flipped": [("out[..., a] = x[..., a] * cs - x[..., b] * sn",
                               "out[..., a] = x[..., a] * cs + x[..., b] * sn"),
                              ("out[..., b] = x[..., b] * cs + x[..., a] * sn",
                               "out[..., b] = x[..., b] * cs - x[..., a] * sn")],
    "rotate-half pairing replaced": [("    return c, c + D // 2\n",
                                      "    return 2 * c, 2 * c + 1\n")],
}


def test_rope_pins_pass_unmutated(tmp_path, monkeypatch):
    monkeypatch.setattr(TR, "rope", load_mutant("rope", [], tmp_path))
    assert run_pins(ROPE_PINS) == []


@pytest.mark.parametrize("mistake", sorted(ROPE_MUTATIONS))
def test_rope_mistake_fails_a_pin(mistake, tmp_path, monkeypatch):
    monkeypatch.setattr(TR, "rope", load_mutant("rope", ROPE_MUTATIONS[mistake], tmp_path))
    assert run_pins(ROPE_PINS), mistake


FP8_PINS = [
    ("table = torch", TF.test_table_matches_torch),
    ("encode = torch cast", TF.test_encode_matches_torch_random),
    ("midpoints to even", TF.test_encode_midpoints_ties_to_even),
    ("exact rings = C oracle", lambda: TF.test_decode_fp8_equals_c_oracle_on_exact_rings(16, 0, 40)),
    ("per-head scales", TF.test_dequantize_applies_per_head_scales),
    ("commit slots and codes", TF.test_kv_commit_fp8_slots_and_codes),
]

FP8_MUTATIONS = {
    "exponent bias": [("(1.0 + m / 8.0) * 2.0 ** (e - 7)", "(1.0 + m / 8.0) * 2.0 ** (e - 8)")],
    "tie rule": [("(lo if lo % 2 == 0 else hi)", "(hi if lo % 2 == 0 else lo)")],
    "K and V scales swapped": [("[which * Hkv:(which + 1) * Hkv]",
                                "[(1 - which) * Hkv:(2 - which) * Hkv]")],
    "encoder drops the sign": [("res[n] = c | (0x80 if", "res[n] = c | (0x00 if")],
    "commit slot off by one": [("slot = (int(pos[b]) + u) % W", "slot = (int(pos[b]) + u + 1) % W")],
}


def test_fp8_pins_pass_unmutated(tmp_path, monkeypatch):
    monkeypatch.setattr(TF, "fp8", load_mutant("fp8", [], tmp_path))
    assert run_pins(FP8_PINS) == []


@pytest.mark.parametrize("mistake", sorted(FP8_MUTATIONS))
def test_fp8_mistake_fails_a_pin(mistake, tmp_path, monkeypatch):
    monkeypatch.setattr(TF, "fp8", load_mutant("fp8", FP8_MUTATIONS[mistake], tmp_path))
    assert run_pins(FP8_PINS), mistake


def test_the_real_oracle_is_back(tmp_path):
    """After the mutants, the package oracle still loads its own library."""
    assert oracle.oracle._lib is None or os.path.basename(
        oracle.oracle.build()) == "liboracle.so"
