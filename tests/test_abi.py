"""Host-side checks of the C ABI: the library loads and exports every symbol
include/swa_sink.h declares, and argument errors are returned before any
launch (these calls never reach the GPU, so they run without one)."""
import ctypes
import os
import re

import pytest

from sliding_window_attention_sink_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "swa_sink.h")


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"SWA_API\s+[\w\s\*]*?\b(swa_sink_\w+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    lib = B.load()
    names = declared_symbols()
    assert len(names) >= 6
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings():
    assert B.swa_sink_version() == 100
    assert B.status_string(0) == "ok"
    for code in (-1, -2, -3, -4, -5):
        assert B.status_string(code) != "unknown status"


FAKE = 0x10000  # a 16-byte aligned address that is never dereferenced


def fwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, cu_seqlens=FAKE, num_seqs=1, max_seqlen=8,
             total_tokens=8, Hq=8, Hkv=2, D=128, window=128, sink=None,
             softmax_scale=0.0, o=FAKE, lse=None, stream=0)
    a.update(kw)
    return B.swa_sink_attn_fwd(**a)


def test_fwd_argument_errors():
    assert fwd(Hq=8, Hkv=3) == -2
    assert fwd(total_tokens=-1) == -2
    assert fwd(num_seqs=-1) == -2
    assert fwd(num_seqs=0) == -2
    assert fwd(max_seqlen=9) == -2
    assert fwd(D=96) == -3
    assert fwd(Hq=256, Hkv=1) == -3
    assert fwd(q=None) == -1
    assert fwd(cu_seqlens=None) == -1
    assert fwd(o=FAKE + 2) == -4
    assert fwd(k=FAKE + 8) == -4
    assert fwd(lse=FAKE + 2) == -4
    assert fwd(total_tokens=0, max_seqlen=0) == 0   # nothing to do, nothing launched


def dec(**kw):
    a = dict(q=FAKE, k_new=FAKE, v_new=FAKE, k_ring=FAKE, v_ring=FAKE, pos=FAKE, B=4,
             n_q=4, Hq=64, Hkv=8, D=128, W=128, sink=None, softmax_scale=0.0, o=FAKE,
             lse=None, stream=0)
    a.update(kw)
    return B.swa_sink_attn_decode(**a)


def test_decode_argument_errors():
    assert dec(n_q=0) == -2
    assert dec(W=0) == -2
    assert dec(Hkv=7) == -2
    assert dec(n_q=9) == -3
    assert dec(W=257) == -3
    assert dec(Hq=128, Hkv=8, n_q=3) == -3   # 48 query rows per kv head
    assert dec(D=80) == -3
    assert dec(pos=None) == -1
    assert dec(k_ring=FAKE + 4) == -4
    assert dec(B=0) == 0


def test_commit_argument_errors():
    a = dict(k_ring=FAKE, v_ring=FAKE, k_new=FAKE, v_new=FAKE, pos=FAKE, n_accept=FAKE,
             B=2, n_q=4, Hkv=8, D=128, W=128, stream=0)
    assert B.swa_sink_kv_commit(**dict(a, n_q=0)) == -2
    assert B.swa_sink_kv_commit(**dict(a, D=32)) == -3
    assert B.swa_sink_kv_commit(**dict(a, n_accept=None)) == -1
    assert B.swa_sink_kv_commit(**dict(a, v_new=FAKE + 1)) == -4
    assert B.swa_sink_kv_commit(**dict(a, B=0)) == 0


def test_header_is_plain_c():
    """The header compiles as C99 with no CUDA or torch headers."""
    import subprocess
    import tempfile
    with tempfile.TemporaryDirectory() as td:
        src = os.path.join(td, "t.c")
        open(src, "w").write('#include "swa_sink.h"\nint main(void){return swa_sink_version()>0?0:1;}\n')
        r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only",
                            "-I", os.path.join(ROOT, "include"), src],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_fwd_noalloc_argument_errors():
    # the slot is checked first, then the arguments exactly as for
    # swa_sink_attn_fwd; none of these calls reaches CUDA
    a = dict(q=FAKE, k=FAKE, v=FAKE, cu_seqlens=FAKE, num_seqs=1, max_seqlen=8,
             total_tokens=8, Hq=8, Hkv=2, D=128, window=128, sink=None,
             softmax_scale=0.0, o=FAKE, lse=None, stream=0)
    assert B.swa_sink_attn_fwd_noalloc(slot=8, **a) == -2
    assert B.swa_sink_attn_fwd_noalloc(slot=-1, **a) == -2
    assert B.swa_sink_attn_fwd_noalloc(slot=0, **dict(a, Hq=8, Hkv=3)) == -2
    assert B.swa_sink_attn_fwd_noalloc(slot=7, **dict(a, D=96)) == -3
    assert B.swa_sink_attn_fwd_noalloc(slot=0, **dict(a, q=None)) == -1
    assert B.swa_sink_attn_fwd_noalloc(slot=0, **dict(a, o=FAKE + 2)) == -4
    assert B.swa_sink_attn_fwd_noalloc(slot=3, **dict(a, total_tokens=0, max_seqlen=0)) == 0


def test_splitkv_workspace_and_argument_errors():
    ws = B.swa_sink_decode_splitkv_workspace(4, 4, 64, 8, 128, 4096, 4000)
    assert ws > 0
    assert B.swa_sink_decode_splitkv_workspace(4, 4, 64, 8, 96, 4096, 4000) == 0
    a = dict(q=FAKE, k_new=FAKE, v_new=FAKE, k_cache=FAKE, v_cache=FAKE, pos=FAKE, B=4, n_q=4,
             Hq=64, Hkv=8, D=128, W=4096, max_ctx=4000, sink=None, softmax_scale=0.0, o=FAKE,
             lse=None, workspace=FAKE, workspace_bytes=ws, stream=0)
    f = B.swa_sink_attn_decode_splitkv
    assert f(**dict(a, W=4000)) == -3          # W not a multiple of 64
    assert f(**dict(a, workspace_bytes=ws - 1)) == -2
    assert f(**dict(a, workspace=None)) == -1
    assert f(**dict(a, workspace=FAKE + 4)) == -4
    assert f(**dict(a, n_q=9)) == -3
    assert f(**dict(a, Hq=64, Hkv=6)) == -2
    assert f(**dict(a, B=-1)) == -2
    assert f(**dict(a, max_ctx=-1)) == -2
    assert f(**dict(a, D=96)) == -3
    assert f(**dict(a, Hq=64, Hkv=4)) == -3   # 4 tokens x 16 heads: 64 query rows per kv head
    assert f(**dict(a, pos=None)) == -1
    assert f(**dict(a, q=FAKE + 8)) == -4
    assert f(**dict(a, pos=FAKE + 2)) == -4
    assert f(**dict(a, lse=FAKE + 2)) == -4
    assert f(**dict(a, sink=FAKE + 1)) == -4
    assert f(**dict(a, B=0)) == 0
    wsf = B.swa_sink_decode_splitkv_workspace
    for bad in (dict(B=-1), dict(n_q=0), dict(Hq=0), dict(Hkv=0), dict(W=0), dict(max_ctx=-1)):
        args = dict(B=4, n_q=4, Hq=64, Hkv=8, D=128, W=4096, max_ctx=4000)
        args.update(bad)
        assert wsf(**args) == 0, bad


def test_splitkv_workspace_of_the_global_layer_decode():
    # 16 sequences x 8 kv heads = 128 units; about 1184 CTAs wanted, so 10
    # ranges each; 16380 cached positions / 10 = 1638, rounded up to a whole
    # 64-position tile: ranges of 1664, 10 of them cover 16380. Each range
    # keeps 32 query rows of D + 4 floats (O, m, and the two sums).
    assert B.swa_sink_decode_splitkv_workspace(16, 4, 64, 8, 128, 16384, 16380) == (
        16 * 8 * 10 * 32 * (128 + 4) * 4)
    # one (sequence, kv head) and a short context: one range per 64 positions
    assert B.swa_sink_decode_splitkv_workspace(1, 1, 8, 1, 64, 4096, 200) == (
        1 * 1 * 4 * 32 * (64 + 4) * 4)


def test_fp8_decode_and_commit_argument_errors():
    a = dict(q=FAKE, k_new=FAKE, v_new=FAKE, k_ring=FAKE, v_ring=FAKE, kv_scale=FAKE, pos=FAKE,
             B=4, n_q=4, Hq=64, Hkv=8, D=128, W=128, sink=None, softmax_scale=0.0, o=FAKE,
             lse=None, stream=0)
    f = B.swa_sink_attn_decode_fp8kv
    assert f(**dict(a, kv_scale=None)) == -1
    assert f(**dict(a, kv_scale=FAKE + 2)) == -4
    assert f(**dict(a, k_ring=FAKE + 8)) == -4
    assert f(**dict(a, W=257)) == -3
    assert f(**dict(a, D=96)) == -3
    assert f(**dict(a, n_q=0)) == -2
    assert f(**dict(a, B=0, kv_scale=None)) == 0
    c = dict(k_ring=FAKE, v_ring=FAKE, k_new=FAKE, v_new=FAKE, kv_scale=FAKE, pos=FAKE,
             n_accept=FAKE, B=2, n_q=4, Hkv=8, D=128, W=128, stream=0)
    g = B.swa_sink_kv_commit_fp8
    assert g(**dict(c, kv_scale=None)) == -1
    assert g(**dict(c, kv_scale=FAKE + 1)) == -4
    assert g(**dict(c, v_ring=FAKE + 8)) == -4
    assert g(**dict(c, D=32)) == -3
    assert g(**dict(c, W=0)) == -2
    assert g(**dict(c, B=0)) == 0


def fwd_rope(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, cu_seqlens=FAKE, num_seqs=1, max_seqlen=8,
             total_tokens=8, Hq=8, Hkv=2, D=128, window=128, sink=None,
             softmax_scale=0.0, rope_base=1e4, rope_interleaved=0, pos0=None,
             k_ring=None, v_ring=None, ring_W=0, workspace=None, workspace_bytes=0,
             o=FAKE, lse=None, stream=0)
    a.update(kw)
    return B.swa_sink_attn_fwd_rope(**a)


def test_fwd_rope_argument_errors():
    assert fwd_rope(rope_base=0.0) == -2
    assert fwd_rope(rope_base=float("inf")) == -2
    assert fwd_rope(rope_base=float("nan")) == -2
    assert fwd_rope(rope_interleaved=2) == -2
    assert fwd_rope(k_ring=FAKE) == -1                     # v_ring missing
    assert fwd_rope(k_ring=FAKE, v_ring=FAKE, ring_W=0) == -2
    assert fwd_rope(k_ring=FAKE + 8, v_ring=FAKE, ring_W=4) == -4
    assert fwd_rope(pos0=FAKE + 2) == -4
    assert fwd_rope(Hq=8, Hkv=3) == -2
    assert fwd_rope(D=96) == -3
    assert fwd_rope(q=None) == -1
    # shapes that need a workspace: a global layer, G = 1
    assert fwd_rope(window=0) == -1
    assert fwd_rope(window=0, workspace=FAKE, workspace_bytes=16) == -2
    assert fwd_rope(window=0, workspace=FAKE + 4, workspace_bytes=1 << 20) == -4
    assert fwd_rope(Hq=2, Hkv=2) == -1
    # a ring shape given a workspace takes the two-pass route: it must be big
    # enough and aligned
    assert fwd_rope(workspace=FAKE, workspace_bytes=16) == -2
    assert fwd_rope(workspace=FAKE + 4, workspace_bytes=1 << 20) == -4
    assert fwd_rope(total_tokens=0, max_seqlen=0) == 0


def test_fwd_rope_workspace_sizes():
    ws = B.swa_sink_attn_fwd_rope_workspace
    # every shape: rotated q (padded to 256 bytes) + rotated k (ring shapes
    # may also be called without it)
    assert ws(32768, 64, 8, 128, 128) == 32768 * 64 * 128 * 2 + 32768 * 8 * 128 * 2
    assert ws(1000, 4, 2, 64, 20) == (1000 * 4 * 64 * 2 + 255) // 256 * 256 + 1000 * 2 * 64 * 2
    q_bytes = 8192 * 64 * 128 * 2
    assert ws(8192, 64, 8, 128, 0) == q_bytes + 8192 * 8 * 128 * 2
    assert ws(300, 2, 2, 64, 128) == (300 * 2 * 64 * 2 + 255) // 256 * 256 + 300 * 2 * 64 * 2
    assert ws(600, 8, 1, 64, 300) > 0          # window too wide for the ring
    assert ws(0, 64, 8, 128, 0) == 0


def bwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, dout=FAKE, lse=FAKE, cu_seqlens=FAKE, num_seqs=1,
             max_seqlen=8, total_tokens=8, Hq=8, Hkv=2, D=128, window=128, sink=None,
             softmax_scale=0.0, dq=FAKE, dk=FAKE, dv=FAKE, dsink=None, workspace=FAKE,
             workspace_bytes=1 << 20, stream=0)
    a.update(kw)
    return B.swa_sink_attn_bwd(**a)


def test_bwd_argument_errors():
    assert bwd(Hq=8, Hkv=3) == -2
    assert bwd(total_tokens=-1) == -2
    assert bwd(max_seqlen=9) == -2
    assert bwd(D=96) == -3
    assert bwd(Hq=96, Hkv=1) == -3          # Hq/Hkv must divide 64
    assert bwd(Hq=128, Hkv=1) == -3         # G = 128 does not divide 64
    assert bwd(lse=None) == -1
    assert bwd(dout=None) == -1
    assert bwd(dk=None) == -1
    assert bwd(workspace=None) == -1
    assert bwd(workspace_bytes=16) == -2
    assert bwd(dq=FAKE + 8) == -4
    assert bwd(lse=FAKE + 2) == -4
    assert bwd(workspace=FAKE + 4) == -4
    assert B.swa_sink_attn_bwd_workspace(8, 8) == 256
    assert B.swa_sink_attn_bwd_workspace(32768, 64) == 32768 * 64 * 4
    assert B.swa_sink_attn_bwd_workspace(0, 64) == 0
