"""Thin ctypes binding of libswasink.so (declared in include/swa_sink.h).

The functions named like the C entry points take torch tensors (or raw
integer device pointers) and only marshal arguments; every step of the
computation runs in the library's CUDA kernels. There is no CPU fallback: if
the library is missing, loading raises.

Convenience wrappers (`attn_fwd`, `attn_fwd_rope`, `attn_decode`, `kv_commit`, ...) allocate the
outputs with torch and raise `SwaSinkError` on a non-zero status.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libswasink.so")

SWA_OK = 0
_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float


class SwaSinkError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (what, status_string(status), status))


def load():
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            "libswasink.so not found at %s; build it with "
            "`python -m sliding_window_attention_sink_b200.build`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    lib.swa_sink_attn_fwd.restype = _i
    lib.swa_sink_attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp,
                                      _f, _vp, _vp, _vp]
    lib.swa_sink_attn_fwd_noalloc.restype = _i
    lib.swa_sink_attn_fwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                              _vp, _f, _vp, _vp, _i, _vp]
    lib.swa_sink_attn_fwd_rope_workspace.restype = ctypes.c_size_t
    lib.swa_sink_attn_fwd_rope_workspace.argtypes = [_i, _i, _i, _i, _i]
    lib.swa_sink_attn_fwd_rope.restype = _i
    lib.swa_sink_attn_fwd_rope.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp,
                                           _f, _f, _i, _vp, _vp, _vp, _i, _vp, ctypes.c_size_t,
                                           _vp, _vp, _vp]
    lib.swa_sink_attn_bwd_workspace.restype = ctypes.c_size_t
    lib.swa_sink_attn_bwd_workspace.argtypes = [_i, _i]
    lib.swa_sink_attn_bwd.restype = _i
    lib.swa_sink_attn_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                      _i, _vp, _f, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    lib.swa_sink_attn_decode.restype = _i
    lib.swa_sink_attn_decode.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                         _i, _vp, _f, _vp, _vp, _vp]
    lib.swa_sink_decode_splitkv_workspace.restype = ctypes.c_size_t
    lib.swa_sink_decode_splitkv_workspace.argtypes = [_i, _i, _i, _i, _i, _i, _i]
    lib.swa_sink_attn_decode_splitkv.restype = _i
    lib.swa_sink_attn_decode_splitkv.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                                 _i, _i, _i, _vp, _f, _vp, _vp, _vp,
                                                 ctypes.c_size_t, _vp]
    lib.swa_sink_kv_commit.restype = _i
    lib.swa_sink_kv_commit.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]
    lib.swa_sink_attn_decode_fp8kv.restype = _i
    lib.swa_sink_attn_decode_fp8kv.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i,
                                               _i, _i, _i, _vp, _f, _vp, _vp, _vp]
    lib.swa_sink_kv_commit_fp8.restype = _i
    lib.swa_sink_kv_commit_fp8.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                           _i, _vp]
    lib.swa_sink_status_string.restype = ctypes.c_char_p
    lib.swa_sink_status_string.argtypes = [_i]
    lib.swa_sink_device_error.restype = _i
    lib.swa_sink_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint), _i]
    lib.swa_sink_version.restype = _i
    lib.swa_sink_version.argtypes = []
    _lib = lib
    return lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def status_string(status):
    return load().swa_sink_status_string(int(status)).decode()


# ---- same names as the C ABI -------------------------------------------------

def swa_sink_attn_fwd(q, k, v, cu_seqlens, num_seqs, max_seqlen, total_tokens, Hq, Hkv, D,
                      window, sink, softmax_scale, o, lse, stream=None):
    return load().swa_sink_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), int(num_seqs), int(max_seqlen),
        int(total_tokens), int(Hq), int(Hkv), int(D), int(window), _ptr(sink),
        float(softmax_scale), _ptr(o), _ptr(lse), _stream(stream))


def swa_sink_attn_fwd_noalloc(q, k, v, cu_seqlens, num_seqs, max_seqlen, total_tokens, Hq, Hkv,
                              D, window, sink, softmax_scale, o, lse, slot, stream=None):
    return load().swa_sink_attn_fwd_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), int(num_seqs), int(max_seqlen),
        int(total_tokens), int(Hq), int(Hkv), int(D), int(window), _ptr(sink),
        float(softmax_scale), _ptr(o), _ptr(lse), int(slot), _stream(stream))


def swa_sink_attn_fwd_rope_workspace(total_tokens, Hq, Hkv, D, window):
    return load().swa_sink_attn_fwd_rope_workspace(int(total_tokens), int(Hq), int(Hkv), int(D),
                                                   int(window))


def swa_sink_attn_fwd_rope(q, k, v, cu_seqlens, num_seqs, max_seqlen, total_tokens, Hq, Hkv, D,
                           window, sink, softmax_scale, rope_base, rope_interleaved, pos0,
                           k_ring, v_ring, ring_W, workspace, workspace_bytes, o, lse,
                           stream=None):
    return load().swa_sink_attn_fwd_rope(
        _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), int(num_seqs), int(max_seqlen),
        int(total_tokens), int(Hq), int(Hkv), int(D), int(window), _ptr(sink),
        float(softmax_scale), float(rope_base), int(rope_interleaved), _ptr(pos0), _ptr(k_ring),
        _ptr(v_ring), int(ring_W), _ptr(workspace), int(workspace_bytes), _ptr(o), _ptr(lse),
        _stream(stream))


def swa_sink_attn_bwd_workspace(total_tokens, Hq):
    return load().swa_sink_attn_bwd_workspace(int(total_tokens), int(Hq))


def swa_sink_attn_bwd(q, k, v, o, dout, lse, cu_seqlens, num_seqs, max_seqlen, total_tokens, Hq,
                      Hkv, D, window, sink, softmax_scale, dq, dk, dv, dsink, workspace,
                      workspace_bytes, stream=None):
    return load().swa_sink_attn_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(cu_seqlens),
        int(num_seqs), int(max_seqlen), int(total_tokens), int(Hq), int(Hkv), int(D),
        int(window), _ptr(sink), float(softmax_scale), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dsink),
        _ptr(workspace), int(workspace_bytes), _stream(stream))


def swa_sink_attn_decode(q, k_new, v_new, k_ring, v_ring, pos, B, n_q, Hq, Hkv, D, W, sink,
                         softmax_scale, o, lse, stream=None):
    return load().swa_sink_attn_decode(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_ring), _ptr(v_ring), _ptr(pos), int(B),
        int(n_q), int(Hq), int(Hkv), int(D), int(W), _ptr(sink), float(softmax_scale),
        _ptr(o), _ptr(lse), _stream(stream))


def swa_sink_decode_splitkv_workspace(B, n_q, Hq, Hkv, D, W, max_ctx):
    return load().swa_sink_decode_splitkv_workspace(int(B), int(n_q), int(Hq), int(Hkv), int(D),
                                                    int(W), int(max_ctx))


def swa_sink_attn_decode_splitkv(q, k_new, v_new, k_cache, v_cache, pos, B, n_q, Hq, Hkv, D, W,
                                 max_ctx, sink, softmax_scale, o, lse, workspace,
                                 workspace_bytes, stream=None):
    return load().swa_sink_attn_decode_splitkv(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(pos), int(B),
        int(n_q), int(Hq), int(Hkv), int(D), int(W), int(max_ctx), _ptr(sink),
        float(softmax_scale), _ptr(o), _ptr(lse), _ptr(workspace), int(workspace_bytes),
        _stream(stream))


def swa_sink_kv_commit(k_ring, v_ring, k_new, v_new, pos, n_accept, B, n_q, Hkv, D, W,
                       stream=None):
    return load().swa_sink_kv_commit(
        _ptr(k_ring), _ptr(v_ring), _ptr(k_new), _ptr(v_new), _ptr(pos), _ptr(n_accept),
        int(B), int(n_q), int(Hkv), int(D), int(W), _stream(stream))


def swa_sink_attn_decode_fp8kv(q, k_new, v_new, k_ring, v_ring, kv_scale, pos, B, n_q, Hq, Hkv,
                               D, W, sink, softmax_scale, o, lse, stream=None):
    return load().swa_sink_attn_decode_fp8kv(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_ring), _ptr(v_ring), _ptr(kv_scale),
        _ptr(pos), int(B), int(n_q), int(Hq), int(Hkv), int(D), int(W), _ptr(sink),
        float(softmax_scale), _ptr(o), _ptr(lse), _stream(stream))


def swa_sink_kv_commit_fp8(k_ring, v_ring, k_new, v_new, kv_scale, pos, n_accept, B, n_q, Hkv,
                           D, W, stream=None):
    return load().swa_sink_kv_commit_fp8(
        _ptr(k_ring), _ptr(v_ring), _ptr(k_new), _ptr(v_new), _ptr(kv_scale), _ptr(pos),
        _ptr(n_accept), int(B), int(n_q), int(Hkv), int(D), int(W), _stream(stream))


def swa_sink_status_string(status):
    return status_string(status)


def swa_sink_device_error(clear=True):
    flags = ctypes.c_uint(0)
    rc = load().swa_sink_device_error(ctypes.byref(flags), 1 if clear else 0)
    if rc != SWA_OK:
        raise SwaSinkError(rc, "swa_sink_device_error")
    return flags.value


def swa_sink_version():
    return load().swa_sink_version()


# ---- convenience wrappers ------------------------------------------------------

def attn_fwd(q, k, v, cu_seqlens, window, sink=None, softmax_scale=0.0, max_seqlen=None,
             out=None, lse=None, want_lse=True, stream=None):
    """q [total,Hq,D], k/v [total,Hkv,D] bf16 CUDA; cu_seqlens int32 CUDA.
    Returns (o, lse) with lse [Hq,total] fp32 (or None)."""
    total, Hq, D = q.shape
    Hkv = k.shape[1]
    num_seqs = cu_seqlens.numel() - 1
    if max_seqlen is None:
        max_seqlen = total
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((Hq, total), dtype=torch.float32, device=q.device)
    rc = swa_sink_attn_fwd(q, k, v, cu_seqlens, num_seqs, max_seqlen, total, Hq, Hkv, D,
                           window, sink, softmax_scale, out, lse, stream)
    if rc != SWA_OK:
        raise SwaSinkError(rc, "swa_sink_attn_fwd")
    return out, lse


def attn_fwd_rope(q, k, v, cu_seqlens, window, rope_base, sink=None, pos0=None,
                  interleaved=False, k_ring=None, v_ring=None, softmax_scale=0.0,
                  max_seqlen=None, out=None, lse=None, want_lse=True, workspace=None,
                  fused=False, stream=None):
    """attn_fwd with RoPE applied to q and k inside the call (q, k are read
    only). pos0: int32 CUDA [num_seqs] first position of each sequence (None:
    0). k_ring / v_ring: bf16 [num_seqs, ring_W, Hkv, D] written with the last
    ring_W tokens of each sequence (rotated K, V), or None. The workspace (a
    uint8 CUDA tensor) is allocated here unless given; fused=True passes none,
    so that shapes of the ring kernel rotate in its shared memory."""
    total, Hq, D = q.shape
    Hkv = k.shape[1]
    num_seqs = cu_seqlens.numel() - 1
    if max_seqlen is None:
        max_seqlen = total
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((Hq, total), dtype=torch.float32, device=q.device)
    need = swa_sink_attn_fwd_rope_workspace(total, Hq, Hkv, D, window)
    if workspace is None and need > 0 and not fused:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ring_W = 0 if k_ring is None else k_ring.shape[1]
    rc = swa_sink_attn_fwd_rope(q, k, v, cu_seqlens, num_seqs, max_seqlen, total, Hq, Hkv, D,
                                window, sink, softmax_scale, rope_base, 1 if interleaved else 0,
                                pos0, k_ring, v_ring, ring_W, workspace,
                                0 if workspace is None else workspace.numel(), out, lse, stream)
    if rc != SWA_OK:
        raise SwaSinkError(rc, "swa_sink_attn_fwd_rope")
    return out, lse


def attn_bwd(q, k, v, o, lse, dout, cu_seqlens, window, sink=None, softmax_scale=0.0,
             max_seqlen=None, want_dsink=True, workspace=None, stream=None):
    """Gradients of attn_fwd: returns (dq, dk, dv, dsink or None) for the
    forward's o and lse and the output gradient dout (bf16)."""
    total, Hq, D = q.shape
    Hkv = k.shape[1]
    num_seqs = cu_seqlens.numel() - 1
    if max_seqlen is None:
        max_seqlen = total
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dsink = (torch.empty((Hq,), dtype=torch.float32, device=q.device) if want_dsink else None)
    need = swa_sink_attn_bwd_workspace(total, Hq)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    rc = swa_sink_attn_bwd(q, k, v, o, dout, lse, cu_seqlens, num_seqs, max_seqlen, total, Hq,
                           Hkv, D, window, sink, softmax_scale, dq, dk, dv, dsink, workspace,
                           workspace.numel(), stream)
    if rc != SWA_OK:
        raise SwaSinkError(rc, "swa_sink_attn_bwd")
    return dq, dk, dv, dsink


def attn_decode(q, k_new, v_new, k_ring, v_ring, pos, sink=None, softmax_scale=0.0, out=None,
                lse=None, want_lse=True, stream=None):
    """q [B,n_q,Hq,D]; k_new/v_new [B,n_q,Hkv,D]; rings [B,W,Hkv,D]; pos int32 [B]."""
    B, n_q, Hq, D = q.shape
    Hkv = k_new.shape[2]
    W = k_ring.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, n_q, Hq), dtype=torch.float32, device=q.device)
    rc = swa_sink_attn_decode(q, k_new, v_new, k_ring, v_ring, pos, B, n_q, Hq, Hkv, D, W,
                              sink, softmax_scale, out, lse, stream)
    if rc != SWA_OK:
        raise SwaSinkError(rc, "swa_sink_attn_decode")
    return out, lse


def attn_decode_splitkv(q, k_new, v_new, k_cache, v_cache, pos, max_ctx, sink=None,
                        softmax_scale=0.0, out=None, lse=None, want_lse=True, workspace=None,
                        stream=None):
    """Like attn_decode over a cache [B,W,Hkv,D] of any W that is a multiple of
    64 (W >= the context: a global layer). The workspace (a uint8 CUDA tensor)
    is allocated here when not given."""
    B, n_q, Hq, D = q.shape
    Hkv = k_new.shape[2]
    W = k_cache.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, n_q, Hq), dtype=torch.float32, device=q.device)
    need = swa_sink_decode_splitkv_workspace(B, n_q, Hq, Hkv, D, W, max_ctx)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    rc = swa_sink_attn_decode_splitkv(q, k_new, v_new, k_cache, v_cache, pos, B, n_q, Hq, Hkv,
                                      D, W, max_ctx, sink, softmax_scale, out, lse, workspace,
                                      workspace.numel(), stream)
    if rc != SWA_OK:
        raise SwaSinkError(rc, "swa_sink_attn_decode_splitkv")
    return out, lse


def kv_commit(k_ring, v_ring, k_new, v_new, pos, n_accept, stream=None):
    B, W, Hkv, D = k_ring.shape
    n_q = k_new.shape[1]
    rc = swa_sink_kv_commit(k_ring, v_ring, k_new, v_new, pos, n_accept, B, n_q, Hkv, D, W,
                            stream)
    if rc != SWA_OK:
        raise SwaSinkError(rc, "swa_sink_kv_commit")


def attn_decode_fp8kv(q, k_new, v_new, k_ring, v_ring, kv_scale, pos, sink=None,
                      softmax_scale=0.0, out=None, lse=None, want_lse=True, stream=None):
    """attn_decode over an E4M3 ring: k_ring / v_ring uint8 codes [B,W,Hkv,D],
    kv_scale fp32 [2*Hkv] (K scales, then V scales)."""
    B, n_q, Hq, D = q.shape
    Hkv = k_new.shape[2]
    W = k_ring.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, n_q, Hq), dtype=torch.float32, device=q.device)
    rc = swa_sink_attn_decode_fp8kv(q, k_new, v_new, k_ring, v_ring, kv_scale, pos, B, n_q, Hq,
                                    Hkv, D, W, sink, softmax_scale, out, lse, stream)
    if rc != SWA_OK:
        raise SwaSinkError(rc, "swa_sink_attn_decode_fp8kv")
    return out, lse


def kv_commit_fp8(k_ring, v_ring, k_new, v_new, kv_scale, pos, n_accept, stream=None):
    B, W, Hkv, D = k_ring.shape
    n_q = k_new.shape[1]
    rc = swa_sink_kv_commit_fp8(k_ring, v_ring, k_new, v_new, kv_scale, pos, n_accept, B, n_q,
                                Hkv, D, W, stream)
    if rc != SWA_OK:
        raise SwaSinkError(rc, "swa_sink_kv_commit_fp8")
