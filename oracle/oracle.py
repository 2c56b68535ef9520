"""ctypes front end of the C oracle (swa_sink_oracle.c).

TEST INFRASTRUCTURE: see the package docstring. Inputs are CPU tensors or
numpy arrays holding bf16 values (their raw 16-bit patterns are passed, so the
oracle sees exactly the bytes the device sees); outputs are float64 numpy
arrays. The math is defined in swa_sink_oracle.c.
"""
import ctypes
import os

import numpy as np

from .build import build

_lib = None
_c_u16p = ctypes.POINTER(ctypes.c_uint16)
_c_i32p = ctypes.POINTER(ctypes.c_int32)
_c_i64p = ctypes.POINTER(ctypes.c_int64)
_c_f64p = ctypes.POINTER(ctypes.c_double)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_prefill.restype = ctypes.c_int
        lib.oracle_prefill.argtypes = [
            _c_u16p, _c_u16p, _c_u16p, _c_i32p, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, _c_f64p, ctypes.c_double,
            _c_f64p, _c_f64p, _c_f64p, ctypes.c_int]
        lib.oracle_prefill_rows.restype = ctypes.c_int
        lib.oracle_prefill_rows.argtypes = [
            _c_u16p, _c_u16p, _c_u16p, _c_i32p, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, _c_f64p, ctypes.c_double,
            _c_i64p, _c_i32p, ctypes.c_int64, _c_f64p, _c_f64p, _c_f64p,
            ctypes.c_int]
        lib.oracle_decode.restype = ctypes.c_int
        lib.oracle_decode.argtypes = [
            _c_u16p, _c_u16p, _c_u16p, _c_u16p, _c_u16p, _c_i32p, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, _c_f64p, ctypes.c_double, _c_f64p, _c_f64p, _c_f64p,
            ctypes.c_int]
        lib.oracle_kv_commit.restype = ctypes.c_int
        lib.oracle_kv_commit.argtypes = [
            _c_u16p, _c_u16p, _c_u16p, _c_u16p, _c_i32p, _c_i32p, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        _lib = lib
    return _lib


def _bits(x):
    """bf16 tensor / uint16 array -> contiguous uint16 numpy array of bits."""
    if hasattr(x, "view") and hasattr(x, "dtype") and "bfloat16" in str(x.dtype):
        import torch
        x = x.detach().to("cpu").contiguous().view(torch.int16).numpy()
    a = np.ascontiguousarray(np.asarray(x))
    if a.dtype == np.int16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError("expected bf16 tensor or uint16 bit array, got %s" % a.dtype)
    return a


def _i32(x):
    if hasattr(x, "numpy"):
        x = x.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _f64_or_none(x):
    if x is None:
        return None
    if hasattr(x, "numpy"):
        x = x.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a, t):
    return None if a is None else a.ctypes.data_as(t)


def _scale(D, scale):
    return (1.0 / np.sqrt(D)) if (scale is None or scale <= 0) else float(scale)


def prefill(q, k, v, cu_seqlens, Hq, Hkv, D, window, sink=None, scale=None,
            nthreads=None, want_wsink=False):
    """Every row. Returns (o [total,Hq,D], lse [Hq,total], wsink or None)."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    cu = _i32(cu_seqlens)
    total = int(cu[-1])
    o = np.empty((total, Hq, D), np.float64)
    lse = np.empty((Hq, total), np.float64)
    ws = np.empty((Hq, total), np.float64) if want_wsink else None
    sk = _f64_or_none(sink)
    rc = lib.oracle_prefill(
        _p(qb, _c_u16p), _p(kb, _c_u16p), _p(vb, _c_u16p), _p(cu, _c_i32p),
        len(cu) - 1, Hq, Hkv, D, int(window), _p(sk, _c_f64p), _scale(D, scale),
        _p(o, _c_f64p), _p(lse, _c_f64p), _p(ws, _c_f64p),
        nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_prefill rejected its arguments (%d)" % rc)
    return o, lse, ws


def prefill_rows(q, k, v, cu_seqlens, Hq, Hkv, D, window, row_tok, row_head,
                 sink=None, scale=None, nthreads=None, want_wsink=False):
    """A sample of (token, head) rows. Returns (o [n,D], lse [n], wsink)."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    cu = _i32(cu_seqlens)
    rt = np.ascontiguousarray(np.asarray(row_tok, dtype=np.int64))
    rh = np.ascontiguousarray(np.asarray(row_head, dtype=np.int32))
    n = rt.shape[0]
    o = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    ws = np.empty((n,), np.float64) if want_wsink else None
    sk = _f64_or_none(sink)
    rc = lib.oracle_prefill_rows(
        _p(qb, _c_u16p), _p(kb, _c_u16p), _p(vb, _c_u16p), _p(cu, _c_i32p),
        len(cu) - 1, Hq, Hkv, D, int(window), _p(sk, _c_f64p), _scale(D, scale),
        _p(rt, _c_i64p), _p(rh, _c_i32p), n, _p(o, _c_f64p), _p(lse, _c_f64p),
        _p(ws, _c_f64p), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_prefill_rows rejected its arguments (%d)" % rc)
    return o, lse, ws


def decode(q, k_new, v_new, k_ring, v_ring, pos, B, n_q, Hq, Hkv, D, W,
           sink=None, scale=None, nthreads=None, want_wsink=False):
    """Returns (o [B,n_q,Hq,D], lse [B,n_q,Hq], wsink or None)."""
    lib = _load()
    qb, knb, vnb = _bits(q), _bits(k_new), _bits(v_new)
    krb, vrb = _bits(k_ring), _bits(v_ring)
    ps = _i32(pos)
    o = np.empty((B, n_q, Hq, D), np.float64)
    lse = np.empty((B, n_q, Hq), np.float64)
    ws = np.empty((B, n_q, Hq), np.float64) if want_wsink else None
    sk = _f64_or_none(sink)
    rc = lib.oracle_decode(
        _p(qb, _c_u16p), _p(knb, _c_u16p), _p(vnb, _c_u16p), _p(krb, _c_u16p),
        _p(vrb, _c_u16p), _p(ps, _c_i32p), B, n_q, Hq, Hkv, D, W,
        _p(sk, _c_f64p), _scale(D, scale), _p(o, _c_f64p), _p(lse, _c_f64p),
        _p(ws, _c_f64p), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_decode rejected its arguments (%d)" % rc)
    return o, lse, ws


def kv_commit(k_ring, v_ring, k_new, v_new, pos, n_accept, B, n_q, Hkv, D, W):
    """Returns new (k_ring, v_ring) uint16 bit arrays; the inputs are untouched."""
    lib = _load()
    kr = _bits(k_ring).copy()
    vr = _bits(v_ring).copy()
    knb, vnb = _bits(k_new), _bits(v_new)
    ps, na = _i32(pos), _i32(n_accept)
    rc = lib.oracle_kv_commit(
        _p(kr, _c_u16p), _p(vr, _c_u16p), _p(knb, _c_u16p), _p(vnb, _c_u16p),
        _p(ps, _c_i32p), _p(na, _c_i32p), B, n_q, Hkv, D, W)
    if rc != 0:
        raise ValueError("oracle_kv_commit rejected its arguments (%d)" % rc)
    return kr, vr
