"""FP8 (E4M3) KV cache: the code <-> value maps and the decode / commit over a
ring of codes, in plain numpy (fp64 for the attention).

TEST INFRASTRUCTURE: see the package docstring.

Sources: the MiMo-V2 blog review (kokolerk.github.io): section 4.3 says
inference as well as training runs in FP8, and section 6 (the V2.5-Pro
release) names the E4M3 format; the MiMo-V3 / HySparse2 news page
(hao.cnyes.com), in its cost comparison at one million tokens, gives KV cache
sizes for an FP8 cache. No page fixes the scale granularity; the reading
taken here is one fp32 scale per kv head for K and one for V, so a ring value
is the E4M3 code's value times that scale.

E4M3 (the OCP FP8 "E4M3FN" format): 1 sign bit, 4 exponent bits (bias 7), 3
mantissa bits; no infinities; S.1111.111 is NaN; the largest finite value is
448; exponent field 0 encodes subnormals m/8 * 2^-6.
"""
import numpy as np


def e4m3_value(code: int) -> float:
    """The value of one E4M3 code, from its bit fields."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_table() -> np.ndarray:
    """float64 [256]: the value of every code (NaN for 0x7F and 0xFF)."""
    return _TABLE.copy()


# the 127 non-negative finite codes 0x00..0x7E have increasing values
_POS = _TABLE[:0x7F]


def e4m3_encode(x) -> np.ndarray:
    """float32 array -> uint8 codes: the nearest finite E4M3 value, ties to the
    code with an even mantissa, magnitudes beyond 448 saturated to 448, NaN to
    0x7F. (The rounding of the one operation x / scale is done in float32 by
    the caller, as the device does.)"""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    out = np.empty(x.shape, dtype=np.uint8)
    flat, res = x.reshape(-1), out.reshape(-1)
    for n, v in enumerate(flat):
        if np.isnan(v):
            res[n] = 0x7F
            continue
        a = min(abs(v), 448.0)
        hi = int(np.searchsorted(_POS, a))  # first code with value >= a
        if hi == 0:
            c = 0
        elif _POS[hi] == a:
            c = hi
        else:
            lo = hi - 1
            dl, dh = a - _POS[lo], _POS[hi] - a
            c = lo if dl < dh else hi if dh < dl else (lo if lo % 2 == 0 else hi)
        res[n] = c | (0x80 if (v < 0 or (v == 0 and np.signbit(v))) else 0)
    return out


def decode_values(q, k_new, v_new, k_ring, v_ring, pos, B, n_q, Hq, Hkv, D, W, sink=None,
                  scale=None):
    """Decode over a ring given as float64 values [B, W, Hkv, D] (q, k_new,
    v_new: float64 arrays of the bf16 inputs). The same operation as the C
    oracle's decode: query t of sequence b (absolute position pos[b] + t)
    sees the ring tokens at positions max(0, pos[b]+t-W+1) .. pos[b]-1 (slot
    p mod W) and the new tokens 0..t; logits a = scale q.k; m = max(s, max a);
    o = sum exp(a - m) v / (exp(s - m) + sum exp(a - m)); lse = m + ln(den).
    Returns (o [B, n_q, Hq, D], lse [B, n_q, Hq])."""
    scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
    G = Hq // Hkv
    q, k_new, v_new = (np.asarray(a, np.float64) for a in (q, k_new, v_new))
    k_ring, v_ring = np.asarray(k_ring, np.float64), np.asarray(v_ring, np.float64)
    s = (np.full(Hq, -np.inf) if sink is None else np.asarray(sink, np.float64))
    o = np.zeros((B, n_q, Hq, D))
    lse = np.zeros((B, n_q, Hq))
    gmap = np.arange(Hq) // G
    for b in range(B):
        P = int(pos[b])
        for t in range(n_q):
            ps = np.arange(max(0, P + t - W + 1), P)
            keys = np.concatenate([k_ring[b, ps % W], k_new[b, :t + 1]], axis=0)  # [n, Hkv, D]
            vals = np.concatenate([v_ring[b, ps % W], v_new[b, :t + 1]], axis=0)
            kh = keys[:, gmap, :]  # [n, Hq, D]
            vh = vals[:, gmap, :]
            a = scale * np.einsum("hd,nhd->hn", q[b, t], kh)  # [Hq, n]
            m = np.maximum(s, a.max(axis=1))
            e = np.exp(a - m[:, None])
            den = np.exp(s - m) + e.sum(axis=1)
            o[b, t] = np.einsum("hn,nhd->hd", e, vh) / den[:, None]
            lse[b, t] = m + np.log(den)
    return o, lse


def dequantize(codes, kv_scale, Hkv, which):
    """Ring codes [B, W, Hkv, D] (uint8) -> float64 values: code value x the
    kv head's scale (which = 0: K scales kv_scale[:Hkv], 1: V scales
    kv_scale[Hkv:])."""
    sc = np.asarray(kv_scale, np.float32).astype(np.float64)[which * Hkv:(which + 1) * Hkv]
    return _TABLE[np.asarray(codes, np.uint8)] * sc[None, None, :, None]


def decode_fp8(q, k_new, v_new, k_codes, v_codes, kv_scale, pos, B, n_q, Hq, Hkv, D, W,
               sink=None, scale=None):
    """Decode over a ring of E4M3 codes with per-kv-head scales."""
    return decode_values(q, k_new, v_new, dequantize(k_codes, kv_scale, Hkv, 0),
                         dequantize(v_codes, kv_scale, Hkv, 1), pos, B, n_q, Hq, Hkv, D, W,
                         sink=sink, scale=scale)


def kv_commit_fp8(k_codes, v_codes, k_new, v_new, kv_scale, pos, n_accept, B, n_q, Hkv, D, W):
    """The accepted new tokens u < n_accept[b] (float32 values of the bf16
    inputs) go to slot (pos[b] + u) mod W as e4m3_encode(x / scale), the
    division rounded in float32. Returns new code arrays."""
    kc, vc = np.array(k_codes, np.uint8), np.array(v_codes, np.uint8)
    sc = np.asarray(kv_scale, np.float32)
    kn, vn = np.asarray(k_new, np.float32), np.asarray(v_new, np.float32)
    for b in range(B):
        for u in range(int(n_accept[b])):
            slot = (int(pos[b]) + u) % W
            for g in range(Hkv):
                kc[b, slot, g] = e4m3_encode(kn[b, u, g] / sc[g])
                vc[b, slot, g] = e4m3_encode(vn[b, u, g] / sc[Hkv + g])
    return kc, vc
