"""fp64 CPU oracle for the gated sliding-window attention core.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  It
shares no code with the CUDA library and never imports it.

The arithmetic lives in ``swa_oracle.c`` (plain C, IEEE fp64, OpenMP over
independent rows); this module marshals numpy arrays, and writes a few steps
out in numpy on top of the C norm/RoPE: the prefill -> ring handoff (dense
and ragged) and the global layers' decode over a full-length cache.  Definitions follow
the ZGCM-1 pages: "7.39B 오픈 모델로 256K 문맥의 … ZGCM-1" (onedev.kr), section
"어떻게 동작하나", and "ZGCM-1: A Fully Open and Extremely Efficient Foundation
Model …" (jaehun.me), sections "How Gated SWA Behaves" and "Why the KV Cache
Shrinks by 6.4×".  The header of ``swa_oracle.c`` lists every reading taken
where the pages are silent.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
(brute force, library special cases, closed forms, finite differences and the
pages' worked numbers under ``tests/golden/``).
"""
import ctypes
import math
import os

import numpy as np

from .build import build as _build

_lib = None

_d = ctypes.c_double
_i = ctypes.c_int
_i64 = ctypes.c_int64
_pd = ctypes.POINTER(ctypes.c_double)
_pu16 = ctypes.POINTER(ctypes.c_uint16)
_pi64 = ctypes.POINTER(ctypes.c_int64)


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(_build())
        L = _lib
        L.oracle_bf16_bits.argtypes = [_d]
        L.oracle_bf16_bits.restype = ctypes.c_uint16
        L.oracle_bf16_value.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_value.restype = _d
        L.oracle_norm_rope.argtypes = [_i64, _i, _i, _i, _d, _d, _pd, _pd, _pd, _pd]
        L.oracle_norm_rope.restype = None
        L.oracle_fwd.argtypes = [_i64, _i64, _i, _i, _i, _i, _i, _d, _d, _d, _i64, _i64,
                                 _pd, _pd, _pd, _pd, _pd, _pd, _pd, _pd]
        L.oracle_fwd.restype = None
        L.oracle_bwd.argtypes = [_i64, _i64, _i, _i, _i, _i, _i, _d, _d, _d,
                                 _pd, _pd, _pd, _pd, _pd, _pd, _pd,
                                 _pd, _pd, _pd, _pd, _pd, _pd]
        L.oracle_bwd.restype = None
        L.oracle_decode.argtypes = [_i64, _i, _i, _i, _i, _i, _d, _d, _d, _pi64,
                                    _pd, _pd, _pd, _pd, _pd, _pd, _pu16, _pu16, _pd]
        L.oracle_decode.restype = None
        L.oracle_kv_bytes_per_token.argtypes = [_i64, _i64, _i64, _i64]
        L.oracle_kv_bytes_per_token.restype = _i64
        L.oracle_threads.argtypes = []
        L.oracle_threads.restype = _i
    return _lib


def _f64(a):
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(_pd)


def _scale(D, scale):
    return 1.0 / math.sqrt(D) if not scale else float(scale)


def threads() -> int:
    """OpenMP threads the oracle uses (``OMP_NUM_THREADS`` or all cores)."""
    return int(lib().oracle_threads())


def bf16_bits(x: float) -> int:
    """Bits of the bf16 nearest to ``x`` (ties to even)."""
    return int(lib().oracle_bf16_bits(float(x)))


def bf16_round_array(x: np.ndarray) -> np.ndarray:
    """Element-wise round-to-nearest-even to bf16, returned as uint16 bits."""
    L = lib()
    flat = np.asarray(x, dtype=np.float64).ravel()
    return np.array([L.oracle_bf16_bits(float(v)) for v in flat], dtype=np.uint16).reshape(np.shape(x))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns (uint16) to fp64."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def e4m3_to_f64(b):
    """Values of FP8 E4M3 bytes (the OCP 8-bit format with 4 exponent bits, bias
    7, and 3 mantissa bits; no infinities, S.1111.111 is NaN), from the
    encoding's definition: normal (1 + m/8) 2^(e-7), subnormal m 2^-9."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    sign = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 7).astype(np.float64)
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def norm_rope(x, w, pos, R, base, eps):
    """RoPE(RMSNorm(x, w), pos) for x [rows, H, D] (fp64), pos [rows]."""
    x, px = _f64(x)
    w, pw = _f64(w)
    pos, pp = _f64(pos)
    rows, H, D = x.shape
    y = np.empty_like(x)
    lib().oracle_norm_rope(rows, H, D, int(R), float(base), float(eps), px, pw, pp,
                           y.ctypes.data_as(_pd))
    return y


def fwd(q, k, v, g, wq, wk, *, W, R, base, eps, scale=0.0, pos0=0, q_begin=0,
        want_lse=True):
    """Gated SWA forward in fp64.

    k, v: [B, T, Hkv, D] at positions pos0 .. pos0+T-1; q, g: [B, T-q_begin, Hq, D]
    (query rows t >= q_begin).  Returns (o [B, T-q_begin, Hq, D], lse [B, T-q_begin, Hq]).
    """
    q, pq = _f64(q)
    k, pk = _f64(k)
    v, pv = _f64(v)
    g, pg = _f64(g)
    wq, pwq = _f64(wq)
    wk, pwk = _f64(wk)
    B, T, Hkv, D = k.shape
    Hq = q.shape[2]
    assert q.shape == (B, T - q_begin, Hq, D) and g.shape == q.shape and v.shape == k.shape
    assert Hq % Hkv == 0 and R % 2 == 0 and R <= D
    assert pos0 == 0 or q_begin >= W - 1, "a chunk must carry each query's whole window"
    o = np.empty(q.shape, dtype=np.float64)
    lse = np.empty((B, T - q_begin, Hq), dtype=np.float64) if want_lse else None
    lib().oracle_fwd(B, T, Hq, Hkv, D, int(W), int(R), float(base), float(eps),
                     _scale(D, scale), int(pos0), int(q_begin), pq, pk, pv, pg, pwq, pwk,
                     o.ctypes.data_as(_pd),
                     lse.ctypes.data_as(_pd) if want_lse else ctypes.cast(None, _pd))
    return o, lse


def fwd_rows(q, k, v, g, wq, wk, b, t0, t1, *, W, R, base, eps, scale=0.0):
    """Forward for query rows [t0, t1) of batch row ``b`` of full tensors.

    q, k, v, g are CPU torch bf16 (or fp64 numpy) tensors [B, T, H, D]; only the
    slices the rows need are upcast, so this scales to very long sequences.
    """
    kb = max(0, t0 - W + 1)

    def sl(x, a, c):
        x = x[b:b + 1, a:c]
        return x.double().numpy() if hasattr(x, "double") else np.asarray(x, np.float64)

    wq_ = wq.double().numpy() if hasattr(wq, "double") else wq
    wk_ = wk.double().numpy() if hasattr(wk, "double") else wk
    return fwd(sl(q, t0, t1), sl(k, kb, t1), sl(v, kb, t1), sl(g, t0, t1), wq_, wk_,
               W=W, R=R, base=base, eps=eps, scale=scale, pos0=kb, q_begin=t0 - kb)


def bwd(q, k, v, g, wq, wk, dO, *, W, R, base, eps, scale=0.0):
    """Exact fp64 backward of :func:`fwd` (positions 0..T-1).

    Returns dq, dk, dv, dg, dwq, dwk.
    """
    q, pq = _f64(q)
    k, pk = _f64(k)
    v, pv = _f64(v)
    g, pg = _f64(g)
    wq, pwq = _f64(wq)
    wk, pwk = _f64(wk)
    dO, pdO = _f64(dO)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    dg = np.empty_like(g)
    dwq = np.empty(D)
    dwk = np.empty(D)
    lib().oracle_bwd(B, T, Hq, Hkv, D, int(W), int(R), float(base), float(eps),
                     _scale(D, scale), pq, pk, pv, pg, pwq, pwk, pdO,
                     dq.ctypes.data_as(_pd), dk.ctypes.data_as(_pd), dv.ctypes.data_as(_pd),
                     dg.ctypes.data_as(_pd), dwq.ctypes.data_as(_pd), dwk.ctypes.data_as(_pd))
    return dq, dk, dv, dg, dwq, dwk


def decode(pos, q, k_new, v_new, g, wq, wk, k_cache_bits, v_cache_bits, *, R, base, eps,
           scale=0.0):
    """One decode step over W-slot rings.

    pos [N] int64; q, g [N, Hq, D]; k_new, v_new [N, Hkv, D] (fp64 values);
    caches [N, Hkv, W, D] as uint16 bf16 bits (copied, not modified).
    Returns (o [N, Hq, D] fp64, k_cache_bits', v_cache_bits').
    """
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    q, pq = _f64(q)
    k_new, pk = _f64(k_new)
    v_new, pv = _f64(v_new)
    g, pg = _f64(g)
    wq, pwq = _f64(wq)
    wk, pwk = _f64(wk)
    kc = np.array(k_cache_bits, dtype=np.uint16, copy=True, order="C")
    vc = np.array(v_cache_bits, dtype=np.uint16, copy=True, order="C")
    N, Hq, D = q.shape
    Hkv, W = kc.shape[1], kc.shape[2]
    o = np.empty_like(q)
    lib().oracle_decode(N, Hq, Hkv, D, W, int(R), float(base), float(eps), _scale(D, scale),
                        pos.ctypes.data_as(_pi64), pq, pk, pv, pg, pwq, pwk,
                        kc.ctypes.data_as(_pu16), vc.ctypes.data_as(_pu16),
                        o.ctypes.data_as(_pd))
    return o, kc, vc


def prefill_to_ring(k, v, wk, k_cache_bits, v_cache_bits, *, R, base, eps):
    """Decode rings after a prefill of T tokens.

    Slot s of ring (b, h) holds the key and value of the latest position
    p <= T-1 with p = s (mod W), the slot a decode step of that position
    writes (jaehun.me review, "Why the KV Cache Shrinks by 6.4x": the window
    layers keep only their last W tokens): k' = RoPE_p(RMSNorm(k_p, wk))
    rounded to bf16, and v_p unchanged.  Slots no position reaches keep their
    bits.  k, v: [B, T, Hkv, D] (fp64 values of bf16 inputs); caches
    [B, Hkv, W, D] as uint16 bf16 bits (copied, not modified).
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    kc = np.array(k_cache_bits, dtype=np.uint16, copy=True, order="C")
    vc = np.array(v_cache_bits, dtype=np.uint16, copy=True, order="C")
    B, T = k.shape[0], k.shape[1]
    W = kc.shape[2]
    for p in range(max(0, T - W), T):  # the last W positions, each to its own slot
        s = p % W
        kp = norm_rope(k[:, p], wk, np.full(B, float(p)), R, base, eps)  # [B, Hkv, D]
        kc[:, :, s, :] = bf16_round_array(kp)
        vc[:, :, s, :] = bf16_round_array(v[:, p])
    return kc, vc


def prefill_to_ring_varlen(k, v, wk, k_cache_bits, v_cache_bits, starts, lens, pos0, *, R, base,
                           eps):
    """Decode rings after ragged or continued prefills.

    Sequence b's lens[b] tokens are rows starts[b] .. of k, v [rows, Hkv, D]
    (fp64 values of bf16 inputs), at positions pos0[b] + i.  As in
    :func:`prefill_to_ring`, slot s of ring b takes the latest of those
    positions p with p = s (mod W): k' = RoPE_p(RMSNorm(k, wk)) rounded to bf16,
    and v.  Slots no position reaches keep their bits.  Returns the new bits.
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    kc = np.array(k_cache_bits, dtype=np.uint16, copy=True, order="C")
    vc = np.array(v_cache_bits, dtype=np.uint16, copy=True, order="C")
    W = kc.shape[2]
    for b in range(kc.shape[0]):
        n, first, p0 = int(lens[b]), int(starts[b]), int(pos0[b])
        for p in range(max(p0, p0 + n - W), p0 + n):  # the last W positions
            row = first + (p - p0)
            kp = norm_rope(k[row][None], wk, np.array([float(p)]), R, base, eps)[0]
            kc[b, :, p % W, :] = bf16_round_array(kp)
            vc[b, :, p % W, :] = bf16_round_array(v[row])
    return kc, vc


def global_decode(pos, q, k_new, v_new, wq, wk, k_cache_bits, v_cache_bits, *, R, base, eps,
                  scale=0.0):
    """One decode step of a global (full causal context, ungated) layer over
    full-length caches.

    The global layers attend over every earlier token and keep every token's
    K and V (onedev.kr summary, "어떻게 동작하나": 5 global layers beside the
    27 window layers; jaehun.me review, "How Gated SWA Behaves": global layers
    skip the gate, and "Why the KV Cache Shrinks by 6.4x": they store the whole
    sequence).  Slot s of a cache holds position s.  For sequence n at position
    p = pos[n]: slot p first receives k' = RoPE_p(RMSNorm(k_new, wk)) rounded
    to bf16 and v_new; then q' = RoPE_p(RMSNorm(q, wq)) attends over slots
    0 .. p (query head h reads KV head h // (Hq / Hkv)): s_j = scale q'.k_j,
    P = softmax(s), o = sum_j P_j v_j.

    pos [N] int64; q [N, Hq, D], k_new, v_new [N, Hkv, D] (fp64 values of bf16
    inputs); caches [N, Hkv, cap, D] as uint16 bf16 bits (copied, not
    modified).  Returns (o [N, Hq, D] fp64, k_cache_bits', v_cache_bits').
    """
    pos = np.asarray(pos, dtype=np.int64)
    q = np.asarray(q, dtype=np.float64)
    k_new = np.asarray(k_new, dtype=np.float64)
    v_new = np.asarray(v_new, dtype=np.float64)
    kc = np.array(k_cache_bits, dtype=np.uint16, copy=True, order="C")
    vc = np.array(v_cache_bits, dtype=np.uint16, copy=True, order="C")
    N, Hq, D = q.shape
    Hkv = kc.shape[1]
    group = Hq // Hkv
    sc = _scale(D, scale)
    o = np.empty_like(q)
    for n in range(N):
        p = int(pos[n])
        at = np.array([float(p)])
        kp = norm_rope(k_new[n][None], wk, at, R, base, eps)[0]  # [Hkv, D]
        kc[n, :, p, :] = bf16_round_array(kp)
        vc[n, :, p, :] = bf16_round_array(v_new[n])
        qp = norm_rope(q[n][None], wq, at, R, base, eps)[0]      # [Hq, D]
        for h in range(Hq):
            kvh = h // group
            keys = bf16_bits_to_f64(kc[n, kvh, :p + 1])          # slots 0 .. p
            vals = bf16_bits_to_f64(vc[n, kvh, :p + 1])
            s = sc * (keys @ qp[h])
            e = np.exp(s - s.max())
            o[n, h] = (e / e.sum()) @ vals
    return o, kc, vc


def kv_bytes_per_token(layers: int, kv_heads: int, head_dim: int, bytes_per_elt: int) -> int:
    """KV-cache bytes per token for ``layers`` layers that keep every token."""
    return int(lib().oracle_kv_bytes_per_token(layers, kv_heads, head_dim, bytes_per_elt))
