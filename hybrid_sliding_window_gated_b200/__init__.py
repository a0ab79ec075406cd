"""Gated sliding-window attention core (ZGCM-1 GatedSWA without projections) on B200.

A thin ctypes binding over ``libswa.so`` (the C ABI in ``include/swa.h``).
This module only marshals arguments: every step of the computation runs in
the library's sm_100a kernels.  If the compiled library is missing, importing
the binding raises, so there is no silent CPU fallback.

PyTorch serves as the owner of device memory and streams: tensors are passed
by ``data_ptr()`` and calls are enqueued on the current CUDA stream.  Before a
pointer is passed, each tensor's dtype, element count, contiguity and device
are checked against what the call reads or writes (``TypeError`` /
``ValueError``); the library itself checks the sizes and alignment.
"""
import ctypes
import os

import torch

__all__ = ["fwd", "fwd_halo", "fwd_fp8", "bwd", "bwd_edges", "bwd_halo", "bwd_noalloc", "bwd_workspace_size", "decode_step", "prefill_to_ring", "prefill_to_ring_varlen",
           "global_fwd", "global_decode_step", "global_decode_workspace_size",
           "get_last_device_error", "SwaError", "Params", "lib", "LIB_PATH"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libswa.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_DEVICE_TIMEOUT = 0, 1, 2, 3, 4
FLAG_FORCE_TIMEOUT = 1


class Params(ctypes.Structure):
    """Mirror of ``swa_params_t``."""
    _fields_ = [("B", ctypes.c_int64), ("T", ctypes.c_int64), ("Hq", ctypes.c_int32),
                ("Hkv", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("window", ctypes.c_int32),
                ("rot_dim", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("rope_base", ctypes.c_double), ("eps", ctypes.c_float), ("scale", ctypes.c_float)]


class SwaError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {lib().swa_error_string(code).decode()} (code {code})")


_lib = None
_vp = ctypes.c_void_p


def lib():
    """The loaded ``libswa.so`` (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m hybrid_sliding_window_gated_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(Params)
        L.swa_fwd.argtypes = [P] + [_vp] * 9
        L.swa_fwd.restype = ctypes.c_int
        L.swa_fwd_halo.argtypes = [P] + [_vp] * 8 + [ctypes.c_int64, _vp, _vp, _vp]
        L.swa_fwd_halo.restype = ctypes.c_int
        L.swa_fwd_fp8.argtypes = [P] + [_vp] * 10
        L.swa_fwd_fp8.restype = ctypes.c_int
        L.swa_bwd.argtypes = [P] + [_vp] * 15 + [ctypes.c_size_t, _vp]
        L.swa_bwd.restype = ctypes.c_int
        L.swa_bwd_edges.argtypes = [P] + [_vp] * 14 + [ctypes.c_int64, _vp, ctypes.c_int64, _vp,
                                                       _vp, ctypes.c_size_t, _vp]
        L.swa_bwd_edges.restype = ctypes.c_int
        L.swa_bwd_halo.argtypes = [P] + [_vp] * 16 + [ctypes.c_int64, _vp, ctypes.c_int64, _vp,
                                                      _vp, ctypes.c_size_t, _vp]
        L.swa_bwd_halo.restype = ctypes.c_int
        L.swa_bwd_noalloc.argtypes = [P] + [_vp] * 15
        L.swa_bwd_noalloc.restype = ctypes.c_int
        L.swa_bwd_workspace_size.argtypes = [P]
        L.swa_bwd_workspace_size.restype = ctypes.c_size_t
        L.swa_decode_step.argtypes = [P] + [_vp] * 11
        L.swa_decode_step.restype = ctypes.c_int
        L.swa_prefill_to_ring.argtypes = [P] + [_vp] * 6
        L.swa_prefill_to_ring.restype = ctypes.c_int
        L.swa_prefill_to_ring_varlen.argtypes = [P] + [_vp] * 9
        L.swa_prefill_to_ring_varlen.restype = ctypes.c_int
        L.swa_global_fwd.argtypes = [P] + [_vp] * 9 + [ctypes.c_int64, _vp]
        L.swa_global_fwd.restype = ctypes.c_int
        L.swa_global_decode_workspace_size.argtypes = [P, ctypes.c_int64]
        L.swa_global_decode_workspace_size.restype = ctypes.c_size_t
        L.swa_global_decode_step.argtypes = [P] + [_vp] * 8 + [ctypes.c_int64, _vp, _vp,
                                                               ctypes.c_size_t, _vp]
        L.swa_global_decode_step.restype = ctypes.c_int
        L.swa_error_string.argtypes = [ctypes.c_int]
        L.swa_error_string.restype = ctypes.c_char_p
        L.swa_get_last_device_error.argtypes = [_vp, ctypes.POINTER(ctypes.c_int)]
        L.swa_get_last_device_error.restype = ctypes.c_int
        L.swa_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc, where):
    if rc != OK:
        raise SwaError(rc, where)


def _need(where, device, **tensors):
    """Host-side check of the tensors a call hands to the library: each entry is
    name=(tensor, dtype, elements the call reads or writes).  A non-empty tensor
    must be a contiguous CUDA tensor on `device` with the dtype and at least
    that many elements; the kernels take its pointer and the sizes in the
    parameter block, so anything else would be misread or overrun."""
    for name, (t, dtype, n) in tensors.items():
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{where}: {name} must be a torch.Tensor")
        if t.dtype != dtype:
            raise TypeError(f"{where}: {name} is {t.dtype}, expected {dtype}")
    used = {name: (t, n) for name, (t, _, n) in tensors.items() if n > 0}
    for name, (t, n) in used.items():
        if t.numel() < n:
            raise ValueError(f"{where}: {name} has {t.numel()} elements, the call needs {n}")
    for name, (t, n) in used.items():
        if not t.is_contiguous():
            raise ValueError(f"{where}: {name} must be contiguous")
    for name, (t, n) in used.items():
        if t.device != device or not t.is_cuda:
            raise ValueError(f"{where}: {name} is on {t.device}, expected a CUDA tensor on "
                             f"the device of the first input")


def make_params(B, T, Hq, Hkv, *, head_dim=128, window=128, rot_dim=42, rope_base=1e4, eps=1e-6,
                scale=0.0, flags=0):
    return Params(B, T, Hq, Hkv, head_dim, window, rot_dim, flags, rope_base, eps, scale)


def fwd(q, k, v, g, wq, wk, *, window=128, rot_dim=42, rope_base=1e4, eps=1e-6, scale=0.0,
        out=None, lse=None, want_lse=False, flags=0, stream=None):
    """o = A_SWA(RoPE(RMSNorm(q)), RoPE(RMSNorm(k)), v) * sigmoid(g).

    q, g: [B,T,Hq,128] bf16; k, v: [B,T,Hkv,128] bf16; wq, wk: [128] fp32 (CUDA).
    Returns o (and lse [B,Hq,T] fp32 when ``want_lse`` or ``lse`` is given).
    """
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    p = make_params(B, T, Hq, Hkv, head_dim=D, window=window, rot_dim=rot_dim,
                    rope_base=rope_base, eps=eps, scale=scale, flags=flags)
    nq, nk = B * T * Hq * D, B * T * Hkv * D
    bf, f32 = torch.bfloat16, torch.float32
    opt = {} if lse is None else {"lse": (lse, f32, B * Hq * T)}
    _need("swa_fwd", q.device, q=(q, bf, nq), k=(k, bf, nk), v=(v, bf, nk), g=(g, bf, nq),
          wq=(wq, f32, D if nq else 0), wk=(wk, f32, D if nq else 0), out=(out, bf, nq), **opt)
    rc = lib().swa_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(wq), _ptr(wk),
                       _ptr(out), _ptr(lse), _stream(stream))
    _check(rc, "swa_fwd")
    return (out, lse) if lse is not None else out


def fwd_halo(q, k, v, g, wq, wk, k_halo, v_halo, pos0, *, window=128, rot_dim=42, rope_base=1e4,
             eps=1e-6, scale=0.0, out=None, lse=None, want_lse=False, flags=0, stream=None):
    """:func:`fwd` for a chunk starting at position pos0 whose previous 127 tokens
    are k_halo, v_halo [B,127,Hkv,128] (swa_fwd_halo); both None: no history."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    p = make_params(B, T, Hq, Hkv, head_dim=D, window=window, rot_dim=rot_dim,
                    rope_base=rope_base, eps=eps, scale=scale, flags=flags)
    nq, nk, nh = B * T * Hq * D, B * T * Hkv * D, B * (window - 1) * Hkv * D
    bf, f32 = torch.bfloat16, torch.float32
    opt = {} if lse is None else {"lse": (lse, f32, B * Hq * T)}
    if k_halo is not None or v_halo is not None:
        opt["k_halo"] = (k_halo, bf, nh if nq else 0)
        opt["v_halo"] = (v_halo, bf, nh if nq else 0)
    _need("swa_fwd_halo", q.device, q=(q, bf, nq), k=(k, bf, nk), v=(v, bf, nk), g=(g, bf, nq),
          wq=(wq, f32, D if nq else 0), wk=(wk, f32, D if nq else 0), out=(out, bf, nq), **opt)
    rc = lib().swa_fwd_halo(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(wq),
                            _ptr(wk), _ptr(k_halo), _ptr(v_halo), int(pos0), _ptr(out), _ptr(lse),
                            _stream(stream))
    _check(rc, "swa_fwd_halo")
    return (out, lse) if lse is not None else out


def fwd_fp8(q8, k8, v8, qkv_scale, g, wq, wk, *, window=128, rot_dim=42, rope_base=1e4,
            eps=1e-6, scale=0.0, out=None, lse=None, want_lse=False, flags=0, stream=None):
    """:func:`fwd` with q, k, v in FP8 E4M3 (swa_fwd_fp8): q8 [B,T,Hq,128], k8,
    v8 [B,T,Hkv,128] as torch.float8_e4m3fn or uint8 bytes; qkv_scale [3] fp32
    (CUDA) with the values q = q8 * qkv_scale[0], k = k8 * qkv_scale[1],
    v = v8 * qkv_scale[2]; g, wq, wk as in :func:`fwd`."""
    B, T, Hq, D = q8.shape
    Hkv = k8.shape[2]
    if out is None:
        out = torch.empty(q8.shape, dtype=torch.bfloat16, device=q8.device)
    if want_lse and lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q8.device)
    byte = lambda t: t.view(torch.uint8) if t.dtype == torch.float8_e4m3fn else t
    q8, k8, v8 = byte(q8), byte(k8), byte(v8)
    p = make_params(B, T, Hq, Hkv, head_dim=D, window=window, rot_dim=rot_dim,
                    rope_base=rope_base, eps=eps, scale=scale, flags=flags)
    nq, nk = B * T * Hq * D, B * T * Hkv * D
    bf, f32, u8 = torch.bfloat16, torch.float32, torch.uint8
    opt = {} if lse is None else {"lse": (lse, f32, B * Hq * T)}
    _need("swa_fwd_fp8", q8.device, q=(q8, u8, nq), k=(k8, u8, nk), v=(v8, u8, nk),
          qkv_scale=(qkv_scale, f32, 3 if nq else 0), g=(g, bf, nq),
          wq=(wq, f32, D if nq else 0), wk=(wk, f32, D if nq else 0), out=(out, bf, nq), **opt)
    rc = lib().swa_fwd_fp8(ctypes.byref(p), _ptr(q8), _ptr(k8), _ptr(v8), _ptr(qkv_scale),
                           _ptr(g), _ptr(wq), _ptr(wk), _ptr(out), _ptr(lse), _stream(stream))
    _check(rc, "swa_fwd_fp8")
    return (out, lse) if lse is not None else out


def bwd_workspace_size(B, T, Hq, Hkv, *, head_dim=128, window=128, rot_dim=42):
    p = make_params(B, T, Hq, Hkv, head_dim=head_dim, window=window, rot_dim=rot_dim)
    return int(lib().swa_bwd_workspace_size(ctypes.byref(p)))


def _need_bwd(where, q, k, v, g, wq, wk, lse, dO, grads, **extra):
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    nq, nk = B * T * Hq * D, B * T * Hkv * D
    nw = D if nq else 0
    bf, f32 = torch.bfloat16, torch.float32
    dq, dk, dv, dg, dwq, dwk = grads
    _need(where, q.device, q=(q, bf, nq), k=(k, bf, nk), v=(v, bf, nk), g=(g, bf, nq),
          wq=(wq, f32, nw), wk=(wk, f32, nw), lse=(lse, f32, B * Hq * T), dO=(dO, bf, nq),
          dq=(dq, bf, nq), dk=(dk, bf, nk), dv=(dv, bf, nk), dg=(dg, bf, nq),
          dwq=(dwq, f32, nw), dwk=(dwk, f32, nw), **extra)


def bwd(q, k, v, g, wq, wk, lse, dO, *, window=128, rot_dim=42, rope_base=1e4, eps=1e-6,
        scale=0.0, workspace=None, grads=None, flags=0, stream=None):
    """Gradients (dq, dk, dv, dg, dwq, dwk) of sum(o * dO) for the forward above."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    p = make_params(B, T, Hq, Hkv, head_dim=D, window=window, rot_dim=rot_dim,
                    rope_base=rope_base, eps=eps, scale=scale, flags=flags)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(g),
                 torch.zeros(D, dtype=torch.float32, device=q.device),
                 torch.zeros(D, dtype=torch.float32, device=q.device))
    dq, dk, dv, dg, dwq, dwk = grads
    nbytes = int(lib().swa_bwd_workspace_size(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    _need_bwd("swa_bwd", q, k, v, g, wq, wk, lse, dO, grads,
              workspace=(workspace, torch.uint8, nbytes))
    rc = lib().swa_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(wq), _ptr(wk),
                       _ptr(lse), _ptr(dO), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dwq),
                       _ptr(dwk), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "swa_bwd")
    return grads


def bwd_edges(q, k, v, g, wq, wk, lse, dO, n_lo, n_hi, *, window=128, rot_dim=42,
              rope_base=1e4, eps=1e-6, scale=0.0, workspace=None, grads=None, stream=None):
    """:func:`bwd`, plus fp32 copies of dk and dv for the first ``n_lo`` and the
    last ``n_hi`` tokens of every sequence (swa_bwd_edges).  Returns
    ``(grads, dkv_lo, dkv_hi)`` with dkv_* of shape [B, n, Hkv, 2, 128]
    (dk, dv) or None when n is 0."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    p = make_params(B, T, Hq, Hkv, head_dim=D, window=window, rot_dim=rot_dim,
                    rope_base=rope_base, eps=eps, scale=scale)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(g),
                 torch.zeros(D, dtype=torch.float32, device=q.device),
                 torch.zeros(D, dtype=torch.float32, device=q.device))
    dq, dk, dv, dg, dwq, dwk = grads
    nbytes = int(lib().swa_bwd_workspace_size(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    lo = torch.empty((B, n_lo, Hkv, 2, D), dtype=torch.float32, device=q.device) if n_lo else None
    hi = torch.empty((B, n_hi, Hkv, 2, D), dtype=torch.float32, device=q.device) if n_hi else None
    extra = {"workspace": (workspace, torch.uint8, nbytes)}
    if lo is not None:
        extra["dkv_lo"] = (lo, torch.float32, lo.numel())
    if hi is not None:
        extra["dkv_hi"] = (hi, torch.float32, hi.numel())
    _need_bwd("swa_bwd_edges", q, k, v, g, wq, wk, lse, dO, grads, **extra)
    rc = lib().swa_bwd_edges(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(wq),
                             _ptr(wk), _ptr(lse), _ptr(dO), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg),
                             _ptr(dwq), _ptr(dwk), n_lo, _ptr(lo), n_hi, _ptr(hi),
                             _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "swa_bwd_edges")
    return grads, lo, hi


def bwd_halo(q, k, v, g, wq, wk, lse, dO, k_halo, v_halo, pos0, n_hi=0, *, window=128,
             rot_dim=42, rope_base=1e4, eps=1e-6, scale=0.0, workspace=None, grads=None,
             stream=None):
    """The backward of :func:`fwd_halo` (swa_bwd_halo).  Returns (grads, dkv_halo,
    dkv_hi): this chunk's fp32 share of the halo keys' dk, dv [B,127,Hkv,2,128],
    and its own last n_hi rows' dk, dv in fp32 (None when n_hi is 0)."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    p = make_params(B, T, Hq, Hkv, head_dim=D, window=window, rot_dim=rot_dim,
                    rope_base=rope_base, eps=eps, scale=scale)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(g),
                 torch.zeros(D, dtype=torch.float32, device=q.device),
                 torch.zeros(D, dtype=torch.float32, device=q.device))
    dq, dk, dv, dg, dwq, dwk = grads
    nbytes = int(lib().swa_bwd_workspace_size(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    halo = torch.empty((B, window - 1, Hkv, 2, D), dtype=torch.float32, device=q.device)
    hi = torch.empty((B, n_hi, Hkv, 2, D), dtype=torch.float32, device=q.device) if n_hi else None
    nh = B * (window - 1) * Hkv * D
    extra = {"workspace": (workspace, torch.uint8, nbytes),
             "k_halo": (k_halo, torch.bfloat16, nh), "v_halo": (v_halo, torch.bfloat16, nh)}
    if hi is not None:
        extra["dkv_hi"] = (hi, torch.float32, hi.numel())
    _need_bwd("swa_bwd_halo", q, k, v, g, wq, wk, lse, dO, grads, **extra)
    rc = lib().swa_bwd_halo(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(wq),
                            _ptr(wk), _ptr(lse), _ptr(dO), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg),
                            _ptr(dwq), _ptr(dwk), _ptr(k_halo), _ptr(v_halo), int(pos0),
                            _ptr(halo), n_hi, _ptr(hi), _ptr(workspace), workspace.numel(),
                            _stream(stream))
    _check(rc, "swa_bwd_halo")
    return grads, halo, hi


def bwd_noalloc(q, k, v, g, wq, wk, lse, dO, *, window=128, rot_dim=42, rope_base=1e4,
                eps=1e-6, scale=0.0, grads=None, stream=None):
    """As :func:`bwd`, with the library's fixed device scratch instead of a workspace."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    p = make_params(B, T, Hq, Hkv, head_dim=D, window=window, rot_dim=rot_dim,
                    rope_base=rope_base, eps=eps, scale=scale)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(g),
                 torch.zeros(D, dtype=torch.float32, device=q.device),
                 torch.zeros(D, dtype=torch.float32, device=q.device))
    dq, dk, dv, dg, dwq, dwk = grads
    _need_bwd("swa_bwd_noalloc", q, k, v, g, wq, wk, lse, dO, grads)
    rc = lib().swa_bwd_noalloc(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(wq),
                               _ptr(wk), _ptr(lse), _ptr(dO), _ptr(dq), _ptr(dk), _ptr(dv),
                               _ptr(dg), _ptr(dwq), _ptr(dwk), _stream(stream))
    _check(rc, "swa_bwd_noalloc")
    return grads


def decode_step(pos, q, k_new, v_new, g, wq, wk, k_cache, v_cache, *, rot_dim=42, rope_base=1e7,
                eps=1e-6, scale=0.0, out=None, flags=0, stream=None):
    """One decode step; updates the [N,Hkv,128,128] rings in place, returns o [N,Hq,128]."""
    N, Hq, D = q.shape
    Hkv, W = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    p = make_params(N, 1, Hq, Hkv, head_dim=D, window=W, rot_dim=rot_dim, rope_base=rope_base,
                    eps=eps, scale=scale, flags=flags)
    nq, nk = N * Hq * D, N * Hkv * D
    bf, f32 = torch.bfloat16, torch.float32
    _need("swa_decode_step", q.device, pos=(pos, torch.int64, N), q=(q, bf, nq),
          k_new=(k_new, bf, nk), v_new=(v_new, bf, nk), g=(g, bf, nq),
          wq=(wq, f32, D if N else 0), wk=(wk, f32, D if N else 0),
          k_cache=(k_cache, bf, nk * W), v_cache=(v_cache, bf, nk * W), out=(out, bf, nq))
    rc = lib().swa_decode_step(ctypes.byref(p), _ptr(pos), _ptr(q), _ptr(k_new), _ptr(v_new),
                               _ptr(g), _ptr(wq), _ptr(wk), _ptr(k_cache), _ptr(v_cache), _ptr(out),
                               _stream(stream))
    _check(rc, "swa_decode_step")
    return out


def prefill_to_ring(k, v, wk, k_cache, v_cache, *, Hq, rot_dim=42, rope_base=1e7, eps=1e-6,
                    stream=None):
    """Fill the [B,Hkv,128,128] decode rings from a prefill's k, v [B,T,Hkv,128]
    (swa_prefill_to_ring), so decode_step can continue at position T."""
    B, T, Hkv, D = k.shape
    W = k_cache.shape[2]
    p = make_params(B, T, Hq, Hkv, head_dim=D, window=W, rot_dim=rot_dim, rope_base=rope_base,
                    eps=eps)
    nk = B * T * Hkv * D if T else 0
    nr = B * Hkv * W * D if T else 0
    bf = torch.bfloat16
    _need("swa_prefill_to_ring", k.device, k=(k, bf, nk), v=(v, bf, nk),
          wk=(wk, torch.float32, D if nk else 0), k_cache=(k_cache, bf, nr),
          v_cache=(v_cache, bf, nr))
    rc = lib().swa_prefill_to_ring(ctypes.byref(p), _ptr(k), _ptr(v), _ptr(wk), _ptr(k_cache),
                                   _ptr(v_cache), _stream(stream))
    _check(rc, "swa_prefill_to_ring")


def global_fwd(q, k, v, wq, wk, k_cache, v_cache, *, rot_dim=42, rope_base=1e4, eps=1e-6,
               scale=0.0, out=None, lse=None, want_lse=False, flags=0, stream=None):
    """Global causal GQA layer over positions 0..T-1 (swa_global_fwd): no window,
    no gate.  q: [B,T,Hq,128]; k, v: [B,T,Hkv,128] bf16; wq, wk: [128] fp32.
    Fills slots 0..T-1 of k_cache, v_cache [B,Hkv,cap,128] (cap >= T) with k'
    and v and returns o (and lse [B,Hq,T] when asked)."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    cap = k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    p = make_params(B, T, Hq, Hkv, head_dim=D, window=0, rot_dim=rot_dim, rope_base=rope_base,
                    eps=eps, scale=scale, flags=flags)
    nq, nk = B * T * Hq * D, B * T * Hkv * D
    nc = B * Hkv * cap * D if nq else 0
    bf, f32 = torch.bfloat16, torch.float32
    opt = {} if lse is None else {"lse": (lse, f32, B * Hq * T)}
    _need("swa_global_fwd", q.device, q=(q, bf, nq), k=(k, bf, nk), v=(v, bf, nk),
          wq=(wq, f32, D if nq else 0), wk=(wk, f32, D if nq else 0), out=(out, bf, nq),
          k_cache=(k_cache, bf, nc), v_cache=(v_cache, bf, nc), **opt)
    rc = lib().swa_global_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(wq), _ptr(wk),
                              _ptr(out), _ptr(lse), _ptr(k_cache), _ptr(v_cache), cap,
                              _stream(stream))
    _check(rc, "swa_global_fwd")
    return (out, lse) if lse is not None else out


def global_decode_workspace_size(N, Hq, Hkv, cap, *, head_dim=128, rot_dim=42):
    p = make_params(N, 1, Hq, Hkv, head_dim=head_dim, window=0, rot_dim=rot_dim)
    return int(lib().swa_global_decode_workspace_size(ctypes.byref(p), cap))


def global_decode_step(pos, q, k_new, v_new, wq, wk, k_cache, v_cache, *, rot_dim=42,
                       rope_base=1e7, eps=1e-6, scale=0.0, out=None, workspace=None, flags=0,
                       stream=None):
    """One decode step of a global layer (swa_global_decode_step): writes k', v at
    slot pos[n] of the [N,Hkv,cap,128] caches and returns o [N,Hq,128]."""
    N, Hq, D = q.shape
    Hkv, cap = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    p = make_params(N, 1, Hq, Hkv, head_dim=D, window=0, rot_dim=rot_dim, rope_base=rope_base,
                    eps=eps, scale=scale, flags=flags)
    nbytes = int(lib().swa_global_decode_workspace_size(ctypes.byref(p), cap))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    nq, nk = N * Hq * D, N * Hkv * D
    bf, f32 = torch.bfloat16, torch.float32
    _need("swa_global_decode_step", q.device, pos=(pos, torch.int64, N), q=(q, bf, nq),
          k_new=(k_new, bf, nk), v_new=(v_new, bf, nk), wq=(wq, f32, D if N else 0),
          wk=(wk, f32, D if N else 0), k_cache=(k_cache, bf, nk * cap),
          v_cache=(v_cache, bf, nk * cap), out=(out, bf, nq),
          workspace=(workspace, torch.uint8, nbytes if N else 0))
    rc = lib().swa_global_decode_step(ctypes.byref(p), _ptr(pos), _ptr(q), _ptr(k_new),
                                      _ptr(v_new), _ptr(wq), _ptr(wk), _ptr(k_cache),
                                      _ptr(v_cache), cap, _ptr(out), _ptr(workspace),
                                      workspace.numel(), _stream(stream))
    _check(rc, "swa_global_decode_step")
    return out


def prefill_to_ring_varlen(k, v, wk, k_cache, v_cache, starts, lens, pos0=None, *, Hq,
                           rot_dim=42, rope_base=1e7, eps=1e-6, stream=None):
    """The ring handoff for a ragged or continued prefill (swa_prefill_to_ring_varlen):
    k, v [T, Hkv, 128] rows (packed, or a padded batch flattened); sequence b's
    lens[b] tokens start at row starts[b], at position pos0[b] (0 if None);
    rings [B, Hkv, 128, 128]."""
    T, Hkv, D = k.shape
    B, W = k_cache.shape[0], k_cache.shape[2]
    p = make_params(B, T, Hq, Hkv, head_dim=D, window=W, rot_dim=rot_dim, rope_base=rope_base,
                    eps=eps)
    i64, bf = torch.int64, torch.bfloat16
    nk = T * Hkv * D
    nr = B * Hkv * W * D
    extra = {} if pos0 is None else {"pos0": (pos0, i64, B)}
    _need("swa_prefill_to_ring_varlen", k_cache.device, starts=(starts, i64, B),
          lens=(lens, i64, B), k=(k, bf, nk), v=(v, bf, nk),
          wk=(wk, torch.float32, D if B else 0), k_cache=(k_cache, bf, nr),
          v_cache=(v_cache, bf, nr), **extra)
    rc = lib().swa_prefill_to_ring_varlen(ctypes.byref(p), _ptr(starts), _ptr(lens), _ptr(pos0),
                                          _ptr(k), _ptr(v), _ptr(wk), _ptr(k_cache),
                                          _ptr(v_cache), _stream(stream))
    _check(rc, "swa_prefill_to_ring_varlen")


def get_last_device_error(stream=None):
    """(code, site): SWA_OK or SWA_ERR_DEVICE_TIMEOUT with the raw site word; clears it."""
    site = ctypes.c_int(0)
    rc = lib().swa_get_last_device_error(_stream(stream), ctypes.byref(site))
    return rc, site.value
