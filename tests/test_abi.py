"""The C-ABI library loads, exports every declared entry point and rejects bad
arguments on the host (no GPU compute is needed for any of these checks)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import hybrid_sliding_window_gated_b200 as swa
from hybrid_sliding_window_gated_b200 import build as swa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    swa_build.build()
    return swa.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "swa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(swa_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert {"swa_fwd", "swa_bwd", "swa_decode_step", "swa_bwd_workspace_size",
            "swa_prefill_to_ring"} <= set(names)
    out = subprocess.check_output(["nm", "-D", "--defined-only", swa.LIB_PATH], text=True)
    exported = set(re.findall(r" T (swa_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(L, n)


def test_error_strings_and_version(L):
    for code in range(5):
        assert L.swa_error_string(code)
    assert b"sm_100a" in L.swa_version()


def _params(**kw):
    base = dict(B=1, T=256, Hq=4, Hkv=1)
    base.update(kw)
    B, T, Hq, Hkv = base.pop("B"), base.pop("T"), base.pop("Hq"), base.pop("Hkv")
    return swa.make_params(B, T, Hq, Hkv, **base)


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=6, Hkv=4), swa.ERR_INVALID_ARG),         # Hq not a multiple of Hkv
    (dict(rot_dim=41), swa.ERR_INVALID_ARG),          # odd rotary dims
    (dict(rot_dim=256), swa.ERR_INVALID_ARG),         # more rotary dims than head dims
    (dict(T=-1), swa.ERR_INVALID_ARG),
    (dict(eps=-1.0), swa.ERR_INVALID_ARG),
    (dict(head_dim=64), swa.ERR_UNSUPPORTED),         # tensor-core path is built for 128
    (dict(window=64), swa.ERR_UNSUPPORTED),
    (dict(rot_dim=40), swa.ERR_UNSUPPORTED),
    (dict(B=1 << 20, T=1 << 21), swa.ERR_UNSUPPORTED),  # 2^41 tokens: size products overflow
])
def test_bad_shapes_rejected_before_any_launch(L, kw, code):
    p = _params(**kw)
    nul = ctypes.c_void_p(0)
    assert L.swa_fwd(ctypes.byref(p), *([nul] * 9)) == code
    assert L.swa_bwd(ctypes.byref(p), *([nul] * 15), 0, nul) == code
    assert L.swa_bwd_workspace_size(ctypes.byref(p)) == 0


def test_null_pointers_rejected(L):
    p = _params()
    nul = ctypes.c_void_p(0)
    assert L.swa_fwd(ctypes.byref(p), *([nul] * 9)) == swa.ERR_INVALID_ARG
    assert L.swa_fwd(None, *([nul] * 9)) == swa.ERR_INVALID_ARG


def test_empty_problem_is_a_no_op(L):
    p = _params(T=0)
    nul = ctypes.c_void_p(0)
    assert L.swa_fwd(ctypes.byref(p), *([nul] * 9)) == swa.OK


def test_misaligned_pointer_rejected(L):
    p = _params()
    good = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 2)
    args = [good] * 9
    args[0] = bad
    assert L.swa_fwd(ctypes.byref(p), *args) == swa.ERR_INVALID_ARG


def test_decode_host_checks(L):
    nul = ctypes.c_void_p(0)
    good = ctypes.c_void_p(1 << 20)
    # more than 8 query heads per KV head: the decode kernel's row budget
    assert L.swa_decode_step(ctypes.byref(_params(Hq=16, Hkv=1)), *([good] * 11)) == \
        swa.ERR_UNSUPPORTED
    assert L.swa_decode_step(ctypes.byref(_params(window=64)), *([good] * 11)) == \
        swa.ERR_UNSUPPORTED
    assert L.swa_decode_step(ctypes.byref(_params()), *([nul] * 11)) == swa.ERR_INVALID_ARG
    assert L.swa_decode_step(ctypes.byref(_params(B=0)), *([nul] * 11)) == swa.OK
    args = [good] * 11
    args[0] = ctypes.c_void_p((1 << 20) + 4)  # positions must be 8-byte aligned
    assert L.swa_decode_step(ctypes.byref(_params()), *args) == swa.ERR_INVALID_ARG
    args = [good] * 11
    args[7] = ctypes.c_void_p((1 << 20) + 8)  # ring must be 16-byte aligned
    assert L.swa_decode_step(ctypes.byref(_params()), *args) == swa.ERR_INVALID_ARG


def test_bwd_host_checks(L):
    p = _params(B=1, T=256, Hq=4, Hkv=1)
    need = L.swa_bwd_workspace_size(ctypes.byref(p))
    assert need >= 256 * 4 * 128 * 2 + 256 * 4 * 4
    good = ctypes.c_void_p(1 << 20)
    args = [good] * 15
    assert L.swa_bwd(ctypes.byref(p), *args, need - 1, None) == swa.ERR_INVALID_ARG
    args[14] = ctypes.c_void_p((1 << 20) + 16)  # workspace must be 256-byte aligned
    assert L.swa_bwd(ctypes.byref(p), *args, need, None) == swa.ERR_INVALID_ARG
    for i in (0, 1, 3, 7, 8, 9, 10, 11):  # rows in 32-byte accesses: 16-byte alignment is not enough
        args = [good] * 15
        args[i] = ctypes.c_void_p((1 << 20) + 16)
        assert L.swa_bwd(ctypes.byref(p), *args, need, None) == swa.ERR_INVALID_ARG
    nul = ctypes.c_void_p(0)
    assert L.swa_bwd(ctypes.byref(_params(T=0)), *([nul] * 15), 0, nul) == swa.OK


def test_bwd_edges_host_checks(L):
    p = _params(B=1, T=256, Hq=4, Hkv=1)
    need = L.swa_bwd_workspace_size(ctypes.byref(p))
    good = ctypes.c_void_p(1 << 20)
    nul = ctypes.c_void_p(0)
    i64 = ctypes.c_int64

    def call(n_lo, lo, n_hi, hi, params=p):
        return L.swa_bwd_edges(ctypes.byref(params), *([good] * 14), i64(n_lo), lo, i64(n_hi), hi,
                               good, need, None)
    assert call(-1, good, 0, nul) == swa.ERR_INVALID_ARG      # negative count
    assert call(0, nul, 257, good) == swa.ERR_INVALID_ARG     # more rows than T
    assert call(5, nul, 0, nul) == swa.ERR_INVALID_ARG        # rows but no buffer
    assert call(5, ctypes.c_void_p((1 << 20) + 4), 0, nul) == swa.ERR_INVALID_ARG  # fp32 pairs
    assert L.swa_bwd_edges(ctypes.byref(_params(T=0)), *([nul] * 14), i64(0), nul, i64(0), nul,
                           nul, 0, None) == swa.OK


def test_prefill_to_ring_host_checks(L):
    nul = ctypes.c_void_p(0)
    good = ctypes.c_void_p(1 << 20)
    p = _params(B=2, T=300, Hq=8, Hkv=2)
    assert L.swa_prefill_to_ring(ctypes.byref(p), *([nul] * 5), nul) == swa.ERR_INVALID_ARG
    assert L.swa_prefill_to_ring(ctypes.byref(_params(B=0)), *([nul] * 5), nul) == swa.OK
    assert L.swa_prefill_to_ring(ctypes.byref(_params(T=0)), *([nul] * 5), nul) == swa.OK
    assert L.swa_prefill_to_ring(ctypes.byref(_params(window=64)), *([good] * 5), nul) == \
        swa.ERR_UNSUPPORTED
    args = [good] * 5
    args[3] = ctypes.c_void_p((1 << 20) + 8)  # rings must be 16-byte aligned
    assert L.swa_prefill_to_ring(ctypes.byref(p), *args, nul) == swa.ERR_INVALID_ARG


# ------------------------------------------- the Python binding's own checks

def _prefill_cpu(B=1, T=64, Hq=4, Hkv=1):
    bf = torch.bfloat16
    return dict(q=torch.zeros(B, T, Hq, 128, dtype=bf), k=torch.zeros(B, T, Hkv, 128, dtype=bf),
                v=torch.zeros(B, T, Hkv, 128, dtype=bf), g=torch.zeros(B, T, Hq, 128, dtype=bf),
                wq=torch.ones(128), wk=torch.ones(128))


def test_binding_rejects_tensors_the_kernels_would_misread():
    """Checked on the host before the library is called: dtype, element count,
    contiguity, then a CUDA device (the CPU tensors here fail that last one)."""
    d = _prefill_cpu()
    with pytest.raises(ValueError, match="CUDA"):
        swa.fwd(**d)
    with pytest.raises(TypeError, match="q is torch.float32"):
        swa.fwd(**dict(d, q=d["q"].float()))
    with pytest.raises(ValueError, match="k has 4096 elements"):
        swa.fwd(**dict(d, k=d["k"][:, :32].contiguous()))
    with pytest.raises(ValueError, match="contiguous"):
        swa.fwd(**dict(d, g=d["g"].transpose(1, 2).contiguous().transpose(1, 2)))
    with pytest.raises(ValueError, match="lse"):
        swa.fwd(**d, lse=torch.empty(1, 4, 63))
    lse = torch.zeros(1, 4, 64)
    with pytest.raises(TypeError, match="dO is torch.float32"):
        swa.bwd(*d.values(), lse, torch.zeros(1, 64, 4, 128))
    with pytest.raises(TypeError, match="workspace"):
        swa.bwd(*d.values(), lse, d["q"].clone(), workspace=torch.empty(10, dtype=torch.int32),
                grads=(d["q"].clone(), d["k"].clone(), d["v"].clone(), d["g"].clone(),
                       torch.zeros(128), torch.zeros(128)))


def test_binding_checks_decode_and_ring_tensors():
    bf = torch.bfloat16
    N, Hq, Hkv = 3, 8, 2
    x = dict(pos=torch.zeros(N, dtype=torch.int64), q=torch.zeros(N, Hq, 128, dtype=bf),
             k_new=torch.zeros(N, Hkv, 128, dtype=bf), v_new=torch.zeros(N, Hkv, 128, dtype=bf),
             g=torch.zeros(N, Hq, 128, dtype=bf), wq=torch.ones(128), wk=torch.ones(128),
             k_cache=torch.zeros(N, Hkv, 128, 128, dtype=bf),
             v_cache=torch.zeros(N, Hkv, 128, 128, dtype=bf))
    with pytest.raises(TypeError, match="pos is torch.int32"):
        swa.decode_step(**dict(x, pos=x["pos"].int()))
    with pytest.raises(ValueError, match="v_cache has"):
        swa.decode_step(**dict(x, v_cache=x["v_cache"][:2].contiguous()))
    with pytest.raises(ValueError, match="CUDA"):
        swa.decode_step(**x)
    d = _prefill_cpu(B=N, T=200, Hq=Hq, Hkv=Hkv)
    with pytest.raises(ValueError, match="k_cache has"):
        swa.prefill_to_ring(d["k"], d["v"], d["wk"], x["k_cache"][:, :1].contiguous(),
                            x["v_cache"], Hq=Hq)
    with pytest.raises(TypeError, match="wk is torch.bfloat16"):
        swa.prefill_to_ring(d["k"], d["v"], d["wk"].bfloat16(), x["k_cache"], x["v_cache"], Hq=Hq)


def test_binding_passes_empty_problems_through():
    """Empty problems skip the tensor checks and reach the library, which
    returns without touching a pointer."""
    bf = torch.bfloat16
    e = dict(q=torch.zeros(1, 0, 4, 128, dtype=bf), k=torch.zeros(1, 0, 1, 128, dtype=bf),
             v=torch.zeros(1, 0, 1, 128, dtype=bf), g=torch.zeros(1, 0, 4, 128, dtype=bf),
             wq=torch.ones(128), wk=torch.ones(128))
    swa.build.build()
    assert swa.fwd(**e, stream=_NullStream()).shape == (1, 0, 4, 128)


class _NullStream:
    cuda_stream = 0


def test_global_layer_host_checks(L):
    good = ctypes.c_void_p(1 << 20)
    nul = ctypes.c_void_p(0)
    i64 = ctypes.c_int64
    p = _params(B=1, T=256, Hq=8, Hkv=2, window=0)

    def fwd(params, cap, lse=nul, q=good):
        return L.swa_global_fwd(ctypes.byref(params), q, good, good, good, good, good, lse,
                                good, good, i64(cap), None)
    assert fwd(_params(B=1, T=256, Hq=8, Hkv=2), 256) == swa.ERR_INVALID_ARG  # window must be 0
    assert fwd(p, 255) == swa.ERR_INVALID_ARG                               # cache shorter than T
    assert fwd(p, 256, q=ctypes.c_void_p((1 << 20) + 8)) == swa.ERR_INVALID_ARG
    assert fwd(p, 256, lse=ctypes.c_void_p((1 << 20) + 2)) == swa.ERR_INVALID_ARG
    assert fwd(_params(B=1, T=0, Hq=8, Hkv=2, window=0), 0) == swa.OK
    assert fwd(_params(B=1, T=256, Hq=8, Hkv=2, window=0, head_dim=64), 256) == swa.ERR_UNSUPPORTED

    pd = _params(B=4, T=1, Hq=8, Hkv=2, window=0)
    need = L.swa_global_decode_workspace_size(ctypes.byref(pd), i64(5000))
    assert need >= 4 * 2 * 3 * 4 * 128 * 4   # 3 chunks of 2048 slots x 4 heads x 128 dims fp32
    assert L.swa_global_decode_workspace_size(ctypes.byref(pd), i64(0)) == 0

    def dec(params, cap, ws_bytes, ws=good, pos=good):
        # pos, then q, k_new, v_new, wq, wk, k_cache, v_cache
        return L.swa_global_decode_step(ctypes.byref(params), pos, *([good] * 7), i64(cap), good,
                                        ws, ws_bytes, None)
    assert dec(pd, 5000, need - 1) == swa.ERR_INVALID_ARG
    assert dec(pd, 5000, need, ws=ctypes.c_void_p((1 << 20) + 16)) == swa.ERR_INVALID_ARG
    assert dec(pd, 5000, need, pos=ctypes.c_void_p((1 << 20) + 4)) == swa.ERR_INVALID_ARG
    assert dec(_params(B=4, T=1, Hq=32, Hkv=2, window=0), 5000, need) == swa.ERR_UNSUPPORTED
    assert dec(pd, 0, need) == swa.ERR_INVALID_ARG
    assert dec(_params(B=0, T=1, Hq=8, Hkv=2, window=0), 5000, 0) == swa.OK
