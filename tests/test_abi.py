"""The C-ABI library loads, exports every declared entry point and rejects bad
arguments on the host (no GPU compute is needed for any of these checks)."""
import ctypes
import os
import re
import subprocess

import pytest

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
