"""Shared helpers for the GPU parity tests (comparison metrics, input staging)."""
import numpy as np
import torch

# Tolerances for bf16 I/O with fp32 accumulation: max-abs error and relative
# Frobenius error of each output tensor against the fp64 oracle.
MAX_ABS = 2e-2
REL_FRO = 5e-3


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = got - ref
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    fro = float(np.sqrt((d * d).sum()) / max(np.sqrt((ref * ref).sum()), 1e-300))
    return max_abs, fro


# A reference whose entries are all below this is zero up to fp64 rounding
# (e.g. dq of a one-token sequence, where P = 1 makes dS vanish exactly): the
# relative Frobenius error is undefined there and only the max-abs bound applies.
ZERO_REF = 1e-9


def assert_parity(got, ref, what, max_abs=MAX_ABS, rel_fro=REL_FRO):
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    ma, fr = errors(got, ref)
    if np.size(ref) and np.abs(ref).max() <= ZERO_REF:
        assert ma <= max_abs, f"{what}: max_abs={ma:.3e} (zero reference)"
        return ma, 0.0
    assert ma <= max_abs and fr <= rel_fro, f"{what}: max_abs={ma:.3e} rel_fro={fr:.3e}"
    return ma, fr


def to_f64(t):
    return t.detach().float().cpu().double().numpy()
