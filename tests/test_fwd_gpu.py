"""GPU forward parity: swa_fwd (through the C ABI) against the fp64 oracle.

Small shapes are compared element by element on every output.  The
layer-shape and long-context configurations run at full size in the launch
configuration the benchmark times, and are compared on every row too: the
oracle recomputes them in chunks of consecutive query rows while the test
accumulates max|delta|, sum(delta^2) and sum(ref^2) in fp64, so no full fp64
copy of the output is ever held.
"""
import math

import numpy as np
import pytest
import torch

import hybrid_sliding_window_gated_b200 as swa
import oracle
import workloads
from swa_testutil import assert_parity, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
# lse is a smooth maximum of the scores, so its error is bounded by the score
# error, which bf16 rounding of q' and k' (relative 2^-9 per element) keeps
# well under 2e-2 for unit-RMS rows.
LSE_ATOL = 2e-2


def run_gpu(inp, cfg, want_lse=True):
    return swa.fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["wq"], inp["wk"],
                   window=cfg.W, rot_dim=cfg.R, rope_base=cfg.base, eps=cfg.eps,
                   want_lse=want_lse)


def oracle_full(inp, cfg):
    f = lambda t: t.float().cpu().double().numpy()
    return oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["g"]), f(inp["wq"]),
                      f(inp["wk"]), W=cfg.W, R=cfg.R, base=cfg.base, eps=cfg.eps)


def check_full(cfg, device=DEV, inp=None):
    inp = workloads.prefill_inputs(cfg, device="cpu") if inp is None else inp
    o_ref, lse_ref = oracle_full(inp, cfg)
    dinp = {k: v.to(device) for k, v in inp.items()}
    o, lse = run_gpu(dinp, cfg)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    assert_parity(to_f64(o), o_ref, "o")
    # lse [B,Hq,T] vs oracle [B,T,Hq]
    np.testing.assert_allclose(to_f64(lse), lse_ref.transpose(0, 2, 1), rtol=0, atol=LSE_ATOL)
    return o, lse


def test_tiny_config_full():
    check_full(workloads.TINY)


@pytest.mark.parametrize("B,T,Hq,Hkv", [
    (1, 1, 4, 1), (1, 127, 4, 1), (1, 128, 4, 1), (1, 129, 4, 1), (2, 300, 8, 2),
    (1, 520, 2, 2), (1, 700, 3, 1), (3, 257, 8, 8), (1, 1000, 32, 8),
])
def test_shapes_and_ragged_tails(B, T, Hq, Hkv):
    check_full(workloads.custom_prefill(B, T, Hq, Hkv, base=1e4, g_std=2.0, seed=B * 1000 + T))


@pytest.mark.parametrize("rot_dim", [0, 32, 48])
def test_other_rot_dims(rot_dim):
    check_full(workloads.custom_prefill(1, 300, 4, 2, base=1e4, seed=7, R=rot_dim))


def test_large_rope_base_and_positions():
    check_full(workloads.custom_prefill(1, 2000, 4, 1, base=1e7, seed=8))


def test_saturated_gate_gives_zero_and_ungated():
    cfg = workloads.custom_prefill(1, 300, 4, 1, seed=9)
    inp = {k: v.to(DEV) for k, v in workloads.prefill_inputs(cfg).items()}
    inp["g"] = torch.full_like(inp["g"], float("-inf"))
    o = run_gpu(inp, cfg, want_lse=False)
    assert torch.count_nonzero(o).item() == 0


def test_saturated_gate_open_gives_ungated_attention():
    """g = +inf: sigmoid is exactly 1, so o is the plain window attention."""
    cfg = workloads.custom_prefill(2, 300, 8, 2, seed=10)
    inp = workloads.prefill_inputs(cfg)
    inp["g"] = torch.full_like(inp["g"], float("inf"))
    check_full(cfg, inp=inp)


@pytest.mark.parametrize("g_mean", [-8.0, -14.0, 8.0])
def test_nearly_shut_gate_keeps_relative_accuracy(g_mean):
    """Gate logits ~ N(g_mean, 1): for g << 0, sigma(g) ~ e^g and o is tiny;
    compared by relative Frobenius error (as well as max-abs)."""
    cfg = workloads.custom_prefill(2, 300, 8, 2, seed=11)
    inp = workloads.prefill_inputs(cfg)
    inp["g"] = (inp["g"].float() + g_mean).bfloat16()
    check_full(cfg, inp=inp)


@pytest.mark.parametrize("B,T,Hq,Hkv,wmax", [(1, 700, 4, 1, 2.5), (2, 300, 8, 2, 2.5),
                                             (1, 260, 4, 2, 6.0)])
def test_exact_two_pass_softmax_branch(B, T, Hq, Hkv, wmax):
    """The forward skips the row-max pass when the norm bound on the scores,
    scale * D * max|wq| * max|wk|, keeps exp2 in range; larger weights (here
    one entry of each set to +-wmax, product above 3.7) take the exact
    two-pass softmax, whose scores then also reach far larger magnitudes."""
    cfg = workloads.custom_prefill(B, T, Hq, Hkv, base=1e4, g_std=2.0, seed=50 + T)
    inp = workloads.prefill_inputs(cfg)
    inp["wq"][5] = wmax
    inp["wk"][77] = -wmax
    inp["wk"][3] = wmax
    check_full(cfg, inp=inp)


def streamed_full_check(cfg, chunk=4096):
    """Every row of a full-size forward against the oracle, chunk by chunk."""
    inp = workloads.prefill_inputs(cfg, device=DEV)
    o, lse = run_gpu(inp, cfg)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    host = {k: v.cpu() for k, v in inp.items()}
    del inp
    o_cpu, lse_cpu = o.cpu(), lse.cpu()
    del o, lse
    max_abs, dd, rr, lse_err = 0.0, 0.0, 0.0, 0.0
    for b in range(cfg.B):
        for t0 in range(0, cfg.T, chunk):
            t1 = min(cfg.T, t0 + chunk)
            ref, lref = oracle.fwd_rows(host["q"], host["k"], host["v"], host["g"], host["wq"],
                                        host["wk"], b, t0, t1, W=cfg.W, R=cfg.R, base=cfg.base,
                                        eps=cfg.eps)
            got = to_f64(o_cpu[b:b + 1, t0:t1])
            assert np.all(np.isfinite(got)), f"non-finite o in b={b} [{t0},{t1})"
            d = got - ref
            max_abs = max(max_abs, float(np.abs(d).max()))
            dd += float((d * d).sum())
            rr += float((ref * ref).sum())
            le = np.abs(to_f64(lse_cpu[b:b + 1, :, t0:t1]) - lref.transpose(0, 2, 1)).max()
            lse_err = max(lse_err, float(le))
    fro = (dd / rr) ** 0.5
    assert max_abs <= 2e-2 and fro <= 5e-3, f"o: max_abs={max_abs:.3e} rel_fro={fro:.3e}"
    assert lse_err <= LSE_ATOL, f"lse: max_abs={lse_err:.3e}"
    return max_abs, fro


def test_layer_shape_every_row():
    streamed_full_check(workloads.LAYER)


def test_long_context_every_row():
    streamed_full_check(workloads.LONG)


def test_forced_timeout_is_reported_and_context_survives():
    cfg = workloads.TINY
    inp = {k: v.to(DEV) for k, v in workloads.prefill_inputs(cfg).items()}
    assert swa.get_last_device_error()[0] == swa.OK
    swa.fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["wq"], inp["wk"], rope_base=cfg.base,
            flags=swa.FLAG_FORCE_TIMEOUT)
    code, site = swa.get_last_device_error()
    assert code == swa.ERR_DEVICE_TIMEOUT and site >= 0x100
    assert swa.get_last_device_error()[0] == swa.OK  # cleared
    check_full(cfg)  # the context is still usable and results are right


def test_training_shape_forward_full():
    """The 1 x 16384 training shape, every output element against the oracle."""
    check_full(workloads.TRAIN)
