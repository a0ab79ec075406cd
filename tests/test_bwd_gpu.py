"""GPU parity of the backward (swa_bwd through the C ABI) against the fp64
oracle's exact chain rule: dq, dk, dv, dg element by element within the bf16
tolerances, dwq and dwk by relative Frobenius error.  The lse the backward
reads comes from the GPU forward, as in training."""
import numpy as np
import pytest
import torch

import hybrid_sliding_window_gated_b200 as swa
import oracle
import workloads
from swa_testutil import REL_FRO, ZERO_REF, assert_parity, errors, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def f64(t):
    return t.detach().float().cpu().double().numpy()


def run_gpu(d, cfg):
    o, lse = swa.fwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], window=cfg.W,
                     rot_dim=cfg.R, rope_base=cfg.base, eps=cfg.eps, want_lse=True)
    grads = swa.bwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], lse, d["dO"], window=cfg.W,
                    rot_dim=cfg.R, rope_base=cfg.base, eps=cfg.eps)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    return grads


def check_bwd(cfg):
    inp = workloads.prefill_inputs(cfg, device="cpu", with_grad_out=True)
    ref = oracle.bwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]), f64(inp["wq"]),
                     f64(inp["wk"]), f64(inp["dO"]), W=cfg.W, R=cfg.R, base=cfg.base, eps=cfg.eps)
    got = run_gpu({k: v.to(DEV) for k, v in inp.items()}, cfg)
    for name, x, r in zip(["dq", "dk", "dv", "dg"], got[:4], ref[:4]):
        assert_parity(to_f64(x), r, name)
    for name, x, r in zip(["dwq", "dwk"], got[4:], ref[4:]):
        if np.abs(r).max() <= ZERO_REF:
            assert np.abs(to_f64(x)).max() <= 1e-4, name
            continue
        fro = errors(to_f64(x), r)[1]
        assert fro <= REL_FRO, f"{name}: rel_fro={fro:.3e}"


def test_tiny_config_backward():
    check_bwd(workloads.TINY)


def check_bwd_scaled(cfg, do_scale=None, v_scale=1.0, row_scale=None):
    """The backward at other magnitudes of dO and v than N(0, 1).  dO and v are
    rescaled in fp32 and rounded to bf16 again (the oracle reads the same
    bits); dO either by one factor or by a factor per (token, head) row.
    Every gradient is compared by relative Frobenius error (max-abs bounds
    mean nothing at these scales) and by max-abs error relative to the
    product of the input scales it carries."""
    inp = workloads.prefill_inputs(cfg, device="cpu", with_grad_out=True)
    if do_scale is not None:
        inp["dO"] = (inp["dO"].float() * do_scale).bfloat16()
    if row_scale is not None:
        inp["dO"] = (inp["dO"].float() * row_scale[..., None]).bfloat16()
    inp["v"] = (inp["v"].float() * v_scale).bfloat16()
    ref = oracle.bwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]), f64(inp["wq"]),
                     f64(inp["wk"]), f64(inp["dO"]), W=cfg.W, R=cfg.R, base=cfg.base, eps=cfg.eps)
    got = run_gpu({k: v.to(DEV) for k, v in inp.items()}, cfg)
    s_do = 1.0 if do_scale is None else do_scale
    carried = {"dq": s_do * v_scale, "dk": s_do * v_scale, "dv": s_do, "dg": s_do * v_scale}
    for name, x, r in zip(["dq", "dk", "dv", "dg"], got[:4], ref[:4]):
        x = to_f64(x)
        assert np.all(np.isfinite(x)), name
        ma, fro = errors(x, r)
        assert fro <= REL_FRO, f"{name}: rel_fro={fro:.3e}"
        if row_scale is None:
            assert ma <= 2e-2 * carried[name], f"{name}: max_abs={ma:.3e}"
    for name, x, r in zip(["dwq", "dwk"], got[4:], ref[4:]):
        fro = errors(to_f64(x), r)[1]
        assert fro <= REL_FRO, f"{name}: rel_fro={fro:.3e}"
    return got, ref


@pytest.mark.parametrize("do_scale", [1e-3, 1e-5, 1e-7, 1e-12, 1e3, 1e6])
def test_backward_at_upstream_gradient_scales(do_scale):
    """Upstream gradients of training are far below N(0, 1) per element; fp16
    staging of dA and dS without a scale would sink them into its subnormals."""
    check_bwd_scaled(workloads.custom_prefill(1, 700, 8, 2, seed=41, backward=True),
                     do_scale=do_scale)


@pytest.mark.parametrize("v_scale,do_scale", [(1e-3, None), (1e-3, 1e-5), (30.0, 1e-4),
                                              (1e-4, 1.0)])
def test_backward_at_value_scales(v_scale, do_scale):
    """Small v makes dP and dS small too: dS is staged with a scale from max|v|.
    (v itself is staged in fp16, exactly for |v| >= 2^-14; below, its absolute
    error is at most 2^-25, which the smallest scale here keeps well inside
    the bound.)"""
    check_bwd_scaled(workloads.custom_prefill(1, 520, 4, 1, seed=42, backward=True),
                     do_scale=do_scale, v_scale=v_scale)


def test_backward_with_row_magnitudes_spanning_six_decades():
    """dO rows (token, head) scaled by 10^-U(0, 6): each query row is staged
    with its own scale, so the smallest rows' dq keeps its relative accuracy;
    the key-major pass shares one scale per key tile."""
    cfg = workloads.custom_prefill(2, 600, 8, 2, seed=43, backward=True)
    gen = torch.Generator().manual_seed(44)
    rs = 10.0 ** (-6.0 * torch.rand((cfg.B, cfg.T, cfg.Hq), generator=gen))
    got, ref = check_bwd_scaled(cfg, row_scale=rs)
    small = (rs < 1e-4).numpy()
    assert small.sum() > 100
    fro = errors(to_f64(got[0])[small], ref[0][small])[1]
    assert fro <= REL_FRO, f"dq of the rows under 1e-4: rel_fro={fro:.3e}"


@pytest.mark.parametrize("g_mean", [-8.0, 8.0])
def test_backward_with_nearly_shut_or_open_gates(g_mean):
    """Gate logits ~ N(+-8, 1): sigma or 1 - sigma is ~3e-4, where a sigmoid
    formed as 1/2 + tanh/2 (or sigma (1 - sigma) formed by cancellation)
    loses its relative accuracy; dA = dO sigma and dg = dO A sigma (1 - sigma)
    are compared by relative Frobenius error."""
    cfg = workloads.custom_prefill(1, 600, 8, 2, seed=45, backward=True)
    inp = workloads.prefill_inputs(cfg, device="cpu", with_grad_out=True)
    inp["g"] = (inp["g"].float() + g_mean).bfloat16()
    ref = oracle.bwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]), f64(inp["wq"]),
                     f64(inp["wk"]), f64(inp["dO"]), W=cfg.W, R=cfg.R, base=cfg.base, eps=cfg.eps)
    got = run_gpu({k: v.to(DEV) for k, v in inp.items()}, cfg)
    for name, x, r in zip(["dq", "dk", "dv", "dg", "dwq", "dwk"], got, ref):
        fro = errors(to_f64(x), r)[1]
        assert fro <= REL_FRO, f"{name}: rel_fro={fro:.3e}"


def test_training_shape_backward_at_gradient_scale_1e_6():
    cfg = workloads.TRAIN
    check_bwd_scaled(cfg, do_scale=1e-6)


@pytest.mark.parametrize("B,T,Hq,Hkv", [
    (1, 1, 4, 1), (1, 127, 4, 1), (1, 128, 4, 1), (1, 129, 4, 1), (2, 300, 8, 2),
    (1, 520, 2, 2), (1, 700, 3, 1), (3, 257, 8, 8), (1, 1000, 32, 8),
])
def test_backward_shapes_and_ragged_tails(B, T, Hq, Hkv):
    check_bwd(workloads.custom_prefill(B, T, Hq, Hkv, base=1e4, seed=B * 1000 + T + 7,
                                       backward=True))


@pytest.mark.parametrize("B,T,Hq,Hkv", [(40, 384, 6, 2), (50, 300, 2, 2)])
def test_backward_odd_pair_counts_inside_a_cta(B, T, Hq, Hkv):
    """More key tiles than CTAs, with an odd group size: the last key tile of
    each (sequence, kv head) chain meets an odd number of (query tile, head)
    pairs, and chains meet inside one CTA's range of tiles, so the key-major
    pass's alternation of pairs between its warpgroups changes phase there."""
    check_bwd(workloads.custom_prefill(B, T, Hq, Hkv, base=1e4, seed=B * 1000 + T + 11,
                                       backward=True))


@pytest.mark.parametrize("rot_dim", [0, 32, 48])
def test_backward_other_rot_dims(rot_dim):
    check_bwd(workloads.custom_prefill(1, 300, 4, 2, base=1e4, seed=17, R=rot_dim, backward=True))


def test_backward_large_rope_base():
    check_bwd(workloads.custom_prefill(1, 2000, 4, 1, base=1e7, seed=18, backward=True))


def test_training_shape_backward():
    check_bwd(workloads.TRAIN)


def test_weight_gradients_accumulate():
    """dwq and dwk are added into the caller's buffers."""
    cfg = workloads.custom_prefill(1, 256, 4, 1, seed=19, backward=True)
    d = {k: v.to(DEV) for k, v in workloads.prefill_inputs(cfg, with_grad_out=True).items()}
    g1 = run_gpu(d, cfg)
    o, lse = swa.fwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], want_lse=True)
    dwq0 = torch.full_like(g1[4], 1.5)
    dwk0 = torch.full_like(g1[5], -2.0)
    grads = (torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["v"]),
             torch.empty_like(d["g"]), dwq0.clone(), dwk0.clone())
    swa.bwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], lse, d["dO"], grads=grads)
    torch.cuda.synchronize()
    torch.testing.assert_close(grads[4] - dwq0, g1[4], rtol=1e-4, atol=1e-4)
    torch.testing.assert_close(grads[5] - dwk0, g1[5], rtol=1e-4, atol=1e-4)


def _small_inputs():
    cfg = workloads.custom_prefill(1, 200, 4, 1, seed=23, backward=True)
    d = {k: v.to(DEV) for k, v in workloads.prefill_inputs(cfg, with_grad_out=True).items()}
    return cfg, d


def test_values_beyond_fp16_range_are_reported():
    """The backward stages v and dA in fp16; a value past its range is refused."""
    cfg, d = _small_inputs()
    o, lse = swa.fwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], want_lse=True)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    d["v"][0, 5, 0, 7] = 1.0e6
    swa.bwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], lse, d["dO"])
    assert swa.get_last_device_error()[0] == swa.ERR_INVALID_ARG
    assert swa.get_last_device_error()[0] == swa.OK  # cleared


def test_upstream_gradient_beyond_the_staging_range_is_reported():
    """dA = dO * sigmoid(g) is staged in fp16 after a per-row power-of-two
    scale; a finite |dO| >= 2^63 is beyond what that scale covers and is refused."""
    cfg, d = _small_inputs()
    o, lse = swa.fwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], want_lse=True)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    d["dO"][0, 150, 2, 100] = -1.0e20
    swa.bwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], lse, d["dO"])
    assert swa.get_last_device_error()[0] == swa.ERR_INVALID_ARG
    assert swa.get_last_device_error()[0] == swa.OK


def test_weights_beyond_fp16_operands_are_reported():
    cfg, d = _small_inputs()
    o, lse = swa.fwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], want_lse=True)
    d["wk"][3] = 1.0e4
    swa.bwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], lse, d["dO"])
    assert swa.get_last_device_error()[0] == swa.ERR_INVALID_ARG
    # the context still computes correct gradients afterwards
    check_bwd(workloads.TINY)


def test_forced_timeout_is_reported_and_context_survives():
    cfg, d = _small_inputs()
    o, lse = swa.fwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], want_lse=True)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    swa.bwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], lse, d["dO"],
            flags=swa.FLAG_FORCE_TIMEOUT)
    code, site = swa.get_last_device_error()
    assert code == swa.ERR_DEVICE_TIMEOUT and site >= 0x100
    assert swa.get_last_device_error()[0] == swa.OK
    check_bwd(workloads.TINY)


@pytest.mark.parametrize("n_lo,n_hi", [(127, 127), (0, 50), (300, 0), (1, 299)])
def test_edge_rows_in_fp32(n_lo, n_hi):
    """swa_bwd_edges: the fp32 copies of the first n_lo and last n_hi rows of dk
    and dv round to exactly the bf16 rows the same call writes, and match the
    oracle; the other outputs equal swa_bwd's bit for bit."""
    cfg = workloads.custom_prefill(2, 300, 8, 2, seed=46, backward=True)
    inp = workloads.prefill_inputs(cfg, device="cpu", with_grad_out=True)
    d = {k: v.to(DEV) for k, v in inp.items()}
    o, lse = swa.fwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], want_lse=True)
    plain = swa.bwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], lse, d["dO"])
    grads, lo, hi = swa.bwd_edges(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], lse, d["dO"],
                                  n_lo, n_hi)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    for a, b in zip(grads[:4], plain[:4]):
        assert torch.equal(a, b)
    ref = oracle.bwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]), f64(inp["wq"]),
                     f64(inp["wk"]), f64(inp["dO"]), W=cfg.W, R=cfg.R, base=cfg.base, eps=cfg.eps)
    T = cfg.T
    for buf, rows in ((lo, slice(0, n_lo)), (hi, slice(T - n_hi, T))):
        if buf is None:
            continue
        for j, (name, full) in enumerate((("dk", grads[1]), ("dv", grads[2]))):
            assert torch.equal(buf[:, :, :, j].to(torch.bfloat16), full[:, rows]), name
            assert_parity(to_f64(buf[:, :, :, j]), ref[1 + j][:, rows], f"{name} edge rows")
