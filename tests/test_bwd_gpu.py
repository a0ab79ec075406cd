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


def test_upstream_gradient_beyond_fp16_range_is_reported():
    """dA = dO * sigmoid(g) is staged in fp16 too: a dO past its range is refused."""
    cfg, d = _small_inputs()
    o, lse = swa.fwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], want_lse=True)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    d["dO"][0, 150, 2, 100] = -2.0e5
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
