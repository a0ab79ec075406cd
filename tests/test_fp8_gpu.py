"""GPU parity of the forward with FP8 E4M3 q, k, v (swa_fwd_fp8 through the C
ABI) against the fp64 oracle on the dequantised inputs: the E4M3 bytes
decoded by the oracle (pinned against torch and the encoding), times each
tensor's factor.  The tolerances are the bf16 path's: every E4M3 value is
exact in bf16 and the factors fold into per-row factors."""
import numpy as np
import pytest
import torch

import hybrid_sliding_window_gated_b200 as swa
import oracle
import workloads
from swa_testutil import assert_parity, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
LSE_ATOL = 2e-2


def dequant(x8, s):
    return oracle.e4m3_to_f64(x8.view(torch.uint8).cpu().numpy()) * float(s)


def run(x, cfg):
    d = {k: v.to(DEV) for k, v in x.items()}
    o, lse = swa.fwd_fp8(d["q8"], d["k8"], d["v8"], d["qkv_scale"], d["g"], d["wq"], d["wk"],
                         window=cfg.W, rot_dim=cfg.R, rope_base=cfg.base, eps=cfg.eps,
                         want_lse=True)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    return o, lse


def check(cfg, x=None):
    x = workloads.fp8_prefill_inputs(cfg) if x is None else x
    o, lse = run(x, cfg)
    s = x["qkv_scale"].tolist()
    f = lambda t: t.float().double().numpy()
    o_ref, lse_ref = oracle.fwd(dequant(x["q8"], s[0]), dequant(x["k8"], s[1]),
                                dequant(x["v8"], s[2]), f(x["g"]), f(x["wq"]), f(x["wk"]),
                                W=cfg.W, R=cfg.R, base=cfg.base, eps=cfg.eps)
    assert_parity(to_f64(o), o_ref, "fp8 o")
    np.testing.assert_allclose(to_f64(lse), lse_ref.transpose(0, 2, 1), rtol=0, atol=LSE_ATOL)
    return o


@pytest.mark.parametrize("B,T,Hq,Hkv", [
    (1, 1, 4, 1), (1, 129, 4, 1), (2, 300, 8, 2), (1, 700, 3, 1), (1, 1000, 32, 8),
])
def test_fp8_shapes_and_ragged_tails(B, T, Hq, Hkv):
    check(workloads.custom_prefill(B, T, Hq, Hkv, base=1e4, g_std=2.0, seed=80 + T))


def test_fp8_tiny_config():
    check(workloads.TINY)


@pytest.mark.parametrize("rot_dim", [0, 32, 48])
def test_fp8_other_rot_dims(rot_dim):
    check(workloads.custom_prefill(1, 300, 4, 2, base=1e4, seed=81, R=rot_dim))


def test_fp8_exact_two_pass_branch():
    cfg = workloads.custom_prefill(1, 400, 4, 1, base=1e4, seed=82)
    x = workloads.fp8_prefill_inputs(cfg)
    x["wq"][5] = 2.5
    x["wk"][77] = -2.5
    check(cfg, x)


def test_fp8_small_and_large_factors():
    """Factors far from 1 (the values' scale lives in the factor only)."""
    cfg = workloads.custom_prefill(2, 300, 8, 2, base=1e4, seed=83)
    x = workloads.fp8_prefill_inputs(cfg)
    x["qkv_scale"] = x["qkv_scale"] * torch.tensor([1e-3, 40.0, 2.0 ** -12])
    check(cfg, x)


def test_fp8_equals_bf16_path_on_representable_inputs():
    """With power-of-two factors the dequantised values are bf16 numbers, and
    swa_fwd on them computes the same thing as swa_fwd_fp8 on the bytes."""
    cfg = workloads.custom_prefill(2, 500, 8, 2, base=1e4, seed=84)
    x = workloads.fp8_prefill_inputs(cfg)
    x["qkv_scale"] = torch.tensor([2.0 ** -7, 2.0 ** -6, 2.0 ** -7])
    o8, _ = run(x, cfg)
    s = x["qkv_scale"].tolist()
    bf = {n: (x[n + "8"].float() * s[i]).bfloat16().to(DEV) for i, n in enumerate("qkv")}
    d = {k: x[k].to(DEV) for k in ("g", "wq", "wk")}
    ob = swa.fwd(bf["q"], bf["k"], bf["v"], d["g"], d["wq"], d["wk"], rope_base=cfg.base)
    torch.cuda.synchronize()
    assert_parity(to_f64(o8), to_f64(ob), "fp8 vs bf16 path", max_abs=1.6e-2, rel_fro=2e-3)


def test_fp8_layer_shape_every_row():
    """The 4 x 4096 layer shape in FP8, every row against the oracle in chunks."""
    cfg = workloads.LAYER
    x = workloads.fp8_prefill_inputs(cfg)
    o, lse = run(x, cfg)
    s = x["qkv_scale"].tolist()
    deq = {n: dequant(x[n + "8"], s[i]) for i, n in enumerate("qkv")}
    g = x["g"].float().double().numpy()
    wq, wk = x["wq"].double().numpy(), x["wk"].double().numpy()
    o_cpu, lse_cpu = o.cpu(), lse.cpu()
    max_abs, dd, rr = 0.0, 0.0, 0.0
    for b in range(cfg.B):
        for t0 in range(0, cfg.T, 2048):
            t1 = t0 + 2048
            ref, lref = oracle.fwd_rows(deq["q"], deq["k"], deq["v"], g, wq, wk, b, t0, t1,
                                        W=cfg.W, R=cfg.R, base=cfg.base, eps=cfg.eps)
            dlt = to_f64(o_cpu[b:b + 1, t0:t1]) - ref
            max_abs = max(max_abs, float(np.abs(dlt).max()))
            dd += float((dlt * dlt).sum())
            rr += float((ref * ref).sum())
            np.testing.assert_allclose(to_f64(lse_cpu[b:b + 1, :, t0:t1]),
                                       lref.transpose(0, 2, 1), rtol=0, atol=LSE_ATOL)
    fro = (dd / rr) ** 0.5
    assert max_abs <= 2e-2 and fro <= 5e-3, (max_abs, fro)
