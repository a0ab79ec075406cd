"""GPU parity of the global causal GQA layers (swa_global_fwd and
swa_global_decode_step through the C ABI) against the fp64 oracle.

The prefill's reference is the oracle's forward with a window past the
sequence (full causal attention, pinned against causal SDPA) and the gate
open (g = +inf gives sigmoid 1); the decode's is oracle.global_decode (pinned
against a dense softmax over the cache, the window decode below position 127,
and the causal prefill row).  Outputs within the bf16 bounds; the cache the
prefill writes: V bit for bit, K' within one bf16 step of the oracle's."""
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


def bits(t):
    return t.detach().cpu().view(torch.int16).numpy().astype(np.uint16)


def f64(t):
    return t.detach().float().cpu().double().numpy()


def oracle_global(inp, cfg, rows=None):
    g_open = np.full(tuple(inp["q"].shape), np.inf)
    if rows is None:
        return oracle.fwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), g_open, f64(inp["wq"]),
                          f64(inp["wk"]), W=cfg.T + 1, R=cfg.R, base=cfg.base, eps=cfg.eps)
    b, t0, t1 = rows
    return oracle.fwd_rows(inp["q"], inp["k"], inp["v"], torch.full_like(inp["q"], float("inf")),
                           inp["wq"], inp["wk"], b, t0, t1, W=cfg.T + 1, R=cfg.R, base=cfg.base,
                           eps=cfg.eps)


def run_prefill(inp, cfg, cap=None, kc=None, vc=None, flags=0):
    B, T, Hkv = cfg.B, cfg.T, cfg.Hkv
    cap = T if cap is None else cap
    d = {k: v.to(DEV) for k, v in inp.items()}
    if kc is None:
        kc = torch.zeros((B, Hkv, cap, 128), dtype=torch.bfloat16, device=DEV)
        vc = torch.zeros_like(kc)
    o, lse = swa.global_fwd(d["q"], d["k"], d["v"], d["wq"], d["wk"], kc, vc, rot_dim=cfg.R,
                            rope_base=cfg.base, eps=cfg.eps, want_lse=True, flags=flags)
    return o, lse, kc, vc


def check_prefill(cfg, inp=None, cap=None):
    inp = workloads.prefill_inputs(cfg) if inp is None else inp
    o, lse, kc, vc = run_prefill(inp, cfg, cap)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    o_ref, lse_ref = oracle_global(inp, cfg)
    assert_parity(to_f64(o), o_ref, "global o")
    np.testing.assert_allclose(to_f64(lse), lse_ref.transpose(0, 2, 1), rtol=0, atol=LSE_ATOL)
    # the cache: v bit for bit, k' within one bf16 step, zeros to the end of the tile
    T = cfg.T
    kref = oracle.norm_rope(f64(inp["k"]).reshape(-1, cfg.Hkv, 128), f64(inp["wk"]),
                            np.tile(np.arange(T, dtype=np.float64), cfg.B), cfg.R, cfg.base,
                            cfg.eps).reshape(cfg.B, T, cfg.Hkv, 128).transpose(0, 2, 1, 3)
    gk = bits(kc)[:, :, :T]
    assert np.array_equal(bits(vc)[:, :, :T], bits(inp["v"]).transpose(0, 2, 1, 3))
    rk = oracle.bf16_round_array(kref)
    gkv, rkv = oracle.bf16_bits_to_f64(gk), oracle.bf16_bits_to_f64(rk)
    # fp32 against fp64 lands on the neighbouring bf16 value at most, except
    # where the rotation nearly cancels: there the fp32 error of unit-scale
    # terms (about 1e-7) exceeds one step of the tiny result
    assert np.all(np.abs(gkv - rkv) <= np.abs(rkv) * 2.0 ** -7 + 1e-6)
    assert np.mean(gk == rk) > 0.95
    end = min(kc.shape[2], -(-T // 128) * 128)
    assert not bits(kc)[:, :, T:end].any() and not bits(vc)[:, :, T:end].any()
    return o


@pytest.mark.parametrize("B,T,Hq,Hkv", [
    (1, 1, 4, 1), (1, 127, 4, 1), (1, 128, 4, 1), (1, 129, 4, 1), (2, 300, 8, 2),
    (1, 700, 3, 1), (1, 1000, 32, 8), (2, 2100, 8, 2), (3, 257, 6, 2),
])
def test_global_prefill_shapes_and_ragged_tails(B, T, Hq, Hkv):
    check_prefill(workloads.custom_prefill(B, T, Hq, Hkv, base=1e4, seed=70 + T))


def test_global_prefill_cache_larger_than_sequence_keeps_other_slots():
    cfg = workloads.custom_prefill(2, 200, 8, 2, base=1e4, seed=71)
    inp = workloads.prefill_inputs(cfg)
    gen = torch.Generator().manual_seed(3)
    kc0 = (torch.randn((2, 2, 600, 128), generator=gen) * 9).bfloat16().to(DEV)
    vc0 = (torch.randn((2, 2, 600, 128), generator=gen) * 9).bfloat16().to(DEV)
    kc, vc = kc0.clone(), vc0.clone()
    o, lse, kc, vc = run_prefill(inp, cfg, kc=kc, vc=vc)
    torch.cuda.synchronize()
    assert torch.equal(kc[:, :, 256:], kc0[:, :, 256:]) and torch.equal(vc[:, :, 256:], vc0[:, :, 256:])
    o_ref, _ = oracle_global(inp, cfg)
    assert_parity(to_f64(o), o_ref, "global o")


@pytest.mark.parametrize("rot_dim", [0, 32, 48])
def test_global_prefill_other_rot_dims(rot_dim):
    check_prefill(workloads.custom_prefill(1, 400, 4, 2, base=1e4, seed=72, R=rot_dim))


def test_global_prefill_exact_two_pass_branch():
    """Norm weights whose score bound leaves exp2's range: the first pass finds
    each row's maximum over all key tiles, the second uses it."""
    cfg = workloads.custom_prefill(1, 600, 4, 1, base=1e4, seed=73)
    inp = workloads.prefill_inputs(cfg)
    inp["wq"][5] = 3.0
    inp["wk"][77] = -3.0
    inp["wk"][3] = 3.0
    check_prefill(cfg, inp=inp)


def test_global_prefill_training_shape_sampled_rows():
    """1 x 16384, 32 / 8 heads, in the launch configuration the benchmark
    times; rows across tiles, including the last, against the oracle."""
    cfg = workloads.custom_prefill(1, 16384, 32, 8, base=1e4, seed=74)
    inp = workloads.prefill_inputs(cfg, device=DEV)
    o, lse, kc, vc = run_prefill(inp, cfg)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    host = {k: v.cpu() for k, v in inp.items()}
    o_cpu, lse_cpu = o.cpu(), lse.cpu()
    for t0, t1 in [(0, 40), (8100, 8200), (16384 - 70, 16384)]:
        ref, lref = oracle_global(host, cfg, rows=(0, t0, t1))
        assert_parity(to_f64(o_cpu[:, t0:t1]), ref, f"global o rows [{t0},{t1})")
        np.testing.assert_allclose(to_f64(lse_cpu[:, :, t0:t1]), lref.transpose(0, 2, 1),
                                   rtol=0, atol=LSE_ATOL)


def _decode_inputs(N, Hq, Hkv, cap, seed, nan_tail=True):
    gen = torch.Generator().manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=gen).bfloat16()
    x = {"q": r(N, Hq, 128), "k": r(N, Hkv, 128), "v": r(N, Hkv, 128),
         "wq": 1 + 0.1 * torch.randn(128, generator=gen),
         "wk": 1 + 0.1 * torch.randn(128, generator=gen),
         "k_cache": r(N, Hkv, cap, 128), "v_cache": r(N, Hkv, cap, 128)}
    return x


def run_decode(x, pos, R=42, base=1e7):
    d = {k: v.to(DEV) for k, v in x.items()}
    kc, vc = d["k_cache"].clone(), d["v_cache"].clone()
    pos_d = torch.tensor(pos, dtype=torch.int64, device=DEV)
    o = swa.global_decode_step(pos_d, d["q"], d["k"], d["v"], d["wq"], d["wk"], kc, vc,
                               rot_dim=R, rope_base=base)
    torch.cuda.synchronize()
    return o, kc, vc


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 2), (6, 2), (8, 1)])
def test_global_decode_positions_across_chunks(Hq, Hkv):
    """Positions at the ends of 128-key tiles and 2048-key chunks; the cache
    slots after each position are NaN, which must not reach the output."""
    cap = 6000
    pos = [0, 1, 127, 128, 2047, 2048, 2049, 4095, 5999]
    N = len(pos)
    x = _decode_inputs(N, Hq, Hkv, cap, seed=Hq * 10 + Hkv)
    for n, p in enumerate(pos):
        x["k_cache"][n, :, p + 1:] = float("nan")
        x["v_cache"][n, :, p + 1:] = float("nan")
    o, kc, vc = run_decode(x, pos)
    assert swa.get_last_device_error()[0] == swa.OK
    o_ref, kr, vr = oracle.global_decode(np.array(pos), f64(x["q"]), f64(x["k"]), f64(x["v"]),
                                         f64(x["wq"]), f64(x["wk"]), bits(x["k_cache"]),
                                         bits(x["v_cache"]), R=42, base=1e7, eps=1e-6)
    assert_parity(to_f64(o), o_ref, "global decode o")
    gk, gv = bits(kc), bits(vc)
    assert np.array_equal(gv, vr)
    for n, p in enumerate(pos):  # only slot p was written; k' within one bf16 step
        others = [i for i in range(cap) if i != p]
        assert np.array_equal(gk[n][:, others], bits(x["k_cache"])[n][:, others])
        a, b = oracle.bf16_bits_to_f64(gk[n][:, p]), oracle.bf16_bits_to_f64(kr[n][:, p])
        assert np.all(np.abs(a - b) <= np.abs(b) * 2.0 ** -7 + 1e-6)


def test_global_decode_long_context_batch():
    """64 sequences at positions spread over 32K slots, 32 / 8 heads."""
    cap, N = 32768, 64
    rng = np.random.default_rng(9)
    pos = sorted(int(p) for p in rng.integers(1, cap, N))
    x = _decode_inputs(N, 32, 8, cap, seed=11)
    o, kc, vc = run_decode(x, pos)
    assert swa.get_last_device_error()[0] == swa.OK
    sel = [0, 17, 40, 63]
    o_ref, _, _ = oracle.global_decode(np.array(pos)[sel], f64(x["q"][sel]), f64(x["k"][sel]),
                                       f64(x["v"][sel]), f64(x["wq"]), f64(x["wk"]),
                                       bits(x["k_cache"][sel]), bits(x["v_cache"][sel]), R=42,
                                       base=1e7, eps=1e-6)
    assert_parity(to_f64(o[sel]), o_ref, "global decode o (sampled sequences)")


def test_global_prefill_then_decode_continues_the_sequence():
    """Prefill T tokens into the caches, then decode token T: its output is
    row T of the causal forward over T + 1 tokens."""
    T = 300
    cfg = workloads.custom_prefill(2, T + 1, 8, 2, base=1e7, seed=75)
    inp = workloads.prefill_inputs(cfg)
    o_ref, _ = oracle_global(inp, cfg)
    d = {k: v.to(DEV) for k, v in inp.items()}
    pre = {x: d[x][:, :T].contiguous() for x in ("q", "k", "v")}
    kc = torch.zeros((2, 2, 1000, 128), dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    o_pre = swa.global_fwd(pre["q"], pre["k"], pre["v"], d["wq"], d["wk"], kc, vc, rot_dim=cfg.R,
                           rope_base=cfg.base, eps=cfg.eps)
    pos = torch.full((2,), T, dtype=torch.int64, device=DEV)
    o_dec = swa.global_decode_step(pos, d["q"][:, T].contiguous(), d["k"][:, T].contiguous(),
                                   d["v"][:, T].contiguous(), d["wq"], d["wk"], kc, vc,
                                   rot_dim=cfg.R, rope_base=cfg.base, eps=cfg.eps)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    assert_parity(to_f64(o_pre), o_ref[:, :T], "prefill rows")
    assert_parity(to_f64(o_dec), o_ref[:, T], "decode row after the prefill")


def test_global_decode_bad_position_is_reported_and_skipped():
    x = _decode_inputs(3, 8, 2, 500, seed=12)
    d = {k: v.to(DEV) for k, v in x.items()}
    o = torch.full_like(d["q"], 3.0)
    pos = torch.tensor([10, 500, -1], dtype=torch.int64, device=DEV)
    swa.global_decode_step(pos, d["q"], d["k"], d["v"], d["wq"], d["wk"], d["k_cache"],
                           d["v_cache"], out=o)
    code, _ = swa.get_last_device_error()
    assert code == swa.ERR_INVALID_ARG
    assert swa.get_last_device_error()[0] == swa.OK
    assert torch.all(o[1:] == 3.0)
    assert torch.all(torch.isfinite(o[0]))


def test_global_forced_timeouts_are_reported_and_context_survives():
    cfg = workloads.custom_prefill(1, 300, 4, 1, base=1e4, seed=76)
    inp = workloads.prefill_inputs(cfg)
    assert swa.get_last_device_error()[0] == swa.OK
    run_prefill(inp, cfg, flags=swa.FLAG_FORCE_TIMEOUT)
    code, site = swa.get_last_device_error()
    assert code == swa.ERR_DEVICE_TIMEOUT and site >= 0x100
    x = _decode_inputs(2, 4, 1, 300, seed=13)
    d = {k: v.to(DEV) for k, v in x.items()}
    pos = torch.tensor([5, 299], dtype=torch.int64, device=DEV)
    swa.global_decode_step(pos, d["q"], d["k"], d["v"], d["wq"], d["wk"], d["k_cache"],
                           d["v_cache"], flags=swa.FLAG_FORCE_TIMEOUT)
    code, site = swa.get_last_device_error()
    assert code == swa.ERR_DEVICE_TIMEOUT and site >= 0x100
    assert swa.get_last_device_error()[0] == swa.OK
    check_prefill(cfg, inp=inp)
