"""GPU parity of the decode step (swa_decode_step through the C ABI) against
the fp64 oracle: attention output within the bf16 tolerances, ring writes
bit-exact (slot index, the untouched slots, the V slot) and the K slot equal
to the oracle's bf16-rounded k' up to one rounding step."""
import numpy as np
import pytest
import torch

import hybrid_sliding_window_gated_b200 as swa
import oracle
import workloads
from swa_testutil import assert_parity, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def bits(t):
    return t.detach().cpu().view(torch.int16).numpy().astype(np.uint16)


def f64(t):
    return t.detach().float().cpu().double().numpy()


def run_both(inp, R, base, eps=1e-6):
    """Decode on the GPU (copies of the rings) and in the oracle."""
    d = {k: v.to(DEV) for k, v in inp.items()}
    kc, vc = d["k_cache"].clone(), d["v_cache"].clone()
    o = swa.decode_step(d["pos"], d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], kc, vc,
                        rot_dim=R, rope_base=base, eps=eps)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    o_ref, kc_ref, vc_ref = oracle.decode(
        inp["pos"].numpy(), f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
        f64(inp["wq"]), f64(inp["wk"]), bits(inp["k_cache"]), bits(inp["v_cache"]), R=R,
        base=base, eps=eps)
    return o, kc, vc, o_ref, kc_ref, vc_ref


def check_rings(pos, kc_in, vc_in, kc, vc, kc_ref, vc_ref):
    kc_in, vc_in, kc, vc = bits(kc_in), bits(vc_in), bits(kc), bits(vc)
    W = kc.shape[2]
    for n, p in enumerate(pos.tolist()):
        s = p % W
        others = [i for i in range(W) if i != s]
        assert np.array_equal(kc[n][:, others], kc_in[n][:, others]), f"seq {n}: K slots touched"
        assert np.array_equal(vc[n][:, others], vc_in[n][:, others]), f"seq {n}: V slots touched"
        assert np.array_equal(vc[n][:, s], vc_ref[n][:, s]), f"seq {n}: V slot is not v_new"
        # k' computed in fp32 vs fp64 may round to the neighbouring bf16 value
        got = oracle.bf16_bits_to_f64(kc[n][:, s])
        ref = oracle.bf16_bits_to_f64(kc_ref[n][:, s])
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -7 + 1e-30), f"seq {n}: K slot"
        assert np.mean(kc[n][:, s] == kc_ref[n][:, s]) > 0.95


def test_decode_config_one_layer():
    cfg = workloads.DECODE
    inp = workloads.decode_layer_inputs(cfg, layer=0)
    o, kc, vc, o_ref, kc_ref, vc_ref = run_both(inp, cfg.R, cfg.base)
    assert_parity(to_f64(o), o_ref, "decode o")
    check_rings(inp["pos"], inp["k_cache"], inp["v_cache"], kc, vc, kc_ref, vc_ref)


@pytest.mark.parametrize("Hq,Hkv,R", [(4, 1, 42), (8, 8, 42), (16, 2, 42), (8, 2, 0), (8, 2, 32),
                                      (8, 2, 48)])
def test_decode_group_sizes_and_rot_dims(Hq, Hkv, R):
    cfg = workloads.Decode("decode test", N=7, layers=1, Hq=Hq, Hkv=Hkv, base=1e4, seed=11, R=R)
    inp = workloads.decode_layer_inputs(cfg, layer=3)
    inp["pos"] = torch.tensor([0, 1, 64, 126, 127, 128, 262143], dtype=torch.int64)
    o, kc, vc, o_ref, kc_ref, vc_ref = run_both(inp, R, cfg.base)
    assert_parity(to_f64(o), o_ref, f"decode o {Hq}/{Hkv} R={R}")
    check_rings(inp["pos"], inp["k_cache"], inp["v_cache"], kc, vc, kc_ref, vc_ref)


def test_sequential_decode_reproduces_prefill():
    """Decoding tokens 0..T-1 one by one, starting from rings full of garbage,
    gives the prefill rows: the ring keeps exactly the last 128 tokens."""
    cfg = workloads.custom_prefill(2, 300, 8, 2, base=1e4, g_std=1.0, seed=21)
    inp = workloads.prefill_inputs(cfg)
    o_ref, _ = oracle.fwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                          f64(inp["wq"]), f64(inp["wk"]), W=cfg.W, R=cfg.R, base=cfg.base,
                          eps=cfg.eps)
    d = {k: v.to(DEV) for k, v in inp.items()}
    gen = torch.Generator(device="cpu").manual_seed(5)
    kc = (torch.randn((2, 2, 128, 128), generator=gen) * 50).to(torch.bfloat16).to(DEV)
    vc = (torch.randn((2, 2, 128, 128), generator=gen) * 50).to(torch.bfloat16).to(DEV)
    outs = []
    for t in range(cfg.T):
        pos = torch.full((2,), t, dtype=torch.int64, device=DEV)
        outs.append(swa.decode_step(pos, d["q"][:, t].contiguous(), d["k"][:, t].contiguous(),
                                    d["v"][:, t].contiguous(), d["g"][:, t].contiguous(), d["wq"],
                                    d["wk"], kc, vc, rot_dim=cfg.R, rope_base=cfg.base))
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    o = torch.stack(outs, dim=1)
    assert_parity(to_f64(o), o_ref, "sequential decode vs prefill")


def test_negative_position_is_reported_and_skipped():
    cfg = workloads.Decode("decode test", N=3, layers=1, Hq=8, Hkv=2, base=1e4, seed=12)
    inp = workloads.decode_layer_inputs(cfg, layer=0)
    inp["pos"] = torch.tensor([300, -1, 7], dtype=torch.int64)
    d = {k: v.to(DEV) for k, v in inp.items()}
    kc, vc = d["k_cache"].clone(), d["v_cache"].clone()
    o = torch.full_like(d["q"], 3.0)
    swa.decode_step(d["pos"], d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], kc, vc,
                    rope_base=cfg.base, out=o)
    code, site = swa.get_last_device_error()
    assert code == swa.ERR_INVALID_ARG
    assert swa.get_last_device_error()[0] == swa.OK
    assert torch.all(o[1] == 3.0)
    assert torch.equal(kc[1], d["k_cache"][1]) and torch.equal(vc[1], d["v_cache"][1])
    keep = [0, 2]
    o_ref, _, _ = oracle.decode(inp["pos"].numpy()[keep], f64(inp["q"])[keep], f64(inp["k"])[keep],
                                f64(inp["v"])[keep], f64(inp["g"])[keep], f64(inp["wq"]),
                                f64(inp["wk"]), bits(inp["k_cache"])[keep],
                                bits(inp["v_cache"])[keep], R=42, base=cfg.base, eps=1e-6)
    assert_parity(to_f64(o[keep]), o_ref, "decode o beside a bad position")


def test_saturated_gate_gives_zero():
    cfg = workloads.Decode("decode test", N=4, layers=1, Hq=8, Hkv=2, base=1e4, seed=13)
    inp = {k: v.to(DEV) for k, v in workloads.decode_layer_inputs(cfg, layer=0).items()}
    inp["g"] = torch.full_like(inp["g"], float("-inf"))
    o = swa.decode_step(inp["pos"], inp["q"], inp["k"], inp["v"], inp["g"], inp["wq"], inp["wk"],
                        inp["k_cache"], inp["v_cache"], rope_base=cfg.base)
    assert torch.count_nonzero(o).item() == 0


def test_open_gate_gives_ungated_attention():
    """g = +inf: sigmoid is exactly 1 and o is the plain attention over the ring."""
    cfg = workloads.Decode("decode test", N=6, layers=1, Hq=8, Hkv=2, base=1e7, seed=15)
    inp = workloads.decode_layer_inputs(cfg, layer=0)
    inp["g"] = torch.full_like(inp["g"], float("inf"))
    o, kc, vc, o_ref, kc_ref, vc_ref = run_both(inp, cfg.R, cfg.base)
    assert_parity(to_f64(o), o_ref, "decode o with g = +inf")


def test_forced_timeout_is_reported_and_context_survives():
    """A wait that nothing completes ends by its time limit; the kernel drains
    its copies, reports the site, and the next call computes correctly."""
    cfg = workloads.Decode("decode test", N=5, layers=1, Hq=8, Hkv=2, base=1e4, seed=14)
    inp = workloads.decode_layer_inputs(cfg, layer=0)
    d = {k: v.to(DEV) for k, v in inp.items()}
    assert swa.get_last_device_error()[0] == swa.OK
    kc, vc = d["k_cache"].clone(), d["v_cache"].clone()
    swa.decode_step(d["pos"], d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], kc, vc,
                    rope_base=cfg.base, flags=swa.FLAG_FORCE_TIMEOUT)
    code, site = swa.get_last_device_error()
    assert code == swa.ERR_DEVICE_TIMEOUT and site >= 0x100
    assert swa.get_last_device_error()[0] == swa.OK
    o, kc2, vc2, o_ref, kc_ref, vc_ref = run_both(inp, 42, cfg.base)
    assert_parity(to_f64(o), o_ref, "decode o after a forced timeout")


@pytest.mark.parametrize("T", [1, 77, 128, 300])
def test_prefill_to_ring_matches_oracle(T):
    """swa_prefill_to_ring: V slots bit-exact, K slots within one bf16 step of
    the oracle's k', slots no position reaches untouched."""
    cfg = workloads.custom_prefill(2, T, 8, 2, base=1e7, g_std=1.0, seed=30 + T)
    inp = workloads.prefill_inputs(cfg)
    gen = torch.Generator(device="cpu").manual_seed(T)
    kc0 = (torch.randn((2, 2, 128, 128), generator=gen) * 50).to(torch.bfloat16)
    vc0 = (torch.randn((2, 2, 128, 128), generator=gen) * 50).to(torch.bfloat16)
    d = {k: v.to(DEV) for k, v in inp.items()}
    kc, vc = kc0.to(DEV), vc0.to(DEV)
    swa.prefill_to_ring(d["k"], d["v"], d["wk"], kc, vc, Hq=8, rot_dim=cfg.R, rope_base=cfg.base,
                        eps=cfg.eps)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    kr, vr = oracle.prefill_to_ring(f64(inp["k"]), f64(inp["v"]), f64(inp["wk"]), bits(kc0),
                                    bits(vc0), R=cfg.R, base=cfg.base, eps=cfg.eps)
    got_k, got_v = bits(kc), bits(vc)
    assert np.array_equal(got_v, vr)
    reached = min(T, 128)
    assert np.array_equal(got_k[:, :, reached:], bits(kc0)[:, :, reached:])
    gk = oracle.bf16_bits_to_f64(got_k[:, :, :reached])
    rk = oracle.bf16_bits_to_f64(kr[:, :, :reached])
    assert np.all(np.abs(gk - rk) <= np.abs(rk) * 2.0 ** -7 + 1e-30)
    assert np.mean(got_k[:, :, :reached] == kr[:, :, :reached]) > 0.95


def test_prefill_then_decode_continues_the_sequence():
    """Prefill T tokens (forward + ring handoff), then decode token T: the
    decode row equals row T of the oracle's forward over T + 1 tokens."""
    T = 200
    cfg = workloads.custom_prefill(2, T + 1, 8, 2, base=1e7, g_std=1.0, seed=33)
    inp = workloads.prefill_inputs(cfg)
    o_ref, _ = oracle.fwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                          f64(inp["wq"]), f64(inp["wk"]), W=cfg.W, R=cfg.R, base=cfg.base,
                          eps=cfg.eps)
    d = {k: v.to(DEV) for k, v in inp.items()}
    pre = {x: d[x][:, :T].contiguous() for x in ("q", "k", "v", "g")}
    o_pre = swa.fwd(pre["q"], pre["k"], pre["v"], pre["g"], d["wq"], d["wk"], rot_dim=cfg.R,
                    rope_base=cfg.base, eps=cfg.eps)
    kc = torch.zeros((2, 2, 128, 128), dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    swa.prefill_to_ring(pre["k"], pre["v"], d["wk"], kc, vc, Hq=8, rot_dim=cfg.R,
                        rope_base=cfg.base, eps=cfg.eps)
    pos = torch.full((2,), T, dtype=torch.int64, device=DEV)
    o_dec = swa.decode_step(pos, d["q"][:, T].contiguous(), d["k"][:, T].contiguous(),
                            d["v"][:, T].contiguous(), d["g"][:, T].contiguous(), d["wq"], d["wk"],
                            kc, vc, rot_dim=cfg.R, rope_base=cfg.base, eps=cfg.eps)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    assert_parity(to_f64(o_pre), o_ref[:, :T], "prefill rows")
    assert_parity(to_f64(o_dec), o_ref[:, T], "decode row after the ring handoff")


def _varlen_case(lens, pos0, seed, Hkv=2):
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
    rows = int(sum(lens))
    gen = torch.Generator(device="cpu").manual_seed(seed)
    k = torch.randn((max(rows, 1), Hkv, 128), generator=gen).bfloat16()
    v = torch.randn((max(rows, 1), Hkv, 128), generator=gen).bfloat16()
    wk = 1 + 0.1 * torch.randn(128, generator=gen)
    B = len(lens)
    kc0 = (torch.randn((B, Hkv, 128, 128), generator=gen) * 50).bfloat16()
    vc0 = (torch.randn((B, Hkv, 128, 128), generator=gen) * 50).bfloat16()
    return starts, k, v, wk, kc0, vc0


@pytest.mark.parametrize("pos0", [None, [5, 0, 1000, 130, 7, 0, 64]])
def test_prefill_to_ring_varlen_matches_oracle(pos0):
    """Ragged lengths below, at and above the window, packed in one row array,
    optionally continuing at positions > 0: V slots bit-exact, K' slots within
    one bf16 step, unreached slots untouched (they keep the noise)."""
    lens = [0, 1, 77, 127, 128, 129, 300]
    starts, k, v, wk, kc0, vc0 = _varlen_case(lens, pos0, seed=41)
    dev = lambda t: t.to(DEV)
    i64 = lambda x: torch.tensor(x, dtype=torch.int64, device=DEV)
    kc, vc = dev(kc0), dev(vc0)
    swa.prefill_to_ring_varlen(dev(k), dev(v), dev(wk), kc, vc, i64(starts), i64(lens),
                               None if pos0 is None else i64(pos0), Hq=8, rope_base=1e7)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    kr, vr = oracle.prefill_to_ring_varlen(f64(k), f64(v), f64(wk), bits(kc0), bits(vc0), starts,
                                           lens, [0] * 7 if pos0 is None else pos0, R=42,
                                           base=1e7, eps=1e-6)
    assert np.array_equal(bits(vc), vr)
    gk, rk = oracle.bf16_bits_to_f64(bits(kc)), oracle.bf16_bits_to_f64(kr)
    assert np.all(np.abs(gk - rk) <= np.abs(rk) * 2.0 ** -7 + 1e-6)
    same = bits(kc0) == kr  # slots the oracle left alone are bit-identical on the GPU too
    assert np.array_equal(bits(kc)[same], kr[same])


def test_padded_ragged_batch_prefill_handoff_then_decode():
    """A serving batch padded to Tmax = 300 with true lengths 50, 300, 129:
    swa_fwd on the padded batch (causal rows do not see the padding after
    them), the varlen handoff with each sequence's true length, then one
    decode step per sequence at its own next position, against the oracle's
    forward over that sequence's len + 1 tokens."""
    lens, Tmax, Hq, Hkv = [50, 300, 129], 300, 8, 2
    cfg = workloads.custom_prefill(3, Tmax + 1, Hq, Hkv, base=1e7, g_std=1.0, seed=43)
    inp = workloads.prefill_inputs(cfg)
    d = {k: v.to(DEV) for k, v in inp.items()}
    pre = {x: d[x][:, :Tmax].contiguous() for x in ("q", "k", "v", "g")}
    o_pre = swa.fwd(pre["q"], pre["k"], pre["v"], pre["g"], d["wq"], d["wk"], rot_dim=cfg.R,
                    rope_base=cfg.base, eps=cfg.eps)
    kc = torch.zeros((3, Hkv, 128, 128), dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    i64 = lambda x: torch.tensor(x, dtype=torch.int64, device=DEV)
    swa.prefill_to_ring_varlen(pre["k"].view(-1, Hkv, 128), pre["v"].view(-1, Hkv, 128), d["wk"],
                               kc, vc, i64([0, Tmax, 2 * Tmax]), i64(lens), Hq=Hq, rot_dim=cfg.R,
                               rope_base=cfg.base, eps=cfg.eps)
    # each sequence's next token is row len[b] of its inputs
    idx = torch.tensor(lens, device=DEV)
    nxt = {x: d[x][torch.arange(3, device=DEV), idx].contiguous() for x in ("q", "k", "v", "g")}
    o_dec = swa.decode_step(i64(lens), nxt["q"], nxt["k"], nxt["v"], nxt["g"], d["wq"], d["wk"],
                            kc, vc, rot_dim=cfg.R, rope_base=cfg.base, eps=cfg.eps)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    for b, n in enumerate(lens):
        sl = {x: f64(inp[x][b:b + 1, :n + 1]) for x in ("q", "k", "v", "g")}
        o_ref, _ = oracle.fwd(sl["q"], sl["k"], sl["v"], sl["g"], f64(inp["wq"]), f64(inp["wk"]),
                              W=cfg.W, R=cfg.R, base=cfg.base, eps=cfg.eps)
        assert_parity(to_f64(o_pre[b:b + 1, :n]), o_ref[:, :n], f"padded prefill rows, seq {b}")
        assert_parity(to_f64(o_dec[b]), o_ref[0, n], f"decode after the ragged handoff, seq {b}")


def test_prefill_to_ring_varlen_bad_lengths_are_reported():
    lens = [10, 20]
    starts, k, v, wk, kc0, vc0 = _varlen_case(lens, None, seed=44)
    i64 = lambda x: torch.tensor(x, dtype=torch.int64, device=DEV)
    kc, vc = kc0.to(DEV), vc0.to(DEV)
    swa.prefill_to_ring_varlen(k.to(DEV), v.to(DEV), wk.to(DEV), kc, vc, i64([0, 25]), i64(lens),
                               Hq=4)  # rows 25 .. 44 of 30: past the end
    code, _ = swa.get_last_device_error()
    assert code == swa.ERR_INVALID_ARG
    assert swa.get_last_device_error()[0] == swa.OK
    assert torch.equal(kc[1], kc0[1].to(DEV)) and torch.equal(vc[1], vc0[1].to(DEV))
    assert not torch.equal(kc[0], kc0[0].to(DEV))  # the valid sequence was written
