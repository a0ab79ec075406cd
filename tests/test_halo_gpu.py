"""GPU parity of the chunked forward and backward with the previous chunk's
halo given by pointer (swa_fwd_halo, swa_bwd_halo): a chunk [s, s + T) of
longer sequences, its 127 earlier tokens as the halo, against the oracle's
forward over the whole sequences (rows s .. s + T - 1) and its backward."""
import numpy as np
import pytest
import torch

import hybrid_sliding_window_gated_b200 as swa
import oracle
import workloads
from swa_testutil import assert_parity, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
W = 128


def f64(t):
    return t.detach().float().cpu().double().numpy()


@pytest.mark.parametrize("B,L,s,T,Hq,Hkv", [
    (1, 400, 127, 200, 4, 1), (2, 700, 300, 400, 8, 2), (1, 500, 200, 1, 4, 1),
    (1, 600, 130, 100, 3, 1), (2, 1200, 1000, 129, 32, 8), (1, 300, 173, 127, 4, 2),
])
def test_forward_chunk_with_halo_equals_rows_of_the_whole(B, L, s, T, Hq, Hkv):
    cfg = workloads.custom_prefill(B, L, Hq, Hkv, base=1e4, g_std=2.0, seed=90 + s + T)
    inp = workloads.prefill_inputs(cfg)
    d = {k: v.to(DEV) for k, v in inp.items()}
    ch = {x: d[x][:, s:s + T].contiguous() for x in ("q", "k", "v", "g")}
    hk = d["k"][:, s - W + 1:s].contiguous()
    hv = d["v"][:, s - W + 1:s].contiguous()
    o, lse = swa.fwd_halo(ch["q"], ch["k"], ch["v"], ch["g"], d["wq"], d["wk"], hk, hv, s,
                          want_lse=True)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    sl = lambda x, a, b: f64(inp[x][:, a:b])
    o_ref, lse_ref = oracle.fwd(sl("q", s, s + T), sl("k", s - W + 1, s + T),
                                sl("v", s - W + 1, s + T), sl("g", s, s + T), f64(inp["wq"]),
                                f64(inp["wk"]), W=W, R=42, base=1e4, eps=1e-6, pos0=s - W + 1,
                                q_begin=W - 1)
    assert_parity(to_f64(o), o_ref, "chunk o")
    np.testing.assert_allclose(to_f64(lse), lse_ref.transpose(0, 2, 1), rtol=0, atol=2e-2)


def test_forward_position_offset_without_history():
    """pos0 without a halo shifts every position: RoPE makes scores depend on
    position differences only, so the output matches positions from 0."""
    cfg = workloads.custom_prefill(2, 300, 8, 2, base=1e4, seed=95)
    inp = workloads.prefill_inputs(cfg)
    d = {k: v.to(DEV) for k, v in inp.items()}
    o = swa.fwd_halo(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], None, None, 5000)
    torch.cuda.synchronize()
    o_ref, _ = oracle.fwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                          f64(inp["wq"]), f64(inp["wk"]), W=W, R=42, base=1e4, eps=1e-6)
    assert_parity(to_f64(o), o_ref, "o at positions from 5000")


def test_forward_halo_argument_checks():
    cfg = workloads.custom_prefill(1, 200, 4, 1, seed=96)
    d = {k: v.to(DEV) for k, v in workloads.prefill_inputs(cfg).items()}
    hk = torch.zeros((1, W - 1, 1, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(swa.SwaError):  # a halo needs pos0 >= 127
        swa.fwd_halo(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], hk, hk, 100)


@pytest.mark.parametrize("B,L,s,Hq,Hkv", [(1, 500, 200, 4, 1), (2, 900, 300, 8, 2),
                                          (1, 700, 127, 3, 1), (2, 1400, 1000, 32, 8)])
def test_backward_two_chunks_with_halo_equal_the_whole(B, L, s, Hq, Hkv):
    """A sequence split at s: the first chunk's backward gives its own rows
    (its last 127 keys' dk, dv in fp32 too); the second chunk's halo backward
    gives its rows and, in fp32, its share of those 127 keys.  The two shares
    summed and rounded once, and every other row, against the oracle's
    backward of the whole; the weight gradients as the sum of the shares."""
    cfg = workloads.custom_prefill(B, L, Hq, Hkv, base=1e4, seed=97 + s, backward=True)
    inp = workloads.prefill_inputs(cfg, with_grad_out=True)
    d = {k: v.to(DEV) for k, v in inp.items()}
    a = {x: d[x][:, :s].contiguous() for x in ("q", "k", "v", "g", "dO")}
    b = {x: d[x][:, s:].contiguous() for x in ("q", "k", "v", "g", "dO")}
    hk, hv = a["k"][:, -(W - 1):].contiguous(), a["v"][:, -(W - 1):].contiguous()
    oa, la = swa.fwd(a["q"], a["k"], a["v"], a["g"], d["wq"], d["wk"], want_lse=True)
    ob, lb = swa.fwd_halo(b["q"], b["k"], b["v"], b["g"], d["wq"], d["wk"], hk, hv, W - 1,
                          want_lse=True)
    ga, _, tail = swa.bwd_edges(a["q"], a["k"], a["v"], a["g"], d["wq"], d["wk"], la, a["dO"],
                                0, W - 1)
    gb, back, _ = swa.bwd_halo(b["q"], b["k"], b["v"], b["g"], d["wq"], d["wk"], lb, b["dO"],
                               hk, hv, W - 1)
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK
    tot = tail + back
    dk = torch.cat([ga[1][:, :s - (W - 1)], tot[:, :, :, 0].bfloat16(), gb[1]], dim=1)
    dv = torch.cat([ga[2][:, :s - (W - 1)], tot[:, :, :, 1].bfloat16(), gb[2]], dim=1)
    dq = torch.cat([ga[0], gb[0]], dim=1)
    dg = torch.cat([ga[3], gb[3]], dim=1)
    ref = oracle.bwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]), f64(inp["wq"]),
                     f64(inp["wk"]), f64(inp["dO"]), W=W, R=42, base=1e4, eps=1e-6)
    for name, x, r in (("dq", dq, ref[0]), ("dk", dk, ref[1]), ("dv", dv, ref[2]),
                       ("dg", dg, ref[3])):
        assert_parity(to_f64(x), r, f"stitched {name}")
    for name, i in (("dwq", 4), ("dwk", 5)):
        got = to_f64(ga[i]) + to_f64(gb[i])
        fro = np.sqrt(((got - ref[i]) ** 2).sum() / (ref[i] ** 2).sum())
        assert fro <= 5e-3, (name, fro)
