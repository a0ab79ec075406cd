"""Pins of the fp64 oracle against things other than itself.

Each test checks the oracle against what the pages or the mathematics fix:
an independent dense brute force (torch fp64, RoPE written as a complex
rotation), PyTorch's causal SDPA for windows >= T, closed forms (window 1,
saturated gates, RMSNorm of the mean square), invariants of RoPE, central
finite differences and torch autograd for the backward, the pages' worked
numbers under tests/golden, and brute force for the decode ring.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden

F64 = torch.float64


# ----------------------------------------------------------------- helpers

def rand_inputs(B, T, Hq, Hkv, D, seed, g_std=1.0, bf16=True):
    rng = np.random.default_rng(seed)

    def r(*s, std=1.0):
        x = rng.standard_normal(s) * std
        if bf16:  # values on the bf16 grid, as the library receives them
            x = torch.tensor(x, dtype=torch.float32).bfloat16().double().numpy()
        return x

    q, k, v = r(B, T, Hq, D), r(B, T, Hkv, D), r(B, T, Hkv, D)
    g = r(B, T, Hq, D, std=g_std)
    wq = 1.0 + 0.1 * rng.standard_normal(D)
    wk = 1.0 + 0.1 * rng.standard_normal(D)
    return q, k, v, g, wq, wk


def brute_norm_rope(x, w, pos, R, base, eps):
    """RMSNorm then partial RoPE written as a complex rotation (independent form)."""
    x = torch.as_tensor(x, dtype=F64)
    y = x / torch.sqrt((x * x).mean(-1, keepdim=True) + eps) * torch.as_tensor(w, dtype=F64)
    if R == 0:
        return y
    half = R // 2
    inv = torch.tensor([base ** (-2.0 * j / R) for j in range(half)], dtype=F64)
    ang = torch.as_tensor(pos, dtype=F64)[:, None] * inv[None, :]  # [T, half]
    rot = torch.polar(torch.ones_like(ang), ang)[None, :, None, :]
    z = torch.complex(y[..., :half], y[..., half:R]) * rot
    return torch.cat([z.real, z.imag, y[..., R:]], dim=-1)


def brute_fwd(q, k, v, g, wq, wk, W, R, base, eps, gate=True):
    """Dense T x T masked softmax attention, fp64."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    pos = np.arange(T, dtype=np.float64)
    qp = brute_norm_rope(q, wq, pos, R, base, eps)
    kp = brute_norm_rope(k, wk, pos, R, base, eps)
    kp = kp.repeat_interleave(Hq // Hkv, dim=2)
    vv = torch.as_tensor(v, dtype=F64).repeat_interleave(Hq // Hkv, dim=2)
    s = torch.einsum("bihd,bjhd->bhij", qp, kp) / math.sqrt(D)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    allowed = (j <= i) & (j >= i - W + 1)
    s = s.masked_fill(~allowed, float("-inf"))
    p = torch.softmax(s, dim=-1)
    a = torch.einsum("bhij,bjhd->bihd", p, vv)
    if gate:
        a = a * torch.sigmoid(torch.as_tensor(g, dtype=F64))
    return a.numpy()


def run_oracle(q, k, v, g, wq, wk, W, R=42, base=1e4, eps=1e-6):
    return oracle.fwd(q, k, v, g, wq, wk, W=W, R=R, base=base, eps=eps)


# ------------------------------------------------------------- forward pins

@pytest.mark.parametrize("B,T,Hq,Hkv,W", [
    (1, 1, 4, 1, 128), (2, 5, 4, 2, 3), (1, 127, 4, 1, 128), (1, 129, 8, 2, 128),
    (2, 200, 4, 1, 64), (1, 300, 4, 1, 128), (1, 40, 8, 8, 7), (1, 33, 2, 1, 1),
])
def test_fwd_matches_dense_bruteforce(B, T, Hq, Hkv, W):
    q, k, v, g, wq, wk = rand_inputs(B, T, Hq, Hkv, 128, seed=T * 7 + W, g_std=2.0)
    o, lse = run_oracle(q, k, v, g, wq, wk, W)
    ref = brute_fwd(q, k, v, g, wq, wk, W, 42, 1e4, 1e-6)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    assert np.all(np.isfinite(lse))


def test_fwd_other_head_dim_and_rot_dim():
    q, k, v, g, wq, wk = rand_inputs(1, 50, 4, 2, 64, seed=3)
    o, _ = oracle.fwd(q, k, v, g, wq, wk, W=16, R=20, base=500.0, eps=1e-5)
    ref = brute_fwd(q, k, v, g, wq, wk, 16, 20, 500.0, 1e-5)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_window_ge_T_is_causal_sdpa():
    """Window >= T reduces to full causal attention (library routine)."""
    B, T, Hq, Hkv, D, R, base, eps = 2, 96, 4, 2, 128, 42, 1e4, 1e-6
    q, k, v, g, wq, wk = rand_inputs(B, T, Hq, Hkv, D, seed=11)
    o, _ = run_oracle(q, k, v, g, wq, wk, W=128)
    pos = np.arange(T, dtype=np.float64)
    qp = brute_norm_rope(q, wq, pos, R, base, eps).transpose(1, 2)
    kp = brute_norm_rope(k, wk, pos, R, base, eps).transpose(1, 2)
    vv = torch.as_tensor(v, dtype=F64).transpose(1, 2)
    kp = kp.repeat_interleave(Hq // Hkv, dim=1)
    vv = vv.repeat_interleave(Hq // Hkv, dim=1)
    a = torch.nn.functional.scaled_dot_product_attention(qp, kp, vv, is_causal=True)
    ref = (a.transpose(1, 2) * torch.sigmoid(torch.as_tensor(g, dtype=F64))).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_window_one_is_v_times_gate_and_ignores_q_k_w():
    B, T, Hq, Hkv, D = 1, 20, 4, 2, 128
    q, k, v, g, wq, wk = rand_inputs(B, T, Hq, Hkv, D, seed=5, g_std=2.0)
    o, lse = run_oracle(q, k, v, g, wq, wk, W=1)
    expect = np.repeat(v, Hq // Hkv, axis=2) / (1.0 + np.exp(-g))
    np.testing.assert_allclose(o, expect, rtol=1e-15, atol=0)
    q2, k2, _, _, wq2, wk2 = rand_inputs(B, T, Hq, Hkv, D, seed=99)
    o2, _ = run_oracle(q2, k2, v, g, wq2, wk2, W=1)
    assert np.array_equal(o, o2)


def test_saturated_gates():
    B, T, Hq, Hkv, D = 1, 64, 4, 1, 128
    q, k, v, g, wq, wk = rand_inputs(B, T, Hq, Hkv, D, seed=6)
    o, _ = run_oracle(q, k, v, np.full_like(g, -np.inf), wq, wk, W=16)
    assert np.all(o == 0.0)  # a closed gate gives exactly zero
    o, _ = run_oracle(q, k, v, np.full_like(g, np.inf), wq, wk, W=16)
    ref = brute_fwd(q, k, v, g, wq, wk, 16, 42, 1e4, 1e-6, gate=False)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_lse_is_log_normaliser():
    """lse = log sum_j exp(s_j) over the window, via torch.logsumexp."""
    B, T, Hq, Hkv, D, W = 1, 70, 4, 1, 128, 32
    q, k, v, g, wq, wk = rand_inputs(B, T, Hq, Hkv, D, seed=8)
    _, lse = run_oracle(q, k, v, g, wq, wk, W=W)
    pos = np.arange(T, dtype=np.float64)
    qp = brute_norm_rope(q, wq, pos, 42, 1e4, 1e-6)
    kp = brute_norm_rope(k, wk, pos, 42, 1e4, 1e-6).repeat_interleave(Hq // Hkv, dim=2)
    s = torch.einsum("bihd,bjhd->bihj", qp, kp) / math.sqrt(D)
    i = torch.arange(T)[:, None, None]
    j = torch.arange(T)[None, None, :]
    s = s.masked_fill(~((j <= i) & (j >= i - W + 1))[None], float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), rtol=0, atol=1e-12)


def test_gate_worked_example():
    """The element-wise gate example of the 'How Gated SWA Behaves' section."""
    gold = read_golden("gate_example.txt")
    W = int(gold["window"])
    a = np.array(gold["attention_output"])
    sg = np.array(gold["sigma_g"])
    D = 128
    # window 1: the attention output is v itself, so v carries the printed output
    v = np.zeros((1, 1, 1, D))
    v[0, 0, 0, :3] = a
    g = np.zeros((1, 1, 1, D))
    g[0, 0, 0, :3] = np.log(sg / (1 - sg))
    q = np.ones((1, 1, 1, D))
    o, _ = oracle.fwd(q, q.copy(), v, g, np.ones(D), np.ones(D), W=1, R=42, base=1e4, eps=1e-6)
    np.testing.assert_allclose(o[0, 0, 0, :3], gold["gated_output"], rtol=1e-12)


def test_window_includes_self_worked_example():
    """Window 4: the 4th token sees exactly tokens 1..4 (itself included)."""
    gold = read_golden("gate_example.txt")
    W, qi, seen = int(gold["window"]), int(gold["query_index"]), int(gold["keys_seen"])
    B, T, Hq, Hkv, D = 1, 8, 1, 1, 128
    q, k, v, g, wq, wk = rand_inputs(B, T, Hq, Hkv, D, seed=12)
    o0, _ = run_oracle(q, k, v, g, wq, wk, W=W)
    depends = []
    for j in range(T):
        v2 = v.copy()
        v2[0, j] += 1.0
        o1, _ = run_oracle(q, k, v2, g, wq, wk, W=W)
        depends.append(not np.array_equal(o0[0, qi], o1[0, qi]))
    assert depends == [j <= qi and j > qi - seen for j in range(T)]
    assert sum(depends) == seen


def test_long_positions_chunked_equals_full():
    """fwd_rows (a chunk at an offset) equals rows of the full computation."""
    B, T, Hq, Hkv, D, W = 1, 400, 4, 1, 128, 128
    q, k, v, g, wq, wk = rand_inputs(B, T, Hq, Hkv, D, seed=13)
    o_full, lse_full = oracle.fwd(q, k, v, g, wq, wk, W=W, R=42, base=1e7, eps=1e-6)
    o, lse = oracle.fwd_rows(q, k, v, g, wq, wk, 0, 250, 300, W=W, R=42, base=1e7, eps=1e-6)
    np.testing.assert_array_equal(o, o_full[:, 250:300])
    np.testing.assert_array_equal(lse, lse_full[:, 250:300])


# ------------------------------------------------------ norm and RoPE pins

def test_rmsnorm_mean_square_closed_form():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((50, 3, 128)) * rng.uniform(0.01, 10, (50, 3, 1))
    eps = 1e-6
    y = oracle.norm_rope(x, np.ones(128), np.zeros(50), 0, 1e4, eps)
    ms = (x * x).mean(-1)
    np.testing.assert_allclose((y * y).mean(-1), ms / (ms + eps), rtol=1e-13)
    # scaling x by c changes only how much eps weighs: N(cx) = N(x) sqrt((ms+eps)/(ms+eps/c^2))
    c = 3.0
    y3 = oracle.norm_rope(c * x, np.ones(128), np.zeros(50), 0, 1e4, eps)
    np.testing.assert_allclose(y3, y * np.sqrt((ms + eps) / (ms + eps / c ** 2))[..., None],
                               rtol=1e-13)


def test_rope_invariants():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 2, 128))
    w = 1 + 0.1 * rng.standard_normal(128)
    pos = rng.integers(0, 262144, 64).astype(np.float64)
    for base in (1e4, 1e7):
        y0 = oracle.norm_rope(x, w, pos, 0, base, 1e-6)
        y = oracle.norm_rope(x, w, pos, 42, base, 1e-6)
        assert np.array_equal(y[..., 42:], y0[..., 42:])      # pass-through dims untouched
        np.testing.assert_allclose(y[..., :21] ** 2 + y[..., 21:42] ** 2,
                                   y0[..., :21] ** 2 + y0[..., 21:42] ** 2, rtol=1e-12)
        yz = oracle.norm_rope(x, w, np.zeros(64), 42, base, 1e-6)
        assert np.array_equal(yz, y0)                        # identity at position 0
        ref = brute_norm_rope(x[None], w, pos, 42, base, 1e-6)[0].numpy()
        np.testing.assert_allclose(y, ref, rtol=0, atol=1e-9)  # complex-rotation form


def test_rope_relative_position_invariance():
    rng = np.random.default_rng(3)
    xq = rng.standard_normal((1, 1, 128))
    xk = rng.standard_normal((1, 1, 128))
    w = np.ones(128)
    for base in (1e4, 1e7):
        for (p, j, c) in [(10, 3, 0), (10, 3, 1000), (500, 400, 250000)]:
            qa = oracle.norm_rope(xq, w, np.array([p + c], float), 42, base, 1e-6)
            ka = oracle.norm_rope(xk, w, np.array([j + c], float), 42, base, 1e-6)
            qb = oracle.norm_rope(xq, w, np.array([p], float), 42, base, 1e-6)
            kb = oracle.norm_rope(xk, w, np.array([j], float), 42, base, 1e-6)
            assert abs((qa * ka).sum() - (qb * kb).sum()) < 1e-9


# ----------------------------------------------------------- backward pins

def _loss(q, k, v, g, wq, wk, dO, W, R, base, eps):
    o, _ = oracle.fwd(q, k, v, g, wq, wk, W=W, R=R, base=base, eps=eps, want_lse=False)
    return float((o * dO).sum())


def test_bwd_central_finite_differences():
    B, T, Hq, Hkv, D, W, R, base, eps = 1, 12, 2, 1, 16, 5, 6, 100.0, 1e-6
    q, k, v, g, wq, wk = rand_inputs(B, T, Hq, Hkv, D, seed=21, bf16=False)
    dO = np.random.default_rng(22).standard_normal(q.shape)
    grads = oracle.bwd(q, k, v, g, wq, wk, dO, W=W, R=R, base=base, eps=eps)
    args = [q, k, v, g, wq, wk]
    h = 1e-6
    for a, gr in zip(args, grads):
        num = np.empty_like(a)
        flat = a.reshape(-1)
        for idx in range(flat.size):
            old = flat[idx]
            flat[idx] = old + h
            lp = _loss(*args, dO, W, R, base, eps)
            flat[idx] = old - h
            lm = _loss(*args, dO, W, R, base, eps)
            flat[idx] = old
            num.reshape(-1)[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(gr, num, rtol=1e-6, atol=1e-7)


def test_bwd_matches_torch_autograd():
    B, T, Hq, Hkv, D, W, R, base, eps = 2, 150, 4, 2, 128, 128, 42, 1e4, 1e-6
    q, k, v, g, wq, wk = rand_inputs(B, T, Hq, Hkv, D, seed=31)
    dO = np.random.default_rng(32).standard_normal(q.shape)
    grads = oracle.bwd(q, k, v, g, wq, wk, dO, W=W, R=R, base=base, eps=eps)
    ts = [torch.tensor(a, dtype=F64, requires_grad=True) for a in (q, k, v, g, wq, wk)]
    tq, tk, tv, tg, twq, twk = ts
    pos = np.arange(T, dtype=np.float64)
    qp = brute_norm_rope(tq, twq, pos, R, base, eps)
    kp = brute_norm_rope(tk, twk, pos, R, base, eps).repeat_interleave(Hq // Hkv, dim=2)
    vv = tv.repeat_interleave(Hq // Hkv, dim=2)
    s = torch.einsum("bihd,bjhd->bhij", qp, kp) / math.sqrt(D)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    s = s.masked_fill(~((j <= i) & (j >= i - W + 1)), float("-inf"))
    o = torch.einsum("bhij,bjhd->bihd", torch.softmax(s, -1), vv) * torch.sigmoid(tg)
    (o * torch.tensor(dO)).sum().backward()
    for gr, t in zip(grads, ts):
        np.testing.assert_allclose(gr, t.grad.numpy(), rtol=1e-9, atol=1e-11)


# ------------------------------------------------------------- decode pins

def _fill_ring(k, v, wk, p, W, R, base, eps, rng):
    """Ring state before decoding position p: positions p-W+1 .. p-1 hold
    bf16(k') and v; every other slot holds noise that must be ignored."""
    Hkv, D = k.shape[2], k.shape[3]
    kc = oracle.bf16_round_array(rng.standard_normal((1, Hkv, W, D)) * 50)
    vc = oracle.bf16_round_array(rng.standard_normal((1, Hkv, W, D)) * 50)
    for ps in range(max(0, p - W + 1), p):
        kp = oracle.norm_rope(k[0, ps][None], wk, np.array([ps], float), R, base, eps)
        kc[0, :, ps % W] = oracle.bf16_round_array(kp[0])
        vc[0, :, ps % W] = oracle.bf16_round_array(v[0, ps])
    return kc, vc


@pytest.mark.parametrize("p", [0, 5, 126, 127, 128, 300])
def test_decode_equals_prefill_row(p):
    W, R, base, eps, Hq, Hkv, D = 128, 42, 1e7, 1e-6, 4, 2, 128
    q, k, v, g, wq, wk = rand_inputs(1, p + 1, Hq, Hkv, D, seed=40 + p)
    rng = np.random.default_rng(p)
    kc, vc = _fill_ring(k, v, wk, p, W, R, base, eps, rng)
    o_dec, kc2, vc2 = oracle.decode(np.array([p]), q[:, p], k[:, p], v[:, p], g[:, p], wq, wk,
                                    kc, vc, R=R, base=base, eps=eps)
    o_pre, _ = oracle.fwd(q, k, v, g, wq, wk, W=W, R=R, base=base, eps=eps)
    # cached keys are bf16-rounded k', so agreement is to bf16 precision
    np.testing.assert_allclose(o_dec[0], o_pre[0, p], rtol=0, atol=2e-2)
    assert np.abs(o_dec[0] - o_pre[0, p]).mean() < 2e-3
    # ring indexing: only slot p mod W changes; v copied bit for bit
    s = p % W
    untouched = [i for i in range(W) if i != s]
    assert np.array_equal(kc2[:, :, untouched], kc[:, :, untouched])
    assert np.array_equal(vc2[:, :, untouched], vc[:, :, untouched])
    assert np.array_equal(vc2[0, :, s], oracle.bf16_round_array(v[0, p]))
    kp = oracle.norm_rope(k[0, p][None], wk, np.array([p], float), R, base, eps)
    assert np.array_equal(kc2[0, :, s], oracle.bf16_round_array(kp[0]))


@pytest.mark.parametrize("T", [1, 50, 128, 131, 260])
def test_prefill_to_ring_equals_sequential_decode(T):
    """The rings after a prefill of T tokens hold what T decode steps
    (positions 0..T-1) leave behind, starting from the same noise; slots no
    position reaches keep the noise."""
    W, R, base, eps, Hq, Hkv, D, B = 128, 42, 1e7, 1e-6, 4, 2, 128, 2
    q, k, v, g, wq, wk = rand_inputs(B, T, Hq, Hkv, D, seed=60 + T)
    rng = np.random.default_rng(T)
    kc0 = oracle.bf16_round_array(rng.standard_normal((B, Hkv, W, D)) * 50)
    vc0 = oracle.bf16_round_array(rng.standard_normal((B, Hkv, W, D)) * 50)
    kc, vc = kc0, vc0
    for t in range(T):
        _, kc, vc = oracle.decode(np.full(B, t), q[:, t], k[:, t], v[:, t], g[:, t], wq, wk,
                                  kc, vc, R=R, base=base, eps=eps)
    kr, vr = oracle.prefill_to_ring(k, v, wk, kc0, vc0, R=R, base=base, eps=eps)
    assert np.array_equal(kr, kc) and np.array_equal(vr, vc)
    if T < W:
        assert np.array_equal(kr[:, :, T:], kc0[:, :, T:])
        assert np.array_equal(vr[:, :, T:], vc0[:, :, T:])


@pytest.mark.parametrize("case", ["ragged", "continued"])
def test_prefill_to_ring_varlen_equals_sequential_decode(case):
    """Ragged sequences (lengths 0, 1, 77, 127, 128, 129, 300) packed in one
    row array, some continuing at positions > 0: each ring equals what
    decode steps at that sequence's positions leave behind, from the same
    noise; with every length T and positions from 0 it is the dense handoff."""
    W, R, base, eps, Hq, Hkv, D = 128, 42, 1e7, 1e-6, 4, 2, 128
    lens = [0, 1, 77, 127, 128, 129, 300]
    pos0 = [0] * 7 if case == "ragged" else [5, 0, 1000, 130, 7, 0, 64]
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    rows = int(sum(lens))
    rng = np.random.default_rng(70)
    bf = lambda x: oracle.bf16_bits_to_f64(oracle.bf16_round_array(x))
    k, v = bf(rng.standard_normal((rows, Hkv, D))), bf(rng.standard_normal((rows, Hkv, D)))
    q, g = bf(rng.standard_normal((rows, Hq, D))), bf(rng.standard_normal((rows, Hq, D)))
    wq, wk = 1 + 0.1 * rng.standard_normal(D), 1 + 0.1 * rng.standard_normal(D)
    B = len(lens)
    kc0 = oracle.bf16_round_array(rng.standard_normal((B, Hkv, W, D)) * 50)
    vc0 = oracle.bf16_round_array(rng.standard_normal((B, Hkv, W, D)) * 50)
    kr, vr = oracle.prefill_to_ring_varlen(k, v, wk, kc0, vc0, starts, lens, pos0, R=R, base=base,
                                           eps=eps)
    for b in range(B):
        kc, vc = kc0[b:b + 1], vc0[b:b + 1]
        for i in range(lens[b]):
            r = starts[b] + i
            _, kc, vc = oracle.decode(np.array([pos0[b] + i]), q[r][None], k[r][None], v[r][None],
                                      g[r][None], wq, wk, kc, vc, R=R, base=base, eps=eps)
        assert np.array_equal(kr[b:b + 1], kc) and np.array_equal(vr[b:b + 1], vc), b
    # every length T from position 0 in a padded layout: the dense handoff
    T = 140
    kd = bf(rng.standard_normal((3, T, Hkv, D)))
    vd = bf(rng.standard_normal((3, T, Hkv, D)))
    ka, va = oracle.prefill_to_ring(kd, vd, wk, kc0[:3], vc0[:3], R=R, base=base, eps=eps)
    kb, vb = oracle.prefill_to_ring_varlen(kd.reshape(-1, Hkv, D), vd.reshape(-1, Hkv, D), wk,
                                           kc0[:3], vc0[:3], [0, T, 2 * T], [T] * 3, [0] * 3,
                                           R=R, base=base, eps=eps)
    assert np.array_equal(ka, kb) and np.array_equal(va, vb)


def test_decode_matches_dense_over_ring_contents():
    """Decode output = dense softmax over the ring's keys (positions known)."""
    W, R, base, eps, Hq, Hkv, D, N = 128, 42, 1e7, 1e-6, 8, 2, 128, 3
    rng = np.random.default_rng(50)
    bf = lambda x: oracle.bf16_bits_to_f64(oracle.bf16_round_array(x))
    q, g = bf(rng.standard_normal((N, Hq, D))), bf(rng.standard_normal((N, Hq, D)))
    kn, vn = bf(rng.standard_normal((N, Hkv, D))), bf(rng.standard_normal((N, Hkv, D)))
    wq, wk = 1 + 0.1 * rng.standard_normal(D), 1 + 0.1 * rng.standard_normal(D)
    kc = oracle.bf16_round_array(rng.standard_normal((N, Hkv, W, D)))
    vc = oracle.bf16_round_array(rng.standard_normal((N, Hkv, W, D)))
    pos = np.array([200000, 70, 129])
    o, kc2, vc2 = oracle.decode(pos, q, kn, vn, g, wq, wk, kc, vc, R=R, base=base, eps=eps)
    for n in range(N):
        p = int(pos[n])
        qp = brute_norm_rope(q[n][None, None], wq, np.array([p], float), R, base, eps)[0, 0]
        keys = torch.tensor(oracle.bf16_bits_to_f64(kc2[n]))   # [Hkv, W, D]
        vals = torch.tensor(oracle.bf16_bits_to_f64(vc2[n]))
        slot_pos = torch.tensor([p - ((p - s) % W) for s in range(W)])
        for h in range(Hq):
            s_ = keys[h // (Hq // Hkv)] @ qp[h] / math.sqrt(D)
            s_ = s_.masked_fill(slot_pos < 0, float("-inf"))
            a = torch.softmax(s_, 0) @ vals[h // (Hq // Hkv)]
            ref = a * torch.sigmoid(torch.tensor(g[n, h]))
            np.testing.assert_allclose(o[n, h], ref.numpy(), rtol=0, atol=1e-12)


# ------------------------------------------------------ global-layer decode

def _global_caches(k, v, wk, p, cap, R, base, eps, rng):
    """Full-length caches whose slots 0 .. p-1 hold the prefill's bf16 k' and
    v (positions = slots), the rest noise."""
    B, Hkv, D = k.shape[0], k.shape[2], k.shape[3]
    kc = oracle.bf16_round_array(rng.standard_normal((B, Hkv, cap, D)) * 50)
    vc = oracle.bf16_round_array(rng.standard_normal((B, Hkv, cap, D)) * 50)
    for t in range(p):
        kp = oracle.norm_rope(k[:, t], wk, np.full(B, float(t)), R, base, eps)
        kc[:, :, t] = oracle.bf16_round_array(kp)
        vc[:, :, t] = oracle.bf16_round_array(v[:, t])
    return kc, vc


def test_global_decode_matches_dense_over_cache_contents():
    """Global decode = a dense softmax over slots 0 .. p of the cache after
    the new key is written (brute-force norm/RoPE, torch softmax)."""
    R, base, eps, Hq, Hkv, D, N, cap = 42, 1e7, 1e-6, 8, 2, 128, 3, 700
    rng = np.random.default_rng(80)
    bf = lambda x: oracle.bf16_bits_to_f64(oracle.bf16_round_array(x))
    q = bf(rng.standard_normal((N, Hq, D)))
    kn, vn = bf(rng.standard_normal((N, Hkv, D))), bf(rng.standard_normal((N, Hkv, D)))
    wq, wk = 1 + 0.1 * rng.standard_normal(D), 1 + 0.1 * rng.standard_normal(D)
    kc = oracle.bf16_round_array(rng.standard_normal((N, Hkv, cap, D)))
    vc = oracle.bf16_round_array(rng.standard_normal((N, Hkv, cap, D)))
    pos = np.array([699, 0, 130])
    o, kc2, vc2 = oracle.global_decode(pos, q, kn, vn, wq, wk, kc, vc, R=R, base=base, eps=eps)
    for n in range(N):
        p = int(pos[n])
        qp = brute_norm_rope(q[n][None, None], wq, np.array([p], float), R, base, eps)[0, 0]
        kpn = brute_norm_rope(kn[n][None, None], wk, np.array([p], float), R, base, eps)[0, 0]
        keys = torch.tensor(oracle.bf16_bits_to_f64(kc[n]))
        vals = torch.tensor(oracle.bf16_bits_to_f64(vc[n]))
        keys[:, p] = torch.tensor(bf(kpn.numpy()))   # the new token's slot
        vals[:, p] = torch.tensor(vn[n])
        for h in range(Hq):
            s_ = keys[h // (Hq // Hkv), :p + 1] @ qp[h] / math.sqrt(D)
            ref = torch.softmax(s_, 0) @ vals[h // (Hq // Hkv), :p + 1]
            np.testing.assert_allclose(o[n, h], ref.numpy(), rtol=0, atol=1e-12)
        others = [i for i in range(cap) if i != p]
        assert np.array_equal(kc2[n][:, others], kc[n][:, others])
        assert np.array_equal(vc2[n][:, others], vc[n][:, others])
        assert np.array_equal(vc2[n][:, p], oracle.bf16_round_array(vn[n]))


@pytest.mark.parametrize("p", [0, 1, 77, 126])
def test_global_decode_equals_ring_decode_inside_the_window(p):
    """Below position 127 a 128-slot ring holds exactly slots 0 .. p, so the
    global decode equals the window layer's decode with the gate open
    (g = +inf gives sigmoid 1), through the C oracle's own decode."""
    R, base, eps, Hq, Hkv, D, N, cap = 42, 1e4, 1e-6, 4, 1, 128, 2, 300
    q, k, v, g, wq, wk = rand_inputs(N, p + 1, Hq, Hkv, D, seed=90 + p)
    rng = np.random.default_rng(91 + p)
    kc, vc = _global_caches(k, v, wk, p, cap, R, base, eps, rng)
    o, kc2, vc2 = oracle.global_decode(np.full(N, p), q[:, p], k[:, p], v[:, p], wq, wk, kc, vc,
                                       R=R, base=base, eps=eps)
    ginf = np.full((N, Hq, D), np.inf)
    o_ring, kr, vr = oracle.decode(np.full(N, p), q[:, p], k[:, p], v[:, p], ginf, wq, wk,
                                   kc[:, :, :128], vc[:, :, :128], R=R, base=base, eps=eps)
    np.testing.assert_allclose(o, o_ring, rtol=0, atol=1e-12)
    assert np.array_equal(kc2[:, :, :128], kr) and np.array_equal(vc2[:, :, :128], vr)
    if p == 0:  # one key: the output is v_new itself
        np.testing.assert_allclose(o, np.repeat(v[:, 0], Hq // Hkv, axis=1), rtol=0, atol=1e-15)


@pytest.mark.parametrize("p", [5, 200, 600])
def test_global_decode_equals_causal_prefill_row(p):
    """Decoding position p over a cache filled by the prefill gives row p of
    the forward with a window past the sequence (full causal attention,
    pinned against SDPA above) and the gate open; cached keys are bf16, so
    the agreement is to bf16 precision."""
    R, base, eps, Hq, Hkv, D, cap = 42, 1e7, 1e-6, 4, 2, 128, 700
    q, k, v, g, wq, wk = rand_inputs(1, p + 1, Hq, Hkv, D, seed=100 + p)
    rng = np.random.default_rng(101 + p)
    kc, vc = _global_caches(k, v, wk, p, cap, R, base, eps, rng)
    o_dec, _, _ = oracle.global_decode(np.array([p]), q[:, p], k[:, p], v[:, p], wq, wk, kc, vc,
                                       R=R, base=base, eps=eps)
    o_pre, _ = oracle.fwd(q, k, v, np.full_like(g, np.inf), wq, wk, W=p + 10, R=R, base=base,
                          eps=eps)
    np.testing.assert_allclose(o_dec[0], o_pre[0, p], rtol=0, atol=2e-2)
    assert np.abs(o_dec[0] - o_pre[0, p]).mean() < 2e-3


# ---------------------------------------------------------------- FP8 inputs

def test_e4m3_decoding_matches_torch_and_the_encoding():
    """Every one of the 256 byte patterns against torch.float8_e4m3fn, and the
    encoding's fixed points: 1.0, the largest normal 448, the smallest
    subnormal 2^-9, the smallest normal 2^-6, NaN."""
    b = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_to_f64(b)
    ref = torch.from_numpy(b).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan) and nan.sum() == 2
    assert np.array_equal(mine[~nan], ref[~nan])
    assert mine[0x38] == 1.0 and mine[0x7E] == 448.0 and mine[0xFE] == -448.0
    assert mine[0x01] == 2.0 ** -9 and mine[0x08] == 2.0 ** -6 and mine[0x80] == 0.0


# ---------------------------------------------------- rounding and footprint

def test_bf16_rounding_matches_torch_rne():
    rng = np.random.default_rng(60)
    x = np.concatenate([
        rng.standard_normal(4000) * 10.0 ** rng.integers(-40, 38, 4000),
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, -1.00390625, 3.3895e38, 3.4e38,
                  1e-40, 9.2e-41, 2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135, np.inf, -np.inf]),
    ]).astype(np.float32)
    mine = oracle.bf16_round_array(x.astype(np.float64))
    ref = torch.tensor(x).bfloat16().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)
    assert oracle.bf16_bits(float("nan")) & 0x7FC0 == 0x7FC0


def test_kv_footprint_worked_numbers():
    gold = read_golden("kv_footprint.txt")
    H, d, b = int(gold["kv_heads"]), int(gold["head_dim"]), int(gold["bytes_per_elt"])
    full = oracle.kv_bytes_per_token(int(gold["layers_full"]), H, d, b)
    hybrid = oracle.kv_bytes_per_token(int(gold["layers_hybrid_global"]), H, d, b)
    assert full == gold["bytes_per_token_full"] == 128 * 1024
    assert hybrid == gold["bytes_per_token_hybrid"] == 20 * 1024
    n = int(gold["tokens_256k"])
    assert full * n / 2 ** 30 == gold["gib_full_256k"]
    assert hybrid * n / 2 ** 30 == gold["gib_hybrid_256k"]
    assert full / hybrid == gold["reduction"]
    # the 27 window layers add a constant ring per sequence, independent of length
    ring = oracle.kv_bytes_per_token(27, H, d, b) * 128
    assert ring == 27 * 128 * 8 * 128 * 2 * 2
