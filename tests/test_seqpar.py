"""Sequence-parallel forward and backward (hybrid_sliding_window_gated_b200.seqpar)
on CPU: gloo ranks each hold a slice of every sequence, with the fp64 oracle
standing in for the per-rank kernels, and the gathered results must equal the
oracle on the whole sequences.  This checks the exchange logic (halo in,
halo gradients back, weight-gradient reduction, chunk-relative positions);
the kernels themselves are checked on the GPU by the other tests."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle

W, R, BASE, EPS = 128, 42, 1e4, 1e-6
B, HQ, HKV, D = 2, 4, 2, 128
LENGTHS = [150, 200, 131]   # tokens per rank; all but the last hold >= W - 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    g = torch.Generator().manual_seed(77)
    T = sum(LENGTHS)
    r = lambda *s: torch.randn(*s, generator=g, dtype=torch.float64)
    return dict(q=r(B, T, HQ, D), k=r(B, T, HKV, D), v=r(B, T, HKV, D), g=r(B, T, HQ, D),
                wq=1 + 0.1 * r(D), wk=1 + 0.1 * r(D), dO=r(B, T, HQ, D))


def host_fwd(q, k, v, g, wq, wk, *, window, rot_dim, rope_base, eps, scale, want_lse):
    n = lambda t: t.numpy()
    o, lse = oracle.fwd(n(q), n(k), n(v), n(g), n(wq), n(wk), W=window, R=rot_dim,
                        base=rope_base, eps=eps, scale=scale)
    o, lse = torch.from_numpy(o), torch.from_numpy(lse).permute(0, 2, 1).contiguous()
    return (o, lse) if want_lse else o


def host_bwd(q, k, v, g, wq, wk, lse, dO, *, window, rot_dim, rope_base, eps, scale):
    n = lambda t: t.numpy()
    grads = oracle.bwd(n(q), n(k), n(v), n(g), n(wq), n(wk), n(dO), W=window, R=rot_dim,
                       base=rope_base, eps=eps, scale=scale)
    return tuple(torch.from_numpy(x) for x in grads)


def host_bwd_edges(q, k, v, g, wq, wk, lse, dO, n_lo, n_hi, **kw):
    grads = host_bwd(q, k, v, g, wq, wk, lse, dO, **kw)
    dkv = torch.stack([grads[1], grads[2]], dim=3)  # [B, T, Hkv, 2, D]
    T = q.shape[1]
    return grads, (dkv[:, :n_lo] if n_lo else None), (dkv[:, T - n_hi:] if n_hi else None)


def host_fwd_halo(q, k, v, g, wq, wk, hk, hv, pos0, *, window, rot_dim, rope_base, eps, scale,
                  want_lse):
    """The chunk's rows at positions pos0 .., its keys the halo then its own."""
    n = lambda t: t.numpy()
    kk, vv = torch.cat([hk, k], dim=1), torch.cat([hv, v], dim=1)
    o, lse = oracle.fwd(n(q), n(kk), n(vv), n(g), n(wq), n(wk), W=window, R=rot_dim,
                        base=rope_base, eps=eps, scale=scale, pos0=pos0 - (window - 1),
                        q_begin=window - 1)
    o, lse = torch.from_numpy(o), torch.from_numpy(lse).permute(0, 2, 1).contiguous()
    return (o, lse) if want_lse else o


def host_bwd_halo(q, k, v, g, wq, wk, lse, dO, hk, hv, pos0, n_hi, *, window, rot_dim, rope_base,
                  eps, scale):
    """The exact backward of host_fwd_halo: the oracle's backward over the
    chunk with its halo rows in front (positions from 0, so pos0 = W - 1),
    their query, gate and upstream-gradient rows zero, which adds nothing."""
    assert pos0 == window - 1
    n = window - 1
    z = torch.zeros((q.shape[0], n) + tuple(q.shape[2:]), dtype=q.dtype)
    cat = lambda a, b: torch.cat([a, b], dim=1)
    kw = dict(window=window, rot_dim=rot_dim, rope_base=rope_base, eps=eps, scale=scale)
    dq, dk, dv, dg, dwq, dwk = host_bwd(cat(z, q), cat(hk, k), cat(hv, v), cat(z, g), wq, wk,
                                        None, cat(z, dO), **kw)
    dkv = torch.stack([dk, dv], dim=3)
    T = q.shape[1]
    back = dkv[:, :n]
    own = dkv[:, n + T - n_hi:] if n_hi else None
    return (dq[:, n:], dk[:, n:], dv[:, n:], dg[:, n:], dwq, dwk), back, own


def _use_host(seqpar):
    seqpar._local_fwd, seqpar._local_bwd = host_fwd, host_bwd
    seqpar._local_bwd_edges = host_bwd_edges
    seqpar._local_fwd_halo, seqpar._local_bwd_halo = host_fwd_halo, host_bwd_halo


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from hybrid_sliding_window_gated_b200 import seqpar
        _use_host(seqpar)
        x = _inputs()
        s0 = sum(LENGTHS[:rank])
        sl = {k: (v[:, s0:s0 + LENGTHS[rank]].contiguous() if v.dim() == 4 else v)
              for k, v in x.items()}
        kw = dict(window=W, rot_dim=R, rope_base=BASE, eps=EPS)
        o, lse = seqpar.fwd(sl["q"], sl["k"], sl["v"], sl["g"], sl["wq"], sl["wk"],
                            want_lse=True, **kw)
        grads = seqpar.bwd(sl["q"], sl["k"], sl["v"], sl["g"], sl["wq"], sl["wk"], lse, sl["dO"],
                           **kw)
        out[rank] = (o.numpy(), lse.numpy()) + tuple(t.numpy() for t in grads)
    finally:
        dist.destroy_process_group()


def test_three_ranks_equal_the_whole_sequence():
    world = len(LENGTHS)
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = [out[r] for r in range(world)]
    x = {k: v.numpy() for k, v in _inputs().items()}
    o_ref, lse_ref = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], W=W, R=R,
                                base=BASE, eps=EPS)
    g_ref = oracle.bwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], x["dO"], W=W, R=R,
                       base=BASE, eps=EPS)
    cat = lambda i: np.concatenate([r[i] for r in res], axis=1)
    # chunk-relative positions change only the rounding of the rotation angles
    np.testing.assert_allclose(cat(0), o_ref, rtol=0, atol=1e-10)
    np.testing.assert_allclose(np.concatenate([r[1] for r in res], axis=2),
                               lse_ref.transpose(0, 2, 1), rtol=0, atol=1e-10)
    for i, name in zip(range(4), ["dq", "dk", "dv", "dg"]):
        np.testing.assert_allclose(cat(2 + i), g_ref[i], rtol=0, atol=1e-9, err_msg=name)
    for r in res:  # all-reduced weight gradients
        np.testing.assert_allclose(r[6], g_ref[4], rtol=1e-9, atol=1e-9, err_msg="dwq")
        np.testing.assert_allclose(r[7], g_ref[5], rtol=1e-9, atol=1e-9, err_msg="dwk")


def test_single_process_calls_the_kernels_directly(monkeypatch):
    from hybrid_sliding_window_gated_b200 import seqpar
    calls = []
    monkeypatch.setattr(seqpar, "_local_fwd", lambda *a, **k: calls.append("fwd") or "o")
    assert seqpar.fwd(*(torch.zeros(1, 4, 1, 128),) * 4, torch.ones(128), torch.ones(128)) == "o"
    assert calls == ["fwd"]


def _short_rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from hybrid_sliding_window_gated_b200 import seqpar
        seqpar._local_fwd = host_fwd
        T = 100 if rank == 0 else 200   # rank 0 cannot supply rank 1's 127-token halo
        x = {k: (v[:, :T].contiguous() if v.dim() == 4 else v) for k, v in _inputs().items()}
        try:
            seqpar.fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], window=W, rot_dim=R)
            out[rank] = "returned"
        except ValueError:
            out[rank] = "raised"
    finally:
        dist.destroy_process_group()


def test_a_short_rank_makes_every_rank_raise():
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_short_rank_main, args=(2, _free_port(), out), nprocs=2, join=True)
        assert dict(out) == {0: "raised", 1: "raised"}


def test_the_product_path_calls_the_kernel_wrappers():
    import hybrid_sliding_window_gated_b200 as swa
    from hybrid_sliding_window_gated_b200 import seqpar
    assert seqpar._local_fwd is swa.fwd and seqpar._local_bwd is swa.bwd
    assert seqpar._local_bwd_edges is swa.bwd_edges
    assert seqpar._local_fwd_halo is swa.fwd_halo and seqpar._local_bwd_halo is swa.bwd_halo
    src = open(seqpar.__file__).read()
    assert "oracle" not in src


def test_rank_steps_without_a_process_group():
    """rank_fwd / rank_bwd / add_back chained by hand over three chunks equal
    the oracle on the whole sequences (the host computation standing in for
    the kernels, as above)."""
    from hybrid_sliding_window_gated_b200 import seqpar
    old = (seqpar._local_fwd, seqpar._local_bwd, seqpar._local_bwd_edges, seqpar._local_fwd_halo,
           seqpar._local_bwd_halo)
    _use_host(seqpar)
    try:
        x = _inputs()
        kw = dict(window=W, rot_dim=R, rope_base=BASE, eps=EPS)
        outs, halo, s0 = [], None, 0
        for T in LENGTHS:
            sl = {k: (v[:, s0:s0 + T].contiguous() if v.dim() == 4 else v) for k, v in x.items()}
            o, lse = seqpar.rank_fwd(sl["q"], sl["k"], sl["v"], sl["g"], sl["wq"], sl["wk"], halo,
                                     want_lse=True, **kw)
            outs.append((sl, halo, o, lse))
            halo = (sl["k"][:, -(W - 1):], sl["v"][:, -(W - 1):])
            s0 += T
        grads = []
        for r, (sl, halo, o, lse) in enumerate(outs):
            tail = W - 1 if r + 1 < len(outs) else 0
            grads.append(seqpar.rank_bwd(sl["q"], sl["k"], sl["v"], sl["g"], sl["wq"], sl["wk"],
                                         lse, sl["dO"], halo, tail=tail, **kw))
        for r in range(1, len(grads)):
            seqpar.add_back(grads[r - 1][1], grads[r - 1][2], grads[r - 1][7], grads[r][6])
    finally:
        (seqpar._local_fwd, seqpar._local_bwd, seqpar._local_bwd_edges, seqpar._local_fwd_halo,
         seqpar._local_bwd_halo) = old
    n = {k: v.numpy() for k, v in x.items()}
    o_ref, _ = oracle.fwd(n["q"], n["k"], n["v"], n["g"], n["wq"], n["wk"], W=W, R=R, base=BASE,
                          eps=EPS)
    g_ref = oracle.bwd(n["q"], n["k"], n["v"], n["g"], n["wq"], n["wk"], n["dO"], W=W, R=R,
                       base=BASE, eps=EPS)
    np.testing.assert_allclose(np.concatenate([r[2].numpy() for r in outs], axis=1), o_ref,
                               rtol=0, atol=1e-10)
    for i, name in enumerate(["dq", "dk", "dv", "dg"]):
        got = np.concatenate([gr[i].numpy() for gr in grads], axis=1)
        np.testing.assert_allclose(got, g_ref[i], rtol=0, atol=1e-9, err_msg=name)
    np.testing.assert_allclose(sum(gr[4].numpy() for gr in grads), g_ref[4], rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(sum(gr[5].numpy() for gr in grads), g_ref[5], rtol=1e-9, atol=1e-9)
