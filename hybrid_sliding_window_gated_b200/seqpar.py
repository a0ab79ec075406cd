"""Sequence-parallel gated SWA: each rank of a process group holds a contiguous
slice of every sequence's tokens, and the only data exchanged is the window's
halo (the ZGCM-1 window layers attend over the last 128 tokens, token itself
included: onedev.kr summary, "어떻게 동작하나"; jaehun.me review, "How Gated SWA
Behaves").

Rank r holds tokens [s_r, s_r + T_r) of each of the B sequences, in rank order,
with T_r >= W - 1 for every rank but the last.

Forward: rank r receives the last W - 1 tokens of k and v from rank r - 1 and
runs swa_fwd_halo on its own tensors with that halo passed by pointer: the
kernel loads it as the key tile before its first one.  Positions are
chunk-relative (the first own token at W - 1, the halo before it): the
rotation makes each score depend only on the difference of two positions, so
the attention is the same.

Backward: swa_bwd_halo on the same chunk writes, in fp32, this rank's share of
the halo keys' dk and dv; it goes back to rank r - 1, which asked its own
call for its last W - 1 rows in fp32 as well, adds the two shares and rounds
once, as a single-GPU backward rounds those rows.  dq and dg need nothing
from other ranks.  dwq and dwk are sums over tokens, so they are all-reduced
over the group.

Exchanges are point-to-point sends to the next (forward) or previous
(backward) rank through torch.distributed (NCCL between GPUs).  One rank's
step, given the halo it received, is :func:`rank_fwd` / :func:`rank_bwd`, which
need no process group.  No input or output is copied: the halo arrives in its
own [B, W - 1, Hkv, D] buffer, and the per-rank traffic beyond the kernels'
own is the halo (W - 1 rows of k and v in, their fp32 gradients back).
"""
import torch
import torch.distributed as dist

from . import bwd as _kernel_bwd
from . import bwd_edges as _kernel_bwd_edges
from . import bwd_halo as _kernel_bwd_halo
from . import fwd as _kernel_fwd
from . import fwd_halo as _kernel_fwd_halo

# The per-rank computation: the library's kernels.  (The CPU tests of the
# exchange logic replace these with a host implementation.)
_local_fwd = _kernel_fwd
_local_fwd_halo = _kernel_fwd_halo
_local_bwd = _kernel_bwd
_local_bwd_edges = _kernel_bwd_edges
_local_bwd_halo = _kernel_bwd_halo


def _ranks(group):
    if group is None and not dist.is_initialized():
        return 0, 1, (lambda r: r)
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    glob = (lambda r: r) if group is None else (lambda r: dist.get_global_rank(group, r))
    return rank, world, glob


def _exchange(send, recv_like, to_next, group):
    """Send `send` to the next rank (to_next) or the previous one, and receive
    tensors shaped like `recv_like` from the other side; returns them, or None
    at that end of the chain."""
    rank, world, glob = _ranks(group)
    dst = rank + 1 if to_next else rank - 1
    src = rank - 1 if to_next else rank + 1
    reqs, got = [], None
    out = [t.contiguous() for t in send] if 0 <= dst < world else []
    reqs += [dist.isend(t, glob(dst), group=group) for t in out]
    if 0 <= src < world:
        got = [torch.empty_like(t) for t in recv_like]
        reqs += [dist.irecv(x, glob(src), group=group) for x in got]
    for r in reqs:
        r.wait()
    return got


def _halo_in(k, v, halo, group):
    rank, world, _ = _ranks(group)
    if world == 1:
        return None
    # The precondition is agreed by every rank before any exchange, so that
    # all of them raise together rather than one waiting on a send.
    ok = torch.tensor([int(rank + 1 == world or k.shape[1] >= halo)], dtype=torch.int32,
                      device=k.device)
    dist.all_reduce(ok, op=dist.ReduceOp.MIN, group=group)
    if int(ok.item()) == 0:
        raise ValueError(f"every rank but the last must hold at least {halo} tokens")
    tails = [k[:, -halo:], v[:, -halo:]]
    return _exchange(tails, tails, True, group)


def rank_fwd(q, k, v, g, wq, wk, halo, *, window=128, rot_dim=42, rope_base=1e4, eps=1e-6,
             scale=0.0, want_lse=False):
    """One rank's forward, given the halo it received: `halo` is (k, v) of the
    previous rank's last W - 1 tokens, or None on the first rank."""
    kw = dict(window=window, rot_dim=rot_dim, rope_base=rope_base, eps=eps, scale=scale)
    if halo is None:
        return _local_fwd(q, k, v, g, wq, wk, want_lse=want_lse, **kw)
    hk, hv = halo
    return _local_fwd_halo(q, k, v, g, wq, wk, hk.contiguous(), hv.contiguous(), window - 1,
                           want_lse=want_lse, **kw)


def rank_bwd(q, k, v, g, wq, wk, lse, dO, halo, *, tail=0, window=128, rot_dim=42,
             rope_base=1e4, eps=1e-6, scale=0.0):
    """One rank's backward, given the halo it received (as in :func:`rank_fwd`).
    Returns (dq, dk, dv, dg, dwq, dwk, back, own): `back` is this rank's share
    of the gradient of the halo keys, [B, W - 1, Hkv, 2, D] fp32 (dk, dv), which
    belongs to the previous rank's last W - 1 rows (None on the first rank);
    `own` is this rank's share of its own last `tail` keys in the same fp32
    form (None when tail is 0), to which the next rank's `back` is added by
    :func:`add_back`.  dwq and dwk are this rank's share."""
    kw = dict(window=window, rot_dim=rot_dim, rope_base=rope_base, eps=eps, scale=scale)
    if halo is None and tail == 0:
        return tuple(_local_bwd(q, k, v, g, wq, wk, lse, dO, **kw)) + (None, None)
    if halo is None:
        grads, _, own = _local_bwd_edges(q, k, v, g, wq, wk, lse, dO, 0, tail, **kw)
        return tuple(grads) + (None, own)
    hk, hv = halo
    grads, back, own = _local_bwd_halo(q, k, v, g, wq, wk, lse, dO, hk.contiguous(),
                                       hv.contiguous(), window - 1, tail, **kw)
    return tuple(grads) + (back, own)


def add_back(dk, dv, own, back):
    """Write this rank's last W - 1 rows of dk and dv as the sum of its own
    share (`own` from its :func:`rank_bwd`) and the next rank's share (`back`
    from the next rank's :func:`rank_bwd`), both fp32: the sum is rounded to
    dk's dtype once."""
    n = back.shape[1]
    acc = torch.promote_types(own.dtype, torch.float32)
    tot = own.to(acc) + back.to(acc)
    dk[:, -n:] = tot[:, :, :, 0].to(dk.dtype)
    dv[:, -n:] = tot[:, :, :, 1].to(dv.dtype)


def fwd(q, k, v, g, wq, wk, *, group=None, window=128, rot_dim=42, rope_base=1e4, eps=1e-6,
        scale=0.0, want_lse=False):
    """o (and lse [B, Hq, T_r]) for this rank's tokens.  q, g: [B, T_r, Hq, D];
    k, v: [B, T_r, Hkv, D]."""
    halo = _halo_in(k, v, window - 1, group)
    return rank_fwd(q, k, v, g, wq, wk, halo, window=window, rot_dim=rot_dim,
                    rope_base=rope_base, eps=eps, scale=scale, want_lse=want_lse)


def bwd(q, k, v, g, wq, wk, lse, dO, *, group=None, window=128, rot_dim=42, rope_base=1e4,
        eps=1e-6, scale=0.0, reduce_weight_grads=True):
    """(dq, dk, dv, dg, dwq, dwk) for this rank's tokens; lse is this rank's
    rows from :func:`fwd`.  dwq and dwk are the group's totals when
    ``reduce_weight_grads``, else this rank's share."""
    halo_n = window - 1
    rank, world, _ = _ranks(group)
    halo = _halo_in(k, v, halo_n, group)
    tail = halo_n if rank + 1 < world else 0
    dq, dk, dv, dg, dwq, dwk, back, own = rank_bwd(q, k, v, g, wq, wk, lse, dO, halo, tail=tail,
                                                   window=window, rot_dim=rot_dim,
                                                   rope_base=rope_base, eps=eps, scale=scale)
    # the next rank's share of the gradient of this rank's last W - 1 keys,
    # exchanged in fp32 (or wider, for wider inputs)
    wide = torch.promote_types(k.dtype, torch.float32)
    like = [torch.empty((k.shape[0], halo_n, k.shape[2], 2, k.shape[3]), dtype=wide,
                        device=k.device)]
    send = [] if back is None else [back.to(wide)]
    ret = _exchange(send, like, False, group) if world > 1 else None
    if ret is not None:
        add_back(dk, dv, own, ret[0])
    if reduce_weight_grads and world > 1:
        dist.all_reduce(dwq, group=group)
        dist.all_reduce(dwk, group=group)
    return dq, dk, dv, dg, dwq, dwk


__all__ = ["fwd", "bwd", "rank_fwd", "rank_bwd", "add_back"]
