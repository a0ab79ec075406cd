"""Sequence-parallel gated SWA: each rank of a process group holds a contiguous
slice of every sequence's tokens, and the only data exchanged is the window's
halo (the ZGCM-1 window layers attend over the last 128 tokens, token itself
included: onedev.kr summary, "어떻게 동작하나"; jaehun.me review, "How Gated SWA
Behaves").

Rank r holds tokens [s_r, s_r + T_r) of each of the B sequences, in rank order,
with T_r >= W - 1 for every rank but the last.

Forward: rank r receives the last W - 1 tokens of k and v from rank r - 1 and
runs the single-GPU kernels on the chunk [halo, own tokens], whose halo query
rows are zero and whose outputs there are dropped.  The chunk's RoPE positions
start at 0, not at the global position: the rotation makes each score depend
only on the difference of the two positions, so the attention is the same.

Backward: the same chunk, with dO = 0 on the halo rows and their lse set to
log(i + 1), the exact normaliser of a zero query row over its i + 1 keys.  The
halo keys' dk and dv (this rank's queries' share) go back to rank r - 1, which
adds them to its last W - 1 rows; dq and dg need nothing from other ranks.
dwq and dwk are sums over tokens, so they are all-reduced over the group.

Exchanges are point-to-point sends to the next (forward) or previous
(backward) rank through torch.distributed (NCCL between GPUs).
"""
import torch
import torch.distributed as dist

from . import bwd as _kernel_bwd
from . import fwd as _kernel_fwd

# The per-rank computation: the library's kernels.  (The CPU tests of the
# exchange logic replace these two with a host implementation.)
_local_fwd = _kernel_fwd
_local_bwd = _kernel_bwd


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
    # Agreed by every rank before any exchange, so that all of them raise.
    ok = torch.tensor([int(rank + 1 == world or k.shape[1] >= halo)], dtype=torch.int32,
                      device=k.device)
    dist.all_reduce(ok, op=dist.ReduceOp.MIN, group=group)
    if int(ok.item()) == 0:
        raise ValueError(f"every rank but the last must hold at least {halo} tokens")
    tails = [k[:, -halo:], v[:, -halo:]]
    return _exchange(tails, tails, True, group)


def _with_halo(x, halo_rows):
    """[B, T, H, D] -> [B, len + T, H, D] with `halo_rows` (or zeros) in front."""
    return torch.cat([halo_rows, x], dim=1)


def halo_lse(B, Hq, n, device):
    """lse of n zero query rows at chunk positions 0..n-1: log(i + 1)."""
    lse = torch.log(torch.arange(1, n + 1, dtype=torch.float64)).to(torch.float32)
    return lse.to(device).view(1, 1, n).expand(B, Hq, n).contiguous()


def fwd(q, k, v, g, wq, wk, *, group=None, window=128, rot_dim=42, rope_base=1e4, eps=1e-6,
        scale=0.0, want_lse=False):
    """o (and lse [B, Hq, T_r]) for this rank's tokens.  q, g: [B, T_r, Hq, D];
    k, v: [B, T_r, Hkv, D]."""
    halo = window - 1
    kw = dict(window=window, rot_dim=rot_dim, rope_base=rope_base, eps=eps, scale=scale)
    got = _halo_in(k, v, halo, group)
    if got is None:
        return _local_fwd(q, k, v, g, wq, wk, want_lse=want_lse, **kw)
    hk, hv = got
    zq = torch.zeros((q.shape[0], halo) + tuple(q.shape[2:]), dtype=q.dtype, device=q.device)
    o, lse = _local_fwd(_with_halo(q, zq), _with_halo(k, hk), _with_halo(v, hv),
                        _with_halo(g, zq), wq, wk, want_lse=True, **kw)
    o = o[:, halo:].contiguous()
    return (o, lse[:, :, halo:].contiguous()) if want_lse else o


def bwd(q, k, v, g, wq, wk, lse, dO, *, group=None, window=128, rot_dim=42, rope_base=1e4,
        eps=1e-6, scale=0.0, reduce_weight_grads=True):
    """(dq, dk, dv, dg, dwq, dwk) for this rank's tokens; lse is this rank's
    rows from :func:`fwd`.  dwq and dwk are the group's totals when
    ``reduce_weight_grads``, else this rank's share."""
    halo = window - 1
    rank, world, _ = _ranks(group)
    kw = dict(window=window, rot_dim=rot_dim, rope_base=rope_base, eps=eps, scale=scale)
    got = _halo_in(k, v, halo, group)
    if got is None:
        dq, dk, dv, dg, dwq, dwk = _local_bwd(q, k, v, g, wq, wk, lse, dO, **kw)
        back = []
    else:
        hk, hv = got
        B, Hq = q.shape[0], q.shape[2]
        zq = torch.zeros((B, halo) + tuple(q.shape[2:]), dtype=q.dtype, device=q.device)
        lse_c = torch.cat([halo_lse(B, Hq, halo, lse.device).to(lse.dtype), lse], dim=2)
        dq, dk, dv, dg, dwq, dwk = _local_bwd(
            _with_halo(q, zq), _with_halo(k, hk), _with_halo(v, hv), _with_halo(g, zq), wq, wk,
            lse_c, _with_halo(dO, zq), **kw)
        back = [dk[:, :halo], dv[:, :halo]]
        dq, dk, dv, dg = (x[:, halo:].contiguous() for x in (dq, dk, dv, dg))
    # the next rank's share of the gradient of this rank's last W - 1 keys
    ret = _exchange(back, [k[:, -halo:], v[:, -halo:]], False, group) if world > 1 else None
    if ret is not None:  # summed in at least fp32, rounded once
        acc = torch.promote_types(dk.dtype, torch.float32)
        dk[:, -halo:] = (dk[:, -halo:].to(acc) + ret[0].to(acc)).to(dk.dtype)
        dv[:, -halo:] = (dv[:, -halo:].to(acc) + ret[1].to(acc)).to(dv.dtype)
    if reduce_weight_grads and world > 1:
        dist.all_reduce(dwq, group=group)
        dist.all_reduce(dwk, group=group)
    return dq, dk, dv, dg, dwq, dwk


__all__ = ["fwd", "bwd", "halo_lse"]
