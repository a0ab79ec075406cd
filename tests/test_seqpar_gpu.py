"""Sequence sharding through the CUDA kernels on one GPU: one sequence batch
split into three chunks, each chunk's step run by seqpar.rank_fwd /
seqpar.rank_bwd (swa_fwd / swa_bwd_edges on [halo, own tokens]) with the halo
handed over by hand, the halo keys' fp32 gradient shares added to the previous
chunk's own fp32 shares and rounded once, and the stitched results
compared with the fp64 oracle on the whole sequences and with one
full-sequence call of the kernels."""
import numpy as np
import pytest
import torch

import hybrid_sliding_window_gated_b200 as swa
import oracle
import workloads
from hybrid_sliding_window_gated_b200 import seqpar
from swa_testutil import REL_FRO, assert_parity, errors, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("lengths", [[150, 200, 131], [127, 384, 300], [1000, 129, 5]])
def test_three_chunks_equal_the_whole_sequence(lengths):
    W = 128
    cfg = workloads.custom_prefill(2, sum(lengths), 8, 2, base=1e4, seed=60 + lengths[0],
                                   backward=True)
    host = workloads.prefill_inputs(cfg, with_grad_out=True)
    x = {k: v.to(DEV) for k, v in host.items()}
    kw = dict(window=W, rot_dim=cfg.R, rope_base=cfg.base, eps=cfg.eps)
    assert seqpar._local_fwd is swa.fwd and seqpar._local_bwd is swa.bwd
    chunks, halo, s0 = [], None, 0
    for T in lengths:
        sl = {k: (v[:, s0:s0 + T].contiguous() if v.dim() == 4 else v) for k, v in x.items()}
        o, lse = seqpar.rank_fwd(sl["q"], sl["k"], sl["v"], sl["g"], sl["wq"], sl["wk"], halo,
                                 want_lse=True, **kw)
        chunks.append((sl, halo, o, lse))
        halo = (sl["k"][:, -(W - 1):].contiguous(), sl["v"][:, -(W - 1):].contiguous())
        s0 += T
    grads = [seqpar.rank_bwd(sl["q"], sl["k"], sl["v"], sl["g"], sl["wq"], sl["wk"], lse,
                             sl["dO"], halo, tail=(W - 1 if r + 1 < len(chunks) else 0), **kw)
             for r, (sl, halo, o, lse) in enumerate(chunks)]
    for r in range(1, len(grads)):
        seqpar.add_back(grads[r - 1][1], grads[r - 1][2], grads[r - 1][7], grads[r][6])
    torch.cuda.synchronize()
    assert swa.get_last_device_error()[0] == swa.OK

    f = lambda t: t.float().cpu().double().numpy()
    o_ref, lse_ref = oracle.fwd(f(host["q"]), f(host["k"]), f(host["v"]), f(host["g"]),
                                f(host["wq"]), f(host["wk"]), W=W, R=cfg.R, base=cfg.base,
                                eps=cfg.eps)
    g_ref = oracle.bwd(f(host["q"]), f(host["k"]), f(host["v"]), f(host["g"]), f(host["wq"]),
                       f(host["wk"]), f(host["dO"]), W=W, R=cfg.R, base=cfg.base, eps=cfg.eps)
    o = torch.cat([c[2] for c in chunks], dim=1)
    lse = torch.cat([c[3] for c in chunks], dim=2)
    assert_parity(to_f64(o), o_ref, "stitched o")
    np.testing.assert_allclose(to_f64(lse), lse_ref.transpose(0, 2, 1), rtol=0, atol=2e-2)
    for i, name in enumerate(["dq", "dk", "dv", "dg"]):
        got = torch.cat([gr[i] for gr in grads], dim=1)
        assert_parity(to_f64(got), g_ref[i], f"stitched {name}")
    for i, name in ((4, "dwq"), (5, "dwk")):
        got = sum(to_f64(gr[i]) for gr in grads)
        fro = errors(got, g_ref[i])[1]
        assert fro <= REL_FRO, f"{name}: rel_fro={fro:.3e}"

    # and against one full-sequence call of the same kernels
    o_full, lse_full = swa.fwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], want_lse=True,
                               **kw)
    full = swa.bwd(x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"], lse_full, x["dO"], **kw)
    torch.cuda.synchronize()
    assert_parity(to_f64(o), to_f64(o_full), "stitched o vs one call")
    for i, name in enumerate(["dq", "dk", "dv", "dg"]):
        got = torch.cat([gr[i] for gr in grads], dim=1)
        assert_parity(to_f64(got), to_f64(full[i]), f"stitched {name} vs one call")
