"""swa_bwd_noalloc (the backward on the library's fixed device scratch)
against swa_bwd with a caller workspace, on two successive calls: the second
call reuses the scratch the first one filled."""
import ctypes

import pytest
import torch

import hybrid_sliding_window_gated_b200 as swa
import workloads


def test_noalloc_is_exported_and_refuses_oversized_problems():
    L = swa.lib()
    assert hasattr(L, "swa_bwd_noalloc")
    # 1 x 65536 tokens x 32 heads needs ~1 GiB of scratch: more than the fixed 64 MiB
    p = swa.make_params(1, 65536, 32, 8)
    nul = ctypes.c_void_p(0)
    assert L.swa_bwd_noalloc(ctypes.byref(p), *([nul] * 15)) == swa.ERR_UNSUPPORTED
    assert L.swa_bwd_noalloc(ctypes.byref(swa.make_params(1, 0, 4, 1)), *([nul] * 15)) == swa.OK


@pytest.mark.gpu
def test_noalloc_matches_workspace_backward_on_two_calls():
    for seed in (31, 32):
        cfg = workloads.custom_prefill(2, 700, 8, 2, seed=seed, backward=True)
        d = {k: v.to("cuda") for k, v in workloads.prefill_inputs(cfg, with_grad_out=True).items()}
        o, lse = swa.fwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], want_lse=True)
        ref = swa.bwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], lse, d["dO"])
        got = swa.bwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], lse, d["dO"])
        torch.cuda.synchronize()
        assert swa.get_last_device_error()[0] == swa.OK
        for a, b in zip(got[:4], ref[:4]):  # same kernels, same inputs: identical bits
            assert torch.equal(a, b)
        for a, b in zip(got[4:], ref[4:]):  # per-CTA atomics: summation order may differ
            torch.testing.assert_close(a, b, rtol=1e-5, atol=1e-5)
