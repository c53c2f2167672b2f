"""cce_forward_noalloc: the forward pass for callers that cannot allocate.

Code that is handed only its input and output buffers (a plugin, an inference
hook) or that runs where cudaMalloc is forbidden or the allocator is exhausted
cannot provide the workspace cce_forward asks for.  cce_forward_noalloc takes
no workspace: its scratch is a static device array inside the library.  These
checks call it through the C ABI and compare it with cce_forward on the same
inputs, on two calls in a row, and check that it allocates nothing.

This file is collected last on purpose: it must pass on its own in a fresh
process and after every other test.
"""
import numpy as np
import pytest

from linear_cross_entropy_05_b200 import synth

from _gpu_helpers import IGN, LOSS_ABS, to_dev

pytestmark = pytest.mark.gpu


def _with_workspace(L, E, C, y):
    loss, lse = L.forward(E, C, y, IGN)
    return loss.cpu().numpy(), lse.cpu().numpy()


def _without_workspace(L, torch, E, C, y):
    N, D = E.shape
    V = C.shape[0]
    loss = torch.full((N,), float("nan"), device=E.device)
    lse = torch.full((N,), float("nan"), device=E.device)
    L.cce_forward_noalloc(E.data_ptr(), C.data_ptr(), y.data_ptr(), N, D, V, IGN, loss.data_ptr(), lse.data_ptr(),
                          torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return loss.cpu().numpy(), lse.cpu().numpy()


def test_noalloc_forward_matches_workspace_forward_on_two_calls():
    import torch
    import linear_cross_entropy_05_b200 as L
    workloads = [synth.GEMMA2_2B.with_sizes(N=1000, V=20000), synth.LLAMA3_8B.with_sizes(N=700, V=9000)]
    free_before_second = None
    for k, w in enumerate(workloads):
        inp = synth.make_inputs(w)
        E, C, y = to_dev(inp)
        ref_loss, ref_lse = _with_workspace(L, E, C, y)
        torch.cuda.synchronize()
        if k == 1:
            free_before_second, _ = torch.cuda.mem_get_info()
        loss, lse = _without_workspace(L, torch, E, C, y)
        if k == 1:
            free_after_second, _ = torch.cuda.mem_get_info()
            assert free_after_second == free_before_second  # nothing was allocated
        assert np.isfinite(loss).all() and np.isfinite(lse).all()
        assert np.abs(loss - ref_loss).max() <= LOSS_ABS
        assert np.abs(lse - ref_lse).max() <= LOSS_ABS
        assert (loss[inp["y"] == IGN] == 0).all()


def test_noalloc_rejects_problems_beyond_its_scratch():
    import torch
    import linear_cross_entropy_05_b200 as L
    torch.cuda.init()
    # the N = 65536 sweep needs ~20 MiB of partials; the static scratch is 8 MiB
    assert L.cce_forward_workspace_size(65536, 2048, 262144) > (8 << 20)
    st = L.cce_forward_noalloc(0, 0, 0, 65536, 2048, 262144, IGN, 0, 0, 0, check=False)
    assert st == 3  # CCE_ERR_WORKSPACE_TOO_SMALL, nothing launched
