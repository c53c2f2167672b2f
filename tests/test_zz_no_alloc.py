"""cce_forward_noalloc: the forward pass for callers that cannot allocate.

Code that is handed only its input and output buffers (a plugin, an inference
hook) or that runs where cudaMalloc is forbidden or the allocator is exhausted
cannot provide the workspace cce_forward asks for.  cce_forward_noalloc takes
no workspace: its scratch is a static device array inside the library.  These
checks call it through the C ABI and compare it with cce_forward on the same
inputs, on calls in a row, and check that it allocates nothing.

Both entry points run the same kernels with the same split of the
vocabulary on the same inputs, so their outputs must agree bit for bit.

This file is collected last on purpose: it must pass on its own in a fresh
process and after every other test.
"""
import numpy as np
import pytest

from linear_cross_entropy_05_b200 import synth

from _gpu_helpers import IGN, to_dev

pytestmark = pytest.mark.gpu

CCE_ERR_WORKSPACE_TOO_SMALL = 3


def _with_workspace(L, E, C, y):
    loss, lse = L.forward(E, C, y, IGN)
    return loss.cpu().numpy(), lse.cpu().numpy()


def _nan_outputs(torch, N, device):
    return (torch.full((N,), float("nan"), device=device), torch.full((N,), float("nan"), device=device))


def _noalloc_into(L, torch, E, C, y, loss, lse, check=True):
    N, D = E.shape
    V = C.shape[0]
    return L.cce_forward_noalloc(E.data_ptr(), C.data_ptr(), y.data_ptr(), N, D, V, IGN, loss.data_ptr(),
                                 lse.data_ptr(), torch.cuda.current_stream().cuda_stream, check=check)


def test_noalloc_forward_equals_workspace_forward_bitwise_on_calls_in_a_row():
    import torch
    import linear_cross_entropy_05_b200 as L
    # two shapes, then the second shape again: a partial left over from the
    # earlier call would show up as a mismatch
    w1 = synth.GEMMA2_2B.with_sizes(N=1000, V=20000)
    w2 = synth.LLAMA3_8B.with_sizes(N=700, V=9000)
    cases = []
    for w in (w1, w2):
        inp = synth.make_inputs(w)
        E, C, y = to_dev(inp)
        ref = _with_workspace(L, E, C, y)
        cases.append((inp, E, C, y, ref))
    outs = [_nan_outputs(torch, c[1].shape[0], c[1].device) for c in (cases[0], cases[1], cases[1])]
    # The first call on the device is the set-up: CUDA loads this part of the
    # library there (with lazy module loading, at this point), which is when
    # the static scratch array itself takes its 8 MiB.  After it, calls
    # allocate nothing.
    setup_loss, setup_lse = _nan_outputs(torch, cases[0][1].shape[0], cases[0][1].device)
    _noalloc_into(L, torch, cases[0][1], cases[0][2], cases[0][3], setup_loss, setup_lse)
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for (inp, E, C, y, _), (loss, lse) in zip((cases[0], cases[1], cases[1]), outs):
        _noalloc_into(L, torch, E, C, y, loss, lse)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before  # nothing was allocated by the three calls
    for (inp, E, C, y, (ref_loss, ref_lse)), (loss, lse) in zip((cases[0], cases[1], cases[1]), outs):
        got_loss, got_lse = loss.cpu().numpy(), lse.cpu().numpy()
        assert np.isfinite(got_loss).all() and np.isfinite(got_lse).all()
        assert np.array_equal(got_loss.view(np.uint32), ref_loss.view(np.uint32))
        assert np.array_equal(got_lse.view(np.uint32), ref_lse.view(np.uint32))
        assert (got_loss[inp["y"] == IGN] == 0).all()


def test_noalloc_rejects_problems_beyond_its_scratch():
    import torch
    import linear_cross_entropy_05_b200 as L
    torch.cuda.init()
    # 131072 tokens over a 262144-entry vocabulary need ~26 MB of partials;
    # the static scratch is 8 MiB
    assert L.cce_forward_workspace_size(131072, 2048, 262144) > (8 << 20)
    st = L.cce_forward_noalloc(0, 0, 0, 131072, 2048, 262144, IGN, 0, 0, 0, check=False)
    assert st == CCE_ERR_WORKSPACE_TOO_SMALL  # nothing launched


def test_noalloc_wait_that_gives_up_yields_nan_not_stale_partials():
    """After a good call the static array holds valid partials of the same
    shape; a call whose kernel gives up waiting (the test hook withholds every
    copy; each wait ends after 20 ms) must not return them as a loss: its
    outputs are NaN.  The context stays usable."""
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=600, V=9000, D=256)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    ref_loss, ref_lse = _with_workspace(L, E, C, y)
    loss, lse = _nan_outputs(torch, w.N, E.device)
    _noalloc_into(L, torch, E, C, y, loss, lse)
    torch.cuda.synchronize()
    assert np.array_equal(loss.cpu().numpy().view(np.uint32), ref_loss.view(np.uint32))
    L.cce_debug_set_wait_limit_ns(20_000_000)
    L.cce_debug_withhold_loads(True)
    try:
        loss2 = torch.zeros(w.N, device=E.device)
        lse2 = torch.zeros(w.N, device=E.device)
        st = _noalloc_into(L, torch, E, C, y, loss2, lse2, check=False)
        torch.cuda.synchronize()
    finally:
        L.cce_debug_withhold_loads(False)
        L.cce_debug_set_wait_limit_ns(1_000_000_000)
    assert st == 0  # the launch itself succeeded; the failure is in the outputs
    assert np.isnan(loss2.cpu().numpy()).all() and np.isnan(lse2.cpu().numpy()).all()
    # normal again
    loss3, lse3 = _nan_outputs(torch, w.N, E.device)
    _noalloc_into(L, torch, E, C, y, loss3, lse3)
    torch.cuda.synchronize()
    assert np.array_equal(loss3.cpu().numpy().view(np.uint32), ref_loss.view(np.uint32))
    assert np.array_equal(lse3.cpu().numpy().view(np.uint32), ref_lse.view(np.uint32))
