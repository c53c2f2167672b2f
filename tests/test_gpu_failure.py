"""Failure detection on the GPU without a fault: lost arrivals end in a status.

The test hook withholds every TMA copy ("a flag that nothing sets"), so the
tensor-core and epilogue warps wait on data that never comes.  Each bounded
wait must give up after the (shortened) limit, the CTAs must unwind and free
their tensor memory, the call's status must read CCE_ERR_TIMEOUT, and the
context must stay usable: a normal call afterwards matches the oracle.
"""
import numpy as np
import pytest

import oracle
from linear_cross_entropy_05_b200 import synth

from _gpu_helpers import DEFAULT_FWD_ORDER, DEFAULT_FWD_VARIANT, IGN, LOSS_ABS, gpu_backward, gpu_forward, rel_fro, to_dev

pytestmark = pytest.mark.gpu

CCE_ERR_TIMEOUT = 6


def test_withheld_loads_end_with_timeout_status_and_a_usable_context():
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=600, V=9000, D=256)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)           # module loaded, lse for the backward below
    assert st["status"] == 0
    dl = torch.full((w.N,), 1.0 / w.N, device="cuda")
    L.cce_debug_set_wait_limit_ns(20_000_000)       # 20 ms per wait
    L.cce_debug_withhold_loads(True)
    try:
        # single-CTA kernel; CTA-pair kernel with units dealt round-robin and
        # drawn from the two queues (there the ring of published units is
        # never fed either: every reader's wait gives up)
        for variant, order in ((0, 0), (1, 0), (1, 1)):
            L.cce_debug_set_forward_variant(variant)
            L.cce_debug_set_forward_order(order)
            ws = L.Workspace()
            l_t, s_t = L.forward(E, C, y, IGN, workspace=ws)
            st = L.read_status(ws)
            assert st["status"] == CCE_ERR_TIMEOUT and st["flags"] & 1
            # partials were never written: the call's outputs are NaN, not stale values
            assert torch.isnan(l_t).all() and torch.isnan(s_t).all()
        L.cce_debug_set_forward_variant(DEFAULT_FWD_VARIANT)
        L.cce_debug_set_forward_order(DEFAULT_FWD_ORDER)
        # filter off through the stripe kernel and through the fused kernel,
        # filter on (an eps far below every entry: no token block is flat, so
        # the tile kernel recomputes, and waits on, every tile)
        for eps, stripes in ((0.0, True), (0.0, False), (1e-30, None)):
            ws = L.Workspace()
            L.backward(E, C, y, torch.from_numpy(lse).cuda(), dl, eps, IGN, workspace=ws, stripes=stripes)
            st = L.read_status(ws)
            assert st["status"] == CCE_ERR_TIMEOUT and st["flags"] & 1
    finally:
        L.cce_debug_set_forward_variant(DEFAULT_FWD_VARIANT)
        L.cce_debug_set_forward_order(DEFAULT_FWD_ORDER)
        L.cce_debug_withhold_loads(False)
        L.cce_debug_set_wait_limit_ns(1_000_000_000)
    torch.cuda.synchronize()

    # the context is intact and the kernels run normally again
    loss, lse, st = gpu_forward(E, C, y)
    assert st["status"] == 0
    ol, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    assert np.abs(loss - ol).max() <= LOSS_ABS
    dloss = synth.random_dloss(2, w.N)
    dE, dC, st = gpu_backward(E, C, y, lse, dloss, 0.0)
    assert st["status"] == 0
    rE, rC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN)
    assert rel_fro(dE.cpu().numpy(), rE) <= 5e-3
    assert rel_fro(dC.cpu().numpy(), rC) <= 5e-3
