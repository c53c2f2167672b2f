"""GPU parity of the forward pass (loss, lse) against the fp64 oracle."""
import math

import numpy as np
import pytest

import oracle
from linear_cross_entropy_05_b200 import synth

from _gpu_helpers import DEFAULT_FWD_ORDER, DEFAULT_FWD_VARIANT, IGN, LOSS_ABS, MEAN_REL, gpu_forward, mean_of, to_dev

pytestmark = pytest.mark.gpu

# Shapes the oracle finishes in seconds; together they span several tiles in
# both directions, ragged N / V / D tails, the minimal D and a vocabulary of 1.
CASES = [
    synth.TINY,
    synth.TINY.with_sizes(N=300, V=4096 + 77, D=264),
    synth.TINY.with_sizes(N=129, V=257, D=8),
    synth.TINY.with_sizes(N=1, V=1, D=64),
    synth.TINY.with_sizes(N=5, V=300, D=16),
    synth.GEMMA2_2B.with_sizes(N=1000, V=20000),
    synth.LLAMA3_8B.with_sizes(N=700, V=9000),
    synth.SMALL_LARGE_VOCAB.with_sizes(N=2000, V=30000),
    synth.SWEEP.with_sizes(N=512, V=40000),
]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_forward_matches_oracle(w):
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    assert st["status"] == 0 and st["flags"] == 0
    ol, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    assert np.abs(loss - ol).max() <= LOSS_ABS
    assert np.abs(lse - olse).max() <= LOSS_ABS
    m, om = mean_of(loss, inp["y"]), mean_of(ol, inp["y"])
    assert abs(m - om) <= MEAN_REL * abs(om)
    assert (loss[inp["y"] == IGN] == 0).all()


@pytest.mark.parametrize("variant", [0, 1], ids=["single-cta", "cta-pair"])
def test_raw_logit_tiles_match_definition(variant):
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.TINY.with_sizes(N=300, V=4096 + 77, D=264)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    N, D, V = w.N, w.D, w.V
    nv = (V + 255) // 256 * 256
    logits = torch.full((N, nv), float("nan"), device="cuda")
    loss = torch.empty(N, device="cuda")
    lse = torch.empty(N, device="cuda")
    ws = L.Workspace()
    L.cce_debug_set_forward_variant(variant)
    try:
        buf = ws.get(L.cce_forward_workspace_size(N, D, V))
        L.cce_debug_forward_logits(E.data_ptr(), C.data_ptr(), y.data_ptr(), N, D, V, IGN, loss.data_ptr(),
                                   lse.data_ptr(), logits.data_ptr(), buf.data_ptr(), buf.numel(),
                                   torch.cuda.current_stream().cuda_stream)
    finally:
        L.cce_debug_set_forward_variant(DEFAULT_FWD_VARIANT)
    g = logits.cpu().numpy()
    z = oracle.logits(oracle.bf16_bits_to_f64(inp["E"]), oracle.bf16_bits_to_f64(inp["C"]))
    # bf16 x bf16 products are exact in fp32; only the fp32 accumulation rounds
    assert np.abs(g[:, :V] - z).max() <= 1e-5 * max(1.0, np.abs(z).max())
    # the rest of the 32-column group holding column V-1 is zero-filled by TMA
    assert (g[:, V:(V + 31) // 32 * 32] == 0).all()


def test_zero_classifier_gives_log_V():
    w = synth.TINY.with_sizes(N=300, V=5000, D=128)
    inp = synth.make_inputs(w)
    inp["C"][:] = 0
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    assert st["status"] == 0
    np.testing.assert_allclose(loss, math.log(5000), atol=1e-5)
    np.testing.assert_allclose(lse, math.log(5000), atol=1e-5)


def test_extreme_logits_stay_finite():
    # |z| up to ~1e4: the online max shift must keep exp() in range
    w = synth.TINY.with_sizes(N=256, V=3000, D=256)
    w = w.__class__(**{**w.__dict__, "std": 16.0})
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    ol, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    assert np.isfinite(loss).all() and np.isfinite(lse).all()
    assert np.abs(olse).max() > 1e3
    # fp32 keeps ~7 significant digits of values near 1e4
    assert np.abs(lse - olse).max() <= 2e-6 * np.abs(olse).max() + LOSS_ABS


def test_ignored_and_invalid_labels():
    w = synth.TINY.with_sizes(N=200, V=1000, D=64)
    inp = synth.make_inputs(w)
    y = inp["y"]
    y[:50] = IGN
    y[77] = 1000      # == V: invalid
    y[78] = -3        # negative, not ignore_index: invalid
    E, C, yd = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, yd)
    assert st["status"] == 7 and st["flags"] & 2   # CCE_ERR_BAD_LABEL
    assert math.isnan(loss[77]) and math.isnan(loss[78])
    assert (loss[:50] == 0).all()
    ol, olse = oracle.forward(inp["E"], inp["C"], y, IGN)
    ok = np.ones(200, bool)
    ok[[77, 78]] = False
    assert np.abs(loss[ok] - ol[ok]).max() <= LOSS_ABS
    assert np.abs(lse - olse).max() <= LOSS_ABS


def test_all_tokens_ignored():
    w = synth.TINY.with_sizes(N=130, V=600, D=32)
    inp = synth.make_inputs(w)
    inp["y"][:] = IGN
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    assert st["status"] == 0
    assert (loss == 0).all() and np.isfinite(lse).all()
    assert math.isnan(mean_of(loss, inp["y"]))


def test_forward_is_deterministic_and_reuses_workspace():
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=700, V=12000, D=512)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    ws = L.Workspace()
    a = gpu_forward(E, C, y, ws)
    b = gpu_forward(E, C, y, ws)
    assert (a[0] == b[0]).all() and (a[1] == b[1]).all()


def test_workspace_too_small_is_rejected():
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.TINY
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    need = L.cce_forward_workspace_size(w.N, w.D, w.V)
    assert need >= 256 + 8 * w.N
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    out = torch.empty(2, w.N, device="cuda")
    st = L.cce_forward(E.data_ptr(), C.data_ptr(), y.data_ptr(), w.N, w.D, w.V, IGN, out[0].data_ptr(),
                       out[1].data_ptr(), ws.data_ptr(), ws.numel(), 0, check=False)
    assert st == 3


def test_library_allocates_no_device_memory():
    import torch
    w = synth.GEMMA2_2B.with_sizes(N=2048, V=30000, D=1024)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    import linear_cross_entropy_05_b200 as L
    ws = L.Workspace()
    loss, lse = L.forward(E, C, y, IGN, workspace=ws)   # warm-up: module load
    dl = torch.full((w.N,), 1.0 / w.N, device="cuda")
    dE, dC = L.backward(E, C, y, lse, dl, 2.0 ** -12, IGN, workspace=ws)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    L.forward(E, C, y, IGN, workspace=ws, out=(loss, lse))
    L.backward(E, C, y, lse, dl, 2.0 ** -12, IGN, workspace=ws, out=(dE, dC))
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    # the only extra global memory is the caller's workspace: O(N + V)
    fwd = L.cce_forward_workspace_size(w.N, w.D, w.V)
    bwd = L.cce_backward_workspace_size(w.N, w.D, w.V)
    assert ws.buf.numel() == max(fwd, bwd)
    assert fwd <= 512 + 64 * 8 * w.N
    assert bwd <= 4096 + 12 * w.N + 3 * 4 * (w.V // 256 + 64) + 2 * 4 * (w.N // 128 + 64)


@pytest.mark.parametrize("w", [synth.TINY.with_sizes(N=300, V=4096 + 77, D=264),
                               synth.TINY.with_sizes(N=129, V=257, D=8),
                               synth.GEMMA2_2B.with_sizes(N=1000, V=20000)],
                         ids=["ragged", "minimal", "gemma-shaped"])
def test_single_cta_forward_variant_matches_oracle(w):
    # the single-CTA forward kernel is selectable for A/B measurement and must
    # give the same losses as the default CTA-pair kernel (tcgen05 cta_group::2)
    import linear_cross_entropy_05_b200 as L
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    L.cce_debug_set_forward_variant(0)
    try:
        loss1, lse1, st = gpu_forward(E, C, y)
    finally:
        L.cce_debug_set_forward_variant(DEFAULT_FWD_VARIANT)
    assert st["status"] == 0
    loss0, lse0, st = gpu_forward(E, C, y)
    ol, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    assert np.abs(loss1 - ol).max() <= LOSS_ABS and np.abs(lse1 - olse).max() <= LOSS_ABS
    assert np.abs(loss0 - loss1).max() <= 1e-4


@pytest.mark.parametrize("sched", [(1, 1, 1, 0), (37, 0, 3, 7), (64, 2, 2, 0), (5, 3, 0, 7), (0, 0, 0, 7)],
                         ids=["one-split-E-hint", "37-splits-both-hints-7-stages", "64-splits-C-hint",
                              "5-splits-groups-of-3-7-stages", "7-stages"])
def test_forward_schedule_knobs_keep_the_result(sched):
    # the split count (partials per token), the raster group, the L2 hints
    # and the pipeline depth change only the order of work: the loss stays
    # the oracle's
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=1000 + 300, V=20000 + 77, D=512)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    L.cce_debug_set_forward_schedule(*sched)
    try:
        loss, lse, st = gpu_forward(E, C, y)
    finally:
        L.cce_debug_set_forward_schedule(0, 0, 0, 0)
    assert st["status"] == 0 and st["flags"] == 0
    ol, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    assert np.abs(loss - ol).max() <= LOSS_ABS
    assert np.abs(lse - olse).max() <= LOSS_ABS


@pytest.mark.parametrize("shape,sched", [
    ((1300 + 77, 20000 + 77, 512), (37, 0, 0, 0)),  # ragged N and V, an odd number of 256-token blocks
    ((200, 9000 + 5, 256), (5, 0, 0, 0)),           # one token block: one queue is empty
    ((4096 + 100, 30000, 512), (64, 2, 0, 0)),      # raster groups inside each queue, many splits
    ((2048 + 256, 5000, 128), (1, 0, 0, 0)),        # one split: a unit is a whole token block
], ids=["ragged", "one-token-block", "groups-of-2-64-splits", "one-split"])
def test_two_queue_order_gives_the_same_bits(shape, sched):
    # the two-queue order changes which pair computes a unit and when, not
    # how: every unit folds its vocabulary tiles in the same order, so with
    # the same split count the loss, lse and row maxima are bit for bit those
    # of the round-robin order
    import torch
    import linear_cross_entropy_05_b200 as L
    N, V, D = shape
    w = synth.GEMMA2_2B.with_sizes(N=N, V=V, D=D)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    out = {}
    L.cce_debug_set_forward_schedule(*sched)
    try:
        for order in (0, 1, 1):   # the second order-1 call runs with the L2 halves known
            L.cce_debug_set_forward_order(order)
            rm = torch.full((N,), float("nan"), device="cuda")
            loss, lse = L.forward(E, C, y, IGN, row_max=rm)
            out.setdefault(order, []).append((loss, lse, rm))
    finally:
        L.cce_debug_set_forward_order(DEFAULT_FWD_ORDER)
        L.cce_debug_set_forward_schedule(0, 0, 0, 0)
    ref = out[0][0]
    for got in out[1]:
        for a, b in zip(ref, got):
            assert torch.equal(a, b)
    ol, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    assert np.abs(ref[0].cpu().numpy() - ol).max() <= LOSS_ABS


def test_l2_half_probe_finds_two_halves():
    # the probe behind the two-queue order sorts the SMs by where atomics on
    # its eight lines are fast; a B200's L2 is split between its two dies,
    # so it must find two non-empty halves covering (nearly) every SM
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=600, V=5000, D=256)
    E, C, y = to_dev(synth.make_inputs(w))
    L.cce_debug_set_forward_order(1)
    try:
        L.forward(E, C, y, IGN)
    finally:
        L.cce_debug_set_forward_order(DEFAULT_FWD_ORDER)
    torch.cuda.synchronize()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    halves = L.cce_debug_l2_halves(256)
    assert set(halves) <= {0, 1, 2}
    n1, n2 = halves.count(1), halves.count(2)
    print(f"L2 halves: {n1} + {n2} of {sms} SMs")
    assert n1 > 0 and n2 > 0 and n1 + n2 >= sms - 4


def test_forward_ex_writes_each_tokens_largest_logit():
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=700, V=9000 + 77, D=256)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    rm = torch.full((w.N,), float("nan"), device="cuda")
    loss, lse = L.forward(E, C, y, IGN, row_max=rm)
    z = oracle.logits(oracle.bf16_bits_to_f64(inp["E"]), oracle.bf16_bits_to_f64(inp["C"]))   # fp64 [N, V]
    want = z.max(axis=1)
    got = rm.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()                            # ignored rows too
    assert np.abs(got - want).max() <= 1e-4 * max(1.0, float(np.abs(want).max()))
    # the same loss as the plain forward
    loss0, lse0 = L.forward(E, C, y, IGN)
    assert torch.equal(loss, loss0) and torch.equal(lse, lse0)
