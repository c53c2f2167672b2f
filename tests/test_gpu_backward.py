"""GPU parity of the backward pass (dE, dC) against the fp64 oracle."""
import math

import numpy as np
import pytest

import oracle
from linear_cross_entropy_05_b200 import synth

from _gpu_helpers import (GRAD_REL_FILTER_OFF, IGN, filter_on_bar, gpu_backward, gpu_forward, rel_fro,
                          to_dev)

pytestmark = pytest.mark.gpu

EPS = synth.EPS_BF16_FILTER
UNIT = (32, 32)     # the unit of skipped work the kernels count: 32 tokens x 32 vocabulary entries
ELEM = (1, 1)       # the filter itself: every entry kept or dropped on its own

CASES_OFF = [
    synth.TINY,
    synth.TINY.with_sizes(N=300, V=4096 + 77, D=264),
    synth.TINY.with_sizes(N=129, V=257, D=8),
    synth.TINY.with_sizes(N=3, V=1, D=64),
    synth.GEMMA2_2B.with_sizes(N=600, V=9000),
    synth.LLAMA3_8B.with_sizes(N=400, V=6000),
    synth.SMALL_LARGE_VOCAB.with_sizes(N=1500, V=20000),
]
CASES_ON = [
    synth.GEMMA2_2B.with_sizes(N=1000, V=20000),
    synth.LLAMA3_8B.with_sizes(N=700, V=9000),
    synth.SMALL_LARGE_VOCAB.with_sizes(N=2000, V=30000),
    synth.SWEEP.with_sizes(N=512, V=40000),
    synth.TINY.with_sizes(N=300, V=4096 + 77, D=264),
]


def _run(w, eps, dloss_seed=99, stripes=None):
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    assert st["status"] == 0
    dloss = synth.random_dloss(dloss_seed, w.N)
    dE, dC, st = gpu_backward(E, C, y, lse, dloss, eps, stripes=stripes)
    _, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    return inp, dloss, olse, dE.cpu().numpy(), dC.cpu().numpy(), st


@pytest.mark.parametrize("stripes", [True, False], ids=["stripes", "fused-tiles"])
@pytest.mark.parametrize("w", CASES_OFF, ids=[w.name for w in CASES_OFF])
def test_backward_filter_off_matches_exact_gradient(w, stripes):
    # both dense paths: softmax-gradient stripes (the default with the filter
    # off) and the fused per-tile kernel
    inp, dloss, olse, gE, gC, st = _run(w, 0.0, stripes=stripes)
    assert st["status"] == 0 and st["flags"] == 0
    n_tiles = -(-w.N // 32) * -(-w.V // 32)
    assert st["live_tiles"] == n_tiles and st["dead_tiles"] == 0 and st["pruned_tiles"] == 0
    assert st["logit_tiles"] == -(-w.N // 128) * -(-w.V // 256)   # every 128 x 256 logit tile recomputed
    rE, rC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN)
    if w.V == 1:  # one class: the gradient is exactly zero
        assert np.abs(gE).max() < 1e-6 and np.abs(gC).max() < 1e-6
        return
    assert rel_fro(gE, rE) <= GRAD_REL_FILTER_OFF
    assert rel_fro(gC, rC) <= GRAD_REL_FILTER_OFF
    ign = inp["y"] == IGN
    assert (gE[ign] == 0).all()


@pytest.mark.parametrize("w", CASES_ON, ids=[w.name for w in CASES_ON])
def test_backward_filter_on(w):
    inp, dloss, olse, gE, gC, st = _run(w, EPS)
    assert st["status"] == 0 and st["flags"] == 0
    fE, fC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, filter_eps=EPS, tile=ELEM)
    live = oracle.tile_live_map(inp["E"], inp["C"], inp["y"], olse, IGN, EPS, UNIT)
    xE, xC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN)
    # same live units as the oracle's (the decision sits at |P - onehot| =
    # eps; fp32 vs fp64 may flip a unit exactly at the edge)
    assert abs(st["live_tiles"] - int(live.sum())) <= max(1, live.size // 1000)
    assert st["live_tiles"] + st["dead_tiles"] + st["pruned_tiles"] == live.size
    # tight against the element-filtered oracle; the filter-on bar against
    # the exact gradient
    assert rel_fro(gE, fE) <= GRAD_REL_FILTER_OFF
    assert rel_fro(gC, fC) <= GRAD_REL_FILTER_OFF
    bar = filter_on_bar(w.V)
    assert rel_fro(gE, xE) <= bar
    assert rel_fro(gC, xC) <= bar


def test_filter_threshold_edges():
    # a huge eps kills every tile except those holding a label (|P - 1| ~ 1);
    # eps above 1 kills every tile
    w = synth.GEMMA2_2B.with_sizes(N=512, V=8192, D=256)
    inp, dloss, olse, gE, gC, st = _run(w, 0.5)
    live_o = oracle.tile_live_map(inp["E"], inp["C"], inp["y"], olse, IGN, 0.5, UNIT)
    assert st["live_tiles"] == int(live_o.sum())
    yt = {(i // 32, int(inp["y"][i]) // 32) for i in range(w.N)}
    assert st["live_tiles"] == len(yt)
    # every block is flat here: the label entries are formed directly and no
    # logit tile is recomputed
    assert st["logit_tiles"] == 0 and st["flat_units"] == st["live_tiles"]
    fE, fC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, filter_eps=0.5, tile=ELEM)
    assert rel_fro(gE, fE) <= GRAD_REL_FILTER_OFF and rel_fro(gC, fC) <= GRAD_REL_FILTER_OFF
    inp, dloss, olse, gE, gC, st = _run(w, 2.0)
    assert st["live_tiles"] == 0 and (gE == 0).all() and (gC == 0).all()


def test_non_flat_blocks_are_recomputed_densely():
    # token rows with large norms make their blocks' softmax peaky: the
    # Cauchy-Schwarz pre-pass cannot clear them, so those blocks are visited
    # in full and non-label tiles there can be live
    w = synth.GEMMA2_2B.with_sizes(N=640, V=12000, D=256)
    inp = synth.make_inputs(w)
    E = oracle.bf16_bits_to_f64(inp["E"])
    E[128:256] *= 120.0          # block 1: logits with std ~ 1.5
    E[300] *= 300.0              # one row of block 2
    inp["E"] = synth.round_to_bf16_bits(E.astype(np.float32))
    Ed, Cd, yd = to_dev(inp)
    loss, lse, st = gpu_forward(Ed, Cd, yd)
    dloss = synth.random_dloss(4, w.N)
    dE, dC, st = gpu_backward(Ed, Cd, yd, lse, dloss, EPS)
    assert st["status"] == 0
    _, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    fE, fC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, filter_eps=EPS, tile=ELEM)
    live = oracle.tile_live_map(inp["E"], inp["C"], inp["y"], olse, IGN, EPS, UNIT)
    nvu = -(-w.V // 32)
    label_tiles = {(i // 32, int(inp["y"][i]) // 32) for i in range(w.N)}
    assert int(live.sum()) > len(label_tiles)            # the peaky blocks have live non-label tiles
    assert st["live_tiles"] + st["dead_tiles"] >= 2 * 4 * nvu  # blocks 1 and 2 visited in full
    # the other blocks are flat: their label units come from the flat-row kernel
    assert 0 < st["flat_units"] < st["live_tiles"]
    assert st["logit_tiles"] % -(-w.V // 256) == 0 and st["logit_tiles"] >= 2 * -(-w.V // 256)
    assert abs(st["live_tiles"] - int(live.sum())) <= max(2, live.size // 1000)
    assert rel_fro(dE.cpu().numpy(), fE) <= GRAD_REL_FILTER_OFF
    assert rel_fro(dC.cpu().numpy(), fC) <= GRAD_REL_FILTER_OFF


def test_zero_classifier_closed_form():
    # C = 0: P = 1/V, dE_i = dloss_i (mean_v C_v - C_y) = 0,
    # dC_v = (1/V) sum_i dloss_i E_i - sum_{i: y_i = v} dloss_i E_i
    w = synth.TINY.with_sizes(N=300, V=1000, D=64)
    inp = synth.make_inputs(w)
    inp["C"][:] = 0
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    dloss = synth.random_dloss(5, w.N)
    dE, dC, st = gpu_backward(E, C, y, lse, dloss, 0.0)
    E64 = oracle.bf16_bits_to_f64(inp["E"])
    want = np.tile((dloss[:, None] * E64).sum(0) / w.V, (w.V, 1))
    for i in range(w.N):
        want[inp["y"][i]] -= dloss[i] * E64[i]
    assert np.abs(dE.cpu().numpy()).max() == 0.0
    assert rel_fro(dC.cpu().numpy(), want) <= GRAD_REL_FILTER_OFF


def test_gradient_identity_at_scale():
    # <E, dE> = <C, dC> = sum G * z holds for any (filtered) G
    import torch
    w = synth.GEMMA2_2B.with_sizes(N=4096, V=64000)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    dE, dC, st = gpu_backward(E, C, y, lse, synth.mean_dloss(inp["y"]), EPS)
    a = float((E.double() * dE.double()).sum())
    b = float((C.double() * dC.double()).sum())
    assert abs(a - b) <= 1e-2 * max(abs(a), abs(b))


def test_backward_repeatable_within_atomic_reordering():
    w = synth.GEMMA2_2B.with_sizes(N=600, V=9000, D=512)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    dl = synth.random_dloss(3, w.N)
    a = gpu_backward(E, C, y, lse, dl, 0.0)
    b = gpu_backward(E, C, y, lse, dl, 0.0)
    assert rel_fro(a[0].cpu().numpy(), b[0].cpu().numpy()) < 1e-6
    assert rel_fro(a[1].cpu().numpy(), b[1].cpu().numpy()) < 1e-6


def test_autograd_wrapper_matches_oracle():
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.LLAMA3_8B.with_sizes(N=500, V=7000, D=256)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    E.requires_grad_(True)
    C.requires_grad_(True)
    out = L.linear_cross_entropy(E, C, y, IGN, filter_eps=0.0)
    out.backward()
    ol, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    keep = inp["y"] != IGN
    assert abs(float(out) - ol[keep].mean()) <= 1e-4 * abs(ol[keep].mean())
    rE, rC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, synth.mean_dloss(inp["y"]), IGN)
    # the wrapper returns bf16 gradients (the dtype of E and C)
    assert rel_fro(E.grad.float().cpu().numpy(), rE) <= 1e-2
    assert rel_fro(C.grad.float().cpu().numpy(), rC) <= 1e-2


@pytest.mark.parametrize("variant", [1, 2, 3], ids=["2stages-2buffers", "8-epilogue-warps", "lsu-reductions"])
@pytest.mark.parametrize("eps", [0.0, EPS], ids=["filter-off", "filter-on"])
def test_backward_kernel_variants_match_oracle(variant, eps):
    # the alternative buffering / epilogue-warp layouts (selectable for A/B
    # measurement) must give the default kernel's results
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=700, V=12000 + 77)
    L.cce_debug_set_backward_variant(variant)
    try:
        inp, dloss, olse, gE, gC, st = _run(w, eps, stripes=False)
    finally:
        L.cce_debug_set_backward_variant(0)
    assert st["status"] == 0
    fE, fC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, filter_eps=eps, tile=ELEM)
    assert rel_fro(gE, fE) <= GRAD_REL_FILTER_OFF
    assert rel_fro(gC, fC) <= GRAD_REL_FILTER_OFF


@pytest.mark.parametrize("eps", [0.0, EPS], ids=["filter-off", "filter-on"])
def test_labels_at_vocabulary_edges(eps):
    # labels 0 and V-1 (the last, ragged vocabulary tile) and a token block
    # whose labels all fall in one tile
    w = synth.GEMMA2_2B.with_sizes(N=300, V=5000 + 77, D=256)
    inp = synth.make_inputs(w)
    y = inp["y"]
    y[:40] = 0
    y[40:80] = w.V - 1
    y[128:256] = w.V - 1
    E, C, yd = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, yd)
    ol, olse = oracle.forward(inp["E"], inp["C"], y, IGN)
    assert np.abs(loss - ol).max() <= 1e-2
    dloss = synth.random_dloss(12, w.N)
    dE, dC, st = gpu_backward(E, C, yd, lse, dloss, eps)
    assert st["status"] == 0
    fE, fC = oracle.backward(inp["E"], inp["C"], y, olse, dloss, IGN, filter_eps=eps, tile=ELEM)
    assert rel_fro(dE.cpu().numpy(), fE) <= GRAD_REL_FILTER_OFF
    assert rel_fro(dC.cpu().numpy(), fC) <= GRAD_REL_FILTER_OFF
    # the label rows of dC carry the one-hot part
    gC = dC.cpu().numpy()
    assert rel_fro(gC[[0, w.V - 1]], fC[[0, w.V - 1]]) <= GRAD_REL_FILTER_OFF


def test_trace_hook_and_run_time_tile_dealing():
    # CTAs draw work items from a global counter: over all CTAs every logit
    # tile is drawn exactly once, each tile's stamps are ordered, and the
    # traced live masks add up to the live-unit counter
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=1000, V=20000)
    inp = synth.make_inputs(w)
    E64 = oracle.bf16_bits_to_f64(inp["E"])
    E64[256:384] *= 120.0        # a peaky block, which the pre-pass cannot clear: its tiles are recomputed
    inp["E"] = synth.round_to_bf16_bits(E64.astype(np.float32))
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cap = 64
    tr = torch.zeros(sms * cap * 4, dtype=torch.int64, device="cuda")
    L.cce_debug_set_backward_trace(tr.data_ptr(), cap)
    try:
        dE, dC, st = gpu_backward(E, C, y, lse, synth.random_dloss(6, w.N), EPS)
    finally:
        L.cce_debug_set_backward_trace(0, 1)
    assert st["status"] == 0
    t = tr.view(sms, cap, 4).cpu().numpy()
    tiles, live = 0, 0
    for b in range(sms):
        k = 0
        while k < cap - 1 and t[b, k, 1] > 0:
            assert t[b, k, 0] <= t[b, k, 1] <= t[b, k, 2] <= t[b, k + 1, 0]
            live += bin(int(t[b, k, 3]) & 0xFFFFFFFF).count("1")
            k += 1
        tiles += k
    assert tiles == st["logit_tiles"] > 0
    # the traced masks hold the units the tile kernel formed; the flat-row
    # kernel forms the rest
    assert live + st["flat_units"] == st["live_tiles"]


@pytest.mark.parametrize("side", [-1, 1], ids=["eps-just-below-P", "eps-just-above-P"])
def test_filter_decision_at_the_threshold(side):
    # one softmax entry P sits 1 % away from eps: its 32 x 32 unit must be
    # live when eps < P and dead when eps > P (every other entry of that unit
    # is ~1/V, far below eps), exactly as the oracle's unit filter decides
    w = synth.TINY.with_sizes(N=64, V=300, D=16)
    inp = synth.make_inputs(w)
    E = np.zeros((w.N, w.D), np.float32)
    C = np.zeros((w.V, w.D), np.float32)
    E[5, 0] = 1.0
    C[200, 0] = 1.125                    # bf16-exact logit z[5, 200] = 1.125, all others 0
    inp["E"] = synth.round_to_bf16_bits(E)
    inp["C"] = synth.round_to_bf16_bits(C)
    inp["y"] = np.zeros(w.N, np.int64)   # every label in column 0 (unit column 0)
    ea = np.exp(1.125)
    P = ea / (ea + w.V - 1)
    eps = P * (1.0 + 0.01 * side)
    Ed, Cd, yd = to_dev(inp)
    loss, lse, st = gpu_forward(Ed, Cd, yd)
    dloss = synth.random_dloss(7, w.N)
    dE, dC, st = gpu_backward(Ed, Cd, yd, lse, dloss, eps)
    assert st["status"] == 0
    _, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    fE, fC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, filter_eps=eps, tile=ELEM)
    live = oracle.tile_live_map(inp["E"], inp["C"], inp["y"], olse, IGN, eps, UNIT)
    assert bool(live[0, 200 // 32]) == (side < 0)
    assert st["live_tiles"] == int(live.sum()) == 2 + (side < 0)   # two label units (+ the edge unit)
    assert rel_fro(dE.cpu().numpy(), fE) <= GRAD_REL_FILTER_OFF
    assert rel_fro(dC.cpu().numpy(), fC) <= GRAD_REL_FILTER_OFF


@pytest.mark.parametrize("slices", [2, 6])
def test_reduce_prefetch_keeps_the_results(slices):
    # the L2 prefetch of the reduction targets is a hint: same gradients
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=1000, V=20000)
    L.cce_debug_set_reduce_prefetch(slices)
    try:
        inp, dloss, olse, gE, gC, st = _run(w, EPS)
    finally:
        L.cce_debug_set_reduce_prefetch(0)
    assert st["status"] == 0
    fE, fC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, filter_eps=EPS, tile=ELEM)
    assert rel_fro(gE, fE) <= GRAD_REL_FILTER_OFF
    assert rel_fro(gC, fC) <= GRAD_REL_FILTER_OFF


@pytest.mark.parametrize("eps", [0.0, EPS], ids=["filter-off", "filter-on"])
def test_l2_hints_keep_the_results(eps):
    # eviction priorities are hints: the fused kernel's gradients are unchanged
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=800, V=12000)
    L.cce_debug_set_l2_hints(True)
    try:
        inp, dloss, olse, gE, gC, st = _run(w, eps, stripes=False)
    finally:
        L.cce_debug_set_l2_hints(False)
    assert st["status"] == 0
    fE, fC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, filter_eps=eps, tile=ELEM)
    assert rel_fro(gE, fE) <= GRAD_REL_FILTER_OFF
    assert rel_fro(gC, fC) <= GRAD_REL_FILTER_OFF


def test_row_max_bound_finds_flat_blocks_cauchy_schwarz_cannot():
    # E scaled x10: the softmax is still spread out (max_v P ~ 1.7e-4 < eps),
    # but |E_i| max_v |C_v| ~ 10 is far above lse + ln eps ~ 1.1, so the
    # Cauchy-Schwarz pre-pass recomputes every tile; the forward's exact
    # row maxima prove the blocks flat.  Both give the element-filtered
    # gradient.  A peaky block (x120) stays non-flat either way.
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=900, V=12000 + 77, D=256)
    inp = synth.make_inputs(w)
    E64 = oracle.bf16_bits_to_f64(inp["E"]) * 10.0
    E64[256:384] *= 12.0                    # one block with a peaky softmax
    inp["E"] = synth.round_to_bf16_bits(E64.astype(np.float32))
    E, C, y = to_dev(inp)
    rm = torch.empty(w.N, device="cuda")
    loss, lse = L.forward(E, C, y, IGN, row_max=rm)
    dloss = synth.random_dloss(23, w.N)
    dl = torch.from_numpy(dloss).cuda()
    n_vt = -(-w.V // 256)
    ws0, ws1 = L.Workspace(), L.Workspace()
    cE, cC = L.backward(E, C, y, lse, dl, EPS, IGN, workspace=ws0)                # Cauchy-Schwarz
    s0 = L.read_status(ws0)
    rE, rC = L.backward(E, C, y, lse, dl, EPS, IGN, workspace=ws1, row_max=rm)    # row maxima
    s1 = L.read_status(ws1)
    assert s0["status"] == 0 and s1["status"] == 0
    assert s0["logit_tiles"] == -(-w.N // 128) * n_vt          # nothing provably flat
    assert s1["logit_tiles"] == n_vt                             # only the peaky block is visited
    assert s1["flat_units"] > 0
    assert s0["live_tiles"] == s1["live_tiles"]                  # the same live units either way
    _, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    fE, fC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, filter_eps=EPS, tile=ELEM)
    for gE, gC in ((cE, cC), (rE, rC)):
        assert rel_fro(gE.cpu().numpy(), fE) <= GRAD_REL_FILTER_OFF
        assert rel_fro(gC.cpu().numpy(), fC) <= GRAD_REL_FILTER_OFF


def test_row_max_flag_without_fresh_maxima_visits_every_tile():
    # CCE_BWD_ROW_MAX when cce_backward_prepare_rows has not stored maxima for
    # this call (a fresh workspace, or maxima already used by a previous
    # call): every block is treated as not flat -- the exact path, slower
    import torch
    import linear_cross_entropy_05_b200 as L
    from linear_cross_entropy_05_b200 import _native as N_
    w = synth.GEMMA2_2B.with_sizes(N=500, V=6000, D=256)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    rm = torch.empty(w.N, device="cuda")
    loss, lse = L.forward(E, C, y, IGN, row_max=rm)
    dl = torch.from_numpy(synth.random_dloss(24, w.N)).cuda()
    dE = torch.empty((w.N, w.D), device="cuda")
    dC = torch.empty((w.V, w.D), device="cuda")
    ws = L.Workspace()
    buf = ws.get(L.cce_backward_workspace_size_ex(w.N, w.D, w.V, L.CCE_BWD_ROW_MAX))
    buf.zero_()
    stream = torch.cuda.current_stream().cuda_stream

    def run():
        N_.cce_backward_ex(E.data_ptr(), C.data_ptr(), y.data_ptr(), lse.data_ptr(), dl.data_ptr(), w.N, w.D, w.V,
                           IGN, EPS, L.CCE_BWD_ROW_MAX, dE.data_ptr(), dC.data_ptr(), buf.data_ptr(), buf.numel(),
                           stream)
        return L.read_status(ws)

    n_tiles = -(-w.N // 128) * -(-w.V // 256)
    assert run()["logit_tiles"] == n_tiles                       # never prepared
    ref = (dE.clone(), dC.clone())
    N_.cce_backward_prepare_rows(rm.data_ptr(), w.N, w.D, w.V, buf.data_ptr(), buf.numel(), stream)
    st = run()
    assert st["logit_tiles"] == 0 and st["flat_units"] > 0      # every block flat with the maxima
    assert rel_fro(dE.cpu().numpy(), ref[0].cpu().numpy()) <= GRAD_REL_FILTER_OFF
    assert rel_fro(dC.cpu().numpy(), ref[1].cpu().numpy()) <= GRAD_REL_FILTER_OFF
    assert run()["logit_tiles"] == n_tiles                       # maxima serve one call only
