"""The dense backward through softmax-gradient stripes (CCE_BWD_STRIPES, the
binding's default with the filter off) against the exact fp64 gradient, on
shapes that exercise its task order: several stripes with buffer reuse, a
ragged last stripe, D not a multiple of 64, token counts that need more than
one launch (beyond 16384 tokens), gradient accumulation; and the property
that each dC tile is written by exactly one task (bitwise repeatable)."""
import numpy as np
import pytest

import oracle
from linear_cross_entropy_05_b200 import synth

from _gpu_helpers import GRAD_REL_FILTER_OFF, IGN, gpu_forward, rel_fro, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    synth.GEMMA2_2B.with_sizes(N=700, V=16 * 256 * 4 + 77, D=264),   # 5 stripes: buffers reused, ragged tail
    synth.LLAMA3_8B.with_sizes(N=16384 + 300, V=3000, D=64),          # two launches (token super-blocks)
    synth.SMALL_LARGE_VOCAB.with_sizes(N=513, V=2048, D=896),         # exactly one stripe
]


def _exact(inp, dloss):
    _, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    return oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN)


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_stripe_backward_matches_exact_gradient(w):
    import torch
    import linear_cross_entropy_05_b200 as L
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    assert st["status"] == 0
    dloss = synth.random_dloss(17, w.N)
    dl = torch.from_numpy(dloss).cuda()
    ws = L.Workspace()
    dE, dC = L.backward(E, C, y, torch.from_numpy(lse).cuda(), dl, 0.0, IGN, workspace=ws, stripes=True)
    st = L.read_status(ws)
    assert st["status"] == 0 and st["flags"] == 0
    assert st["live_tiles"] == -(-w.N // 32) * -(-w.V // 32)
    assert st["logit_tiles"] == -(-w.N // 128) * -(-w.V // 256)
    rE, rC = _exact(inp, dloss)
    assert rel_fro(dE.cpu().numpy(), rE) <= GRAD_REL_FILTER_OFF
    assert rel_fro(dC.cpu().numpy(), rC) <= GRAD_REL_FILTER_OFF
    ign = inp["y"] == IGN
    if ign.any():
        assert float(dE[torch.from_numpy(ign).cuda()].abs().max()) == 0.0


def test_stripe_backward_dC_written_once_and_accumulation():
    import torch
    import linear_cross_entropy_05_b200 as L
    w = CASES[0]
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    lse_t = torch.from_numpy(lse).cuda()
    dl = torch.from_numpy(synth.random_dloss(18, w.N)).cuda()
    ws = L.Workspace()
    dE1, dC1 = L.backward(E, C, y, lse_t, dl, 0.0, IGN, workspace=ws, stripes=True)
    dE2, dC2 = L.backward(E, C, y, lse_t, dl, 0.0, IGN, workspace=ws, stripes=True)
    # every dC tile comes from one task that sums over all tokens in a fixed order
    assert torch.equal(dC1.view(torch.int32), dC2.view(torch.int32))
    assert float((dE1 - dE2).abs().max()) <= 1e-6 * float(dE1.abs().max())
    # accumulation: prior + this call's gradients
    pE = torch.randn_like(dE1)
    pC = torch.randn_like(dC1)
    aE, aC = pE.clone(), pC.clone()
    L.backward(E, C, y, lse_t, dl, 0.0, IGN, workspace=ws, out=(aE, aC), accumulate=True, stripes=True)
    assert float((aE - (pE + dE1)).abs().max()) <= 1e-5
    assert float((aC - (pC + dC1)).abs().max()) <= 1e-5
    assert L.read_status(ws)["status"] == 0


@pytest.mark.parametrize("vt", [1, 4, 8, 12], ids=["1-tile", "4-tiles", "8-tiles", "12-tiles"])
def test_stripe_width_knob_keeps_the_result(vt):
    # narrower and ragged stripe widths (the default is 16 tiles of 256):
    # more stripes, more buffer reuse, the same gradient
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=600, V=9 * 256 + 77, D=264)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    dloss = synth.random_dloss(19, w.N)
    L.cce_debug_set_stripe_params(0, 0, vt)
    try:
        ws = L.Workspace()
        dE, dC = L.backward(E, C, y, torch.from_numpy(lse).cuda(), torch.from_numpy(dloss).cuda(), 0.0, IGN,
                            workspace=ws, stripes=True)
        st = L.read_status(ws)
    finally:
        L.cce_debug_set_stripe_params(0, 0, 0)
    assert st["status"] == 0 and st["flags"] == 0
    rE, rC = _exact(inp, dloss)
    assert rel_fro(dE.cpu().numpy(), rE) <= GRAD_REL_FILTER_OFF
    assert rel_fro(dC.cpu().numpy(), rC) <= GRAD_REL_FILTER_OFF


@pytest.mark.parametrize("order", [(1, 4, 2), (1, 1, 1), (1, 64, 1)], ids=["g4-lag2", "g1-lag1", "one-group"])
def test_stripe_task_order_keeps_the_bits(order):
    # the interleaved task order runs the same tasks: in the deterministic
    # (stripe-ordered) mode the gradients are bit for bit those of the
    # default order, and they match the exact gradient
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=1300, V=5 * 4096 + 77, D=264)   # 6 stripes, 6 token blocks
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    lse_t = torch.from_numpy(lse).cuda()
    dloss = synth.random_dloss(20, w.N)
    dl = torch.from_numpy(dloss).cuda()
    ref = L.backward(E, C, y, lse_t, dl, 0.0, IGN, workspace=L.Workspace(), stripes=True, deterministic=True)
    L.cce_debug_set_stripe_order(*order)
    try:
        ws = L.Workspace()
        got = L.backward(E, C, y, lse_t, dl, 0.0, IGN, workspace=ws, stripes=True, deterministic=True)
        st = L.read_status(ws)
        fast = L.backward(E, C, y, lse_t, dl, 0.0, IGN, workspace=ws, stripes=True)
    finally:
        L.cce_debug_set_stripe_order(0, 4, 2)
    assert st["status"] == 0 and st["flags"] == 0
    assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
    rE, rC = _exact(inp, dloss)
    assert rel_fro(fast[0].cpu().numpy(), rE) <= GRAD_REL_FILTER_OFF
    assert rel_fro(fast[1].cpu().numpy(), rC) <= GRAD_REL_FILTER_OFF


@pytest.mark.parametrize("deterministic", [False, True], ids=["atomic", "stripe-ordered"])
def test_stripes_with_the_entry_filter(deterministic):
    # CCE_BWD_STRIPES with filter_eps > 0: the pre-pass sends flat blocks to
    # the flat-row kernel; the stripe kernel recomputes the 256-token blocks
    # that hold a block that is not flat, zeroes the entries below eps (and
    # the flat blocks' rows) in G, and skips the all-zero G tiles in the dC
    # and dE products; the result is the element-filtered gradient, on a head
    # whose scaled rows make blocks 1 and 2 (of six) non-flat
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=700, V=3 * 4096 + 77, D=264)
    inp = synth.make_inputs(w)
    E64 = oracle.bf16_bits_to_f64(inp["E"])
    E64[128:384] *= 120.0
    inp["E"] = synth.round_to_bf16_bits(E64.astype(np.float32))
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    lse_t = torch.from_numpy(lse).cuda()
    dloss = synth.random_dloss(21, w.N)
    dl = torch.from_numpy(dloss).cuda()
    eps = synth.EPS_BF16_FILTER
    ws = L.Workspace()
    dE, dC = L.backward(E, C, y, lse_t, dl, eps, IGN, workspace=ws, stripes=True, deterministic=deterministic)
    st = L.read_status(ws)
    assert st["status"] == 0 and st["flags"] == 0
    n_vt = -(-w.V // 256)
    if deterministic:
        # stripe order alone, no flat-row path: every tile recomputed
        assert st["logit_tiles"] == -(-w.N // 128) * n_vt and st["flat_units"] == 0
    else:
        assert st["logit_tiles"] == 4 * n_vt      # the two 256-token blocks holding blocks 1 and 2
        assert st["flat_units"] > 0
    _, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    fE, fC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, filter_eps=eps, tile=(1, 1))
    # live (some entry kept), dead (recomputed, none kept) and pruned (flat
    # blocks' units without a label entry) add up to all units
    live = oracle.tile_live_map(inp["E"], inp["C"], inp["y"], olse, IGN, eps, (32, 32))
    assert st["live_tiles"] + st["dead_tiles"] + st["pruned_tiles"] == live.size
    assert abs(st["live_tiles"] - int(live.sum())) <= max(2, live.size // 1000)
    assert rel_fro(dE.cpu().numpy(), fE) <= GRAD_REL_FILTER_OFF
    assert rel_fro(dC.cpu().numpy(), fC) <= GRAD_REL_FILTER_OFF
    # the default filtered path gives the same gradient up to the bf16
    # rounding of G, which each path does in its own order (each is ~1.7e-3
    # from the oracle)
    gE, gC = L.backward(E, C, y, lse_t, dl, eps, IGN, workspace=L.Workspace())
    assert rel_fro(dE.cpu().numpy(), gE.cpu().numpy()) <= GRAD_REL_FILTER_OFF
    assert rel_fro(dC.cpu().numpy(), gC.cpu().numpy()) <= GRAD_REL_FILTER_OFF
    if deterministic:
        dE2, dC2 = L.backward(E, C, y, lse_t, dl, eps, IGN, workspace=ws, stripes=True, deterministic=True)
        assert torch.equal(dE, dE2) and torch.equal(dC, dC2)


def test_stripes_with_the_filter_on_a_flat_head_recompute_nothing():
    # every block flat: the stripe kernel skips every recompute task and
    # every dC / dE product; the gradient comes from the flat-row kernel
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=16384 + 300, V=12000, D=256)   # two token super-blocks
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    dloss = synth.random_dloss(25, w.N)
    ws = L.Workspace()
    dE, dC = L.backward(E, C, y, torch.from_numpy(lse).cuda(), torch.from_numpy(dloss).cuda(),
                        synth.EPS_BF16_FILTER, IGN, workspace=ws, stripes=True)
    st = L.read_status(ws)
    assert st["status"] == 0 and st["flags"] == 0
    assert st["logit_tiles"] == 0 and st["flat_units"] == st["live_tiles"] > 0
    _, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    rows = np.concatenate([np.arange(0, 256), np.arange(w.N - 300, w.N)])
    vrows = np.unique(np.concatenate([inp["y"][inp["y"] != IGN][:200], [0, w.V - 1]]))
    fE, fC = oracle.backward_sampled(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, rows, vrows,
                                     filter_eps=synth.EPS_BF16_FILTER, tile=(1, 1))
    assert rel_fro(dE[torch.from_numpy(rows).cuda()].cpu().numpy(), fE) <= GRAD_REL_FILTER_OFF
    assert rel_fro(dC[torch.from_numpy(vrows).cuda()].cpu().numpy(), fC) <= GRAD_REL_FILTER_OFF


def test_stripes_with_the_filter_accumulate():
    # CCE_BWD_ACCUMULATE through the filtered stripe path: the stripes add
    # their dC tiles (instead of storing them) and the flat-row kernel adds
    # on top; the result is the prior contents plus this call's gradient
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=700, V=2 * 4096 + 77, D=264)
    inp = synth.make_inputs(w)
    E64 = oracle.bf16_bits_to_f64(inp["E"])
    E64[128:256] *= 120.0                   # one block that is not flat
    inp["E"] = synth.round_to_bf16_bits(E64.astype(np.float32))
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    lse_t = torch.from_numpy(lse).cuda()
    dl = torch.from_numpy(synth.random_dloss(26, w.N)).cuda()
    eps = synth.EPS_BF16_FILTER
    gE, gC = L.backward(E, C, y, lse_t, dl, eps, IGN, workspace=L.Workspace(), stripes=True)
    gen = torch.Generator().manual_seed(4)
    pE = (torch.randn(gE.shape, generator=gen) * float(gE.abs().max())).cuda()
    pC = (torch.randn(gC.shape, generator=gen) * float(gC.abs().max())).cuda()
    aE, aC = pE.clone(), pC.clone()
    ws = L.Workspace()
    L.backward(E, C, y, lse_t, dl, eps, IGN, workspace=ws, out=(aE, aC), accumulate=True, stripes=True)
    assert L.read_status(ws)["status"] == 0
    assert rel_fro((aE - pE).cpu().numpy(), gE.cpu().numpy()) < 1e-5
    assert rel_fro((aC - pC).cpu().numpy(), gC.cpu().numpy()) < 1e-5


@pytest.mark.parametrize("eps", [0.0, synth.EPS_BF16_FILTER], ids=["filter-off", "filter-on"])
def test_stripes_with_bf16_outputs(eps):
    # CCE_BWD_STRIPES | CCE_BWD_BF16_GRADS: fp32 scratch sums rounded once to
    # bf16; with accumulate the old bf16 values are added before rounding
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=700, V=2 * 4096 + 77, D=264)
    inp = synth.make_inputs(w)
    E64 = oracle.bf16_bits_to_f64(inp["E"])
    E64[128:256] *= 120.0                   # one block that is not flat
    inp["E"] = synth.round_to_bf16_bits(E64.astype(np.float32))
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    lse_t = torch.from_numpy(lse).cuda()
    dloss = synth.random_dloss(27, w.N)
    dl = torch.from_numpy(dloss).cuda()
    ws = L.Workspace()
    bE, bC = L.backward(E, C, y, lse_t, dl, eps, IGN, workspace=ws, stripes=True, bf16_grads=True)
    assert bE.dtype == torch.bfloat16 and bC.dtype == torch.bfloat16
    assert L.read_status(ws)["status"] == 0
    fE, fC = L.backward(E, C, y, lse_t, dl, eps, IGN, workspace=L.Workspace(), stripes=True)   # fp32
    # one rounding to bf16 of the same kind of sum: within a bf16 step
    assert rel_fro(bE.float().cpu().numpy(), fE.cpu().numpy()) < 4e-3
    assert rel_fro(bC.float().cpu().numpy(), fC.cpu().numpy()) < 4e-3
    _, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    oE, oC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, filter_eps=eps, tile=(1, 1))
    assert rel_fro(bE.float().cpu().numpy(), oE) <= 1e-2
    assert rel_fro(bC.float().cpu().numpy(), oC) <= 1e-2
    # accumulation into existing bf16 gradients
    gen = torch.Generator().manual_seed(5)
    pE = (torch.randn(bE.shape, generator=gen) * float(bE.float().abs().max())).to(torch.bfloat16).cuda()
    pC = (torch.randn(bC.shape, generator=gen) * float(bC.float().abs().max())).to(torch.bfloat16).cuda()
    aE, aC = pE.clone(), pC.clone()
    L.backward(E, C, y, lse_t, dl, eps, IGN, workspace=ws, out=(aE, aC), accumulate=True, stripes=True,
               bf16_grads=True)
    wE, wC = (pE.float() + fE).to(torch.bfloat16), (pC.float() + fC).to(torch.bfloat16)
    assert rel_fro(aE.float().cpu().numpy(), wE.float().cpu().numpy()) < 4e-3
    assert rel_fro(aC.float().cpu().numpy(), wC.float().cpu().numpy()) < 4e-3
