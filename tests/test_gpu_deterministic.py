"""Deterministic (fixed-point accumulated) backward and bf16 gradient outputs."""
import numpy as np
import pytest

import oracle
from linear_cross_entropy_05_b200 import synth

from _gpu_helpers import GRAD_REL_FILTER_OFF, GRAD_REL_FILTER_ON, IGN, gpu_forward, rel_fro, to_dev

pytestmark = pytest.mark.gpu

EPS = synth.EPS_BF16_FILTER
CASES = [
    (synth.TINY.with_sizes(N=300, V=4096 + 77, D=264), 0.0),
    (synth.GEMMA2_2B.with_sizes(N=1000, V=20000), EPS),
    (synth.LLAMA3_8B.with_sizes(N=700, V=9000), EPS),
    (synth.SMALL_LARGE_VOCAB.with_sizes(N=1500, V=20000), 0.0),
    # flat blocks with D = 264: the flat-row kernel's last dC piece is a
    # ragged 8-value tail (fp32 and int64 bulk reduce-adds)
    (synth.GEMMA2_2B.with_sizes(N=500, V=6000, D=264), EPS),
]


def _bwd(E, C, y, lse, dl, eps, **kw):
    import torch
    import linear_cross_entropy_05_b200 as L
    ws = L.Workspace()
    dE, dC = L.backward(E, C, y, lse, dl, eps, IGN, workspace=ws, **kw)
    st = L.read_status(ws)
    assert st["status"] == 0 and st["flags"] == 0
    return dE, dC, st


@pytest.mark.parametrize("stripes", [None, False], ids=["default-path", "fixed-point"])
@pytest.mark.parametrize("w,eps", CASES, ids=[c[0].name + ("-filter" if c[1] else "") for c in CASES])
def test_deterministic_backward_is_bitwise_reproducible_and_matches_oracle(w, eps, stripes):
    # with the filter off the default path is the stripe kernel summing in
    # stripe order; stripes=False (and the filter on) take the int64
    # fixed-point accumulation
    import torch
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    dloss = synth.random_dloss(8, w.N)
    dl = torch.from_numpy(dloss).cuda()
    lse_t = torch.from_numpy(lse).cuda()
    a = _bwd(E, C, y, lse_t, dl, eps, deterministic=True, stripes=stripes)
    b = _bwd(E, C, y, lse_t, dl, eps, deterministic=True, stripes=stripes)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])       # same bits
    assert a[2]["live_tiles"] == b[2]["live_tiles"]
    ref = _bwd(E, C, y, lse_t, dl, eps)                               # atomic fp32 accumulation
    assert rel_fro(a[0].cpu().numpy(), ref[0].cpu().numpy()) < 1e-5
    assert rel_fro(a[1].cpu().numpy(), ref[1].cpu().numpy()) < 1e-5
    _, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    oE, oC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, filter_eps=eps)
    assert rel_fro(a[0].cpu().numpy(), oE) <= GRAD_REL_FILTER_OFF
    assert rel_fro(a[1].cpu().numpy(), oC) <= GRAD_REL_FILTER_OFF


@pytest.mark.parametrize("w,eps", CASES[:2] + CASES[4:], ids=["ragged", "gemma-shaped-filter", "flat-D264-filter"])
def test_bf16_gradient_outputs(w, eps):
    import torch
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    dloss = synth.random_dloss(9, w.N)
    dl = torch.from_numpy(dloss).cuda()
    lse_t = torch.from_numpy(lse).cuda()
    gE, gC, _ = _bwd(E, C, y, lse_t, dl, eps, bf16_grads=True)
    assert gE.dtype == torch.bfloat16 and gC.dtype == torch.bfloat16
    fE, fC, _ = _bwd(E, C, y, lse_t, dl, eps, deterministic=True, stripes=False)
    # the bf16 outputs are the deterministic fp32 results rounded once
    assert torch.equal(gE, fE.to(torch.bfloat16)) or rel_fro(gE.float().cpu().numpy(), fE.cpu().numpy()) < 4e-3
    _, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    oE, oC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, filter_eps=eps)
    tol = GRAD_REL_FILTER_OFF if eps <= 0 else GRAD_REL_FILTER_ON
    assert rel_fro(gE.float().cpu().numpy(), oE) <= tol
    assert rel_fro(gC.float().cpu().numpy(), oC) <= tol


def test_deterministic_scale_edges():
    # all-zero upstream gradient: exact zeros; a large dloss scale stays in range
    import torch
    w = synth.GEMMA2_2B.with_sizes(N=500, V=6000, D=256)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    lse_t = torch.from_numpy(lse).cuda()
    z = torch.zeros(w.N, device="cuda")
    dE, dC, _ = _bwd(E, C, y, lse_t, z, 0.0, deterministic=True)
    assert (dE == 0).all() and (dC == 0).all()
    big = torch.full((w.N,), 1e4, device="cuda")
    dE, dC, _ = _bwd(E, C, y, lse_t, big, 0.0, deterministic=True)
    rE, rC, _ = _bwd(E, C, y, lse_t, big, 0.0)
    assert torch.isfinite(dE).all() and torch.isfinite(dC).all()
    assert rel_fro(dE.cpu().numpy(), rE.cpu().numpy()) < 1e-5
    assert rel_fro(dC.cpu().numpy(), rC.cpu().numpy()) < 1e-5


@pytest.mark.parametrize("mode", ["atomic", "deterministic", "bf16"])
def test_accumulate_adds_this_calls_gradients(mode):
    # CCE_BWD_ACCUMULATE: no zeroing pass; the call adds its gradients to
    # whatever dE and dC hold
    import torch
    w = synth.GEMMA2_2B.with_sizes(N=600, V=9000, D=256)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    dl = torch.from_numpy(synth.random_dloss(12, w.N)).cuda()
    lse_t = torch.from_numpy(lse).cuda()
    kw = {"atomic": {}, "deterministic": {"deterministic": True}, "bf16": {"bf16_grads": True}}[mode]
    gE, gC, _ = _bwd(E, C, y, lse_t, dl, EPS, **kw)          # this call's gradients alone
    # prior contents of the size of the gradients (seeded, generated on the host)
    gen = torch.Generator().manual_seed(3)
    rE = (torch.randn(gE.shape, generator=gen) * float(gE.float().abs().max())).to(gE.dtype).cuda()
    rC = (torch.randn(gC.shape, generator=gen) * float(gC.float().abs().max())).to(gC.dtype).cuda()
    aE, aC = rE.clone(), rC.clone()
    _bwd(E, C, y, lse_t, dl, EPS, out=(aE, aC), accumulate=True, **kw)
    if mode == "deterministic":
        # one fp32 add of the same fixed-point sum per entry: bit for bit
        assert torch.equal(aE, rE + gE) and torch.equal(aC, rC + gC)
        zE, zC = torch.zeros_like(gE), torch.zeros_like(gC)
        for _ in range(2):
            _bwd(E, C, y, lse_t, dl, EPS, out=(zE, zC), accumulate=True, **kw)
        assert torch.equal(zE, 2 * gE) and torch.equal(zC, 2 * gC)   # doubling is exact in fp32
    elif mode == "bf16":
        # old + this call's sum, rounded once to bf16: the same as rounding
        # old + (the fp32 deterministic sum) except where the fp32 rounding of
        # the sum moves a bf16 tie, and then by one bf16 step at most
        fE, fC, _ = _bwd(E, C, y, lse_t, dl, EPS, deterministic=True)
        for a, r, f in ((aE, rE, fE), (aC, rC, fC)):
            want = (r.float() + f).to(torch.bfloat16)
            off = a != want
            assert off.float().mean().item() < 1e-3
            assert ((a.float() - want.float()).abs()[off] <= want.float().abs()[off] * 2.0 ** -7).all()
    else:
        for a, r, g in ((aE, rE, gE), (aC, rC, gC)):
            assert rel_fro((a - r).cpu().numpy(), g.cpu().numpy()) < 1e-5


@pytest.mark.parametrize("eps", [0.0, synth.EPS_BF16_FILTER])
def test_prepared_backward_equals_unprepared(eps):
    """cce_backward_prepare on a second stream while the forward runs, then
    the backward with CCE_BWD_PREPARED: the same bits (deterministic mode) and
    the same filter counters as a backward that computes max_v |C_v| itself."""
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=900, V=20000)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    dl = torch.from_numpy(synth.random_dloss(5, w.N)).cuda()
    ws_f, ws_a, ws_b = L.Workspace(), L.Workspace(), L.Workspace()
    side = torch.cuda.Stream()
    main = torch.cuda.current_stream()
    ready = torch.cuda.Event()
    side.wait_stream(main)
    L.backward_prepare(C, w.N, ws_b, deterministic=True, stream=side)
    ready.record(side)
    loss, lse = L.forward(E, C, y, IGN, workspace=ws_f)
    main.wait_event(ready)
    # (the fixed-point path, which uses max_v |C_v| with the filter on or off)
    dE_p, dC_p = L.backward(E, C, y, lse, dl, eps, IGN, workspace=ws_b, deterministic=True, prepared=True,
                            stripes=False)
    st_p = L.read_status(ws_b)
    dE, dC = L.backward(E, C, y, lse, dl, eps, IGN, workspace=ws_a, deterministic=True, stripes=False)
    st = L.read_status(ws_a)
    assert st_p["status"] == 0 and st["status"] == 0
    for k in ("live_tiles", "dead_tiles", "pruned_tiles", "logit_tiles"):
        assert st_p[k] == st[k]
    assert torch.equal(dE_p.view(torch.int32), dE.view(torch.int32))
    assert torch.equal(dC_p.view(torch.int32), dC.view(torch.int32))


@pytest.mark.parametrize("bf16", [False, True], ids=["fp32", "bf16-grads"])
def test_fixed_point_with_flat_and_non_flat_blocks(bf16):
    # peaky rows keep one token block out of the flat set: its tiles go
    # through the tile kernel's int64 reductions while the flat blocks'
    # label entries go through the flat-row kernel's int64 bulk adds; the
    # result is bitwise repeatable and matches the element-filtered oracle
    import torch
    w = synth.GEMMA2_2B.with_sizes(N=640, V=12000, D=256)
    inp = synth.make_inputs(w)
    E64 = oracle.bf16_bits_to_f64(inp["E"])
    E64[128:256] *= 120.0
    inp["E"] = synth.round_to_bf16_bits(E64.astype(np.float32))
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    dloss = synth.random_dloss(9, w.N)
    dl = torch.from_numpy(dloss).cuda()
    lse_t = torch.from_numpy(lse).cuda()
    kw = dict(deterministic=not bf16, bf16_grads=bf16)
    a = _bwd(E, C, y, lse_t, dl, EPS, **kw)
    b = _bwd(E, C, y, lse_t, dl, EPS, **kw)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    st = a[2]
    assert 0 < st["flat_units"] < st["live_tiles"] and st["logit_tiles"] > 0
    _, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    fE, fC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, filter_eps=EPS, tile=(1, 1))
    bar = 1e-2 if bf16 else GRAD_REL_FILTER_OFF      # bf16 outputs: one more rounding
    assert rel_fro(a[0].float().cpu().numpy(), fE) <= bar
    assert rel_fro(a[1].float().cpu().numpy(), fC) <= bar
