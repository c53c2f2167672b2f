"""Vocabulary-parallel form: shards of C on one GPU, merged, against the
unsharded path and the oracle.  (Each shard would live on its own GPU; the
exchange is an all-gather of the [3, N] statistics and an all-reduce of dE.)"""
import numpy as np
import pytest

import oracle
from linear_cross_entropy_05_b200 import synth

from _gpu_helpers import GRAD_REL_FILTER_OFF, IGN, LOSS_ABS, filter_on_bar, gpu_backward, gpu_forward, \
    rel_fro, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    (synth.GEMMA2_2B.with_sizes(N=1000, V=20077), [0, 7001, 14500, 20077]),
    (synth.LLAMA3_8B.with_sizes(N=700, V=9000), [0, 4096, 9000]),
    (synth.TINY.with_sizes(N=300, V=4173, D=264), [0, 1, 2000, 4173]),     # a one-row shard
]


def _shards(w, bounds, C):
    return [(bounds[k], C[bounds[k]:bounds[k + 1]].contiguous()) for k in range(len(bounds) - 1)]


@pytest.mark.parametrize("w,bounds", CASES, ids=[c[0].name for c in CASES])
def test_sharded_forward_merge_matches_unsharded(w, bounds):
    import torch
    import linear_cross_entropy_05_b200 as L
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    stats = torch.stack([L.forward_shard(E, Cs, y, off, IGN) for off, Cs in _shards(w, bounds, C)])
    loss, lse = L.merge_shards(stats, y, w.V, IGN)
    ref_loss, ref_lse, _ = gpu_forward(E, C, y)
    assert np.abs(loss.cpu().numpy() - ref_loss).max() <= 1e-4
    assert np.abs(lse.cpu().numpy() - ref_lse).max() <= 1e-4
    ol, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    assert np.abs(loss.cpu().numpy() - ol).max() <= LOSS_ABS
    assert (loss.cpu().numpy()[inp["y"] == IGN] == 0).all()


@pytest.mark.parametrize("eps", [0.0, synth.EPS_BF16_FILTER], ids=["filter-off", "filter-on"])
@pytest.mark.parametrize("w,bounds", CASES[:2], ids=[c[0].name for c in CASES[:2]])
def test_sharded_backward_assembles_the_full_gradient(w, bounds, eps):
    import torch
    import linear_cross_entropy_05_b200 as L
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, _ = gpu_forward(E, C, y)
    lse_t = torch.from_numpy(lse).cuda()
    dloss = synth.random_dloss(21, w.N)
    dl = torch.from_numpy(dloss).cuda()
    dE = torch.zeros_like(E, dtype=torch.float32)
    dCs = []
    for off, Cs in _shards(w, bounds, C):
        dEp, dCp = L.backward_shard(E, Cs, y, lse_t, dl, off, eps, IGN)
        dE += dEp
        dCs.append(dCp)
    dC = torch.cat(dCs)
    _, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)
    if eps == 0.0:
        rE, rC, _ = gpu_backward(E, C, y, lse, dloss, 0.0)
        assert rel_fro(dE.cpu().numpy(), rE.cpu().numpy()) < 1e-5
        assert rel_fro(dC.cpu().numpy(), rC.cpu().numpy()) < 1e-5
        oE, oC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN)
        assert rel_fro(dE.cpu().numpy(), oE) <= GRAD_REL_FILTER_OFF
        assert rel_fro(dC.cpu().numpy(), oC) <= GRAD_REL_FILTER_OFF
    else:
        # the filter decides entry by entry, so the shards together drop
        # exactly the entries the unsharded filter drops: tight against the
        # element-filtered oracle, and the filter-on bar against the exact one
        fE, fC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, filter_eps=eps, tile=(1, 1))
        assert rel_fro(dE.cpu().numpy(), fE) <= GRAD_REL_FILTER_OFF
        assert rel_fro(dC.cpu().numpy(), fC) <= GRAD_REL_FILTER_OFF
        xE, xC = oracle.backward(inp["E"], inp["C"], inp["y"], olse, dloss, IGN)
        assert rel_fro(dE.cpu().numpy(), xE) <= filter_on_bar(w.V)
        assert rel_fro(dC.cpu().numpy(), xC) <= filter_on_bar(w.V)


def test_single_shard_helper_equals_unsharded_path():
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.GEMMA2_2B.with_sizes(N=600, V=9000)
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, dE, dC = L.vocab_parallel_forward_backward(E, C, y, 0, w.V, filter_eps=0.0)
    rl, rlse, _ = gpu_forward(E, C, y)
    rE, rC, _ = gpu_backward(E, C, y, rlse, synth.mean_dloss(inp["y"]), 0.0)
    assert np.abs(loss.cpu().numpy() - rl).max() <= 1e-5
    assert rel_fro(dE.cpu().numpy(), rE.cpu().numpy()) < 1e-5
    assert rel_fro(dC.cpu().numpy(), rC.cpu().numpy()) < 1e-5


def test_merge_flags_labels_outside_the_full_vocabulary():
    import torch
    import linear_cross_entropy_05_b200 as L
    w = synth.TINY.with_sizes(N=200, V=3000, D=64)
    inp = synth.make_inputs(w)
    inp["y"][5] = 3000
    inp["y"][6] = IGN
    E, C, y = to_dev(inp)
    stats = torch.stack([L.forward_shard(E, C[:1500].contiguous(), y, 0), L.forward_shard(E, C[1500:].contiguous(), y, 1500)])
    loss, lse = L.merge_shards(stats, y, w.V, IGN)
    l = loss.cpu().numpy()
    assert np.isnan(l[5]) and l[6] == 0.0 and np.isfinite(np.delete(l, 5)).all()


def test_merge_of_hand_made_statistics():
    # lse = M + log sum_r s_r exp(m_r - M) and loss = lse - sum_r t_r, with
    # shards that hold nothing for a token (m = -inf, s = 0) and an ignored
    # token; float32-exact inputs against fp64
    import torch
    import linear_cross_entropy_05_b200 as L
    inf = np.inf
    m = np.array([[1.0, 2.0, -inf, 0.5, 30.0],
                  [3.0, -inf, -inf, 0.25, -20.0],
                  [-2.0, 1.5, 4.0, 0.5, 29.0]], dtype=np.float32)
    s = np.array([[1.5, 2.0, 0.0, 1.0, 3.0],
                  [2.5, 0.0, 0.0, 7.0, 1.0],
                  [1.0, 4.0, 9.0, 1.0, 2.0]], dtype=np.float32)
    t = np.array([[0.75, 0.0, 0.0, 0.0, 0.0],
                  [0.0, 0.0, 0.0, 0.125, 0.0],
                  [0.0, 1.0, 3.5, 0.0, 28.0]], dtype=np.float32)
    y = np.array([3, 9, 7, 0, IGN], dtype=np.int64)
    stats = torch.from_numpy(np.stack([m, s, t], axis=1)).cuda()        # [R, 3, N]
    loss, lse = L.merge_shards(stats, torch.from_numpy(y).cuda(), 10, IGN)
    m64, s64, t64 = m.astype(np.float64), s.astype(np.float64), t.astype(np.float64)
    M = m64.max(axis=0)
    want_lse = M + np.log((s64 * np.exp(m64 - M)).sum(axis=0))
    want_loss = np.where(y != IGN, want_lse - t64.sum(axis=0), 0.0)
    assert np.abs(lse.cpu().numpy() - want_lse).max() <= 1e-5 * np.abs(want_lse).max()
    assert np.abs(loss.cpu().numpy() - want_loss).max() <= 1e-5 * np.abs(want_loss).max()
    assert loss.cpu().numpy()[4] == 0
