"""The five LLM-head workloads at full size, in the launch configuration the
benchmark times, against the fp64 oracle.

The oracle's full forward of these workloads (every token's loss and lse) is
stored in tests/golden/fullsize_oracle.npz by tests/golden/make_fullsize_oracle.py,
which calls only the oracle and the seeded input generator.  With it:

* forward: every token's loss and lse, and the mean loss over kept tokens,
  are compared at full size (loss within 1e-2 absolute, mean within 1e-4
  relative);
* backward: sampled rows the oracle can form one by one against the EXACT
  gradient (the bar: 1e-2 relative Frobenius with the filter on, 5e-3 with it
  off) and, with the filter on, against the oracle's element-filtered
  gradient (5e-3): at least four whole 128-token blocks of dE (the first, one in the
  middle, a seeded one and the last) and at least sixteen rows of dC (the
  most frequent labels, a label seen once, rows without any kept token, the
  last row, seeded rows, and on the small-model head scaled "peaky" rows);
* identities that hold at any size: <E, dE> = <C, dC> and, with the filter
  off, sum_v dC_v = 0 (every softmax-gradient row sums to zero).
"""
import os

import numpy as np
import pytest

import oracle
from linear_cross_entropy_05_b200 import synth

from _gpu_helpers import (GRAD_REL_FILTER_OFF, GRAD_REL_FILTER_ON, IGN, LOSS_ABS, MEAN_REL, gpu_backward,
                          gpu_forward, rel_fro, to_dev)

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "fullsize_oracle.npz")
GRAD_REL_VS_FILTERED = 5e-3   # GPU with the filter on vs the oracle with the same (element) filter

SWEEPS = [synth.SWEEP.with_sizes(N=n, name=f"long-batch-sweep[N={n}]") for n in synth.SWEEP_NS]
CASES = [(synth.GEMMA2_2B, synth.GEMMA2_2B.filter_eps), (synth.LLAMA3_8B, synth.LLAMA3_8B.filter_eps),
         (synth.SMALL_LARGE_VOCAB, synth.SMALL_LARGE_VOCAB.filter_eps), (synth.SMALL_LARGE_VOCAB, 0.0)] + \
        [(w, w.filter_eps) for w in SWEEPS]
IDS = [w.name + ("" if eps > 0 else "[filter off]") for w, eps in CASES]


def _golden(name):
    with np.load(GOLDEN) as f:
        return f[f"{name}/loss"], f[f"{name}/lse"]


def _dE_rows(N, seed):
    nb = -(-N // 128)
    rng = np.random.default_rng(seed)
    blocks = sorted({0, nb // 2, int(rng.integers(1, nb - 1)), nb - 1})
    return np.concatenate([np.arange(b * 128, min(N, (b + 1) * 128)) for b in blocks])


def _dC_rows(inp, V, seed):
    y = inp["y"]
    counts = np.bincount(y[y != IGN], minlength=V)
    rng = np.random.default_rng(seed)
    picks = list(np.argsort(-counts, kind="stable")[:6])              # most frequent labels
    once = np.nonzero(counts == 1)[0]
    if once.size:
        picks.append(int(once[0]))                                     # a label seen once
    never = np.nonzero(counts == 0)[0]
    if never.size:
        picks += [int(never[0]), int(never[-1])]                       # rows without any kept token
    picks += [V - 1, 7777 % V]
    if inp["peaky_rows"].size:
        picks += [int(inp["peaky_rows"][0]), int(inp["peaky_rows"][-1])]
    picks += list(rng.choice(V, size=6, replace=False))
    rows = np.unique(np.asarray(picks, dtype=np.int64))
    assert rows.size >= 16
    return rows


@pytest.mark.parametrize("w,eps", CASES, ids=IDS)
def test_full_size_against_the_oracle(w, eps):
    import torch
    inp = synth.make_inputs(w)
    ol, olse = _golden(w.name)
    E, C, y = to_dev(inp)

    # ---- forward: every token, and the mean over kept tokens
    loss, lse, st = gpu_forward(E, C, y)
    assert st["status"] == 0 and st["flags"] == 0
    assert np.isfinite(loss).all() and np.isfinite(lse).all()
    assert np.abs(loss.astype(np.float64) - ol).max() <= LOSS_ABS
    assert np.abs(lse.astype(np.float64) - olse).max() <= LOSS_ABS
    keep = inp["y"] != IGN
    o_mean = ol[keep].mean()
    assert abs(loss[keep].astype(np.float64).mean() - o_mean) <= MEAN_REL * abs(o_mean)

    # ---- backward (mean-reduction dloss, as a training step uses)
    dloss = synth.mean_dloss(inp["y"])
    dE, dC, st = gpu_backward(E, C, y, lse, dloss, eps)
    assert st["status"] == 0 and st["flags"] == 0
    n_units = -(-w.N // 32) * -(-w.V // 32)
    if eps > 0:
        assert st["live_tiles"] + st["dead_tiles"] + st["pruned_tiles"] == n_units
    else:
        assert st["live_tiles"] == n_units and st["pruned_tiles"] == 0

    rE = _dE_rows(w.N, 11)
    rC = _dC_rows(inp, w.V, 12)
    gE = dE[torch.from_numpy(rE).cuda()].cpu().numpy()
    gC = dC[torch.from_numpy(rC).cuda()].cpu().numpy()
    xE, xC = oracle.backward_sampled(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, rE, rC, filter_eps=0.0)
    bar = GRAD_REL_FILTER_ON if eps > 0 else GRAD_REL_FILTER_OFF
    assert rel_fro(gE, xE) <= bar
    assert rel_fro(gC, xC) <= bar
    if eps > 0:
        fE, fC = oracle.backward_sampled(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, rE, rC,
                                         filter_eps=eps, tile=(1, 1))
        assert rel_fro(gE, fE) <= GRAD_REL_VS_FILTERED
        assert rel_fro(gC, fC) <= GRAD_REL_VS_FILTERED

    # ---- identities at full size
    a = float((E.double() * dE.double()).sum())
    b = float((C.double() * dC.double()).sum())
    assert abs(a - b) <= 1e-2 * max(abs(a), abs(b))
    if eps == 0:
        col = dC.double().sum(0)
        assert float(col.norm()) <= 1e-3 * float(dC.double().norm())
