"""Pins for the fp64 oracle, independent of the oracle's own code.

Each test fixes the oracle to something other than itself: closed forms,
invariants of the softmax gradient, central finite differences, a library
cross-entropy with autograd, a hand-worked example, brute-force loops on tiny
inputs, and planted mistakes that the pins must catch.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from linear_cross_entropy_05_b200 import synth

HERE = os.path.dirname(os.path.abspath(__file__))
IGN = -100


def _bits(x):
    return synth.round_to_bf16_bits(np.asarray(x, dtype=np.float32))


# --------------------------------------------------------------------------
# decoding / rounding of the shared inputs
# --------------------------------------------------------------------------

def test_bf16_decode_known_patterns():
    bits = np.array([0x3F80, 0xC000, 0x0000, 0x3F81, 0x8000, 0x4049], dtype=np.uint16)
    got = oracle.bf16_bits_to_f64(bits)
    assert got.tolist() == [1.0, -2.0, 0.0, 1.0078125, -0.0, 3.140625]


def test_bf16_rounding_ties_to_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -9, 3.14159265], dtype=np.float32)
    assert synth.round_to_bf16_bits(x).tolist() == [0x3F80, 0x3F80, 0x3F82, 0xBF80, 0x4049]


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------

@pytest.mark.parametrize("V", [1, 7, 4096, 4096 + 77])
def test_zero_classifier_gives_log_V(V):
    rng = np.random.default_rng(1)
    N, D = 9, 16
    E = rng.standard_normal((N, D))
    C = np.zeros((V, D))
    y = rng.integers(0, V, N)
    loss, lse = oracle.forward_f64(E, C, y, IGN)
    np.testing.assert_allclose(loss, math.log(V), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, math.log(V), rtol=0, atol=1e-12)
    dloss = rng.random(N) + 0.5
    dE, dC = oracle.backward_f64(E, C, y, lse, dloss, IGN)
    # dE_i = dloss_i * (mean_v C_v - C_{y_i}) = 0 because C = 0
    np.testing.assert_allclose(dE, 0.0, atol=1e-14)
    # dC_v = (1/V) sum_i dloss_i E_i - sum_{i: y_i = v} dloss_i E_i
    want = np.tile((dloss[:, None] * E).sum(0) / V, (V, 1))
    for i in range(N):
        want[y[i]] -= dloss[i] * E[i]
    np.testing.assert_allclose(dC, want, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("alpha", [0.5, 4.0, 30.0, 700.0])
def test_dominant_target_logit(alpha):
    # row i: z_{i,y_i} = alpha, every other logit 0 => loss = log(1 + (V-1) e^-alpha)
    V, D, N = 11, 5, 3
    E = np.eye(N, D)
    y = np.array([2, 7, 10])
    C = np.zeros((V, D))
    for i in range(N):
        C[y[i]] = alpha * E[i]
    loss, lse = oracle.forward_f64(E, C, y, IGN)
    want = math.log1p((V - 1) * math.exp(-alpha))
    # loss = lse - z_y cancels: fp64 keeps it to a few ulps of alpha
    np.testing.assert_allclose(loss, want, rtol=1e-12, atol=4e-16 * (1.0 + alpha))
    np.testing.assert_allclose(lse, alpha + want, rtol=1e-12)


def test_vocab_of_one_has_zero_loss_and_gradient():
    rng = np.random.default_rng(2)
    E = rng.standard_normal((6, 4))
    C = rng.standard_normal((1, 4))
    y = np.zeros(6, dtype=np.int64)
    loss, lse = oracle.forward_f64(E, C, y, IGN)
    np.testing.assert_allclose(loss, 0.0, atol=1e-14)
    dE, dC = oracle.backward_f64(E, C, y, lse, np.ones(6), IGN)
    np.testing.assert_allclose(dE, 0.0, atol=1e-14)
    np.testing.assert_allclose(dC, 0.0, atol=1e-14)


def test_worked_example_fixture():
    with open(os.path.join(HERE, "golden", "worked_example_2x2x3.json")) as f:
        g = json.load(f)
    E = np.array(g["E"])
    C = np.array(g["C"])
    y = np.array(g["y"])
    loss, lse = oracle.forward_f64(E, C, y, g["ignore_index"])
    np.testing.assert_allclose(loss, g["loss"], rtol=1e-14)
    np.testing.assert_allclose(lse, g["lse"], rtol=1e-14)
    dE, dC = oracle.backward_f64(E, C, y, lse, np.array(g["dloss"]), g["ignore_index"])
    np.testing.assert_allclose(dE, g["dE"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(dC, g["dC"], rtol=1e-13, atol=1e-15)
    # the same example through the bf16-bits entry point (0 and 1 are exact in bf16)
    l2, s2 = oracle.forward(_bits(E), _bits(C), y, g["ignore_index"])
    np.testing.assert_allclose(l2, g["loss"], rtol=1e-14)


# --------------------------------------------------------------------------
# invariants
# --------------------------------------------------------------------------

def test_softmax_rows_sum_to_one_and_gradient_rows_to_zero():
    rng = np.random.default_rng(3)
    z = rng.standard_normal((7, 33)) * 5
    y = rng.integers(0, 33, 7)
    y[3] = IGN
    lse = z.max(1) + np.log(np.exp(z - z.max(1, keepdims=True)).sum(1))
    P, Dm, G = oracle.softmax_grad_f64(z, lse, y, np.full(7, 2.0), IGN)
    np.testing.assert_allclose(P.sum(1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(Dm.sum(1), 0.0, atol=1e-14)
    np.testing.assert_allclose(G.sum(1), 0.0, atol=1e-14)
    assert np.all(Dm[3] == 0.0) and np.all(G[3] == 0.0)


def test_gradient_identities():
    # sum_v dC_v = sum_i (sum_v G_iv) E_i = 0 and <E, dE> = <C, dC> = sum G*z
    rng = np.random.default_rng(4)
    N, D, V = 13, 6, 29
    E = rng.standard_normal((N, D))
    C = rng.standard_normal((V, D))
    y = rng.integers(0, V, N)
    y[5] = IGN
    loss, lse = oracle.forward_f64(E, C, y, IGN)
    dE, dC = oracle.backward_f64(E, C, y, lse, rng.random(N), IGN)
    np.testing.assert_allclose(dC.sum(0), 0.0, atol=1e-12)
    assert abs((E * dE).sum() - (C * dC).sum()) < 1e-11
    assert np.all(dE[5] == 0.0)


def test_ignored_and_invalid_labels():
    rng = np.random.default_rng(5)
    E = rng.standard_normal((4, 3))
    C = rng.standard_normal((5, 3))
    y = np.array([0, IGN, 4, 5])  # 5 is out of range
    loss, lse = oracle.forward_f64(E, C, y, IGN)
    assert loss[1] == 0.0
    assert math.isnan(loss[3])
    assert np.isfinite(lse).all()
    assert math.isnan(oracle.mean_loss(np.zeros(3), np.array([IGN] * 3), IGN))
    np.testing.assert_allclose(oracle.mean_loss(np.array([1.0, 5.0, 3.0]), np.array([0, IGN, 2]), IGN), 2.0)


# --------------------------------------------------------------------------
# finite differences and an independent library
# --------------------------------------------------------------------------

def test_central_finite_differences():
    rng = np.random.default_rng(6)
    N, D, V = 5, 4, 7
    E = rng.standard_normal((N, D))
    C = rng.standard_normal((V, D))
    y = rng.integers(0, V, N)
    y[2] = IGN
    dloss = rng.random(N) + 0.5

    def f(E_, C_):
        l, _ = oracle.forward_f64(E_, C_, y, IGN)
        return float((dloss * l).sum())

    _, lse = oracle.forward_f64(E, C, y, IGN)
    dE, dC = oracle.backward_f64(E, C, y, lse, dloss, IGN)
    h = 1e-6
    for (X, dX, which) in ((E, dE, 0), (C, dC, 1)):
        num = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            Xp = X.copy(); Xp[idx] += h
            Xm = X.copy(); Xm[idx] -= h
            num[idx] = (f(Xp, C) - f(Xm, C)) / (2 * h) if which == 0 else (f(E, Xp) - f(E, Xm)) / (2 * h)
        np.testing.assert_allclose(dX, num, rtol=1e-6, atol=1e-8)


def test_matches_torch_cross_entropy_and_autograd():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(7)
    N, D, V = 24, 16, 50
    E = rng.standard_normal((N, D)) * 0.7
    C = rng.standard_normal((V, D)) * 0.7
    y = rng.integers(0, V, N)
    y[[1, 9]] = IGN
    dloss = rng.random(N) + 0.25
    loss, lse = oracle.forward_f64(E, C, y, IGN)
    Et = torch.tensor(E, dtype=torch.float64, requires_grad=True)
    Ct = torch.tensor(C, dtype=torch.float64, requires_grad=True)
    yt = torch.tensor(y)
    lt = torch.nn.functional.cross_entropy(Et @ Ct.T, yt, ignore_index=IGN, reduction="none")
    np.testing.assert_allclose(loss, lt.detach().numpy(), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, torch.logsumexp(Et @ Ct.T, 1).detach().numpy(), rtol=1e-14)
    (lt * torch.tensor(dloss)).sum().backward()
    dE, dC = oracle.backward_f64(E, C, y, lse, dloss, IGN)
    np.testing.assert_allclose(dE, Et.grad.numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dC, Ct.grad.numpy(), rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------------------
# tile filter: brute force on tiny inputs
# --------------------------------------------------------------------------

def _brute_filtered(E, C, y, dloss, eps, Bn, Bv):
    N, D = E.shape
    V = C.shape[0]
    z = [[sum(E[i, d] * C[v, d] for d in range(D)) for v in range(V)] for i in range(N)]
    lse = [math.log(sum(math.exp(z[i][v]) for v in range(V))) for i in range(N)]
    Dm = [[0.0] * V for _ in range(N)]
    for i in range(N):
        if y[i] == IGN:
            continue
        for v in range(V):
            Dm[i][v] = math.exp(z[i][v] - lse[i]) - (1.0 if v == y[i] else 0.0)
    nt_r, nt_v = -(-N // Bn), -(-V // Bv)
    live = np.zeros((nt_r, nt_v), dtype=bool)
    for a in range(nt_r):
        for b in range(nt_v):
            for i in range(a * Bn, min(N, (a + 1) * Bn)):
                for v in range(b * Bv, min(V, (b + 1) * Bv)):
                    if abs(Dm[i][v]) >= eps:
                        live[a, b] = True
    dE = np.zeros((N, D))
    dC = np.zeros((V, D))
    for i in range(N):
        for v in range(V):
            if not live[i // Bn, v // Bv]:
                continue
            g = dloss[i] * Dm[i][v]
            for d in range(D):
                dE[i, d] += g * C[v, d]
                dC[v, d] += g * E[i, d]
    return np.array(lse), live, dE, dC


@pytest.mark.parametrize("eps", [0.02, 0.1])
@pytest.mark.parametrize("tile", [(2, 4), (1, 1)], ids=["2x4-tiles", "elements"])
def test_tile_filter_against_brute_force(eps, tile):
    rng = np.random.default_rng(8)
    N, D, V = 7, 3, 11
    Bn, Bv = tile
    E = rng.standard_normal((N, D)) * 1.5
    C = rng.standard_normal((V, D)) * 1.5
    y = rng.integers(0, V, N)
    y[4] = IGN
    dloss = rng.random(N) + 0.5
    lse_b, live_b, dE_b, dC_b = _brute_filtered(E, C, y, dloss, eps, Bn, Bv)
    _, lse = oracle.forward_f64(E, C, y, IGN)
    np.testing.assert_allclose(lse, lse_b, rtol=1e-13)
    dE, dC, live = oracle.backward_f64(E, C, y, lse, dloss, IGN, filter_eps=eps, tile=(Bn, Bv),
                                       return_live=True)
    assert live.shape == live_b.shape and (live == live_b).all()
    assert 0 < live.sum() < live.size  # the case really filters something
    np.testing.assert_allclose(dE, dE_b, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dC, dC_b, rtol=1e-12, atol=1e-14)


def _decode_bits(bits):
    # bf16 is the upper half of an fp32 (decoding pinned by test_bf16_decode_known_patterns)
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def _tile_map_case():
    rng = np.random.default_rng(21)
    N, D, V, Bn, Bv = 13, 3, 19, 2, 3          # ragged in both directions
    E_bits = _bits(rng.standard_normal((N, D)) * 3.0)
    C_bits = _bits(rng.standard_normal((V, D)) * 3.0)
    y = rng.integers(0, V, N)
    y[[2, 9]] = IGN
    return E_bits, C_bits, y, Bn, Bv


@pytest.mark.parametrize("rows_per_block", [None, 1, 5])
@pytest.mark.parametrize("eps", [0.03, 0.1])
def test_tile_live_map_against_brute_force(monkeypatch, rows_per_block, eps):
    """oracle.tile_live_map (bf16 inputs, the caller's lse) against a
    brute-force enumeration of |P - onehot| >= eps per tile; rows_per_block
    forces the oracle's row blocking to cut the rows every 2 or 4 tokens (not
    only at the end), so a wrong block boundary shows."""
    E_bits, C_bits, y, Bn, Bv = _tile_map_case()
    E, C = _decode_bits(E_bits), _decode_bits(C_bits)
    lse_b, live_b, _, _ = _brute_filtered(E, C, y, np.ones(len(y)), eps, Bn, Bv)
    if rows_per_block is not None:
        monkeypatch.setattr(oracle, "_rows_per_block", lambda V, budget_elems=0: rows_per_block)
    live = oracle.tile_live_map(E_bits, C_bits, y, lse_b, IGN, eps, tile=(Bn, Bv))
    assert live.shape == live_b.shape == (7, 7)
    assert (live == live_b).all()
    assert 0 < live.sum() < live.size


@pytest.mark.parametrize("mutation", ["scaled_difference", "rows_shifted", "columns_shifted"])
def test_tile_live_map_pin_catches_planted_mistakes(monkeypatch, mutation):
    E_bits, C_bits, y, Bn, Bv = _tile_map_case()
    E, C = _decode_bits(E_bits), _decode_bits(C_bits)
    eps = 0.03
    lse_b, live_b, _, _ = _brute_filtered(E, C, y, np.ones(len(y)), eps, Bn, Bv)
    real_sg = oracle.softmax_grad_f64
    real_map = oracle.tile_live_map_f64
    if mutation == "scaled_difference":     # liveness decided on dloss-scaled entries (dloss = 0.3)
        monkeypatch.setattr(oracle, "softmax_grad_f64",
                            lambda z, lse, yy, dl, ign: tuple(x * (0.3 if k else 1.0)
                                                               for k, x in enumerate(real_sg(z, lse, yy, dl, ign))))
    elif mutation == "rows_shifted":        # tile rows anchored one token late
        monkeypatch.setattr(oracle, "tile_live_map_f64",
                            lambda Dm, r0, bn, bv, e: real_map(np.vstack([np.zeros((1, Dm.shape[1])), Dm])[:-1],
                                                               r0, bn, bv, e))
    elif mutation == "columns_shifted":     # vocabulary tiles anchored one column late
        monkeypatch.setattr(oracle, "tile_live_map_f64",
                            lambda Dm, r0, bn, bv, e: real_map(np.hstack([np.zeros((Dm.shape[0], 1)), Dm])[:, :-1],
                                                               r0, bn, bv, e))
    live = oracle.tile_live_map(E_bits, C_bits, y, lse_b, IGN, eps, tile=(Bn, Bv))
    assert live.shape != live_b.shape or not (live == live_b).all(), f"{mutation} went unnoticed"


def test_element_filter_defaults_and_keeps_only_large_entries():
    # the default filter works element by element: the filtered G equals the
    # exact G with every |P - onehot| < eps entry set to zero
    rng = np.random.default_rng(13)
    N, D, V = 6, 4, 9
    E = rng.standard_normal((N, D))
    C = rng.standard_normal((V, D))
    y = rng.integers(0, V, N)
    y[2] = IGN
    dloss = rng.random(N) + 0.5
    _, lse = oracle.forward_f64(E, C, y, IGN)
    eps = 0.05
    z = E @ C.T
    P = np.exp(z - lse[:, None])
    Dm = P.copy()
    for i in range(N):
        if y[i] == IGN:
            Dm[i] = 0.0
        else:
            Dm[i, y[i]] -= 1.0
    G = np.where(np.abs(Dm) >= eps, Dm, 0.0) * dloss[:, None]
    assert 0 < (np.abs(Dm) >= eps).sum() < Dm.size - N   # the case really drops entries
    dE, dC = oracle.backward_f64(E, C, y, lse, dloss, IGN, filter_eps=eps)
    np.testing.assert_allclose(dE, G @ C, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(dC, G.T @ E, rtol=1e-12, atol=1e-15)


def test_sampled_backward_matches_full():
    w = synth.TINY.with_sizes(N=300, V=1000, D=64)
    inp = synth.make_inputs(w)
    E, C, y = inp["E"], inp["C"], inp["y"]
    y = y.copy(); y[[3, 200]] = IGN
    dloss = synth.random_dloss(11, w.N)
    loss, lse = oracle.forward(E, C, y, IGN)
    loss_s, lse_s = oracle.forward(E, C, y, IGN, rows=[5, 299, 3])
    np.testing.assert_allclose(loss_s, loss[[5, 299, 3]], rtol=1e-14)
    for eps, tile in ((0.0, (128, 256)), (2e-3, (128, 256)), (1e-3, (64, 128)), (1e-3, (1, 1)), (3e-4, (1, 1))):
        dE, dC = oracle.backward(E, C, y, lse, dloss, IGN, filter_eps=eps, tile=tile)
        rE = [0, 129, 299, 3]
        rC = [0, 255, 256, 999, int(y[7])]
        sE, sC = oracle.backward_sampled(E, C, y, lse, dloss, IGN, rE, rC, filter_eps=eps, tile=tile)
        np.testing.assert_allclose(sE, dE[rE], rtol=1e-11, atol=1e-15)
        np.testing.assert_allclose(sC, dC[rC], rtol=1e-11, atol=1e-15)


# --------------------------------------------------------------------------
# planted mistakes: the pins above must catch each one
# --------------------------------------------------------------------------

def _run_pins():
    """Run a compact subset of the pins; return True if all pass."""
    try:
        test_worked_example_fixture()
        test_central_finite_differences()
        test_zero_classifier_gives_log_V(7)
        test_gradient_identities()
        return True
    except AssertionError:
        return False


@pytest.mark.parametrize("mutation", ["transposed_dC", "dropped_onehot", "sign_flip", "no_dloss",
                                      "lse_without_max_shift_back", "wrong_label_column"])
def test_planted_mistakes_are_caught(monkeypatch, mutation):
    assert _run_pins()
    real_sg = oracle.softmax_grad_f64
    real_fw = oracle.forward_f64
    real_bw = oracle.backward_f64
    if mutation == "dropped_onehot":
        def sg(z, lse, y, dloss, ign):
            P = np.exp(z - lse[:, None]); Dm = P.copy()
            Dm[y == ign] = 0.0
            return P, Dm, Dm * dloss[:, None]
        monkeypatch.setattr(oracle, "softmax_grad_f64", sg)
    elif mutation == "sign_flip":
        def sg(z, lse, y, dloss, ign):
            P, Dm, G = real_sg(z, lse, y, dloss, ign)
            return P, -Dm, -G
        monkeypatch.setattr(oracle, "softmax_grad_f64", sg)
    elif mutation == "no_dloss":
        def sg(z, lse, y, dloss, ign):
            return real_sg(z, lse, y, np.ones_like(dloss), ign)
        monkeypatch.setattr(oracle, "softmax_grad_f64", sg)
    elif mutation == "transposed_dC":
        def bw(E, C, y, lse, dloss, ign, *a, **k):
            dE, dC = real_bw(E, C, y, lse, dloss, ign, *a, **k)
            return dE, dC[::-1].copy()
        monkeypatch.setattr(oracle, "backward_f64", bw)
    elif mutation == "lse_without_max_shift_back":
        monkeypatch.setattr(oracle, "_lse_of_rows",
                            lambda z: np.log(np.exp(z - z.max(1)[:, None]).sum(1)))
    elif mutation == "wrong_label_column":
        def fw(E, C, y, ign, rows=None):
            yy = np.where(y == ign, y, (y + 1) % C.shape[0])
            return real_fw(E, C, yy, ign, rows)
        monkeypatch.setattr(oracle, "forward_f64", fw)
    assert not _run_pins(), f"planted mistake {mutation} went unnoticed"
