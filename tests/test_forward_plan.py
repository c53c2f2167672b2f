"""Host-side launch planning of the forward (no GPU needed): how many
vocabulary splits, raster groups and CTAs `cce_forward` chooses, for a GPU
with a given number of SMs, under both unit orders of the CTA-pair kernel."""
import ctypes

import pytest

from linear_cross_entropy_05_b200 import synth

SMS = 148   # B200
BN = 256


def _plan(L, N, D, V, sms=SMS):
    return L.cce_debug_forward_plan(N, D, V, sms)


def _shapes():
    out = [(w.name, w.N, w.D, w.V) for w in synth.WORKLOADS.values()]
    out += [(f"sweep-N{n}", n, synth.SWEEP.D, synth.SWEEP.V) for n in synth.SWEEP_NS]
    out += [("small-case", 2048, 2304, 32768), ("one-tile", 300, 64, 200)]
    return out


@pytest.fixture
def L():
    import linear_cross_entropy_05_b200 as L
    yield L
    L.cce_debug_set_forward_order(1)
    L.cce_debug_set_forward_schedule(0, 0, 0, 0)
    L.cce_debug_set_forward_variant(1)


def _max_pair_tiles(n_mblk, n_vtile, s, workers, group_m):
    # units dealt round-robin (unit u to worker u % workers), units ordered
    # split-major inside raster groups of group_m token blocks
    load = [0] * workers
    u = 0
    for g0 in range(0, n_mblk, group_m):
        gm = min(group_m, n_mblk - g0)
        for r in range(s):
            tiles = (r + 1) * n_vtile // s - r * n_vtile // s
            for _ in range(gm):
                load[u % workers] += tiles
                u += 1
    return max(load)


@pytest.mark.parametrize("name,N,D,V", _shapes(), ids=[s[0] for s in _shapes()])
def test_two_queue_plan_takes_short_units_over_the_balanced_floor(L, name, N, D, V):
    p = _plan(L, N, D, V)
    assert p["pair"]
    assert p["n_mblk"] == -(-N // 256) and p["n_vtile"] == -(-V // BN)
    s = p["n_split"]
    assert 1 <= s <= min(128, p["n_vtile"])
    # units of at most ~8 vocabulary tiles, unless 128 splits (or one split
    # per tile) is the limit
    assert -(-p["n_vtile"] // s) <= 8 or s == 128 or s == p["n_vtile"]
    # the split count of the round-robin order (chosen for balance) is the floor
    L.cce_debug_set_forward_order(0)
    s_rr = _plan(L, N, D, V)["n_split"]
    L.cce_debug_set_forward_order(1)
    assert s >= min(s_rr, p["n_vtile"])
    # raster groups of ~24 MB of E rows (256-row blocks of bf16) per L2 half
    block = 256 * D * 2
    assert 1 <= p["group_m"] <= p["n_mblk"]
    assert p["group_m"] == 1 or p["group_m"] * block <= (24 << 20)
    assert p["group_m"] == p["n_mblk"] or (p["group_m"] + 1) * block > (24 << 20)
    # one CTA pair per two SMs, fewer if there are fewer units
    assert p["grid"] == 2 * min(p["n_mblk"] * s, SMS // 2)


@pytest.mark.parametrize("name,N,D,V", _shapes()[:6], ids=[s[0] for s in _shapes()[:6]])
def test_round_robin_plan_minimises_the_most_loaded_pair(L, name, N, D, V):
    L.cce_debug_set_forward_order(0)
    p = _plan(L, N, D, V)
    s, workers = p["n_split"], SMS // 2
    assert 1 <= s <= 64
    assert p["group_m"] == 1 or p["group_m"] * 256 * D * 2 <= (48 << 20)
    if p["n_mblk"] * 64 <= (1 << 16):
        # exact: the fewest splits reaching the smallest most-loaded pair
        loads = {c: _max_pair_tiles(p["n_mblk"], p["n_vtile"], c, workers, p["group_m"])
                 for c in range(1, min(64, p["n_vtile"]) + 1)}
        best = min(loads.values())
        assert loads[s] == best and all(loads[c] > best for c in range(1, s))


def test_workloads_plan_as_measured(L):
    # the split counts the measured DRAM traffic and times were taken with
    assert _plan(L, 8192, 2304, 256000)["n_split"] == 125
    assert _plan(L, 16384, 4096, 128256)["n_split"] == 63
    assert _plan(L, 65536, 2048, 262144)["n_split"] == 128
    assert _plan(L, 2048, 2304, 32768)["n_split"] == 64
    L.cce_debug_set_forward_order(0)
    assert _plan(L, 8192, 2304, 256000)["n_split"] == 37


def test_knobs_and_the_single_cta_kernel(L):
    L.cce_debug_set_forward_schedule(40, 4, 0, 0)
    p = _plan(L, 8192, 2304, 256000)
    assert p["n_split"] == 40 and p["group_m"] == 4
    L.cce_debug_set_forward_schedule(0, 0, 0, 0)
    L.cce_debug_set_forward_variant(0)
    p = _plan(L, 8192, 2304, 256000)
    assert not p["pair"] and p["n_mblk"] == 64 and p["grid"] == min(64 * p["n_split"], SMS)
    assert p["n_split"] <= 64   # the two-queue order is a CTA-pair order


def test_invalid_plans_are_refused():
    from linear_cross_entropy_05_b200._native import load_library
    lib = load_library()
    out = (ctypes.c_int * 6)()
    assert lib.cce_debug_forward_plan(8192, 2304, 256000, 0, out) == -1
    assert lib.cce_debug_forward_plan(8192, 2304, 256000, 148, None) == -1
    assert lib.cce_debug_forward_plan(8192, 2303, 256000, 148, out) == -1   # D not a multiple of 8
    assert lib.cce_debug_forward_plan(0, 2304, 256000, 148, out) == -1
