"""Task order of the dense stripe backward (CCE_BWD_STRIPES), decoded on the
host by the library itself (no GPU): every task appears exactly once, and
every task comes after the tasks whose outputs it reads -- the property that
lets persistent CTA pairs take tasks in this order without deadlock:

* a dC tile task B(s, vt, dc) after every recompute task A(s, m2, vt);
* a dE tile task C(s, m2, dc) after every A(s, m2, vt) of its stripe;
* A(s, ...) after every B and C task of stripe s - nbuf (it overwrites
  their stripe buffer)."""
import pytest

END, A, B, C = -1, 0, 1, 2


@pytest.fixture(scope="module")
def lib():
    from linear_cross_entropy_05_b200 import build, _native
    build.build()
    return _native


PLANS = [
    # n_m2, n_vtile, n_dc, vt_per_s, nbuf
    (32, 1000, 9, 8, 3),        # Gemma-2-2B-shaped head, 8192 tokens
    (64, 594, 4, 8, 3),         # small-model head, one 16384-token launch
    (1, 1, 1, 8, 3),            # one tile
    (3, 17, 2, 8, 3),           # ragged last stripe
    (5, 16, 3, 8, 3),           # two full stripes
    (2, 9, 1, 8, 3),            # two stripes, the second of one tile
    (4, 40, 2, 8, 2),           # two buffers
    (7, 25, 5, 4, 3),
]


ORDERS = [(0, 4, 2), (1, 4, 2), (1, 1, 1), (1, 3, 5), (1, 64, 1)]   # (order, token blocks per group, lag)


@pytest.mark.parametrize("order", ORDERS, ids=[f"order{o}-g{g}-lag{l}" for o, g, l in ORDERS])
@pytest.mark.parametrize("plan", PLANS, ids=[str(p) for p in PLANS])
def test_stripe_schedule_is_complete_and_ordered(lib, plan, order):
    n_m2, n_vt, n_dc, vps, nbuf = plan
    tasks = lib.cce_debug_stripe_schedule(*plan, *order)
    n_s = -(-n_vt // vps)
    nbuf = min(nbuf, n_s)
    assert tasks[-1][0] == END
    body = [tuple(int(x) for x in t) for t in tasks[:-1]]
    assert all(t[0] in (A, B, C) for t in body)
    pos = {}
    for i, t in enumerate(body):
        assert t not in pos, f"task {t} twice"
        pos[t] = i

    def stripe_of(vt):
        return vt // vps

    want_A = {(A, stripe_of(vt), m2, vt) for m2 in range(n_m2) for vt in range(n_vt)}
    want_B = {(B, stripe_of(vt), vt, dc) for vt in range(n_vt) for dc in range(n_dc)}
    want_C = {(C, s, m2, dc) for s in range(n_s) for m2 in range(n_m2) for dc in range(n_dc)}
    assert set(pos) == want_A | want_B | want_C
    last_A_of_vt = {vt: max(pos[(A, stripe_of(vt), m2, vt)] for m2 in range(n_m2)) for vt in range(n_vt)}
    for (k, s, a, b), i in pos.items():
        if k == B:
            assert last_A_of_vt[a] < i
        elif k == C:
            for vt in range(s * vps, min(n_vt, (s + 1) * vps)):
                assert pos[(A, s, a, vt)] < i
        elif s >= nbuf:
            s0 = s - nbuf
            for vt in range(s0 * vps, min(n_vt, (s0 + 1) * vps)):
                for dc in range(n_dc):
                    assert pos[(B, s0, vt, dc)] < i
            for m2 in range(n_m2):
                for dc in range(n_dc):
                    assert pos[(C, s0, m2, dc)] < i
    # the deterministic mode sums each dE tile in stripe order
    for s in range(1, n_s):
        for m2 in range(n_m2):
            for dc in range(n_dc):
                assert pos[(C, s - 1, m2, dc)] < pos[(C, s, m2, dc)]


def test_stripe_schedule_rejects_bad_sizes(lib):
    from linear_cross_entropy_05_b200._native import CCEError
    with pytest.raises(CCEError):
        lib.cce_debug_stripe_schedule(0, 4, 1, 8, 3)
    with pytest.raises(CCEError):
        lib.cce_debug_stripe_schedule(4, 4, 1, 8, 3, 1, 4, 0)     # lag 0: a dE task right after its inputs
    from linear_cross_entropy_05_b200 import _native
    lib_c = _native.load_library()
    assert lib_c.cce_debug_set_stripe_order(2, 4, 2) == 1
    assert lib_c.cce_debug_set_stripe_order(1, 0, 2) == 1
    assert lib_c.cce_debug_set_stripe_order(1, 4, 2) == 0
    assert lib_c.cce_debug_set_stripe_order(0, 4, 2) == 0
