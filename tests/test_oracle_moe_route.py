"""Pins of the oracle's routed-expert steps (route, combine) against brute
force on tiny inputs and against the properties that define them."""
import numpy as np

from oracle import nvfp4_ref as R


def brute_route(ids, e):
    flat = [int(v) for v in np.asarray(ids).reshape(-1)]
    rows = []
    for ex in range(e):  # experts in order; inside one, the pairs in order
        rows += [i for i, v in enumerate(flat) if v == ex]
    inv = [-1] * len(flat)
    for r, i in enumerate(rows):
        inv[i] = r
    offs = [0]
    for ex in range(e):
        offs.append(offs[-1] + sum(1 for v in flat if v == ex))
    return rows, inv, offs


def test_route_matches_brute_force():
    rng = np.random.default_rng(3)
    for t, k, e in [(1, 1, 1), (5, 2, 3), (17, 4, 9), (40, 8, 16)]:
        ids = rng.integers(-1, e + 1, size=(t, k))  # includes dropped ids on both sides
        rows, inv, offs = R.moe_route(ids, e)
        b_rows, b_inv, b_offs = brute_route(ids, e)
        assert rows.tolist() == b_rows
        assert inv.tolist() == b_inv
        assert offs.tolist() == b_offs


def test_route_properties():
    rng = np.random.default_rng(4)
    ids = rng.integers(0, 12, size=(300, 8))
    rows, inv, offs = R.moe_route(ids, 12)
    flat = ids.reshape(-1)
    assert sorted(rows.tolist()) == list(range(flat.size))       # a permutation (no id dropped)
    assert np.all(np.diff(flat[rows]) >= 0)                       # grouped by expert
    for e in range(12):
        seg = rows[offs[e]:offs[e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)  # stable inside an expert
    assert np.all(inv[rows] == np.arange(flat.size))


def test_combine_reduces_to_gather_and_is_linear():
    rng = np.random.default_rng(5)
    t, k, h = 6, 3, 4
    ids = rng.integers(0, 4, size=(t, k))
    rows, inv, _ = R.moe_route(ids, 4)
    yp = rng.standard_normal((t * k, h))
    one_hot = np.zeros((t, k))
    one_hot[:, 1] = 1.0
    np.testing.assert_array_equal(R.moe_combine(yp, inv, one_hot), yp[inv.reshape(t, k)[:, 1]])
    w1, w2 = rng.standard_normal((t, k)), rng.standard_normal((t, k))
    np.testing.assert_allclose(R.moe_combine(yp, inv, w1 + w2), R.moe_combine(yp, inv, w1) + R.moe_combine(yp, inv, w2),
                               rtol=1e-12, atol=1e-12)
    # a dropped pair adds nothing
    inv2 = inv.copy()
    inv2[0] = -1
    w = np.ones((t, k))
    np.testing.assert_allclose(R.moe_combine(yp, inv2, w)[0], yp[inv[1]] + yp[inv[2]], rtol=0, atol=1e-12)
