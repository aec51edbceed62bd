"""Pins of the beacon-query oracle (online k-means; BeaconKV, Key ideas) against facts that do not come
from the oracle itself: exact cluster means, fp64 sums, the tie and seeding rules, and planted mistakes."""
import numpy as np
import pytest

from oracle import beacon as ob


def _clusters(rng, centers, per, spread):
    pts, lab = [], []
    for i, ctr in enumerate(centers):
        pts.append(ctr + spread * rng.standard_normal((per, len(ctr))))
        lab += [i] * per
    return np.vstack(pts).astype(np.float32), np.array(lab)


def test_distances_match_fp64_sums():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((40, 64)).astype(np.float32)
    c = rng.standard_normal((7, 64)).astype(np.float32)
    d = ob.distances_f32(q, c)
    ref = ((q[:, None, :].astype(np.float64) - c[None, :, :]) ** 2).sum(-1)
    assert d.dtype == np.float32
    assert np.max(np.abs(d - ref) / ref) < 1e-5


def test_separated_clusters_give_their_means():
    """Four far-apart groups, seeded by one point of each: every point joins its own group and every beacon
    ends at the group's fp64 mean (to fp32 rounding)."""
    rng = np.random.default_rng(2)
    centers = np.array([[10, 0, 0], [0, 10, 0], [0, 0, 10], [-10, -10, -10]], dtype=np.float64)
    pts, lab = _clusters(rng, centers, 50, 0.3)
    seeds = pts[[0, 50, 100, 150]]
    rest = np.delete(pts, [0, 50, 100, 150], axis=0)
    rest_lab = np.delete(lab, [0, 50, 100, 150])
    c, n, a = ob.beacon_update(np.zeros((4, 3), np.float32), np.zeros(4, int), seeds)
    assert n.tolist() == [1, 1, 1, 1] and np.array_equal(c, seeds)
    c, n, a = ob.beacon_update(c, n, rest)
    assert np.array_equal(a, rest_lab)
    assert n.tolist() == [50, 50, 50, 50]
    for i in range(4):
        assert np.allclose(c[i], pts[lab == i].astype(np.float64).mean(0), rtol=0, atol=2e-5)


def test_running_mean_over_batches():
    """One beacon fed many batches holds the mean of all points ever fed (fp64 reference)."""
    rng = np.random.default_rng(3)
    c, n = np.zeros((1, 16), np.float32), np.zeros(1, int)
    seen = []
    for m in (1, 7, 30, 2, 61):
        q = (3.0 + rng.standard_normal((m, 16))).astype(np.float32)
        seen.append(q)
        c, n, a = ob.beacon_update(c, n, q)
        assert (a == 0).all()
    allq = np.vstack(seen).astype(np.float64)
    assert n[0] == len(allq)
    assert np.allclose(c[0], allq.mean(0), rtol=1e-5, atol=1e-5)


def test_ties_go_to_the_lower_beacon_and_idle_beacons_stay_exact():
    c = np.array([[1, 1], [1, 1], [5, 5]], np.float32)
    n = np.array([3, 3, 2])
    q = np.array([[1.5, 0.5], [0.5, 1.5], [1, 1]], np.float32)
    c2, n2, a = ob.beacon_update(c, n, q)
    assert a.tolist() == [0, 0, 0]
    assert n2.tolist() == [6, 3, 2]
    assert np.array_equal(c2[1], c[1]) and np.array_equal(c2[2], c[2])


def test_seeding_takes_the_first_queries_in_order():
    """Empty beacons 1 and 3 take queries 0 and 1; beacons with counts keep theirs."""
    c = np.array([[0, 0], [9, 9], [100, 0], [9, 9]], np.float32)
    n = np.array([2, 0, 1, 0])
    q = np.array([[50, 50], [-50, 50], [0.5, 0], [99, 1]], np.float32)
    c2, n2, a = ob.beacon_update(c, n, q)
    assert a.tolist() == [1, 3, 0, 2]
    assert np.array_equal(c2[1], q[0]) and np.array_equal(c2[3], q[1])
    assert n2.tolist() == [3, 1, 2, 1]


def test_fewer_queries_than_beacons_and_no_queries():
    c = np.zeros((4, 2), np.float32)
    n = np.zeros(4, int)
    c2, n2, a = ob.beacon_update(c, n, np.array([[1, 2]], np.float32))
    assert a.tolist() == [0] and n2.tolist() == [1, 0, 0, 0] and c2[0].tolist() == [1, 2]
    c3, n3, a3 = ob.beacon_update(c2, n2, np.zeros((0, 2), np.float32))
    assert len(a3) == 0 and np.array_equal(c3, c2) and np.array_equal(n3, n2)


@pytest.mark.parametrize("mistake", ["argmax", "drop_old_mass", "count_off_by_one", "tie_upper"])
def test_planted_mistakes_are_caught(mistake, monkeypatch):
    """Each plausible mistake, planted in the oracle, fails at least one pin above."""
    orig_update, orig_dist = ob.beacon_update, ob.distances_f32

    def bad_update(c, n, q):
        c0 = np.array(c, np.float32)
        n0 = np.array(n)
        if mistake == "argmax":
            monkeypatch.setattr(ob, "distances_f32", lambda q_, c_: -orig_dist(q_, c_))
            try:
                return orig_update(c0, n0, q)
            finally:
                monkeypatch.setattr(ob, "distances_f32", orig_dist)
        c2, n2, a = orig_update(c0, n0, q)
        if mistake == "drop_old_mass":
            for b in range(len(n0)):
                sel = a == b
                if sel.any():
                    c2[b] = q[sel].astype(np.float64).mean(0)
        elif mistake == "count_off_by_one":
            n2 = n2 + (n2 > 0)
        elif mistake == "tie_upper":
            d = orig_dist(q, c0)
            a = len(n0) - 1 - np.argmin(d[:, ::-1], axis=1)
        return c2, n2, a

    monkeypatch.setattr(ob, "beacon_update", bad_update)
    pins = [test_separated_clusters_give_their_means, test_running_mean_over_batches,
            test_ties_go_to_the_lower_beacon_and_idle_beacons_stay_exact, test_seeding_takes_the_first_queries_in_order,
            test_fewer_queries_than_beacons_and_no_queries]
    failed = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed >= 1
