"""Pins of the step-aware ranking oracle ("StepKV: Step-Aware KV Cache Compression for LLM Agents", abstract)
against a hand-worked example, limits, closed forms, brute force and planted mistakes."""
import json
import os

import numpy as np
import pytest

from oracle import stepkv as sk

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "stepkv_hand_example.json")


def _case(rng, n=400, steps=9, span=3000):
    start = np.concatenate([[0], np.sort(rng.choice(np.arange(1, span), steps - 1, replace=False))])
    pos = rng.choice(span, n, replace=False)
    s = rng.exponential(size=n) * (rng.random(n) < 0.8)
    return s, pos, start


def test_hand_example():
    g = json.load(open(GOLDEN))
    assert sk.step_of(g["slot_pos"], g["step_start"]).tolist() == g["steps"]
    assert np.allclose(sk.step_utility(g["scores"], g["slot_pos"], g["step_start"]), g["utility"], rtol=0, atol=1e-12)
    assert np.allclose(sk.combined_scores(g["scores"], g["slot_pos"], g["step_start"], g["beta"]), g["combined"],
                       rtol=0, atol=1e-12)


def test_step_assignment_by_brute_force():
    rng = np.random.default_rng(1)
    s, pos, start = _case(rng)
    k = sk.step_of(pos, start)
    for p, kk in zip(pos, k):
        want = max(j for j in range(len(start)) if start[j] <= p)
        assert kk == want


def test_limits_of_beta():
    """beta = 0 ranks by token saliency alone; beta = 1 by the step mean alone (np.bincount means)."""
    rng = np.random.default_rng(2)
    s, pos, start = _case(rng)
    assert np.array_equal(sk.combined_scores(s, pos, start, 0.0), s)
    k = sk.step_of(pos, start)
    means = np.bincount(k, weights=s, minlength=len(start)) / np.maximum(np.bincount(k, minlength=len(start)), 1)
    assert np.allclose(sk.combined_scores(s, pos, start, 1.0), means[k], rtol=1e-14, atol=0)


@pytest.mark.parametrize("beta", [0.25, 0.5, 0.9])
def test_step_mean_of_the_combined_score_is_the_utility(beta):
    """Averaged over a step, (1 - beta) s + beta U gives U back (closed form), for every beta."""
    rng = np.random.default_rng(3)
    s, pos, start = _case(rng)
    c = sk.combined_scores(s, pos, start, beta)
    k = sk.step_of(pos, start)
    u = sk.step_utility(s, pos, start)
    for j in np.unique(k):
        assert abs(c[k == j].mean() - u[j]) < 1e-12 * max(1.0, abs(u[j]))


def test_slot_order_does_not_matter():
    """Compaction permutes slots: each entry's combined score follows the entry, not its slot."""
    rng = np.random.default_rng(4)
    s, pos, start = _case(rng)
    perm = rng.permutation(len(s))
    assert np.allclose(sk.combined_scores(s[perm], pos[perm], start, 0.5), sk.combined_scores(s, pos, start, 0.5)[perm],
                       rtol=1e-14, atol=0)


def test_empty_steps_have_zero_utility():
    u = sk.step_utility([1.0, 2.0], [0, 1], [0, 5, 9])
    assert u.tolist() == [1.5, 0.0, 0.0]


@pytest.mark.parametrize("mistake", ["sum_not_mean", "boundary_left", "beta_swapped", "global_mean"])
def test_planted_mistakes_are_caught(mistake, monkeypatch):
    orig_util, orig_step, orig_comb = sk.step_utility, sk.step_of, sk.combined_scores
    if mistake == "sum_not_mean":
        def util(scores, pos, start):
            k = orig_step(pos, start)
            return np.bincount(k, weights=np.asarray(scores, float), minlength=len(start))
        monkeypatch.setattr(sk, "step_utility", util)
    elif mistake == "boundary_left":
        monkeypatch.setattr(sk, "step_of", lambda pos, start: np.maximum(
            np.searchsorted(np.asarray(start), np.asarray(pos), side="left") - 1, 0))
    elif mistake == "beta_swapped":
        monkeypatch.setattr(sk, "combined_scores", lambda s, p, st, b: orig_comb(s, p, st, 1.0 - b))
    else:
        monkeypatch.setattr(sk, "step_utility", lambda scores, pos, start: np.full(len(start), np.mean(scores)))
    failed = 0
    for pin in (test_hand_example, test_step_assignment_by_brute_force, test_limits_of_beta):
        try:
            pin()
        except AssertionError:
            failed += 1
    for pin in (test_step_mean_of_the_combined_score_is_the_utility,):
        try:
            pin(0.25)
        except AssertionError:
            failed += 1
    assert failed >= 1
