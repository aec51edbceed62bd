"""Pins of the decode-step oracle (paged attention with the scores folded in; ActKV Dissected, Component 3)
against library routines and closed forms, plus planted mistakes."""
import math

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

from oracle import decode as od


def _case(rng, G=4, n=300, D=64):
    q = rng.standard_normal((G, D))
    k = rng.standard_normal((n, D))
    v = rng.standard_normal((n, D))
    pos = rng.permutation(n + 40)[:n]
    return q, k, v, pos


def test_output_and_lse_match_scipy():
    """The output is scipy's softmax over the visible keys times V; the LSE is scipy's logsumexp."""
    rng = np.random.default_rng(5)
    q, k, v, pos = _case(rng)
    qpos = int(np.sort(pos)[200])                  # about two thirds of the keys visible
    out, lse, inc = od.decode_step(q, k, v, qpos, pos)
    vis = pos <= qpos
    l = (q @ k[vis].T) / math.sqrt(q.shape[1])
    assert np.allclose(lse, logsumexp(l, axis=1), rtol=0, atol=1e-12)
    assert np.allclose(out, softmax(l, axis=1) @ v[vis], rtol=1e-12, atol=1e-12)
    assert np.all(inc[~vis] == 0)
    assert abs(inc.sum() - q.shape[0]) < 1e-12     # each head's probabilities sum to one


def test_dominant_key_and_uniform_keys():
    """One key far above the rest takes all the weight; identical keys share it equally (closed forms)."""
    D = 8
    q = np.ones((2, D))
    k = np.zeros((5, D))
    k[3] = 50.0                                     # logit 400/sqrt(8) above the others
    v = np.arange(5 * D, dtype=np.float64).reshape(5, D)
    out, lse, inc = od.decode_step(q, k, v, 10, np.arange(5))
    assert np.allclose(out, v[3][None, :], atol=1e-9)
    assert np.allclose(inc[3], 2.0) and np.allclose(np.delete(inc, 3), 0.0, atol=1e-9)
    k2 = np.tile(np.arange(D, dtype=np.float64), (6, 1))
    out2, lse2, inc2 = od.decode_step(q, k2, v[:5].tolist() + [v[0].tolist()], 99, np.arange(6))
    vv = np.array(v[:5].tolist() + [v[0].tolist()])
    assert np.allclose(out2, vv.mean(0)[None, :]) and np.allclose(inc2, 2.0 / 6)
    assert np.allclose(lse2, (q @ k2[0]) / math.sqrt(D) + math.log(6))


def test_no_visible_key():
    q, k, v, pos = _case(np.random.default_rng(6), n=10)
    out, lse, inc = od.decode_step(q, k, v, -1, pos)
    assert np.all(np.isneginf(lse)) and np.all(out == 0) and np.all(inc == 0)


def test_increment_agrees_with_the_scoring_oracle():
    """One decode query's score increment is the scoring step's per-query term: the decode oracle (output path)
    and the scoring oracle (exp(logit - lse) summed over the group) agree on the same query and LSE."""
    from oracle import path as op
    rng = np.random.default_rng(7)
    q, k, v, pos = _case(rng, G=3, n=250)
    qpos = int(np.sort(pos)[180])
    out, lse, inc = od.decode_step(q, k, v, qpos, pos)
    s = op.scores_from_lse(q[None], k, np.array([qpos]), pos, lse[:, None])
    assert np.allclose(inc, s, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("mistake", ["no_scale", "mask_reversed", "unnormalised"])
def test_planted_mistakes_are_caught(mistake, monkeypatch):
    from oracle import path as op
    orig_logits, orig_vis, orig_step = op.logits, op.visible, od.decode_step
    if mistake == "no_scale":
        monkeypatch.setattr(op, "logits", lambda q, k: orig_logits(q, k) * math.sqrt(np.asarray(q).shape[-1]))
    elif mistake == "mask_reversed":
        monkeypatch.setattr(op, "visible", lambda a, b: orig_vis(a, b) == False)  # noqa: E712
    else:
        def bad(q, k, v, qp, kp):
            out, lse, inc = orig_step(q, k, v, qp, kp)
            return out * np.exp(lse)[:, None], lse, inc
        monkeypatch.setattr(od, "decode_step", bad)
    failed = 0
    for pin in (test_output_and_lse_match_scipy, test_dominant_key_and_uniform_keys):
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed >= 1
