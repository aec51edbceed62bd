"""Pins of the CPU oracle to what the pages and the mathematics fix (no GPU).

Each pin checks the oracle against something other than itself: a hand-derived
closed form, an identity, a library routine (scipy/numpy), brute-force
enumeration, or a constant printed in "ActKV Dissected" (golden fixtures with
their citations under tests/golden/).  ``test_planted_mistakes_are_caught``
plants plausible mistakes into the oracle and checks that some pin fails.
"""
import inspect
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special as sps

from oracle import path

INT32_MAX = 2**31 - 1


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------
# the pins, as plain functions of the oracle module (so a mutated oracle can be
# run through them)
# ---------------------------------------------------------------------------

def pin_constants(P, golden_dir):
    with open(os.path.join(golden_dir, "actkv_constants.json")) as f:
        c = json.load(f)["constants"]
    rp = P.RatchetParams()
    assert rp.top_k == c["confidence_top_k"]["value"]
    assert rp.window == c["pool_window"]["value"]
    assert rp.stride == c["pool_stride"]["value"]
    assert rp.grow_num / rp.grow_den == c["growth"]["value"]
    assert rp.init_budget == c["initial_budget"]["value"]
    assert rp.cap == c["budget_cap"]["value"]
    sig = inspect.signature(P.lrfu_update).parameters
    assert sig["lam"].default == c["lrfu_lambda"]["value"]
    assert sig["hit_mass"].default == c["hit_mass"]["value"]
    # "six doublings of headroom" between the initial budget and the cap
    assert round(math.log2(rp.cap / rp.init_budget)) == c["doublings_of_headroom"]["value"]


def _masked_logits_lib(q, k, q_pos, k_pos):
    """Independent formulation: per-pair dot products with numpy.dot, mask from the causal rule."""
    nq, G, D = q.shape
    n = k.shape[0]
    out = np.full((G, nq, n), -np.inf)
    for j in range(nq):
        for g in range(G):
            for i in range(n):
                if k_pos[i] <= q_pos[j]:
                    out[g, j, i] = float(np.dot(q[j, g], k[i])) / math.sqrt(D)
    return out


def pin_lse_matches_library(P):
    r = _rng(1)
    nq, G, D, n = 5, 3, 16, 40
    q = r.standard_normal((nq, G, D))
    k = r.standard_normal((n, D))
    k_pos = np.arange(n)
    q_pos = np.array([3, 10, 25, 39, INT32_MAX])
    lse = P.attention_lse(q, k, q_pos, k_pos)
    ref = _masked_logits_lib(q, k, q_pos, k_pos)
    np.testing.assert_allclose(lse, sps.logsumexp(ref, axis=2), rtol=0, atol=1e-12)
    # probabilities recovered from the LSE sum to one for every column
    p = np.exp(ref - lse[:, :, None])
    np.testing.assert_allclose(p.sum(axis=2), 1.0, rtol=0, atol=1e-12)


def pin_score_column_mass(P):
    """Sum over keys of the scores = number of (query, head) columns that see a key."""
    r = _rng(2)
    nq, G, D, n = 7, 4, 32, 64
    q = r.standard_normal((nq, G, D))
    k = r.standard_normal((n, D)) * 1.5
    k_pos = r.permutation(n)            # slot order is not position order
    q_pos = np.array([0, 5, 17, 30, 45, 63, INT32_MAX])
    lse = P.attention_lse(q, k, q_pos, k_pos)
    s = P.scores_from_lse(q, k, q_pos, k_pos, lse)
    assert abs(s.sum() - G * nq) < 1e-10
    # and each key's score is the softmax mass it received, computed by scipy
    ref = sps.softmax(_masked_logits_lib(q, k, q_pos, k_pos), axis=2).sum(axis=(0, 1))
    np.testing.assert_allclose(s, ref, rtol=1e-12, atol=1e-14)


def pin_score_hand_example(P):
    """D = 2.  Query a at position 1 sees keys 0, 1 with logits ln 3 and 0 -> p = 3/4, 1/4.
    Query b at position 2 sees keys 0, 1, 2 with logits 0, 0, 5 -> p = (1, 1, e^5) / (2 + e^5)."""
    r2 = math.sqrt(2.0)
    q = np.array([[[r2, 0.0]], [[0.0, r2]]])            # [nq=2, G=1, D=2]
    k = np.array([[math.log(3.0), 0.0], [0.0, 0.0], [5.0, 5.0]])
    k_pos = np.array([0, 1, 2])
    q_pos = np.array([1, 2])
    lse = P.attention_lse(q, k, q_pos, k_pos)
    np.testing.assert_allclose(lse[0], [math.log(4.0), math.log(2.0 + math.exp(5.0))], rtol=1e-14)
    s = P.scores_from_lse(q, k, q_pos, k_pos, lse)
    z = 2.0 + math.exp(5.0)
    np.testing.assert_allclose(s, [0.75 + 1 / z, 0.25 + 1 / z, math.exp(5.0) / z], rtol=1e-13)


def pin_equal_keys_uniform(P):
    """All keys equal: each column spreads 1/n_visible over the keys it sees."""
    D, n, G = 8, 20, 2
    k = np.tile(np.linspace(-1, 1, D), (n, 1))
    q = _rng(3).standard_normal((3, G, D))
    k_pos = np.arange(n)
    q_pos = np.array([4, 11, 19])
    s = P.scores_from_lse(q, k, q_pos, k_pos, P.attention_lse(q, k, q_pos, k_pos))
    expect = np.zeros(n)
    for qp in q_pos:
        expect[: qp + 1] += G / (qp + 1)
    np.testing.assert_allclose(s, expect, rtol=1e-12)


def pin_gqa_linearity(P):
    """A group's score is the sum of its heads' scores taken one head at a time."""
    r = _rng(4)
    q = r.standard_normal((6, 4, 16))
    k = r.standard_normal((30, 16))
    k_pos = np.arange(30)
    q_pos = np.array([2, 9, 9, 20, 29, INT32_MAX])
    lse = P.attention_lse(q, k, q_pos, k_pos)
    s = P.scores_from_lse(q, k, q_pos, k_pos, lse)
    per = sum(P.scores_from_lse(q[:, g:g + 1], k, q_pos, k_pos,
                                P.attention_lse(q[:, g:g + 1], k, q_pos, k_pos)) for g in range(4))
    np.testing.assert_allclose(s, per, rtol=1e-12)


def pin_mask_direction(P):
    """A query never gives mass to a key that comes after it."""
    r = _rng(5)
    q = r.standard_normal((1, 1, 8))
    k = r.standard_normal((10, 8))
    s = P.scores_from_lse(q, k, np.array([4]), np.arange(10), P.attention_lse(q, k, np.array([4]), np.arange(10)))
    assert np.all(s[5:] == 0.0) and np.all(s[:5] > 0.0)


def pin_lrfu_closed_form(P):
    """200 rounds of the update equal LRFU's closed form sum_t h_t 2^(-lam (r - t)) (Lee et al.'s F(x) = (1/2)^(lam x))."""
    r = _rng(6)
    n, rounds = 16, 200
    crf = np.zeros(n)
    hist = []
    for t in range(rounds):
        s = np.where(r.random(n) < 0.3, r.random(n), 0.0)
        hist.append(s)
        crf = P.lrfu_update(crf, s, np.arange(n), lam=0.5, hit_mass=1.0)
    expect = np.zeros(n)
    for t, h in enumerate(hist):
        expect += h * 0.5 ** (0.5 * (rounds - 1 - t))
    np.testing.assert_allclose(crf, expect, rtol=1e-12)


def pin_lrfu_special_cases(P):
    """lam = 0 counts hits (LFU); lam = 1 with binary hits: the latest hit outranks any older history (LRU)."""
    r = _rng(7)
    n = 12
    hits = r.random((30, n)) < 0.4
    lfu = np.zeros(n)
    lru = np.zeros(n)
    for h in hits:
        s = h.astype(float)
        lfu = P.lrfu_update(lfu, s, np.arange(n), lam=0.0, hit_mass=1.0, binary=True)
        lru = P.lrfu_update(lru, s, np.arange(n), lam=1.0, hit_mass=1.0, binary=True)
    lfu_ref = np.zeros(n)
    for h in hits:
        lfu_ref = np.where(h, lfu_ref + 1, lfu_ref)
    np.testing.assert_allclose(lfu, lfu_ref)
    last = hits[-1]
    if last.any() and (~last).any():
        assert lru[last].min() > lru[~last].max()


def _precedes(a, b, key, pos):
    return key[a] > key[b] or (key[a] == key[b] and (pos[a] < pos[b] or (pos[a] == pos[b] and a < b)))


def pin_gate_bruteforce(P):
    """The gate is a prefix of the rank order with the fewest entries whose mass reaches 0.9 of the total."""
    r = _rng(8)
    for trial in range(60):
        n = int(r.integers(1, 11))
        s = np.round(r.random(n) * 8) / 8 * (r.random(n) < 0.85)   # ties and zeros
        pos = r.permutation(n) * 3
        g = P.hit_gate(s, pos, 0.9)
        target = 0.9 * s.sum()
        best = None
        for size in range(0, n + 1):
            if any(s[list(c)].sum() >= target for c in itertools.combinations(range(n), size)):
                best = size
                break
        if target <= 0:
            best = 0
        assert g.sum() == best, (s, g)
        for a in np.flatnonzero(g):
            for b in np.flatnonzero(~g):
                assert _precedes(a, b, s, pos)
    assert P.hit_gate(np.array([0.1, 0.0, 0.5]), np.arange(3), 1.0).tolist() == [True, False, True]


def pin_select_bruteforce(P):
    """Exactly one kept set of size min(B, n) has every kept entry ahead of every dropped one; it is the oracle's."""
    r = _rng(9)
    for trial in range(60):
        n = int(r.integers(1, 12))
        crf = np.round(r.random(n) * 4) / 4
        pos = r.permutation(n) + 100
        B = int(r.integers(0, n + 2))
        keep = P.select_budget(crf, pos, B)
        size = min(B, n)
        ok = [c for c in itertools.combinations(range(n), size)
              if all(_precedes(a, b, crf, pos) for a in c for b in set(range(n)) - set(c))]
        assert len(ok) == 1
        assert set(np.flatnonzero(keep)) == set(ok[0])


def pin_select_protected(P):
    crf = np.array([0.9, 0.1, 0.8, 0.0, 0.7, 0.2])
    lab = np.array([0, 2, 0, 2, 1, 0])
    keep = P.select_budget(crf, np.arange(6), 3, lab, protect_mask=1 << 2)
    assert keep.tolist() == [True, True, False, True, False, False]


def pin_plan_golden(P, golden_dir):
    with open(os.path.join(golden_dir, "plan_hand_example.json")) as f:
        g = json.load(f)
    src, dst, m = P.plan_slots(np.array(g["keep"], dtype=bool), g["n"])
    assert m == g["m"] and src.tolist() == g["moves_src"] and dst.tolist() == g["moves_dst"]
    bt = np.array([7, 3], dtype=np.int64)
    pool = np.arange(8 * 4 * 2, dtype=np.float64).reshape(8, 4, 2)
    row = P.PagedRow(block_table=bt, n=g["n"], slot_pos=np.arange(8), slot_label=np.zeros(8, np.uint8))
    _, _, new, freed = P.compact_row(pool, pool, row, src, dst, m, g["page_size"])
    assert freed == [int(bt[p]) for p in g["freed_logical_pages"]]
    assert new.block_table.tolist() == [7, -1]


def _check_compaction(P, keep, n, page_size, r):
    keep = np.asarray(keep, dtype=bool)
    src, dst, m = P.plan_slots(keep, n)
    assert m == keep[:n].sum() and len(src) == len(dst)
    assert len(set(dst.tolist())) == len(dst) and len(set(src.tolist())) == len(src)
    assert not set(dst.tolist()) & set(src.tolist())
    assert all(d < m and not keep[d] for d in dst) and all(s_ >= m and keep[s_] for s_ in src)
    assert list(src) == sorted(src) and list(dst) == sorted(dst)
    P_ = page_size
    npg = -(-n // P_) + 1
    bt = r.permutation(3 * npg)[:npg]
    pool_k = r.integers(0, 2**16, size=(3 * npg, P_, 4)).astype(np.uint16)
    pool_v = r.integers(0, 2**16, size=(3 * npg, P_, 4)).astype(np.uint16)
    pos = r.permutation(n + 5)[: npg * P_ if npg * P_ <= n + 5 else n + 5]
    pos = np.concatenate([pos, np.zeros(max(0, npg * P_ - len(pos)), dtype=pos.dtype)])
    row = P.PagedRow(block_table=bt.copy(), n=n, slot_pos=pos.copy(), slot_label=(pos % 3).astype(np.uint8))
    k2, v2, new, freed = P.compact_row(pool_k, pool_v, row, src, dst, m, P_)
    # slots [0, m) hold exactly the kept entries (bytes travel with their token position)
    def items(kp, vp, b, p, idx):
        return sorted((int(p[i]), kp[b[i // P_], i % P_].tobytes(), vp[b[i // P_], i % P_].tobytes()) for i in idx)
    before = items(pool_k, pool_v, bt, pos, np.flatnonzero(keep[:n]))
    after = items(k2, v2, np.where(new.block_table < 0, bt, new.block_table), new.slot_pos, range(m))
    assert before == after
    # stayed entries untouched; freed = ceil(n/P) - ceil(m/P) pages, in ascending logical order
    for i in range(m):
        if keep[i]:
            assert new.slot_pos[i] == pos[i]
    assert len(freed) == -(-n // P_) - (-(-m // P_))
    assert freed == [int(bt[p]) for p in range(-(-m // P_), -(-n // P_))]
    assert np.all(new.block_table[-(-m // P_):-(-n // P_)] == -1)
    assert new.n == m


def pin_plan_exhaustive(P):
    r = _rng(10)
    n = 16
    for mask in range(1 << n):
        keep = np.array([(mask >> i) & 1 for i in range(n)], dtype=bool)
        if mask % 97 == 0:
            _check_compaction(P, keep, n, 4, r)
        else:
            src, dst, m = P.plan_slots(keep, n)
            assert len(src) == len(dst) == int((~keep[:m]).sum())


def pin_plan_random_large(P):
    r = _rng(11)
    for n in (1, 15, 16, 17, 257, 1000, 4096):
        for frac in (0.0, 0.1, 0.6, 1.0):
            keep = r.random(n) < frac
            _check_compaction(P, keep, n, 16, r)


def pin_confidence(P):
    V = 128256
    assert abs(P.token_confidence(np.full(V, 3.25)) - math.log(V)) < 1e-12
    a = 1e-4
    z = a * np.arange(V)
    lse = a * V + math.log(-math.expm1(-a * V)) - math.log(math.expm1(a))    # log((e^{aV}-1)/(e^a-1))
    top = a * (V - 1 - 9.5)                                                  # mean of the 20 largest
    assert abs(P.token_confidence(z) - (lse - top)) < 1e-9
    # top-20 tokens at b, rest at 0: c = log(20 + (V - 20) e^-b)
    zz = np.zeros(V)
    zz[:20] = 2.0
    assert abs(P.token_confidence(zz) - math.log(20 + (V - 20) * math.exp(-2.0))) < 1e-12


def pin_min_pool(P):
    c = [1.0] * 200
    c[100] = -5.0
    y = P.min_pool(c, 64, 8)
    assert len(y) == (200 - 64) // 8 + 1
    assert [j for j, v in enumerate(y) if v == -5.0] == list(range(5, 13))
    # a dip at the last step of window 1 (8 * 1 + 63 = 71) is seen by windows 1..8
    c = [1.0] * 200
    c[71] = -5.0
    assert [j for j, v in enumerate(P.min_pool(c, 64, 8)) if v == -5.0] == list(range(1, 9))


def pin_ols(P):
    r = _rng(12)
    for _ in range(20):
        x = np.arange(int(r.integers(2, 40))) + int(r.integers(0, 1000))
        y = r.standard_normal(len(x)) + 0.01 * x
        assert abs(P.ols_slope(x, y) - np.polyfit(x, y, 1)[0]) < 1e-9


def pin_budget_sequence(P, golden_dir):
    with open(os.path.join(golden_dir, "ratchet_budget_sequence.json")) as f:
        seq = json.load(f)["sequence"]
    b = [seq[0]]
    for _ in range(len(seq) - 1):
        b.append(P.grow(b[-1]))
    assert b == seq


def pin_ratchet_rounds(P):
    """Constant confidence never grows the budget; a steady decline grows it at the first fit, once per round."""
    V = 4096
    flat = P.Ratchet(params=P.RatchetParams())
    for _ in range(6):
        flat.round(np.zeros((64, V)))
    assert flat.budget == 512 and flat.expansions == 0
    dec = P.Ratchet(params=P.RatchetParams())
    budgets = []
    for rd in range(6):
        steps = np.zeros((64, V))
        for t in range(64):
            steps[t, :20] = 0.05 * (64 * rd + t)       # c_t = log(20 + (V-20) e^-b_t) falls as b_t grows
        budgets.append(dec.round(steps))
    # round 0: one pooled point (no fit); round 1: 9 points -> grow; round 2: 1 new point -> none; round 3: grow
    assert budgets == [512, 896, 896, 1568, 1568, 2744]
    assert all(b2 >= b1 for b1, b2 in zip(budgets, budgets[1:]))


PINS = [pin_lse_matches_library, pin_score_column_mass, pin_score_hand_example, pin_equal_keys_uniform,
        pin_gqa_linearity, pin_mask_direction, pin_lrfu_closed_form, pin_lrfu_special_cases,
        pin_gate_bruteforce, pin_select_bruteforce, pin_select_protected, pin_plan_exhaustive,
        pin_plan_random_large, pin_confidence, pin_min_pool, pin_ols, pin_ratchet_rounds]
PINS_GOLDEN = [pin_constants, pin_plan_golden, pin_budget_sequence]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(path)


@pytest.mark.parametrize("pin", PINS_GOLDEN, ids=lambda f: f.__name__)
def test_pin_golden(pin, golden_dir):
    pin(path, golden_dir)


# ---------------------------------------------------------------------------
# planted mistakes: each mutation of the oracle must make at least one pin fail
# ---------------------------------------------------------------------------

MUTATIONS = [
    ("visible", ">= np.asarray(k_pos", "<= np.asarray(k_pos"),                        # reversed causal mask
    ("logits", "/ math.sqrt(D)", "/ D"),                                              # wrong scale
    ("logits", '"jgd,id->gji", q, k', '"jgd,id->gji", q[:, ::-1], k'),                  # heads of the group swapped
    ("scores_from_lse", "lse[:, a:b, None]", "lse[::-1, a:b, None]"),                 # wrong head's LSE
    ("scores_from_lse", "np.exp(l - lse", "np.exp(l + lse"),                           # sign of the LSE
    ("attention_lse", "safe + np.log(ssum)", "np.log(ssum)"),                          # dropped max shift
    ("lrfu_update", "2.0 ** (-lam * dt)", "2.0 ** (lam * dt)"),                        # decay sign
    ("hit_gate", "side=\"left\")) + 1", "side=\"left\"))"),                             # off-by-one prefix
    ("rank_order", "np.asarray(pos, dtype=np.int64), -key", "-np.asarray(pos, dtype=np.int64), -key"),  # tie-break
    ("select_budget", "order[:room]", "order[:room + 1]"),                              # one too many kept
    ("plan_slots", "movers = [i for i in range(m, n) if keep[i]]", "movers = [i for i in range(n - 1, m - 1, -1) if keep[i]]"),
    ("compact_row", "first_free, end = -(-m // P), -(-row.n // P)", "first_free, end = m // P, -(-row.n // P)"),
    ("token_confidence", "np.sort(z)[-top_k:]", "np.sort(z)[-top_k + 1:]"),           # top-19
    ("min_pool", "c[stride * j: stride * j + window]", "c[stride * j: stride * j + window - 1]"),
    ("ols_slope", "((x - xb) ** 2).sum()", "((y - yb) ** 2).sum()"),
    ("grow", "budget * num // den", "-(-budget * num // den)"),                        # ceil instead of floor
]


def _run_all_pins(P, golden_dir):
    failed = []
    for pin in PINS:
        try:
            pin(P)
        except Exception:
            failed.append(pin.__name__)
    for pin in PINS_GOLDEN:
        try:
            pin(P, golden_dir)
        except Exception:
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("mut", MUTATIONS, ids=lambda m: m[0] + ":" + m[2][:24])
def test_planted_mistakes_are_caught(mut, monkeypatch, golden_dir):
    name, old, new = mut
    src = inspect.getsource(getattr(path, name))
    assert old in src, f"mutation anchor not found in {name}"
    ns = dict(vars(path))
    exec(compile(src.replace(old, new, 1), f"<mutant {name}>", "exec"), ns)
    monkeypatch.setattr(path, name, ns[name])
    # functions defined in the exec'd namespace look names up there; point them at the module
    for k, v in vars(path).items():
        if callable(v) and getattr(v, "__module__", None) == path.__name__:
            ns[k] = getattr(path, k)
    failed = _run_all_pins(path, golden_dir)
    assert failed, f"planted mistake in {name} was not caught by any pin"
