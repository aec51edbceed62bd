"""Pins of the whole-cache oracle driver (``oracle.cache``) on a hand-built paged cache.

The cache: 2 sequences x 2 layers x 2 KV heads (8 rows), 4 query heads (GQA group 2), head_dim 4,
pages of 4 slots, rows of different lengths whose pages sit at randomly permuted places in a pool
with spare pages.  The test builds every row's logical content itself and places it in the pool,
so each pin compares the driver with something it does not compute:

* row ids follow row = (seq * layers + layer) * kv_heads + head (the C library's layout);
* the V pool holds an identity code per slot (row, logical slot), so a gather through the block
  table must return exactly the codes 0..n-1 of its own row;
* LSE and scores are brute force: one math.exp per (query, head, key) over the visible pairs
  ("ActKV Dissected", Component 3: probabilities are logits minus the LSE; Component 1: the
  score is the attention tallied over the query set);
* the LRFU values and keep masks equal the pinned per-row steps of ``oracle.path`` on the rows'
  logical inputs, with a different budget per sequence;
* compaction equals a single pass of plain slot copies in which every read sees the pool as it
  was before the pass, and the freed list is ordered by row, then by logical page ("ActKV
  Dissected", Component 3: one parallel copy pass, freed blocks returned to the scheduler).

``test_planted_mistakes_are_caught`` plants plausible mistakes in ``oracle.cache`` and requires
each one to fail a pin.
"""
import inspect
import math

import numpy as np
import pytest

from oracle import cache as ocache
from oracle import path as opath

S, L, HKV, HQ, D, P = 2, 2, 2, 4, 4, 4
G = HQ // HKV
ROWS = S * L * HKV
MAX_PAGES = 8
MAX_Q = 4


def _row_id(s, l, h):
    return (s * L + l) * HKV + h


def hand_cache(seed=11):
    """Logical rows, their placement in a permuted pool, and a query set (all host numpy)."""
    rng = np.random.default_rng(seed)
    n = np.array([3, 7, 16, 17, 22, 9, 31, 12], dtype=np.int64)
    pages_needed = [-(-int(x) // P) for x in n]
    num_pages = sum(pages_needed) + 5
    perm = rng.permutation(num_pages)
    bt = np.full((ROWS, MAX_PAGES), -1, dtype=np.int64)
    nxt = 0
    for r in range(ROWS):
        for p in range(pages_needed[r]):
            bt[r, p] = perm[nxt]
            nxt += 1
    spare = sorted(int(x) for x in perm[nxt:])
    k_logical = {r: rng.standard_normal((int(n[r]), D)) for r in range(ROWS)}
    # token positions: distinct, in a shuffled slot order (as after earlier compactions)
    pos = {r: rng.permutation(rng.choice(60, size=int(n[r]), replace=False)).astype(np.int64) for r in range(ROWS)}
    labels = {r: rng.integers(0, 3, size=int(n[r])).astype(np.uint8) for r in range(ROWS)}
    k_pool = rng.standard_normal((num_pages, P, D))          # spare and tail slots hold junk
    v_pool = np.full((num_pages, P, D), -1.0)
    slot_pos = np.full((ROWS, MAX_PAGES * P), -7, dtype=np.int64)
    slot_label = np.full((ROWS, MAX_PAGES * P), 9, dtype=np.uint8)
    for r in range(ROWS):
        for i in range(int(n[r])):
            pg, off = bt[r, i // P], i % P
            k_pool[pg, off] = k_logical[r][i]
            v_pool[pg, off] = [r, i, 0.0, 0.0]                 # identity code of the slot
            slot_pos[r, i] = pos[r][i]
            slot_label[r, i] = labels[r][i]
    num_q = np.array([3, 4], dtype=np.int64)
    q = rng.standard_normal((S, L, MAX_Q, HQ, D))
    q_pos = np.array([[25, 40, 59, 0], [10, 33, 47, 58]], dtype=np.int64)
    return dict(n=n, bt=bt, spare=spare, k_logical=k_logical, pos=pos, labels=labels, k_pool=k_pool,
                v_pool=v_pool, slot_pos=slot_pos, slot_label=slot_label, num_q=num_q, q=q, q_pos=q_pos,
                num_pages=num_pages)


def _geo(C):
    return C.Geometry(S, L, HKV, HQ, P)


def _brute_lse(c, s, l, hq):
    """log sum over visible keys of exp(q.k / sqrt(D)) for every query of head hq (fp64, -inf if none)."""
    h = hq // G
    r = _row_id(s, l, h)
    out = []
    for j in range(int(c["num_q"][s])):
        terms = [float(np.dot(c["q"][s, l, j, hq], c["k_logical"][r][i])) / math.sqrt(D)
                 for i in range(int(c["n"][r])) if c["pos"][r][i] <= c["q_pos"][s, j]]
        if not terms:
            out.append(-math.inf)
            continue
        mx = max(terms)
        out.append(mx + math.log(sum(math.exp(t - mx) for t in terms)))
    return out


def _brute_scores(c, r, lse):
    s, rem = divmod(r, L * HKV)
    l, h = divmod(rem, HKV)
    sc = np.zeros(int(c["n"][r]))
    for i in range(int(c["n"][r])):
        for j in range(int(c["num_q"][s])):
            if c["pos"][r][i] > c["q_pos"][s, j]:
                continue
            for hq in range(h * G, (h + 1) * G):
                lg = float(np.dot(c["q"][s, l, j, hq], c["k_logical"][r][i])) / math.sqrt(D)
                sc[i] += math.exp(lg - lse[s, l, hq, j])
    return sc


# ---------------------------------------------------------------------------
# pins, as functions of the cache module (so that a mutated module can be run through them)
# ---------------------------------------------------------------------------

def pin_coords(C):
    geo = _geo(C)
    assert geo.rows == ROWS and geo.group == G
    for s in range(S):
        for l in range(L):
            for h in range(HKV):
                assert tuple(int(x) for x in geo.coords(_row_id(s, l, h))) == (s, l, h)


def pin_gather(C):
    c = hand_cache()
    for r in range(ROWS):
        n = int(c["n"][r])
        got = C.gather_row(c["v_pool"], c["bt"][r], n, P)
        want = np.array([[r, i, 0.0, 0.0] for i in range(n)])
        assert np.array_equal(got, want), f"row {r}"
        assert np.array_equal(C.gather_row(c["k_pool"], c["bt"][r], n, P), c["k_logical"][r])


def pin_lse_bruteforce(C):
    c = hand_cache()
    geo = _geo(C)
    lse = C.lse_cache(geo, c["k_pool"], c["bt"], c["n"], c["slot_pos"], c["q"], c["q_pos"], c["num_q"], MAX_Q)
    assert lse.shape == (S, L, HQ, MAX_Q)
    for s in range(S):
        for l in range(L):
            for hq in range(HQ):
                want = _brute_lse(c, s, l, hq)
                nq = int(c["num_q"][s])
                np.testing.assert_allclose(lse[s, l, hq, :nq], want, rtol=1e-12, atol=1e-12)
                assert np.all(lse[s, l, hq, nq:] == -np.inf)


def pin_scores_bruteforce(C):
    c = hand_cache()
    geo = _geo(C)
    lse = C.lse_cache(geo, c["k_pool"], c["bt"], c["n"], c["slot_pos"], c["q"], c["q_pos"], c["num_q"], MAX_Q)
    lse32 = lse.astype(np.float32).astype(np.float64)
    sc = C.score_cache(geo, c["k_pool"], c["bt"], c["n"], c["slot_pos"], c["q"], lse32, c["q_pos"], c["num_q"])
    for r in range(ROWS):
        n = int(c["n"][r])
        np.testing.assert_allclose(sc[r, :n], _brute_scores(c, r, lse32), rtol=1e-12, atol=1e-15)
        assert np.all(sc[r, n:] == 0.0)
    # a sampled subset of rows gives the same values on those rows
    sub = C.score_cache(geo, c["k_pool"], c["bt"], c["n"], c["slot_pos"], c["q"], lse32, c["q_pos"], c["num_q"],
                        rows=[6, 1])
    assert np.array_equal(sub[[6, 1]], sc[[6, 1]])


def pin_lrfu_select_rows(C):
    c = hand_cache()
    geo = _geo(C)
    rng = np.random.default_rng(5)
    scores = np.zeros((ROWS, MAX_PAGES * P))
    crf0 = np.zeros((ROWS, MAX_PAGES * P))
    for r in range(ROWS):
        n = int(c["n"][r])
        scores[r, :n] = rng.exponential(size=n)
        crf0[r, :n] = rng.exponential(size=n)
    crf0[:, -1] = 123.0                      # beyond every row's length: left as it was
    crf1, hits = C.lrfu_cache(geo, scores, crf0, c["n"], c["slot_pos"], 0.5, 0.9)
    budget = [5, 11]
    keep, kept = C.select_cache(geo, crf1, c["n"], c["slot_pos"], c["slot_label"], budget)
    keep_p, _ = C.select_cache(geo, crf1, c["n"], c["slot_pos"], c["slot_label"], budget, protect_mask=0b100)
    for r in range(ROWS):
        n = int(c["n"][r])
        s = r // (L * HKV)
        want = opath.lrfu_update(crf0[r, :n], scores[r, :n], c["pos"][r], 0.5, 0.9)
        assert np.array_equal(crf1[r, :n], want), f"row {r}"
        assert np.array_equal(hits[r, :n], opath.hit_gate(scores[r, :n], c["pos"][r], 0.9))
        assert crf1[r, -1] == 123.0
        k = opath.select_budget(want, c["pos"][r], budget[s])
        assert np.array_equal(keep[r, :n].astype(bool), k) and int(kept[r]) == min(budget[s], n)
        assert not keep[r, n:].any()
        kp = opath.select_budget(want, c["pos"][r], budget[s], c["labels"][r], 0b100)
        assert np.array_equal(keep_p[r, :n].astype(bool), kp)


def _random_keeps(c, seed):
    rng = np.random.default_rng(seed)
    keep = np.zeros((ROWS, MAX_PAGES * P), dtype=np.uint8)
    for r in range(ROWS):
        n = int(c["n"][r])
        keep[r, :n] = rng.random(n) < (0.15 + 0.1 * r)
    return keep


def pin_plan_rows(C):
    c = hand_cache()
    geo = _geo(C)
    keep = _random_keeps(c, 3)
    plans = C.plan_cache(geo, keep, c["n"])
    assert sorted(plans) == list(range(ROWS))
    for r in range(ROWS):
        n = int(c["n"][r])
        m = int(keep[r, :n].sum())
        holes = [i for i in range(m) if not keep[r, i]]
        movers = [i for i in range(m, n) if keep[r, i]]
        src, dst, mm = plans[r]
        assert mm == m and list(src) == movers and list(dst) == holes


def pin_compact_single_pass(C):
    c = hand_cache()
    geo = _geo(C)
    keep = _random_keeps(c, 4)
    crf = np.random.default_rng(9).random((ROWS, MAX_PAGES * P))
    plans = C.plan_cache(geo, keep, c["n"])
    k2, v2, bt2, rl2, sp2, sl2, cr2, freed = C.compact_cache(geo, c["k_pool"], c["v_pool"], c["bt"], c["n"],
                                                             c["slot_pos"], c["slot_label"], crf, plans)
    # the single pass written out: every copy reads the pool as it was before the pass
    kw, vw = c["k_pool"].copy(), c["v_pool"].copy()
    sp_w, sl_w, cr_w = c["slot_pos"].copy(), c["slot_label"].copy(), crf.copy()
    bt_w = c["bt"].copy()
    freed_w = []
    for r in range(ROWS):
        n = int(c["n"][r])
        m = int(keep[r, :n].sum())
        holes = [i for i in range(m) if not keep[r, i]]
        movers = [i for i in range(m, n) if keep[r, i]]
        for a, b in zip(movers, holes):
            kw[c["bt"][r, b // P], b % P] = c["k_pool"][c["bt"][r, a // P], a % P]
            vw[c["bt"][r, b // P], b % P] = c["v_pool"][c["bt"][r, a // P], a % P]
            sp_w[r, b], sl_w[r, b], cr_w[r, b] = c["slot_pos"][r, a], c["slot_label"][r, a], crf[r, a]
        for p in range(-(-m // P), -(-n // P)):
            freed_w.append(int(c["bt"][r, p]))
            bt_w[r, p] = -1
        # the row's kept entries are exactly the slots [0, m) after the pass, each once
        codes = sorted(int(x) for x in C.gather_row(v2, bt2[r], m, P)[:, 1]) if m else []
        assert codes == [i for i in range(n) if keep[r, i]], f"row {r}"
        assert int(rl2[r]) == m
    assert np.array_equal(k2, kw) and np.array_equal(v2, vw)
    assert np.array_equal(bt2, bt_w) and np.array_equal(sp2, sp_w) and np.array_equal(sl2, sl_w)
    assert np.array_equal(cr2, cr_w)
    assert list(freed) == freed_w
    # pages of no row are untouched, and the freed count per row is ceil(n/P) - ceil(m/P)
    assert np.array_equal(k2[c["spare"]], c["k_pool"][c["spare"]])
    assert len(freed) == sum(-(-int(c["n"][r]) // P) - (-(-int(keep[r].sum()) // P)) for r in range(ROWS))


PINS = [pin_coords, pin_gather, pin_lse_bruteforce, pin_scores_bruteforce, pin_lrfu_select_rows, pin_plan_rows,
        pin_compact_single_pass]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(ocache)


def test_hand_cache_is_what_the_pins_assume():
    """The layout really is permuted and fragmented, and rows own disjoint pages."""
    c = hand_cache()
    used = c["bt"][c["bt"] >= 0]
    assert len(set(used.tolist())) == len(used)
    assert not np.array_equal(np.sort(used), used)
    assert len(c["spare"]) == 5
    assert any(c["pos"][r][i] > c["q_pos"][r // (L * HKV), 0] for r in range(ROWS) for i in range(int(c["n"][r])))


MUTATIONS = [
    ("Geometry", "return sl // self.num_layers, sl % self.num_layers, h",
     "return sl // self.num_layers, h, sl % self.num_layers"),                       # layer and head swapped
    ("gather_row", "pool[bt_row[i // page_size], i % page_size]",
     "pool[bt_row[i // page_size], (i + 1) % page_size]"),                           # page offset off by one
    ("row_queries", "q[s, l, :nq, h * G:(h + 1) * G, :]", "q[s, l, :nq, h:h + G, :]"),  # wrong head group
    ("lse_cache", "out[s, l, h * G:(h + 1) * G, :nq]", "out[s, l, h:h + G, :nq]"),  # LSE stored for the wrong heads
    ("score_cache", "slot_pos[r, :n], lse[s, l, h * G:(h + 1) * G, :nq]",
     "slot_pos[r, :n], lse[s, l, h * G:(h + 1) * G, ::-1][:, :nq]"),                # queries' LSE misaligned
    ("lrfu_cache", "lam, hit_mass, dt, binary", "hit_mass, lam, dt, binary"),        # parameters swapped
    ("select_cache", "s, _, _ = geo.coords(r)", "_, s, _ = geo.coords(r)"),          # another sequence's budget
    ("compact_cache", "for r in sorted(plans):", "for r in sorted(plans, reverse=True):"),  # freed list row order
    ("compact_cache", "cr[r] = new.crf", "pass"),                                     # CRF not moved with its entry
]


def _run_all_pins(C):
    failed = []
    for pin in PINS:
        try:
            pin(C)
        except Exception:
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("mut", MUTATIONS, ids=lambda m: m[0] + ":" + m[2][:28])
def test_planted_mistakes_are_caught(mut, monkeypatch):
    name, old, new = mut
    src = inspect.getsource(getattr(ocache, name))
    assert old in src, f"mutation anchor not found in {name}"
    ns = dict(vars(ocache))
    exec(compile(src.replace(old, new, 1), f"<mutant {name}>", "exec"), ns)
    monkeypatch.setattr(ocache, name, ns[name])
    for k, v in vars(ocache).items():
        if callable(v) and getattr(v, "__module__", None) == ocache.__name__:
            ns[k] = getattr(ocache, k)
    failed = _run_all_pins(ocache)
    assert failed, f"planted mistake in {name} was not caught by any pin"
