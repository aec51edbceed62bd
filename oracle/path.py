"""CPU oracle of the attention-guided eviction and compaction path (fp64, numpy).

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and the
CPU-baseline leg of the benchmark import this module.  The product path (the
CUDA library and its binding) never calls it, and it shares no code with the
CUDA side: it takes plain numpy arrays and returns plain numpy arrays.

Each function follows one step of the method as the pages state it, with the
plainest reading where they leave a step open.  Sources:

* "ActKV Dissected" (forum write-up of ActKV), sections Summary, Component 1
  (action-attention-guided eviction), Component 2 (budget follows hesitation),
  Component 3 (systems engineering) and Lineage.
* "BeaconKV Compresses KV Cache for Long-Reasoning Models with Beacon Queries",
  section Key ideas (beacon plus recent queries form the query set).

Parity status: every function here is pinned by the non-GPU tests against
closed forms, identities, library routines or brute force; none is
"parity unpinned".
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np

INT32_MAX = 2**31 - 1


# ----------------------------------------------------------------------------
# Step 1: attention probabilities recovered from the log-sum-exp
# ("ActKV Dissected", Component 3: softmax's log-sum-exp is a byproduct of paged
# attention, so per-block probabilities are the current query's logits minus the
# LSE; Component 1: each entry's score is the attention tallied over all action
# tokens).
# ----------------------------------------------------------------------------

def logits(q: np.ndarray, k: np.ndarray) -> np.ndarray:
    """Scaled dot products l[g, j, i] = q[j, g] . k[i] / sqrt(D).

    q: [nq, G, D] query vectors of one GQA group; k: [n, D] keys of the row.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    D = q.shape[-1]
    return np.einsum("jgd,id->gji", q, k, optimize=True) / math.sqrt(D)


def visible(q_pos: np.ndarray, k_pos: np.ndarray) -> np.ndarray:
    """Causal visibility v[j, i]: query j attends to key i iff pos(key) <= pos(query).

    A beacon query carries INT32_MAX and so sees every key.
    """
    return np.asarray(q_pos, dtype=np.int64)[:, None] >= np.asarray(k_pos, dtype=np.int64)[None, :]


def attention_lse(q: np.ndarray, k: np.ndarray, q_pos: np.ndarray, k_pos: np.ndarray,
                  chunk: int = 64) -> np.ndarray:
    """Natural-log LSE over the visible keys: lse[g, j] = log sum_i exp(l[g, j, i]).

    This is the quantity a paged-attention kernel emits beside its output.  A
    column that sees no key gets -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    nq, G, _ = q.shape
    out = np.full((G, nq), -np.inf)
    for a in range(0, nq, chunk):
        b = min(nq, a + chunk)
        l = logits(q[a:b], k)                              # [G, b-a, n]
        vis = visible(q_pos[a:b], k_pos)[None, :, :]       # [1, b-a, n]
        l = np.where(vis, l, -np.inf)
        mx = l.max(axis=2, initial=-np.inf)
        safe = np.where(np.isfinite(mx), mx, 0.0)
        ssum = np.exp(l - safe[:, :, None]).sum(axis=2)
        with np.errstate(divide="ignore"):   # log(0) of a column that sees no key; np.where takes -inf there
            out[:, a:b] = np.where(np.isfinite(mx), safe + np.log(ssum), -np.inf)
    return out


def scores_from_lse(q: np.ndarray, k: np.ndarray, q_pos: np.ndarray, k_pos: np.ndarray,
                    lse: np.ndarray, chunk: int = 64) -> np.ndarray:
    """s[i] = sum over queries j and group heads g of [pos_j >= pos_i] * exp(l[g, j, i] - lse[g, j]).

    lse: [G, nq] as handed to the scorer (the fp32 value the GPU sees, widened).
    """
    q = np.asarray(q, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    nq = q.shape[0]
    n = np.asarray(k).shape[0]
    s = np.zeros(n)
    for a in range(0, nq, chunk):
        b = min(nq, a + chunk)
        l = logits(q[a:b], k)                              # [G, b-a, n]
        vis = visible(q_pos[a:b], k_pos)[None, :, :]
        p = np.where(vis, np.exp(l - lse[:, a:b, None]), 0.0)
        s += p.sum(axis=(0, 1))
    return s


# ----------------------------------------------------------------------------
# Step 2: hit signal and LRFU ("ActKV Dissected", Component 1: entries in the
# top 90% are action-critical; the signal replaces LRFU's hit with "hit by action
# attention", decay coefficient lambda = 0.5).
# ----------------------------------------------------------------------------

def rank_order(key: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """Slots sorted by (key descending, token position ascending, slot ascending)."""
    key = np.asarray(key, dtype=np.float64)
    slot = np.arange(len(key))
    return np.lexsort((slot, np.asarray(pos, dtype=np.int64), -key))


def hit_gate(s: np.ndarray, pos: np.ndarray, hit_mass: float = 0.9) -> np.ndarray:
    """Action-critical mask: the shortest prefix of the rank order whose mass reaches hit_mass * total.

    "Top 90%" is read as cumulative attention mass (a nucleus with p = 0.9).  A
    hit_mass of 1 or more switches the gate off: every entry that received any
    attention (s > 0) is a hit.
    """
    s = np.asarray(s, dtype=np.float64)
    n = len(s)
    if hit_mass >= 1.0:
        return s > 0.0
    order = rank_order(s, pos)
    target = hit_mass * s.sum()
    hits = np.zeros(n, dtype=bool)
    if n == 0 or target <= 0.0:
        return hits
    run = np.cumsum(s[order])
    K = int(np.searchsorted(run, target, side="left")) + 1
    hits[order[:min(K, n)]] = True
    return hits


def lrfu_update(crf: np.ndarray, s: np.ndarray, pos: np.ndarray, lam: float = 0.5, hit_mass: float = 0.9,
                dt: int = 1, binary: bool = False) -> np.ndarray:
    """Combined recency-frequency value after one round: CRF' = h + 2**(-lam*dt) * CRF.

    The hit h of an entry is its score when the gate marks it action-critical
    (or 1 under binary hits) and 0 otherwise.  Rounds are LRFU's time unit.
    """
    gate = hit_gate(s, pos, hit_mass)
    h = np.where(gate, 1.0 if binary else np.asarray(s, dtype=np.float64), 0.0)
    return h + 2.0 ** (-lam * dt) * np.asarray(crf, dtype=np.float64)


def lrfu_closed_form(hits_by_round: Sequence[float], lam: float) -> float:
    """LRFU's closed form after the last round r: sum_t h_t * 2**(-lam*(r - t))."""
    r = len(hits_by_round) - 1
    return sum(h * 2.0 ** (-lam * (r - t)) for t, h in enumerate(hits_by_round))


# ----------------------------------------------------------------------------
# Step 3b: top-budget selection (eviction keeps the top-`budget` entries by CRF,
# ties broken by the lower token index).
# ----------------------------------------------------------------------------

def select_budget(crf: np.ndarray, pos: np.ndarray, budget: int, labels: Optional[np.ndarray] = None,
                  protect_mask: int = 0) -> np.ndarray:
    """Keep mask: protected labels always, then the first budget-minus-protected slots of the rank order."""
    n = len(crf)
    keep = np.zeros(n, dtype=bool)
    if labels is not None and protect_mask:
        prot = ((1 << np.asarray(labels, dtype=np.int64)) & protect_mask) != 0
    else:
        prot = np.zeros(n, dtype=bool)
    keep |= prot
    room = max(int(budget) - int(prot.sum()), 0)
    order = [i for i in rank_order(crf, pos) if not prot[i]]
    keep[np.asarray(order[:room], dtype=np.int64)] = True
    return keep


# ----------------------------------------------------------------------------
# Step 4: conflict-free slot plan ("ActKV Dissected", Component 3: survivors
# outside the target region are paired one-to-one with holes inside it).  The
# target region is the dense prefix [0, m) of the row, m = number kept.
# ----------------------------------------------------------------------------

def plan_slots(keep: np.ndarray, n: int):
    """Moves (src, dst): the j-th kept slot at or after m fills the j-th hole before m."""
    keep = np.asarray(keep[:n], dtype=bool)
    m = int(keep.sum())
    holes = [i for i in range(m) if not keep[i]]
    movers = [i for i in range(m, n) if keep[i]]
    assert len(holes) == len(movers)
    return np.asarray(movers, dtype=np.int64), np.asarray(holes, dtype=np.int64), m


# ----------------------------------------------------------------------------
# Step 5: in-place paged compaction ("ActKV Dissected", Component 3: one parallel
# copy pass, freed blocks returned to the scheduler, no extra KV buffer).
# ----------------------------------------------------------------------------

@dataclass
class PagedRow:
    """One (sequence, layer, KV head) row of the paged cache, as host arrays."""
    block_table: np.ndarray      # [max_pages] int
    n: int
    slot_pos: np.ndarray         # [max_slots]
    slot_label: np.ndarray       # [max_slots]
    crf: Optional[np.ndarray] = None


def compact_row(k_pool: np.ndarray, v_pool: np.ndarray, row: PagedRow, src: np.ndarray, dst: np.ndarray,
                m: int, page_size: int):
    """Gather-based compaction of one row; returns (k_pool', v_pool', row', freed page ids).

    k_pool/v_pool: [num_pages, page_size, D] (any dtype; copied bytewise).  Source
    slots are read from the pool as it was before the pass, which is what a
    conflict-free plan makes the in-place copy equivalent to.
    """
    P = page_size
    k_new, v_new = k_pool.copy(), v_pool.copy()
    bt = row.block_table.copy()
    pos, lab = row.slot_pos.copy(), row.slot_label.copy()
    crf = None if row.crf is None else row.crf.copy()
    for a, b in zip(src.tolist(), dst.tolist()):
        pa, oa = bt[a // P], a % P
        pb, ob = bt[b // P], b % P
        k_new[pb, ob] = k_pool[pa, oa]
        v_new[pb, ob] = v_pool[pa, oa]
        pos[b] = row.slot_pos[a]
        lab[b] = row.slot_label[a]
        if crf is not None:
            crf[b] = row.crf[a]
    first_free, end = -(-m // P), -(-row.n // P)
    freed = [int(bt[p]) for p in range(first_free, end)]
    bt[first_free:end] = -1
    return k_new, v_new, PagedRow(block_table=bt, n=m, slot_pos=pos, slot_label=lab, crf=crf), freed


# ----------------------------------------------------------------------------
# Step 3a: confidence monitor and one-way budget ratchet ("ActKV Dissected",
# Component 2: average negative log-probability of the top-20 tokens of each
# step's output distribution; sliding-window min-pooling with window 64 and
# stride 8; a negative slope of a linear fit grows the budget by 1.75x up to
# 30,000; the budget never shrinks; Summary: initial budget 512).
# ----------------------------------------------------------------------------

def token_confidence(z: np.ndarray, top_k: int = 20) -> float:
    """c = mean over the top_k tokens of -log softmax(z) = LSE(z) - mean(top_k largest z)."""
    z = np.asarray(z, dtype=np.float64)
    mx = z.max()
    lse = mx + math.log(np.exp(z - mx).sum())
    top = np.sort(z)[-top_k:]
    return float(lse - top.mean())


def min_pool(c: Sequence[float], window: int = 64, stride: int = 8) -> List[float]:
    """y_j = min of c over [stride*j, stride*j + window), complete windows only."""
    c = list(c)
    out = []
    j = 0
    while stride * j + window <= len(c):
        out.append(min(c[stride * j: stride * j + window]))
        j += 1
    return out


def ols_slope(x: Sequence[float], y: Sequence[float]) -> float:
    """Least-squares slope sum (x - xbar)(y - ybar) / sum (x - xbar)^2."""
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    xb, yb = x.mean(), y.mean()
    return float(((x - xb) * (y - yb)).sum() / ((x - xb) ** 2).sum())


def grow(budget: int, num: int = 7, den: int = 4, cap: int = 30000) -> int:
    """One ratchet step: floor(budget * 7/4) (1.75 = 7/4 exactly), capped."""
    return min(budget * num // den, cap)


@dataclass
class RatchetParams:
    top_k: int = 20
    window: int = 64
    stride: int = 8
    grow_num: int = 7
    grow_den: int = 4
    init_budget: int = 512
    cap: int = 30000
    min_points: int = 2


@dataclass
class Ratchet:
    """Per-sequence monitor state kept as the full history (plain, not incremental)."""
    params: RatchetParams = field(default_factory=RatchetParams)
    c: List[float] = field(default_factory=list)
    budget: int = 0
    last_expand_step: int = 0
    expansions: int = 0
    last_slope: float = float("nan")
    last_points: int = 0

    def __post_init__(self):
        if self.budget == 0:
            self.budget = self.params.init_budget

    def fit_points(self):
        """Pooled points whose window starts at or after the last expansion: (x = j, y = y_j)."""
        p = self.params
        y = min_pool(self.c, p.window, p.stride)
        pts = [(j, yj) for j, yj in enumerate(y) if p.stride * j >= self.last_expand_step]
        return pts

    def round(self, step_logits: np.ndarray) -> int:
        """Consume one round of decode steps ([steps, vocab]); evaluate the fit once; return the budget."""
        p = self.params
        for z in step_logits:
            self.c.append(token_confidence(z, p.top_k))
        pts = self.fit_points()
        self.last_points = len(pts)
        self.last_slope = float("nan")
        if len(pts) >= p.min_points:
            xs, ys = zip(*pts)
            self.last_slope = ols_slope(xs, ys)
            if self.last_slope < 0.0:
                self.budget = grow(self.budget, p.grow_num, p.grow_den, p.cap)
                self.last_expand_step = len(self.c)
                self.expansions += 1
        return self.budget
