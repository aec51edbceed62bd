"""CPU oracle of beacon-query maintenance (online k-means over past queries).

TEST INFRASTRUCTURE ONLY.  Only the test suite imports this module; the CUDA library
never calls it and shares no code with it.

"BeaconKV Compresses KV Cache for Long-Reasoning Models with Beacon Queries", Key ideas:
the queries that return to distant context fall into a few similarity groups, one
representative per group (a beacon query) stands in for that history, and the beacons
join the recent queries in the query set that scores the cache.  The page does not say
how the groups are found.  Reading adopted: online (mini-batch) k-means, separately for
each (sequence, layer, query head):

* each call brings that group's m new query vectors;
* beacons that have absorbed nothing yet (count 0) are first seeded, in index order, with
  the first new queries (the j-th empty beacon takes query j);
* every new query goes to its nearest beacon among those with a count or a seed (squared
  Euclidean distance; the lower beacon index wins a tie);
* each beacon that drew new queries becomes the mean of everything it has absorbed, old and
  new: c_b <- (c_b * n_b + sum of its new queries) / (n_b + m_b), n_b <- n_b + m_b; a beacon
  that drew nothing keeps its value (a seeded one keeps its seed with count 0 and is seeded
  afresh next time).

Decision precision.  Which beacon a query joins is an integer decided by floating point,
so both sides take that decision in fp32 with one fixed order of operations: the distance
is the sum over d = 0..D-1, in that order, of (q_d - c_d)^2, with the difference, the square
and each partial sum rounded to fp32 separately (no fused multiply-add).  The mean is fp32
in one fixed order too: S = c_b * n_b, then S += q_j for the beacon's new queries in query
order, then c_b = S / (n_b + m_b), each step rounded to fp32.

Parity status: pinned by the non-GPU tests (exact cluster means of separated data,
running means against fp64 means, distances against fp64 sums, tie and seeding rules,
and planted mistakes); not "parity unpinned".
"""
from __future__ import annotations

import numpy as np


def distances_f32(q: np.ndarray, c: np.ndarray) -> np.ndarray:
    """Squared distances [m, B] in fp32, summed over d in order with separate roundings."""
    q = np.asarray(q, dtype=np.float32)
    c = np.asarray(c, dtype=np.float32)
    acc = np.zeros((q.shape[0], c.shape[0]), dtype=np.float32)
    for d in range(q.shape[1]):
        t = np.subtract(q[:, d][:, None], c[None, :, d], dtype=np.float32)
        acc = np.add(acc, np.multiply(t, t, dtype=np.float32), dtype=np.float32)
    return acc


def beacon_update(c: np.ndarray, n: np.ndarray, q: np.ndarray):
    """One call for one group.

    c: [B, D] fp32 beacons, n: [B] int counts, q: [m, D] new queries (fp32 values; bf16 queries
    are passed already widened).  Returns (c', n', assignment [m], -1 where no beacon exists).
    """
    c = np.array(c, dtype=np.float32, copy=True)
    n = np.array(n, dtype=np.int64, copy=True)
    q = np.asarray(q, dtype=np.float32)
    B, m = c.shape[0], q.shape[0]
    live = n > 0
    empty = np.flatnonzero(~live)
    seeds = min(len(empty), m)
    for t in range(seeds):
        c[empty[t]] = q[t]
        live[empty[t]] = True
    a = np.full(m, -1, dtype=np.int64)
    if m == 0 or not live.any():
        return c, n, a
    d = distances_f32(q, c)
    d[:, ~live] = np.inf
    a = np.argmin(d, axis=1)          # first minimum: the lower index wins a tie
    s = np.multiply(c, n[:, None].astype(np.float32), dtype=np.float32)
    for j in range(m):                # query order
        s[a[j]] = np.add(s[a[j]], q[j], dtype=np.float32)
    drawn = np.bincount(a, minlength=B)
    for b in range(B):
        if drawn[b] > 0:              # a beacon that drew nothing keeps its value exactly
            c[b] = np.divide(s[b], np.float32(n[b] + drawn[b]), dtype=np.float32)
    return c, n + drawn, a
