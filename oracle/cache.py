"""Whole-cache driver of the CPU oracle: the per-row steps of ``oracle.path`` applied
to a paged cache laid out as the C library sees it.

TEST INFRASTRUCTURE ONLY (see ``oracle.path``).  Layouts, all host numpy arrays:

* ``k_pool``/``v_pool``: [num_pages, page_size, D]; a page holds page_size tokens of
  one (layer, KV head) row.
* ``block_table``: [rows, max_pages], -1 = no page; row = (seq * layers + layer) * kv_heads + head.
* ``row_len``: [rows]; ``slot_pos``/``slot_label``: [rows, max_pages * page_size].
* queries: ``q`` [S, L, max_q, Hq, D], ``lse`` [S, L, Hq, max_q], ``q_pos`` [S, max_q], ``num_q`` [S].

Parity status: pinned on a hand-built, permuted cache by the non-GPU tests (row-id order,
gathers against per-slot identity codes, LSE and scores by brute force, the per-row steps
against the pinned ``oracle.path`` functions, compaction against a written-out single copy
pass and the freed-list order), with planted mistakes that must each fail a pin.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import numpy as np

from . import path


@dataclass
class Geometry:
    num_seqs: int
    num_layers: int
    num_kv_heads: int
    num_q_heads: int
    page_size: int

    @property
    def rows(self) -> int:
        return self.num_seqs * self.num_layers * self.num_kv_heads

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def coords(self, r: int):
        h = r % self.num_kv_heads
        sl = r // self.num_kv_heads
        return sl // self.num_layers, sl % self.num_layers, h


def gather_row(pool: np.ndarray, bt_row: np.ndarray, n: int, page_size: int) -> np.ndarray:
    """Logical [n, D] view of a row, read page by page through its block table."""
    i = np.arange(n)
    return pool[bt_row[i // page_size], i % page_size]


def row_queries(geo: Geometry, r: int, q, q_pos, num_q):
    s, l, h = geo.coords(r)
    G = geo.group
    nq = int(num_q[s])
    return q[s, l, :nq, h * G:(h + 1) * G, :], q_pos[s, :nq], s, l, h, nq


def lse_cache(geo: Geometry, k_pool, block_table, row_len, slot_pos, q, q_pos, num_q, max_q) -> np.ndarray:
    """LSE of every query column over its row's visible keys: [S, L, Hq, max_q] (fp64, -inf if none)."""
    out = np.full((geo.num_seqs, geo.num_layers, geo.num_q_heads, max_q), -np.inf)
    G = geo.group
    for r in range(geo.rows):
        qr, qp, s, l, h, nq = row_queries(geo, r, q, q_pos, num_q)
        n = int(row_len[r])
        k = gather_row(k_pool, block_table[r], n, geo.page_size).astype(np.float64)
        out[s, l, h * G:(h + 1) * G, :nq] = path.attention_lse(qr, k, qp, slot_pos[r, :n])
    return out


def score_cache(geo: Geometry, k_pool, block_table, row_len, slot_pos, q, lse, q_pos, num_q,
                rows: Optional[List[int]] = None) -> np.ndarray:
    """Scores [rows, max_slots] (fp64; zero beyond each row's length)."""
    max_slots = block_table.shape[1] * geo.page_size
    rows = range(geo.rows) if rows is None else rows
    out = np.zeros((geo.rows, max_slots))
    G = geo.group
    for r in rows:
        qr, qp, s, l, h, nq = row_queries(geo, r, q, q_pos, num_q)
        n = int(row_len[r])
        k = gather_row(k_pool, block_table[r], n, geo.page_size).astype(np.float64)
        out[r, :n] = path.scores_from_lse(qr, k, qp, slot_pos[r, :n], lse[s, l, h * G:(h + 1) * G, :nq])
    return out


def lrfu_cache(geo: Geometry, scores, crf, row_len, slot_pos, lam=0.5, hit_mass=0.9, dt=1, binary=False,
               rows: Optional[List[int]] = None):
    """CRF after one round for every row; slots beyond a row's length are left as they were."""
    out = np.array(crf, dtype=np.float64, copy=True)
    hits = np.zeros(out.shape, dtype=bool)
    for r in (range(geo.rows) if rows is None else rows):
        n = int(row_len[r])
        hits[r, :n] = path.hit_gate(scores[r, :n], slot_pos[r, :n], hit_mass)
        out[r, :n] = path.lrfu_update(crf[r, :n], scores[r, :n], slot_pos[r, :n], lam, hit_mass, dt, binary)
    return out, hits


def select_cache(geo: Geometry, crf, row_len, slot_pos, slot_label, budget, protect_mask=0,
                 rows: Optional[List[int]] = None):
    """Keep mask [rows, max_slots] and kept count per row; budget is per sequence."""
    keep = np.zeros(crf.shape, dtype=np.uint8)
    kept = np.zeros(geo.rows, dtype=np.int64)
    for r in (range(geo.rows) if rows is None else rows):
        s, _, _ = geo.coords(r)
        n = int(row_len[r])
        lab = None if slot_label is None else slot_label[r, :n]
        k = path.select_budget(crf[r, :n], slot_pos[r, :n], int(budget[s]), lab, protect_mask)
        keep[r, :n] = k
        kept[r] = int(k.sum())
    return keep, kept


def plan_cache(geo: Geometry, keep, row_len, rows: Optional[List[int]] = None):
    """Per-row move lists (src, dst) and the new row length m."""
    plans = {}
    for r in (range(geo.rows) if rows is None else rows):
        src, dst, m = path.plan_slots(keep[r], int(row_len[r]))
        plans[r] = (src, dst, m)
    return plans


def compact_cache(geo: Geometry, k_pool, v_pool, block_table, row_len, slot_pos, slot_label, crf, plans):
    """Apply every row's plan; freed pages listed row by row, ascending logical page within a row."""
    P = geo.page_size
    k_new, v_new = k_pool.copy(), v_pool.copy()
    bt, rl = block_table.copy(), row_len.copy()
    sp, sl = slot_pos.copy(), slot_label.copy()
    cr = None if crf is None else crf.copy()
    freed: List[int] = []
    for r in sorted(plans):
        src, dst, m = plans[r]
        row = path.PagedRow(block_table=bt[r], n=int(rl[r]), slot_pos=sp[r], slot_label=sl[r],
                            crf=None if cr is None else cr[r])
        # rows own disjoint pages, so compacting row after row on one pool equals one pass
        k_new, v_new, new, fr = path.compact_row(k_new, v_new, row, src, dst, m, P)
        bt[r], rl[r], sp[r], sl[r] = new.block_table, new.n, new.slot_pos, new.slot_label
        if cr is not None:
            cr[r] = new.crf
        freed.extend(fr)
    return k_new, v_new, bt, rl, sp, sl, cr, np.asarray(freed, dtype=np.int64)
