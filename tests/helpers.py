"""Shared test plumbing: build a seeded workload on the device and hand sampled rows to the oracle.

Inputs come only from the seeded generator (agent_kv_cache_lse_b200.synth) or from torch's
own RNG; the oracle reads those inputs (copied before the path runs), never anything a
CUDA kernel of the library wrote.  Row-local helpers gather only the sampled rows' pages,
so full-size workloads never travel to the host whole.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Optional

import numpy as np
import torch

from agent_kv_cache_lse_b200 import kvc, synth
from oracle import cache as ocache
from oracle import path as opath


def has_gpu() -> bool:
    return torch.cuda.is_available()


@dataclass
class Workload:
    spec: synth.Spec
    layout: synth.Layout
    cache: kvc.Cache
    queries: kvc.QuerySet
    geo: ocache.Geometry

    def row_queries(self, r: int):
        """Host fp64 query vectors [nq, G, D], positions [nq] of row r's group."""
        s, l, h = self.geo.coords(r)
        G = self.geo.group
        nq = int(self.queries.num_q[s])
        q = self.queries.q[s, l, :nq, h * G:(h + 1) * G, :].cpu().to(torch.float64).numpy()
        return q, self.queries.q_pos[s, :nq].cpu().numpy(), s, l, h, nq


def geometry(spec: synth.Spec) -> ocache.Geometry:
    return ocache.Geometry(spec.num_seqs, spec.num_layers, spec.num_kv_heads, spec.num_q_heads, spec.page_size)


def randn_pool(spec: synth.Spec, layout: synth.Layout, seed: int, device="cuda") -> torch.Tensor:
    """A pool of N(0, 1) values from torch's seeded generator, rounded to the spec dtype (fast at any size)."""
    g = torch.Generator(device=device).manual_seed(seed)
    pool = torch.empty((layout.num_pages, spec.page_size, spec.head_dim), dtype=synth.torch_dtype(spec), device=device)
    flat = pool.view(-1)
    step = 1 << 28
    for a in range(0, flat.numel(), step):
        b = min(flat.numel(), a + step)
        flat[a:b] = torch.randn(b - a, generator=g, device=device, dtype=torch.float32).to(pool.dtype)
    return pool


def build(spec: synth.Spec, device="cuda", fill: str = "synth") -> Workload:
    """Seeded workload on the device; fill="randn" draws the pools from torch's generator instead of the
    counter-based one (for caches too large to generate element by element in reasonable time)."""
    layout = synth.make_layout(spec)
    if fill == "randn":
        kp = randn_pool(spec, layout, spec.seed * 2 + 1, device)
        vp = randn_pool(spec, layout, spec.seed * 2 + 2, device)
    else:
        kp = synth.fill_pool(spec, layout, "k", device)
        vp = synth.fill_pool(spec, layout, "v", device)
    qs = synth.make_queries(spec, device)
    lse = torch.full((spec.num_seqs, spec.num_layers, spec.num_q_heads, qs.max_q), float("-inf"),
                     dtype=torch.float32, device=device)
    cache = kvc.Cache(kp, vp, layout.block_table.to(device), layout.row_len.to(device), layout.slot_pos.to(device),
                      layout.slot_label.to(device), spec.num_seqs, spec.num_layers, spec.num_kv_heads)
    queries = kvc.QuerySet(qs.q, lse, qs.q_pos.to(device), qs.num_q.to(device))
    return Workload(spec, layout, cache, queries, geometry(spec))


def _bits(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


@dataclass
class RowSnap:
    """Host copy of one row's state (its own pages only)."""
    n: int
    pages: np.ndarray     # physical page ids of the row's first ceil(n/P) pages
    kbits: np.ndarray     # [npages, P, D] raw bits
    vbits: np.ndarray
    kf: np.ndarray        # [n, D] fp64 logical keys
    bt: np.ndarray        # [max_pages] block-table row
    sp: np.ndarray        # [max_slots]
    sl: np.ndarray


def snap_rows(w: Workload, rows: List[int]) -> Dict[int, RowSnap]:
    c, P = w.cache, w.spec.page_size
    out = {}
    for r in rows:
        n = int(c.row_len[r])
        npg = -(-n // P)
        pages_d = c.block_table[r, :npg].to(torch.int64)
        kp = c.k_pool[pages_d]
        vp = c.v_pool[pages_d]
        kf = kp.reshape(-1, kp.shape[-1])[:n].cpu().to(torch.float64).numpy()
        out[r] = RowSnap(n=n, pages=pages_d.cpu().numpy(), kbits=_bits(kp).cpu().numpy(),
                         vbits=_bits(vp).cpu().numpy(), kf=kf, bt=c.block_table[r].cpu().numpy(),
                         sp=c.slot_pos[r].cpu().numpy(), sl=c.slot_label[r].cpu().numpy())
    return out


def oracle_lse(w: Workload, rows: Optional[List[int]] = None, snaps: Optional[Dict[int, RowSnap]] = None) -> np.ndarray:
    """Oracle LSE (fp64) for the columns of the given rows (all rows when None); -inf elsewhere."""
    rows = list(range(w.spec.rows)) if rows is None else rows
    snaps = snaps or snap_rows(w, rows)
    out = np.full(tuple(w.queries.lse.shape), -np.inf)
    G = w.geo.group
    for r in rows:
        q, qp, s, l, h, nq = w.row_queries(r)
        sn = snaps[r]
        out[s, l, h * G:(h + 1) * G, :nq] = opath.attention_lse(q, sn.kf, qp, sn.sp[:sn.n])
    return out


def set_lse(w: Workload, lse64: np.ndarray, rows: Optional[List[int]] = None):
    """Hand the fp32-rounded oracle LSE to the device (only the given rows' columns when rows is set)."""
    lse32 = torch.from_numpy(lse64.astype(np.float32))
    if rows is None:
        w.queries.lse.copy_(lse32.to(w.queries.lse.device))
        return
    G = w.geo.group
    for r in rows:
        s, l, h = w.geo.coords(r)
        w.queries.lse[s, l, h * G:(h + 1) * G] = lse32[s, l, h * G:(h + 1) * G].to(w.queries.lse.device)


def oracle_scores(w: Workload, lse32: np.ndarray, rows: Optional[List[int]] = None,
                  snaps: Optional[Dict[int, RowSnap]] = None) -> Dict[int, np.ndarray]:
    rows = list(range(w.spec.rows)) if rows is None else rows
    snaps = snaps or snap_rows(w, rows)
    G = w.geo.group
    out = {}
    for r in rows:
        q, qp, s, l, h, nq = w.row_queries(r)
        sn = snaps[r]
        out[r] = opath.scores_from_lse(q, sn.kf, qp, sn.sp[:sn.n], lse32[s, l, h * G:(h + 1) * G, :nq])
    return out


def assert_scores_close(gpu: np.ndarray, orc: np.ndarray, what=""):
    """Tolerance fixed for the scores: |gpu - oracle| <= 1e-6 + 1e-3 |oracle| elementwise."""
    err = np.abs(gpu - orc)
    bad = err > 1e-6 + 1e-3 * np.abs(orc)
    if bad.any():
        i = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} scores out of tolerance, e.g. at {i.tolist()}: "
                             f"gpu {gpu[tuple(i[0])]} oracle {orc[tuple(i[0])]}")
