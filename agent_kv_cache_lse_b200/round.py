"""One eviction round over a paged cache: the C-ABI calls in path order.

``EvictionRound`` owns the per-round device buffers (scores, LRFU values, keep mask,
slot plan, freed-page list, workspace, ratchet state) and enqueues, on the caller's stream:

  kvc_score_from_lse -> (kvc_confidence_ratchet on a second stream | kvc_lrfu_update)
  -> kvc_select_budget -> kvc_plan_slots -> kvc_compact_pages

and, in a round without logits (budget unchanged), kvc_lrfu_select (LRFU update and
top-budget selection in one launch) in place of the middle three.

("ActKV Dissected": Component 2 budget, Component 1 scoring and LRFU, Component 3
slot plan and in-place compaction).  Nothing here computes; it only allocates with
torch and marshals arguments.  The LRFU values persist across rounds (they move with
their entries during compaction), as do the ratchet state and the budget.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import kvc


class EvictionRound:
    KERNELS_PER_ROUND = 8  # ratchet 2, score 1, lrfu 1, select 1, plan 1, compact 2 (7 without logits)

    def __init__(self, cache: kvc.Cache, params: Optional[kvc.KvcRatchetParams] = None,
                 freed_capacity: Optional[int] = None, device="cuda"):
        self.cache = cache
        self.params = params or kvc.ratchet_params()
        rows, ms = cache.rows, cache.max_slots
        dev = torch.device(device)
        self.scores = torch.zeros((rows, ms), dtype=torch.float32, device=dev)
        self.crf = torch.zeros((rows, ms), dtype=torch.float32, device=dev)
        self.keep = torch.zeros((rows, ms), dtype=torch.uint8, device=dev)
        self.kept = torch.zeros(rows, dtype=torch.int32, device=dev)
        self.move_src = torch.zeros((rows, ms), dtype=torch.int32, device=dev)
        self.move_dst = torch.zeros((rows, ms), dtype=torch.int32, device=dev)
        self.num_moves = torch.zeros(rows, dtype=torch.int32, device=dev)
        cap = freed_capacity if freed_capacity is not None else cache.block_table.numel()
        self.freed = torch.full((max(cap, 1),), -1, dtype=torch.int32, device=dev)
        self.num_freed = torch.zeros(1, dtype=torch.int64, device=dev)
        ws = kvc.kvc_compact_workspace_bytes(rows)
        self.workspace = torch.zeros((ws + 7) // 8, dtype=torch.int64, device=dev)
        self.status = torch.zeros(2, dtype=torch.int32, device=dev)
        S = cache.num_seqs
        self.budget = torch.full((S,), self.params.init_budget, dtype=torch.int32, device=dev)
        nb = kvc.kvc_ratchet_state_bytes(S, self.params)
        self.state = torch.zeros(((nb + 15) // 16) * 16, dtype=torch.uint8, device=dev)
        kvc.kvc_ratchet_init(self.state, self.budget, S, self.params)
        self._side = torch.cuda.Stream(device=dev)
        self._fork, self._join = torch.cuda.Event(), torch.cuda.Event()

    def reset_ratchet(self, stream=None):
        kvc.kvc_ratchet_init(self.state, self.budget, self.cache.num_seqs, self.params, stream)

    def run(self, queries: kvc.QuerySet, logits: Optional[torch.Tensor] = None, lam: float = 0.5,
            hit_mass: float = 0.9, score_flags: int = 0, protect_label_mask: int = 0,
            confidence_out: Optional[torch.Tensor] = None, stream=None):
        """Enqueue one round.  logits [S, steps, V] fp32 drive the ratchet (None: budget unchanged).

        With logits, the ratchet runs on a second stream beside the LRFU update (neither needs the other;
        the selection needs both), forked after the scores and joined before the selection."""
        main = stream if stream is not None else torch.cuda.current_stream()
        kvc.kvc_score_from_lse(self.cache, queries, self.scores, score_flags, self.status, main)
        self.run_after_scores(logits, lam, hit_mass, main, protect_label_mask, confidence_out)

    def run_after_scores(self, logits: Optional[torch.Tensor], lam: float = 0.5, hit_mass: float = 0.9, stream=None,
                         protect_label_mask: int = 0, confidence_out: Optional[torch.Tensor] = None):
        """Enqueue the rest of a round on scores already in self.scores: (ratchet | LRFU) -> select + plan (one
        launch) -> compact, or LRFU + select (one launch) -> plan -> compact when there are no logits."""
        c = self.cache
        main = stream if stream is not None else torch.cuda.current_stream()
        if logits is not None:
            # the LRFU update goes first so that its clusters take their SMs before the ratchet's CTAs spread
            self._fork.record(main)
            kvc.kvc_lrfu_update(c, self.scores, self.crf, lam, hit_mass, 1, 0, self.status, main)
            self._side.wait_event(self._fork)
            kvc.kvc_confidence_ratchet(logits, self.state, self.budget, self.params, confidence_out, self.status,
                                       self._side)
            self._join.record(self._side)
            main.wait_event(self._join)
            kvc.kvc_select_plan(c, self.crf, self.budget, self.keep, self.kept, self.move_src, self.move_dst,
                                self.num_moves, protect_label_mask, self.status, main)
        else:
            kvc.kvc_lrfu_select(c, self.scores, self.crf, self.budget, self.keep, self.kept, lam, hit_mass, 1, 0,
                                protect_label_mask, self.status, main)
            kvc.kvc_plan_slots(c, self.keep, self.kept, self.move_src, self.move_dst, self.num_moves, self.status,
                               main)
        kvc.kvc_compact_pages(c, self.move_src, self.move_dst, self.num_moves, self.kept, self.crf, self.freed,
                              self.num_freed, self.workspace, self.status, main)

    def device_status(self):
        return kvc.device_status(self.status)
