"""CPU oracle of step-aware ranking scores (fp64, numpy).

TEST INFRASTRUCTURE ONLY.  Only the test suite imports this module; the CUDA library never
calls it and shares no code with it.

"StepKV: Step-Aware KV Cache Compression for LLM Agents" (abstract): cache entries are tied to
the reasoning step that generated them, each step gets a utility estimated from signals of the
trajectory, that utility is combined with token-level saliency, and the combined scores rank the
prunable tokens globally, the top ones being kept under the budget.  The page gives no formula
for any of these; the readings adopted here, the plainest ones the rest supports:

* steps: a step begins at position 0 and at every position where a reasoning segment begins (a
  ReAct step = thought, action, observation); the caller passes each sequence's ascending step
  start positions, so that the step of an entry is a function of its token position alone and
  survives compaction (which permutes slots and drops entries);
* step of an entry = the last step whose start is at or before the entry's position;
* token saliency = the entry's attention score (the step-1 score of this path);
* step utility U_k = the mean saliency of the row's entries of step k (a trajectory-derived
  signal in the same units as the saliency);
* combined score = (1 - beta) * s_i + beta * U_{step(i)}, beta in [0, 1] (0.5 by default);
* the combined scores rank the row's entries through the same top-budget selection as the
  LRFU values (ties to the lower position, protected labels first).

Parity status: pinned by the non-GPU tests (beta = 0 and beta = 1 limits, the step mean of the
combined score, invariance under slot permutation, a hand example, brute force of the step
assignment, and planted mistakes); not "parity unpinned".
"""
from __future__ import annotations

import numpy as np


def step_of(pos: np.ndarray, step_start: np.ndarray) -> np.ndarray:
    """Index of the last step start at or before each position (step_start ascending, step_start[0] = 0)."""
    return np.searchsorted(np.asarray(step_start, dtype=np.int64), np.asarray(pos, dtype=np.int64),
                           side="right") - 1


def step_utility(scores: np.ndarray, pos: np.ndarray, step_start: np.ndarray) -> np.ndarray:
    """U_k for every step of the table: mean score of the row's entries in step k (0 for a step with none)."""
    s = np.asarray(scores, dtype=np.float64)
    k = step_of(pos, step_start)
    n_steps = len(step_start)
    tot = np.zeros(n_steps)
    cnt = np.zeros(n_steps)
    for i in range(len(s)):
        tot[k[i]] += s[i]
        cnt[k[i]] += 1
    return np.where(cnt > 0, tot / np.maximum(cnt, 1), 0.0)


def combined_scores(scores: np.ndarray, pos: np.ndarray, step_start: np.ndarray, beta: float) -> np.ndarray:
    """(1 - beta) * s_i + beta * U_{step(i)} for the row's entries, in slot order."""
    s = np.asarray(scores, dtype=np.float64)
    u = step_utility(s, pos, step_start)
    return (1.0 - beta) * s + beta * u[step_of(pos, step_start)]
