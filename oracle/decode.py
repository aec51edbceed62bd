"""CPU oracle of one decode step of paged attention with the scores folded in (fp64, numpy).

TEST INFRASTRUCTURE ONLY.  Only the test suite imports this module; the CUDA library never
calls it and shares no code with it.

"ActKV Dissected", Component 3: the softmax log-sum-exp is a byproduct of paged attention,
so the current query's attention probabilities are its logits minus that LSE, with no
gather of the attention matrix and no recompute.  One decode step of one (sequence, layer)
has one query per query head; for the G heads of a KV head's group and the row's keys
(those at or before the query's position):
    l[g, i] = q_g . k_i / sqrt(D)
    lse[g]  = log sum_i exp(l[g, i])
    out[g]  = sum_i exp(l[g, i] - lse[g]) v_i            (the attention output)
    s_i    += sum_g exp(l[g, i] - lse[g])                 (the step's contribution to the scores)
The LSE and the probabilities reuse the functions of oracle.path, which its own pins cover;
the output is pinned by tests/test_decode_pins.py.
"""
from __future__ import annotations

import numpy as np

from . import path


def decode_step(q: np.ndarray, k: np.ndarray, v: np.ndarray, q_pos: int, k_pos: np.ndarray):
    """q: [G, D] the group's query heads; k, v: [n, D]; k_pos: [n].  Returns (out [G, D], lse [G], inc [n])."""
    q = np.asarray(q, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    qp = np.array([q_pos], dtype=np.int64)
    lse = path.attention_lse(q[None], k, qp, k_pos)[:, 0]                 # [G]
    l = path.logits(q[None], k)[:, 0, :]                                   # [G, n]
    vis = path.visible(qp, k_pos)[0]                                       # [n]
    safe = np.where(np.isfinite(lse), lse, 0.0)
    p = np.where(vis[None, :] & np.isfinite(lse)[:, None], np.exp(l - safe[:, None]), 0.0)
    return p @ v, lse, p.sum(axis=0)
