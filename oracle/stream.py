"""CPU oracle of streaming a compacted cache forward: new tokens appended at each row's end.

TEST INFRASTRUCTURE ONLY (see ``oracle.path``).

"KV-streams for Efficient Compaction in Agentic Reinforcement Learning" (abstract): the compacted cache is
carried across rollouts and new tokens stream into it instead of the whole context being prefilled again.
After a compaction every row is a dense prefix [0, n); appending writes token i of the new tokens at slot
n + i.  A row that reaches a logical page it does not hold takes a page from the free-page stack: the
rows in order, each row's new pages in ascending logical order, from the top of the stack (the pages the
call takes are the top ``total`` entries, row r's k-th new page is stack[depth - total + offset_r + k]).
A stack too shallow for the call leaves everything as it was.

Parity status: pinned by the non-GPU tests (a hand-worked example, content and stack invariants on random
caches, the overflow case and planted mistakes).
"""
from __future__ import annotations

from typing import Tuple

import numpy as np


def pages_needed(n: int, count: int, page_size: int) -> int:
    """Logical pages a row of n slots must add to hold count more: ceil((n + count) / P) - ceil(n / P)."""
    return -(-(n + count) // page_size) - (-(-n // page_size))


def append_tokens(k_pool, v_pool, block_table, row_len, slot_pos, slot_label, crf, stack, depth: int,
                  k_new, v_new, new_pos, label: int, seq_of_row, page_size: int):
    """Returns (k_pool', v_pool', block_table', row_len', slot_pos', slot_label', crf', depth', ok).

    k_new/v_new: [rows, count, D]; new_pos: [seqs, count]; seq_of_row: [rows] sequence of each row;
    stack: the free pages, its top at index depth - 1; crf may be None.  ok is False when the stack is
    too shallow (then nothing changes).
    """
    P = page_size
    rows, count = k_new.shape[0], k_new.shape[1]
    need = [pages_needed(int(row_len[r]), count, P) for r in range(rows)]
    total = sum(need)
    out = [a.copy() for a in (k_pool, v_pool, block_table, row_len, slot_pos, slot_label)]
    crf_out = None if crf is None else crf.copy()
    if total > depth:
        return (*out, crf_out, depth, False)
    k2, v2, bt, rl, sp, sl = out
    base = depth - total
    offset = 0
    for r in range(rows):
        n = int(row_len[r])
        first_new = -(-n // P)
        for k in range(need[r]):
            bt[r, first_new + k] = stack[base + offset + k]
        offset += need[r]
        for i in range(count):
            s = n + i
            page = bt[r, s // P]
            k2[page, s % P] = k_new[r, i]
            v2[page, s % P] = v_new[r, i]
            sp[r, s] = new_pos[seq_of_row[r], i]
            sl[r, s] = label
            if crf_out is not None:
                crf_out[r, s] = 0.0
        rl[r] = n + count
    return k2, v2, bt, rl, sp, sl, crf_out, base, True


def logical_rows(pool, block_table, row_len, page_size: int):
    """Each row's content in slot order, read through its block table: list of [n, D] arrays."""
    out = []
    for r in range(block_table.shape[0]):
        n = int(row_len[r])
        i = np.arange(n)
        out.append(pool[block_table[r, i // page_size], i % page_size])
    return out


def check_stack_use(block_table_before, block_table_after, stack, depth_before: int, depth_after: int) -> Tuple[bool, str]:
    """The pages newly entered in the block tables are exactly the stack's top depth_before - depth_after
    entries, each once."""
    new = sorted(int(p) for p in block_table_after[(block_table_before < 0) & (block_table_after >= 0)])
    top = sorted(int(p) for p in stack[depth_after:depth_before])
    if new != top:
        return False, f"new pages {new} != stack top {top}"
    return True, ""
