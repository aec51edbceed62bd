"""Pins of the append oracle (``oracle.stream``): streaming new tokens into a compacted cache.

"KV-streams for Efficient Compaction in Agentic Reinforcement Learning" (abstract): the compacted cache is
carried forward and new tokens stream into it.  The pins: a hand-worked example (page by page), the content
of every row read through its block table equal to its old content followed by the new tokens, the pages
taken equal to the top of the free stack (each once, in row order), the pool untouched outside the new
slots, and a stack too shallow leaving everything as it was.  Planted mistakes must each fail a pin.
"""
import inspect

import numpy as np
import pytest

from oracle import stream as ost

P, D = 4, 3


def _cache(lengths, max_pages, num_pages, seed):
    rng = np.random.default_rng(seed)
    rows = len(lengths)
    perm = rng.permutation(num_pages)
    bt = np.full((rows, max_pages), -1, dtype=np.int64)
    used = 0
    for r, n in enumerate(lengths):
        k = -(-n // P)
        bt[r, :k] = perm[used:used + k]
        used += k
    stack = perm[used:].copy()
    k_pool = rng.standard_normal((num_pages, P, D))
    v_pool = rng.standard_normal((num_pages, P, D))
    sp = rng.integers(0, 1000, (rows, max_pages * P))
    sl = rng.integers(0, 3, (rows, max_pages * P)).astype(np.uint8)
    crf = rng.random((rows, max_pages * P))
    return k_pool, v_pool, bt, np.array(lengths), sp, sl, crf, stack


def pin_hand_example(S):
    # 2 rows of 3 and 8 slots (pages of 4), 3 new tokens each: row 0 fills slot 3 of its page 0 and needs one
    # page for slots 4-5; row 1 needs one page for slots 8-10.  Stack [10, 11, 12, 13] of depth 4: the call
    # takes the top two, row 0 gets 12, row 1 gets 13; the depth drops to 2.
    k_pool = np.zeros((14, P, 1))
    v_pool = np.zeros((14, P, 1))
    bt = np.array([[0, -1, -1], [1, 2, -1]])
    rl = np.array([3, 8])
    sp = np.zeros((2, 12), dtype=np.int64)
    sl = np.zeros((2, 12), dtype=np.uint8)
    stack = np.array([10, 11, 12, 13])
    k_new = np.array([[[1.0], [2.0], [3.0]], [[4.0], [5.0], [6.0]]])
    new_pos = np.array([[100, 101, 102]])
    k2, v2, bt2, rl2, sp2, sl2, _, depth, ok = S.append_tokens(k_pool, v_pool, bt, rl, sp, sl, None, stack, 4, k_new,
                                                                k_new, new_pos, 1, np.array([0, 0]), P)
    assert ok and depth == 2
    assert bt2.tolist() == [[0, 12, -1], [1, 2, 13]]
    assert rl2.tolist() == [6, 11]
    assert k2[0, 3, 0] == 1.0 and k2[12, 0, 0] == 2.0 and k2[12, 1, 0] == 3.0
    assert k2[13, 0, 0] == 4.0 and k2[13, 1, 0] == 5.0 and k2[13, 2, 0] == 6.0
    assert sp2[0, 3:6].tolist() == [100, 101, 102] and sp2[1, 8:11].tolist() == [100, 101, 102]
    assert sl2[0, 3:6].tolist() == [1, 1, 1]


def pin_content_and_stack(S):
    lengths = [0, 1, 3, 4, 5, 8, 13, 16, 2]
    seqs = np.array([0, 0, 0, 1, 1, 1, 2, 2, 2])
    for count in (1, 3, 4, 9):
        k_pool, v_pool, bt, rl, sp, sl, crf, stack = _cache(lengths, 12, 80, seed=count)
        rng = np.random.default_rng(100 + count)
        k_new = rng.standard_normal((len(lengths), count, D))
        v_new = rng.standard_normal((len(lengths), count, D))
        new_pos = rng.integers(1000, 2000, (3, count))
        depth = len(stack)
        before_k = ost.logical_rows(k_pool, bt, rl, P)
        before_v = ost.logical_rows(v_pool, bt, rl, P)
        k2, v2, bt2, rl2, sp2, sl2, crf2, depth2, ok = S.append_tokens(
            k_pool, v_pool, bt, rl, sp, sl, crf, stack, depth, k_new, v_new, new_pos, 2, seqs, P)
        assert ok
        after_k = ost.logical_rows(k2, bt2, rl2, P)
        after_v = ost.logical_rows(v2, bt2, rl2, P)
        for r, n in enumerate(lengths):
            assert np.array_equal(after_k[r], np.concatenate([before_k[r], k_new[r]])), (count, r)
            assert np.array_equal(after_v[r], np.concatenate([before_v[r], v_new[r]])), (count, r)
            assert np.array_equal(sp2[r, n:n + count], new_pos[seqs[r]]) and np.all(sl2[r, n:n + count] == 2)
            assert np.all(crf2[r, n:n + count] == 0.0) and np.array_equal(crf2[r, :n], crf[r, :n])
            assert int(rl2[r]) == n + count
        total = sum(ost.pages_needed(n, count, P) for n in lengths)
        assert depth2 == depth - total
        ok2, why = ost.check_stack_use(bt, bt2, stack, depth, depth2)
        assert ok2, why
        # pages are handed out in row order: row r's new pages come before row r+1's in the stack
        taken = [int(p) for r in range(len(lengths)) for p in bt2[r][(bt[r] < 0) & (bt2[r] >= 0)]]
        assert taken == [int(p) for p in stack[depth2:depth]]
        # no slot of an old page other than the new slots changed
        used_old = set(int(p) for p in bt[bt >= 0])
        for p in used_old:
            for off in range(P):
                owners = [(r, lp) for r in range(len(lengths)) for lp in range(bt.shape[1]) if bt[r, lp] == p]
                r, lp = owners[0]
                s = lp * P + off
                if s < lengths[r]:
                    assert np.array_equal(k2[p, off], k_pool[p, off])


def pin_overflow(S):
    # two rows of 4 slots, 8 new tokens each: 2 pages per row, 4 in all; a stack one page short changes nothing,
    # a stack of exactly 4 pages is emptied
    lengths = [4, 4]
    k_pool, v_pool, bt, rl, sp, sl, crf, stack = _cache(lengths, 4, 6, seed=3)
    assert len(stack) == 4
    k_new = np.ones((2, 8, D))
    pos = np.zeros((1, 8), dtype=np.int64)
    res = S.append_tokens(k_pool, v_pool, bt, rl, sp, sl, crf, stack, 3, k_new, k_new, pos, 0, np.array([0, 0]), P)
    assert res[-1] is False and res[-2] == 3
    assert np.array_equal(res[2], bt) and np.array_equal(res[3], rl) and np.array_equal(res[0], k_pool)
    res = S.append_tokens(k_pool, v_pool, bt, rl, sp, sl, crf, stack, 4, k_new, k_new, pos, 0, np.array([0, 0]), P)
    assert res[-1] is True and res[-2] == 0 and res[3].tolist() == [12, 12]


PINS = [pin_hand_example, pin_content_and_stack, pin_overflow]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(ost)


MUTATIONS = [
    ("append_tokens", "base = depth - total", "base = 0"),                                  # bottom of the stack
    ("append_tokens", "stack[base + offset + k]", "stack[base + total - 1 - offset - k]"),  # rows in reverse order
    ("pages_needed", "-(-(n + count) // page_size) - (-(-n // page_size))",
     "(n + count) // page_size - n // page_size"),                                         # floor instead of ceil
    ("append_tokens", "if total > depth:", "if total > depth + 1:"),                        # overflow off by one
]


@pytest.mark.parametrize("mut", MUTATIONS, ids=lambda m: m[0] + ":" + m[2][:24])
def test_planted_mistakes_are_caught(mut, monkeypatch):
    name, old, new = mut
    src = inspect.getsource(getattr(ost, name))
    assert old in src
    ns = dict(vars(ost))
    exec(compile(src.replace(old, new, 1), f"<mutant {name}>", "exec"), ns)
    monkeypatch.setattr(ost, name, ns[name])
    for k, v in vars(ost).items():
        if callable(v) and getattr(v, "__module__", None) == ost.__name__:
            ns[k] = getattr(ost, k)
    failed = []
    for pin in PINS:
        try:
            pin(ost)
        except Exception:
            failed.append(pin.__name__)
    assert failed, f"planted mistake in {name} was not caught"
