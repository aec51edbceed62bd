"""Streaming new tokens into a compacted cache: kvc_append_tokens against the oracle (oracle.stream), bit for bit.

"KV-streams for Efficient Compaction in Agentic Reinforcement Learning" (abstract): the compacted cache is
carried forward and new tokens stream into it, with pages from the free list.  Rows of lengths at and around
page boundaries, several token counts, a permuted pool; the whole pool, block table, lengths, positions,
labels, LRFU values and stack depth must equal the oracle's.  A stack too shallow changes nothing.
"""
import numpy as np
import pytest
import torch

from agent_kv_cache_lse_b200 import kvc
from oracle import stream as ost

pytestmark = pytest.mark.gpu
DEV = "cuda"
P = 16


def _cache(lengths, max_slots, num_pages, seed, D=128, S=None):
    rows = len(lengths)
    S = S or rows
    mp = -(-max_slots // P)
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    bt = torch.full((rows, mp), -1, dtype=torch.int32)
    used = 0
    for r, n in enumerate(lengths):
        k = -(-n // P)
        bt[r, :k] = perm[used:used + k]
        used += k
    stack = perm[used:].clone()
    kp = torch.randint(-30000, 30000, (num_pages, P, D), dtype=torch.int16, generator=g).view(torch.bfloat16)
    vp = torch.randint(-30000, 30000, (num_pages, P, D), dtype=torch.int16, generator=g).view(torch.bfloat16)
    pos = torch.randint(0, 1 << 20, (rows, mp * P), dtype=torch.int32, generator=g)
    lab = torch.randint(0, 3, (rows, mp * P), dtype=torch.uint8, generator=g)
    cache = kvc.Cache(kp.to(DEV), vp.to(DEV), bt.to(DEV), torch.tensor(lengths, dtype=torch.int32).to(DEV),
                      pos.to(DEV), lab.to(DEV), S, 1, rows // S)
    return cache, stack


@pytest.mark.parametrize("count", [1, 16, 37, 64])
def test_append_parity(count):
    lengths = [0, 1, 15, 16, 17, 100, 255, 256, 4000, 30000, 33]
    rows = len(lengths)
    max_slots = 30000 + 128
    num_pages = sum(-(-n // P) for n in lengths) + rows * (-(-count // P) + 1) + 7
    cache, stack = _cache(lengths, max_slots, num_pages, seed=count)
    g = torch.Generator().manual_seed(100 + count)
    k_new = torch.randint(-30000, 30000, (rows, count, 128), dtype=torch.int16, generator=g).view(torch.bfloat16)
    v_new = torch.randint(-30000, 30000, (rows, count, 128), dtype=torch.int16, generator=g).view(torch.bfloat16)
    new_pos = torch.randint(1 << 20, 1 << 21, (rows, count), dtype=torch.int32, generator=g)
    crf = torch.rand((rows, cache.max_slots), generator=g)
    host = dict(k=cache.k_pool.cpu().view(torch.int16).numpy(), v=cache.v_pool.cpu().view(torch.int16).numpy(),
                bt=cache.block_table.cpu().numpy(), rl=cache.row_len.cpu().numpy(), sp=cache.slot_pos.cpu().numpy(),
                sl=cache.slot_label.cpu().numpy(), crf=crf.numpy().copy())
    pages = torch.full((num_pages,), -1, dtype=torch.int32)
    pages[:len(stack)] = stack
    depth = torch.tensor([len(stack)], dtype=torch.int64)
    ws = torch.zeros(kvc.kvc_append_workspace_bytes(rows) // 8, dtype=torch.int64, device=DEV)
    status = torch.zeros(2, dtype=torch.int32, device=DEV)
    crf_d = crf.to(DEV)
    pages_d, depth_d = pages.to(DEV), depth.to(DEV)
    kvc.kvc_append_tokens(cache, k_new.to(DEV), v_new.to(DEV), new_pos.to(DEV), 2, crf_d, pages_d, depth_d, ws, status)
    torch.cuda.synchronize()
    assert kvc.device_status(status)[0] == 0, kvc.device_status(status)
    want = ost.append_tokens(host["k"], host["v"], host["bt"], host["rl"], host["sp"], host["sl"], host["crf"],
                             pages.numpy(), len(stack), k_new.view(torch.int16).numpy(), v_new.view(torch.int16).numpy(),
                             new_pos.numpy(), 2, np.arange(rows), P)
    k2, v2, bt2, rl2, sp2, sl2, crf2, depth2, ok = want
    assert ok
    assert np.array_equal(cache.k_pool.cpu().view(torch.int16).numpy(), k2)
    assert np.array_equal(cache.v_pool.cpu().view(torch.int16).numpy(), v2)
    assert np.array_equal(cache.block_table.cpu().numpy(), bt2)
    assert np.array_equal(cache.row_len.cpu().numpy(), rl2)
    assert np.array_equal(cache.slot_pos.cpu().numpy(), sp2)
    assert np.array_equal(cache.slot_label.cpu().numpy(), sl2)
    assert np.array_equal(crf_d.cpu().numpy(), crf2)
    assert int(depth_d[0]) == depth2


def test_append_stack_too_shallow_changes_nothing():
    lengths = [16, 16]
    cache, stack = _cache(lengths, 64, 4, seed=9)
    k_new = torch.zeros((2, 40, 128), dtype=torch.bfloat16, device=DEV)
    new_pos = torch.zeros((2, 40), dtype=torch.int32, device=DEV)
    pages = stack.to(DEV)
    depth = torch.tensor([len(stack)], dtype=torch.int64, device=DEV)
    ws = torch.zeros(kvc.kvc_append_workspace_bytes(2) // 8, dtype=torch.int64, device=DEV)
    status = torch.zeros(2, dtype=torch.int32, device=DEV)
    bt0, k0 = cache.block_table.cpu().clone(), cache.k_pool.cpu().clone()
    kvc.kvc_append_tokens(cache, k_new, k_new, new_pos, 1, None, pages, depth, ws, status)
    torch.cuda.synchronize()
    assert kvc.device_status(status)[:2] == (5, -1)
    assert torch.equal(cache.block_table.cpu(), bt0) and torch.equal(cache.k_pool.cpu().view(torch.int16),
                                                                      k0.view(torch.int16))
    assert cache.row_len.cpu().tolist() == [16, 16] and int(depth[0]) == len(stack)
