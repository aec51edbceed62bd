"""The compaction entry point that allocates nothing, against the regular one.

Some callers cannot allocate device memory when they compact: engines whose allocator has
handed all free memory to the KV pool, or foreign-function callers with no access to the host
framework's allocator.  For them
kvc_compact_pages_noalloc keeps its workspace in an array inside the library.  This test
calls both entry points through the C ABI on identical copies of a cache and requires the
same results (compaction is bit-exact), on two calls in a row so that whatever the first
call left in the built-in array cannot leak into the second.  It lives in its own file,
collected last, and also passes when run alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from agent_kv_cache_lse_b200 import kvc

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cache(lengths, max_slots, seed, P=16, D=128):
    rows = len(lengths)
    mp = -(-max_slots // P)
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(rows * mp, generator=g).to(torch.int32)
    bt = torch.full((rows, mp), -1, dtype=torch.int32)
    for r, n in enumerate(lengths):
        bt[r, :-(-n // P)] = perm[r * mp:r * mp + -(-n // P)]
    kp = torch.randint(-30000, 30000, (rows * mp, P, D), dtype=torch.int16, generator=g).view(torch.bfloat16)
    vp = torch.randint(-30000, 30000, (rows * mp, P, D), dtype=torch.int16, generator=g).view(torch.bfloat16)
    pos = torch.stack([torch.randperm(mp * P, generator=g) for _ in range(rows)]).to(torch.int32)
    lab = torch.randint(0, 3, (rows, mp * P), dtype=torch.uint8, generator=g)
    rl = torch.tensor(lengths, dtype=torch.int32)
    keep = (torch.rand((rows, mp * P), generator=g) < 0.3).to(torch.uint8)
    for r, n in enumerate(lengths):
        keep[r, n:] = 0
    return dict(k=kp, v=vp, bt=bt, rl=rl, pos=pos, lab=lab, keep=keep)


def _device_copy(h, rows):
    return kvc.Cache(h["k"].to(DEV), h["v"].to(DEV), h["bt"].to(DEV), h["rl"].to(DEV), h["pos"].to(DEV),
                     h["lab"].to(DEV), rows, 1, 1)


def _plan(c, keep):
    rows, ms = keep.shape
    kept = keep.sum(dim=1).to(torch.int32).to(DEV)
    src = torch.zeros((rows, ms), dtype=torch.int32, device=DEV)
    dst = torch.zeros_like(src)
    nm = torch.zeros(rows, dtype=torch.int32, device=DEV)
    kvc.kvc_plan_slots(c, keep.to(DEV), kept, src, dst, nm)
    return src, dst, nm, kept


@pytest.mark.parametrize("call", [0, 1])
def test_noalloc_matches_regular_compaction(call):
    for rep, seed in enumerate((101 + call, 202 + call)):          # two calls in a row
        lengths = [4097, 33000, 16, 1, 0, 257][: 6 - rep]
        ms = 33008
        h = _cache(lengths, ms, seed)
        rows = len(lengths)
        a, b = _device_copy(h, rows), _device_copy(h, rows)
        src, dst, nm, kept = _plan(a, h["keep"])
        crf0 = torch.rand((rows, ms), generator=torch.Generator().manual_seed(seed)).to(DEV)
        crf_a, crf_b = crf0.clone(), crf0.clone()
        cap = rows * (ms // 16)
        fa = torch.full((cap,), -3, dtype=torch.int32, device=DEV)
        fb = fa.clone()
        na = torch.zeros(1, dtype=torch.int64, device=DEV)
        nb = na.clone()
        sa = torch.zeros(2, dtype=torch.int32, device=DEV)
        sb = sa.clone()
        ws = torch.zeros(kvc.kvc_compact_workspace_bytes(rows) // 8 + 1, dtype=torch.int64, device=DEV)
        kvc.kvc_compact_pages(a, src, dst, nm, kept, crf_a, fa, na, ws, sa)
        kvc.kvc_compact_pages_noalloc(b, src, dst, nm, kept, crf_b, fb, nb, sb)
        torch.cuda.synchronize()
        assert kvc.device_status(sa)[0] == 0 and kvc.device_status(sb)[0] == 0
        for x, y in ((a.k_pool, b.k_pool), (a.v_pool, b.v_pool)):
            assert torch.equal(x.view(torch.int16), y.view(torch.int16))
        for x, y in ((a.block_table, b.block_table), (a.row_len, b.row_len), (a.slot_pos, b.slot_pos),
                     (a.slot_label, b.slot_label), (crf_a, crf_b), (na, nb), (fa, fb)):
            assert torch.equal(x, y)
        assert int(na[0]) > 0


def test_noalloc_rejects_too_many_rows():
    c = kvc.Cache(torch.zeros((1, 16, 128), dtype=torch.bfloat16, device=DEV),
                  torch.zeros((1, 16, 128), dtype=torch.bfloat16, device=DEV),
                  torch.zeros((kvc.NOALLOC_MAX_ROWS + 1, 1), dtype=torch.int32, device=DEV),
                  torch.zeros(kvc.NOALLOC_MAX_ROWS + 1, dtype=torch.int32, device=DEV),
                  torch.zeros((kvc.NOALLOC_MAX_ROWS + 1, 16), dtype=torch.int32, device=DEV), None,
                  kvc.NOALLOC_MAX_ROWS + 1, 1, 1)
    z = torch.zeros(kvc.NOALLOC_MAX_ROWS + 1, dtype=torch.int32, device=DEV)
    with pytest.raises(kvc.KvcError, match="at most"):
        kvc.kvc_compact_pages_noalloc(c, z, z, z, z, None, z, torch.zeros(1, dtype=torch.int64, device=DEV))
