"""Beacon-query maintenance (online k-means; BeaconKV, Key ideas) on the GPU against the oracle: beacons and
counts must match bit for bit, since both sides take every decision in the same fp32 order."""
import numpy as np
import pytest
import torch

from agent_kv_cache_lse_b200 import kvc
from oracle import beacon as ob

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _clustered(gen, S, L, max_q, Hq, D, centers, spread, dtype):
    """Queries drawn around a few centres per group (seeded), in the query-set layout."""
    ctr = torch.randn((S, L, Hq, centers, D), generator=gen) * 3.0
    pick = torch.randint(0, centers, (S, L, max_q, Hq), generator=gen)
    q = torch.empty((S, L, max_q, Hq, D))
    for s in range(S):
        for l in range(L):
            for h in range(Hq):
                q[s, l, :, h] = ctr[s, l, h, pick[s, l, :, h]] + spread * torch.randn((max_q, D), generator=gen)
    return q.to(dtype)


def _oracle_round(c, n, q, num_q):
    S, L, max_q, Hq, D = q.shape
    qf = q.float().numpy()
    c2, n2 = c.copy(), n.copy()
    for s in range(S):
        m = min(max(int(num_q[s]), 0), max_q)
        for l in range(L):
            for h in range(Hq):
                c2[s, l, h], n2[s, l, h], _ = ob.beacon_update(c[s, l, h], n[s, l, h], qf[s, l, :m, h])
    return c2, n2


def _run(q, num_q, beacons, counts, beacon_q=None):
    st = torch.zeros(2, dtype=torch.int32, device=DEV)
    kvc.kvc_beacon_update(q.to(DEV), torch.tensor(num_q, dtype=torch.int32, device=DEV), beacons, counts, beacon_q, st)
    torch.cuda.synchronize()
    assert st.tolist() == [0, 0]


@pytest.mark.parametrize("dtype,D,B", [(torch.bfloat16, 128, 16), (torch.float32, 64, 64), (torch.float32, 37, 8)])
def test_rounds_match_oracle_bitwise(dtype, D, B):
    """Several rounds with state carried: uneven query counts (one below B, one zero), beacons exact.  A head size
    that is not a multiple of 4 takes the distance sums one dimension per load."""
    gen = torch.Generator().manual_seed(7)
    S, L, Hq, max_q = 3, 2, 4, 96
    beacons = torch.zeros((S, L, Hq, B, D), device=DEV)
    counts = torch.zeros((S, L, Hq, B), dtype=torch.int32, device=DEV)
    c = np.zeros((S, L, Hq, B, D), np.float32)
    n = np.zeros((S, L, Hq, B), np.int64)
    for rd, num_q in enumerate([[96, 7, 0], [40, 96, 33], [5, 0, 96], [96, 96, 96]]):
        q = _clustered(gen, S, L, max_q, Hq, D, centers=6, spread=0.7, dtype=dtype)
        _run(q, num_q, beacons, counts)
        c, n = _oracle_round(c, n, q, num_q)
        assert np.array_equal(counts.cpu().numpy(), n), f"round {rd}"
        got = beacons.cpu().numpy()
        assert np.array_equal(got.view(np.uint32), c.view(np.uint32)), \
            f"round {rd}: {np.max(np.abs(got - c))} max difference"


def test_beacon_query_output_and_clamping():
    """beacon_q receives the beacons (bf16, nearest even) in rows 0..B-1 and leaves the other rows alone;
    num_q above max_q is clamped, a negative one counts as zero."""
    gen = torch.Generator().manual_seed(11)
    S, L, Hq, D, B, max_q, out_q = 2, 1, 3, 128, 8, 40, 20
    q = _clustered(gen, S, L, max_q, Hq, D, centers=4, spread=0.5, dtype=torch.bfloat16)
    beacons = torch.zeros((S, L, Hq, B, D), device=DEV)
    counts = torch.zeros((S, L, Hq, B), dtype=torch.int32, device=DEV)
    out = torch.full((S, L, out_q, Hq, D), 7.0, dtype=torch.bfloat16, device=DEV)
    _run(q, [1000, -3], beacons, counts, out)
    c, n = _oracle_round(np.zeros((S, L, Hq, B, D), np.float32), np.zeros((S, L, Hq, B), np.int64), q, [max_q, 0])
    assert np.array_equal(beacons.cpu().numpy(), c) and np.array_equal(counts.cpu().numpy(), n)
    want = torch.from_numpy(c).permute(0, 1, 3, 2, 4).to(torch.bfloat16)      # [S][L][B][Hq][D]
    assert torch.equal(out[:, :, :B].cpu(), want)
    assert bool((out[:, :, B:] == 7.0).all())


def test_ties_and_duplicates():
    """Identical queries and identical beacons: the lower index wins, on both sides alike."""
    S, L, Hq, D, B, max_q = 1, 1, 1, 4, 4, 6
    q = torch.tensor([[1, 1, 1, 1], [1, 1, 1, 1], [2, 2, 2, 2], [1, 1, 1, 1], [2, 2, 2, 2], [0, 0, 0, 0]],
                     dtype=torch.float32).reshape(1, 1, max_q, 1, D)
    beacons = torch.zeros((S, L, Hq, B, D), device=DEV)
    counts = torch.zeros((S, L, Hq, B), dtype=torch.int32, device=DEV)
    _run(q, [max_q], beacons, counts)
    c, n = _oracle_round(np.zeros((S, L, Hq, B, D), np.float32), np.zeros((S, L, Hq, B), np.int64), q, [max_q])
    assert np.array_equal(beacons.cpu().numpy(), c) and np.array_equal(counts.cpu().numpy(), n)
    assert n[0, 0, 0].tolist() == [4, 0, 2, 0]   # duplicate seeds 1 and 3 lose their ties to beacon 0


@pytest.mark.parametrize("max_q,D,B", [(1000, 128, 16), (9000, 32, 8)])
def test_large_batches_match_oracle(max_q, D, B):
    """More queries than fit in shared memory (rounds staged one at a time), and more than the per-beacon lists
    hold (the update scans the assignments instead): the same bits as the oracle."""
    gen = torch.Generator().manual_seed(13)
    S, L, Hq = 1, 1, 2
    q = _clustered(gen, S, L, max_q, Hq, D, centers=5, spread=0.8, dtype=torch.bfloat16)
    beacons = torch.zeros((S, L, Hq, B, D), device=DEV)
    counts = torch.zeros((S, L, Hq, B), dtype=torch.int32, device=DEV)
    c = np.zeros((S, L, Hq, B, D), np.float32)
    n = np.zeros((S, L, Hq, B), np.int64)
    for num_q in ([max_q], [max_q // 3]):
        _run(q, num_q, beacons, counts)
        c, n = _oracle_round(c, n, q, num_q)
        assert np.array_equal(counts.cpu().numpy(), n)
        assert np.array_equal(beacons.cpu().numpy().view(np.uint32), c.view(np.uint32))
