"""Step-isolated parity: each CUDA entry point against the oracle on identical seeded inputs.

Tolerances: scores 1e-6 absolute + 1e-3 relative (fp32); LRFU values to fp32 rounding
(2e-6 relative); selection, slot plan, block table, freed list and the compacted pools
bit-exact; the LSE pass (a stand-in for the attention kernel's byproduct) within
5e-5 absolute; per-step confidence within 3e-5 absolute (fp32 log-sum-exp over the
vocabulary against fp64).
"""
import math

import numpy as np
import pytest
import torch

from agent_kv_cache_lse_b200 import kvc, synth
from oracle import cache as ocache
from oracle import path as opath

from . import helpers as H

pytestmark = pytest.mark.gpu

DEV = "cuda"
HIT = float(np.float32(0.9))   # the fp32 value both sides use


def small_spec(name="small", seed=11, S=1, L=1, Hq=32, Hkv=8, D=128, ctx=(4096 + 99,), budget=512, queries="action",
               dtype="bf16", heavy=0.02):
    return synth.Spec(name=name, seed=seed, num_seqs=S, num_layers=L, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                      dtype=dtype, ctx=list(ctx), budget=budget, heavy_frac=heavy, queries=queries)


# ----------------------------------------------------------------------------- scoring

SCORE_CASES = {
    "llama8b_shape_ragged": dict(ctx=(4096 + 99,)),
    "multi_seq_layer": dict(S=3, L=2, ctx=(1500, 2817, 4000), seed=12),
    "gqa7_beacons": dict(Hq=28, Hkv=4, ctx=(2100,), queries="beacon_recent", seed=13, heavy=0.0),
    "d64": dict(D=64, Hq=8, Hkv=2, ctx=(3000,), seed=14),
    "short_rows": dict(S=2, ctx=(17, 300), seed=15),
}


@pytest.mark.parametrize("case", list(SCORE_CASES), ids=list(SCORE_CASES))
@pytest.mark.parametrize("path", ["tensor", "simt"])
def test_score_parity(case, path):
    spec = small_spec(**SCORE_CASES[case])
    w = H.build(spec)
    lse64 = H.oracle_lse(w)
    H.set_lse(w, lse64)
    scores = torch.full((spec.rows, spec.max_slots), -7.0, device=DEV)
    status = torch.zeros(2, dtype=torch.int32, device=DEV)
    flags = kvc.KVC_SCORE_SIMT if path == "simt" else 0
    kvc.kvc_score_from_lse(w.cache, w.queries, scores, flags, status)
    torch.cuda.synchronize()
    assert kvc.device_status(status)[0] == 0
    orc = H.oracle_scores(w, lse64.astype(np.float32))
    got = scores.cpu().numpy()
    rl = w.layout.row_len.numpy()
    for r in range(spec.rows):
        n = int(rl[r])
        H.assert_scores_close(got[r, :n], orc[r], f"{case} row {r}")
        assert np.all(got[r, n:] == -7.0), "slots beyond the row length must not be written"


def test_score_accumulate_and_lse_flag():
    spec = small_spec(ctx=(1200,), seed=16)
    w = H.build(spec)
    lse64 = H.oracle_lse(w)
    H.set_lse(w, lse64)
    s1 = torch.zeros((spec.rows, spec.max_slots), device=DEV)
    kvc.kvc_score_from_lse(w.cache, w.queries, s1, 0)
    s2 = s1.clone()
    kvc.kvc_score_from_lse(w.cache, w.queries, s2, kvc.KVC_SCORE_ACCUMULATE)
    torch.cuda.synchronize()
    torch.testing.assert_close(s2, 2 * s1, rtol=1e-6, atol=0)
    # COMPUTE_LSE: the library's own LSE pass, then scoring with it
    w.queries.lse.fill_(123.0)
    s3 = torch.zeros_like(s1)
    kvc.kvc_score_from_lse(w.cache, w.queries, s3, kvc.KVC_SCORE_COMPUTE_LSE)
    torch.cuda.synchronize()
    orc = H.oracle_scores(w, lse64.astype(np.float32))
    for r in range(spec.rows):
        n = int(w.layout.row_len[r])
        H.assert_scores_close(s3.cpu().numpy()[r, :n], orc[r], "compute-lse")


@pytest.mark.parametrize("case", ["llama8b_shape_ragged", "gqa7_beacons", "multi_seq_layer"])
def test_query_lse_parity(case):
    spec = small_spec(**SCORE_CASES[case])
    w = H.build(spec)
    lse64 = H.oracle_lse(w)
    status = torch.zeros(2, dtype=torch.int32, device=DEV)
    kvc.kvc_query_lse(w.cache, w.queries, status)
    torch.cuda.synchronize()
    assert kvc.device_status(status)[0] == 0
    got = w.queries.lse.cpu().numpy().astype(np.float64)
    for s in range(spec.num_seqs):
        nq = int(w.queries.num_q[s])
        a, b = got[s, :, :, :nq], lse64[s, :, :, :nq]
        assert np.array_equal(np.isinf(a), np.isinf(b))
        fin = np.isfinite(b)
        assert np.max(np.abs(a[fin] - b[fin])) < 5e-5


# ----------------------------------------------------------------------------- a bare cache for the row steps

def bare_cache(lengths, max_slots, S=None, L=1, P=16, D=128, num_pages=None, seed=0):
    rows = len(lengths)
    S = S or rows
    Hkv = rows // (S * L)
    mp = -(-max_slots // P)
    npages = num_pages or rows * mp
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(npages, generator=g).to(torch.int32)
    bt = torch.full((rows, mp), -1, dtype=torch.int32)
    for r, n in enumerate(lengths):
        k = -(-n // P)
        bt[r, :k] = perm[r * mp:r * mp + k]
    kp = torch.randint(-30000, 30000, (npages, P, D), dtype=torch.int16, generator=g).view(torch.bfloat16)
    vp = torch.randint(-30000, 30000, (npages, P, D), dtype=torch.int16, generator=g).view(torch.bfloat16)
    pos = torch.stack([torch.randperm(mp * P, generator=g) for _ in range(rows)]).to(torch.int32)
    lab = torch.randint(0, 3, (rows, mp * P), dtype=torch.uint8, generator=g)
    rl = torch.tensor(lengths, dtype=torch.int32)
    return kvc.Cache(kp.to(DEV), vp.to(DEV), bt.to(DEV), rl.to(DEV), pos.to(DEV), lab.to(DEV), S, L, Hkv)


def _row_values(rng, n, mode):
    if mode == "lognormal":
        return np.exp(rng.standard_normal(n) * 2).astype(np.float32)
    if mode == "ties":                   # quantised to 2^-10 with k in 0..63
        return (rng.integers(0, 64, n) * 2.0**-10).astype(np.float32)
    if mode == "sparse":
        v = np.exp(rng.standard_normal(n)).astype(np.float32)
        v[rng.random(n) < 0.7] = 0
        return v
    if mode == "equal":
        return np.full(n, 0.25, dtype=np.float32)
    raise ValueError(mode)


# ----------------------------------------------------------------------------- select

@pytest.mark.parametrize("mode", ["lognormal", "ties", "sparse", "equal"])
def test_select_parity(mode):
    rng = np.random.default_rng(21)
    lengths = [0, 1, 15, 16, 17, 255, 256, 1000, 4096 + 5, 33000]
    ms = 33008
    c = bare_cache(lengths, ms, S=len(lengths))
    crf = np.zeros((len(lengths), ms), dtype=np.float32)
    for r, n in enumerate(lengths):
        crf[r, :n] = _row_values(rng, n, mode)
    budgets = np.array([5, 0, 7, 16, 3, 100, 300, 512, 2048, 30000], dtype=np.int32)
    keep = torch.full((len(lengths), ms), 9, dtype=torch.uint8, device=DEV)
    kept = torch.zeros(len(lengths), dtype=torch.int32, device=DEV)
    kvc.kvc_select_budget(c, torch.from_numpy(crf).to(DEV), torch.from_numpy(budgets).to(DEV), keep, kept)
    torch.cuda.synchronize()
    pos = c.slot_pos.cpu().numpy()
    got = keep.cpu().numpy()
    for r, n in enumerate(lengths):
        ok = opath.select_budget(crf[r, :n].astype(np.float64), pos[r, :n], int(budgets[r]))
        assert np.array_equal(got[r, :n].astype(bool), ok), f"row {r} (n={n})"
        assert int(kept[r]) == int(ok.sum())
        assert np.all(got[r, n:] == 9)


def test_select_protected_labels():
    rng = np.random.default_rng(22)
    lengths = [3000, 700]
    c = bare_cache(lengths, 3008, S=2)
    crf = np.zeros((2, 3008), dtype=np.float32)
    for r, n in enumerate(lengths):
        crf[r, :n] = _row_values(rng, n, "ties")
    budgets = torch.tensor([400, 100], dtype=torch.int32, device=DEV)
    keep = torch.zeros((2, 3008), dtype=torch.uint8, device=DEV)
    kept = torch.zeros(2, dtype=torch.int32, device=DEV)
    kvc.kvc_select_budget(c, torch.from_numpy(crf).to(DEV), budgets, keep, kept, protect_label_mask=1 << 2)
    torch.cuda.synchronize()
    pos, lab = c.slot_pos.cpu().numpy(), c.slot_label.cpu().numpy()
    for r, n in enumerate(lengths):
        ok = opath.select_budget(crf[r, :n].astype(np.float64), pos[r, :n], int(budgets[r]), lab[r, :n], 1 << 2)
        assert np.array_equal(keep.cpu().numpy()[r, :n].astype(bool), ok)


# ----------------------------------------------------------------------------- LRFU

@pytest.mark.parametrize("mode", ["lognormal", "ties", "sparse", "equal"])
@pytest.mark.parametrize("variant", ["gate", "binary", "gate_off", "dt3"])
def test_lrfu_parity(mode, variant):
    rng = np.random.default_rng(31)
    lengths = [0, 1, 16, 257, 5000, 33000]
    ms = 33008
    c = bare_cache(lengths, ms, S=len(lengths))
    s = np.zeros((len(lengths), ms), dtype=np.float32)
    crf0 = np.zeros((len(lengths), ms), dtype=np.float32)
    for r, n in enumerate(lengths):
        s[r, :n] = _row_values(rng, n, mode)
        crf0[r, :n] = (rng.random(n) * 3).astype(np.float32)
    crf0[:, -3:] = 5.5
    hit = 1.0 if variant == "gate_off" else HIT
    dt = 3 if variant == "dt3" else 1
    binary = variant == "binary"
    crf = torch.from_numpy(crf0.copy()).to(DEV)
    kvc.kvc_lrfu_update(c, torch.from_numpy(s).to(DEV), crf, 0.5, hit, dt, kvc.KVC_HIT_BINARY if binary else 0)
    torch.cuda.synchronize()
    got = crf.cpu().numpy().astype(np.float64)
    pos = c.slot_pos.cpu().numpy()
    for r, n in enumerate(lengths):
        sr = s[r, :n].astype(np.float64)
        want = opath.lrfu_update(crf0[r, :n].astype(np.float64), sr, pos[r, :n], 0.5, hit, dt, binary)
        gate = opath.hit_gate(sr, pos[r, :n], hit)
        tau = sr[gate].min() if gate.any() else 0.0
        err = np.abs(got[r, :n] - want)
        bad = err > 2e-6 * np.abs(want) + 1e-30
        near = np.abs(sr - tau) <= 1e-4 * tau
        assert np.all(near[bad]), f"row {r}: {int(bad.sum())} LRFU values differ away from the gate threshold"
        assert np.all(got[r, n:] == crf0[r, n:].astype(np.float64))


# ----------------------------------------------------------------------------- plan + compaction

@pytest.mark.parametrize("mode", ["lognormal", "ties", "sparse", "equal"])
def test_lrfu_select_fused_matches_separate(mode):
    """kvc_lrfu_select equals kvc_lrfu_update then kvc_select_budget: LRFU values bit for bit, the same keep
    mask and counts, with protected labels; and the selection it makes equals the oracle's on those values."""
    rng = np.random.default_rng(41)
    lengths = [0, 1, 16, 257, 5000, 33000]
    ms = 33008
    c = bare_cache(lengths, ms, S=len(lengths))
    s = np.zeros((len(lengths), ms), dtype=np.float32)
    crf0 = np.zeros((len(lengths), ms), dtype=np.float32)
    for r, n in enumerate(lengths):
        s[r, :n] = _row_values(rng, n, mode)
        crf0[r, :n] = _row_values(rng, n, mode)
    budgets = torch.tensor([3, 0, 5, 100, 512, 2048], dtype=torch.int32, device=DEV)
    sd = torch.from_numpy(s).to(DEV)
    outs = []
    for fused in (False, True):
        crf = torch.from_numpy(crf0.copy()).to(DEV)
        keep = torch.full((len(lengths), ms), 9, dtype=torch.uint8, device=DEV)
        kept = torch.zeros(len(lengths), dtype=torch.int32, device=DEV)
        st = torch.zeros(2, dtype=torch.int32, device=DEV)
        if fused:
            kvc.kvc_lrfu_select(c, sd, crf, budgets, keep, kept, 0.5, HIT, 1, 0, 1 << 2, st)
        else:
            kvc.kvc_lrfu_update(c, sd, crf, 0.5, HIT, 1, 0, st)
            kvc.kvc_select_budget(c, crf, budgets, keep, kept, 1 << 2, st)
        torch.cuda.synchronize()
        outs.append((crf.cpu().numpy(), keep.cpu().numpy(), kept.cpu().numpy(), st.cpu().tolist()))
    (c0, k0, n0, s0), (c1, k1, n1, s1) = outs
    assert np.array_equal(c0.view(np.uint32), c1.view(np.uint32))
    assert np.array_equal(k0, k1) and np.array_equal(n0, n1) and s0 == s1 == [0, 0]
    pos, lab = c.slot_pos.cpu().numpy(), c.slot_label.cpu().numpy()
    for r, n in enumerate(lengths):
        ok = opath.select_budget(c1[r, :n].astype(np.float64), pos[r, :n], int(budgets[r]), lab[r, :n], 1 << 2)
        assert np.array_equal(k1[r, :n].astype(bool), ok), f"row {r}"


@pytest.mark.parametrize("mode", ["lognormal", "ties", "equal"])
def test_select_plan_fused_matches_separate(mode):
    """kvc_select_plan equals kvc_select_budget then kvc_plan_slots: the same keep mask, counts, move lists and
    move counts, with protected labels; and the plan it makes equals the oracle's on that mask."""
    rng = np.random.default_rng(43)
    lengths = [0, 1, 16, 257, 5000, 33000]
    ms = 33008
    c = bare_cache(lengths, ms, S=len(lengths))
    crf0 = np.zeros((len(lengths), ms), dtype=np.float32)
    for r, n in enumerate(lengths):
        crf0[r, :n] = _row_values(rng, n, mode)
    budgets = torch.tensor([3, 0, 5, 100, 512, 2048], dtype=torch.int32, device=DEV)
    crf = torch.from_numpy(crf0).to(DEV)
    outs = []
    for fused in (False, True):
        keep = torch.full((len(lengths), ms), 9, dtype=torch.uint8, device=DEV)
        kept = torch.zeros(len(lengths), dtype=torch.int32, device=DEV)
        src = torch.full((len(lengths), ms), -7, dtype=torch.int32, device=DEV)
        dst = torch.full((len(lengths), ms), -7, dtype=torch.int32, device=DEV)
        nm = torch.full((len(lengths),), -7, dtype=torch.int32, device=DEV)
        st = torch.zeros(2, dtype=torch.int32, device=DEV)
        if fused:
            kvc.kvc_select_plan(c, crf, budgets, keep, kept, src, dst, nm, 1 << 2, st)
        else:
            kvc.kvc_select_budget(c, crf, budgets, keep, kept, 1 << 2, st)
            kvc.kvc_plan_slots(c, keep, kept, src, dst, nm, st)
        torch.cuda.synchronize()
        outs.append([t.cpu().numpy() for t in (keep, kept, src, dst, nm)] + [st.cpu().tolist()])
    for a, b in zip(outs[0][:5], outs[1][:5]):
        assert np.array_equal(a, b)
    assert outs[0][5] == outs[1][5] == [0, 0]
    keep, kept, src, dst, nm = outs[1][:5]
    for r, n in enumerate(lengths):
        want_src, want_dst, m = opath.plan_slots(keep[r, :n].astype(bool), n)
        assert int(nm[r]) == len(want_src) and int(kept[r]) == m
        assert np.array_equal(src[r, :len(want_src)], want_src) and np.array_equal(dst[r, :len(want_dst)], want_dst)


def _masks(rng, lengths, mode):
    keeps = []
    for n in lengths:
        if mode == "random":
            k = rng.random(n) < rng.random()
        elif mode == "all":
            k = np.ones(n, bool)
        elif mode == "none":
            k = np.zeros(n, bool)
        else:  # tail-heavy: survivors skew to the tail, as the pages note for agent traces
            k = rng.random(n) < np.linspace(0.05, 0.9, n) if n else np.zeros(0, bool)
        keeps.append(k)
    return keeps


@pytest.mark.parametrize("mode", ["random", "all", "none", "tail"])
@pytest.mark.parametrize("D", [128, 64])
def test_plan_compact_parity(mode, D):
    rng = np.random.default_rng(41 + D)
    lengths = [0, 1, 15, 16, 17, 100, 257, 4096, 33000]
    ms = 33008
    c = bare_cache(lengths, ms, S=len(lengths), D=D)
    keeps = _masks(rng, lengths, mode)
    keep = np.zeros((len(lengths), ms), dtype=np.uint8)
    for r, k in enumerate(keeps):
        keep[r, :len(k)] = k
    kept = keep.sum(axis=1).astype(np.int32)
    rows = len(lengths)
    src = torch.full((rows, ms), -5, dtype=torch.int32, device=DEV)
    dst = torch.full((rows, ms), -5, dtype=torch.int32, device=DEV)
    nm = torch.zeros(rows, dtype=torch.int32, device=DEV)
    status = torch.zeros(2, dtype=torch.int32, device=DEV)
    kvc.kvc_plan_slots(c, torch.from_numpy(keep).to(DEV), torch.from_numpy(kept).to(DEV), src, dst, nm, status)
    torch.cuda.synchronize()
    assert kvc.device_status(status)[0] == 0
    geo = ocache.Geometry(rows, 1, 1, 1, 16)
    plans = ocache.plan_cache(geo, keep, np.array(lengths))
    osrc = np.full((rows, ms), 0, dtype=np.int32)
    odst = np.full((rows, ms), 0, dtype=np.int32)
    onm = np.zeros(rows, dtype=np.int32)
    gs, gd = src.cpu().numpy(), dst.cpu().numpy()
    for r in range(rows):
        a, b, m = plans[r]
        assert int(nm[r]) == len(a)
        assert np.array_equal(gs[r, :len(a)], a) and np.array_equal(gd[r, :len(b)], b)
        osrc[r, :len(a)], odst[r, :len(b)], onm[r] = a, b, len(a)
    # compaction from the oracle's plan on both sides; everything bit-exact
    crf0 = rng.random((rows, ms)).astype(np.float32)
    host_k = c.k_pool.cpu().view(torch.int16).numpy()
    host_v = c.v_pool.cpu().view(torch.int16).numpy()
    bt0, rl0 = c.block_table.cpu().numpy(), c.row_len.cpu().numpy()
    sp0, sl0 = c.slot_pos.cpu().numpy(), c.slot_label.cpu().numpy()
    crf = torch.from_numpy(crf0).to(DEV)
    freed = torch.full((rows * (ms // 16),), -9, dtype=torch.int32, device=DEV)
    nfreed = torch.zeros(1, dtype=torch.int64, device=DEV)
    ws = torch.zeros(kvc.kvc_compact_workspace_bytes(rows) // 8 + 1, dtype=torch.int64, device=DEV)
    kvc.kvc_compact_pages(c, torch.from_numpy(osrc).to(DEV), torch.from_numpy(odst).to(DEV),
                          torch.from_numpy(onm).to(DEV), torch.from_numpy(kept).to(DEV), crf, freed, nfreed, ws,
                          status)
    torch.cuda.synchronize()
    assert kvc.device_status(status)[0] == 0
    k2, v2, bt2, rl2, sp2, sl2, cr2, fr2 = ocache.compact_cache(geo, host_k, host_v, bt0, rl0, sp0, sl0,
                                                                crf0, plans)
    assert np.array_equal(c.k_pool.cpu().view(torch.int16).numpy(), k2)
    assert np.array_equal(c.v_pool.cpu().view(torch.int16).numpy(), v2)
    assert np.array_equal(c.block_table.cpu().numpy(), bt2)
    assert np.array_equal(c.row_len.cpu().numpy(), rl2)
    assert np.array_equal(c.slot_pos.cpu().numpy(), sp2)
    assert np.array_equal(c.slot_label.cpu().numpy(), sl2)
    assert np.array_equal(crf.cpu().numpy(), cr2)
    assert int(nfreed[0]) == len(fr2)
    assert np.array_equal(freed.cpu().numpy()[:len(fr2)], fr2)
    # pages freed per row: ceil(n/P) - ceil(m/P)
    assert len(fr2) == sum(-(-n // 16) - (-(-int(m) // 16)) for n, m in zip(lengths, kept))


def test_compact_freed_overflow_keeps_pages():
    lengths = [64, 64]
    c = bare_cache(lengths, 64, S=2)
    keep = np.zeros((2, 64), dtype=np.uint8)
    keep[:, :16] = 1
    kept = np.array([16, 16], dtype=np.int32)
    z = torch.zeros((2, 64), dtype=torch.int32, device=DEV)
    nm = torch.zeros(2, dtype=torch.int32, device=DEV)
    freed = torch.full((4,), -1, dtype=torch.int32, device=DEV)   # row 0 frees 3 pages, row 1 would need 3 more
    nfreed = torch.zeros(1, dtype=torch.int64, device=DEV)
    ws = torch.zeros(8, dtype=torch.int64, device=DEV)
    status = torch.zeros(2, dtype=torch.int32, device=DEV)
    bt0 = c.block_table.cpu().numpy().copy()
    kvc.kvc_compact_pages(c, z, z, nm, torch.from_numpy(kept).to(DEV), None, freed, nfreed, ws, status)
    torch.cuda.synchronize()
    assert kvc.device_status(status)[0] == 5
    assert int(nfreed[0]) == 6
    assert freed.cpu().tolist()[:3] == bt0[0, 1:4].tolist()
    assert np.array_equal(c.block_table.cpu().numpy()[1], bt0[1])      # row 1 keeps its pages
    assert c.row_len.cpu().tolist() == [16, 16]


def test_plan_mismatch_leaves_row_untouched():
    """A row whose kept count disagrees with its keep mask is reported (kept mismatch), gets num_moves = -1 and is
    left exactly as it was by the compaction: block table, row_len, positions and pool bytes; the consistent row
    beside it is compacted as usual."""
    lengths = [64, 64]
    c = bare_cache(lengths, 64, S=2)
    keep = np.zeros((2, 64), dtype=np.uint8)
    keep[0, 40:56] = 1
    keep[1, 30:50] = 1
    kept = np.array([16, 16], dtype=np.int32)          # row 1's mask holds 20 entries
    src = torch.zeros((2, 64), dtype=torch.int32, device=DEV)
    dst = torch.zeros((2, 64), dtype=torch.int32, device=DEV)
    nm = torch.zeros(2, dtype=torch.int32, device=DEV)
    status = torch.zeros(2, dtype=torch.int32, device=DEV)
    kd = torch.from_numpy(kept).to(DEV)
    bt0, rl0, sp0 = c.block_table.cpu().numpy().copy(), c.row_len.cpu().numpy().copy(), c.slot_pos.cpu().numpy().copy()
    k0 = c.k_pool.cpu().view(torch.int16).numpy().copy()
    v0 = c.v_pool.cpu().view(torch.int16).numpy().copy()
    kvc.kvc_plan_slots(c, torch.from_numpy(keep).to(DEV), kd, src, dst, nm, status)
    freed = torch.full((16,), -1, dtype=torch.int32, device=DEV)
    nfreed = torch.zeros(1, dtype=torch.int64, device=DEV)
    ws = torch.zeros(8, dtype=torch.int64, device=DEV)
    kvc.kvc_compact_pages(c, src, dst, nm, kd, None, freed, nfreed, ws, status)
    torch.cuda.synchronize()
    assert kvc.device_status(status)[:2] == (4, 1)
    assert nm.cpu().tolist() == [16, -1]
    bt1 = c.block_table.cpu().numpy()
    assert np.array_equal(bt1[1], bt0[1]) and int(c.row_len[1]) == 64
    assert np.array_equal(c.slot_pos.cpu().numpy()[1], sp0[1])
    pages1 = bt0[1, :4].astype(np.int64)
    assert np.array_equal(c.k_pool.cpu().view(torch.int16).numpy()[pages1], k0[pages1])
    assert np.array_equal(c.v_pool.cpu().view(torch.int16).numpy()[pages1], v0[pages1])
    # row 0: 16 survivors moved into the first page, three pages freed
    assert int(c.row_len[0]) == 16 and int(nfreed[0]) == 3
    assert freed.cpu().tolist()[:3] == bt0[0, 1:4].tolist()
    assert np.array_equal(c.slot_pos.cpu().numpy()[0, :16], sp0[0, 40:56])


# ----------------------------------------------------------------------------- confidence + ratchet

@pytest.mark.parametrize("V", [4096 + 13, 128256])
def test_confidence_parity(V):
    S, T = 2, 64
    spec = synth.Spec(name="logits", seed=51, num_seqs=S, num_layers=1, num_q_heads=1, num_kv_heads=1, head_dim=64,
                      dtype="f32", ctx=[16] * S, budget=512, vocab=V)
    logits = torch.stack([synth.logits(spec, s, 0, T, device=DEV) for s in range(S)])
    logits[1, 5] = 0.75                          # an all-equal step (exercises the exact fallback)
    logits[1, 6, :40] = 9.0                      # ties at the top
    p = kvc.ratchet_params(max_steps=T)
    state = torch.zeros(kvc.kvc_ratchet_state_bytes(S, p), dtype=torch.uint8, device=DEV)
    budget = torch.zeros(S, dtype=torch.int32, device=DEV)
    conf = torch.zeros((S, T), device=DEV)
    kvc.kvc_ratchet_init(state, budget, S, p)
    kvc.kvc_confidence_ratchet(logits, state, budget, p, conf)
    torch.cuda.synchronize()
    lg = logits.cpu().numpy()
    want = np.array([[opath.token_confidence(lg[s, t]) for t in range(T)] for s in range(S)])
    assert np.max(np.abs(conf.cpu().numpy() - want)) < 3e-5
    assert abs(want[1, 5] - math.log(V)) < 1e-9


def _trend_logits(S, T, V, rounds, slope_sign):
    """Top-20 logits at b_t, the rest near 0: c_t = log(20 + V' e^-b_t) falls as b_t rises."""
    out = []
    for rd in range(rounds):
        z = torch.zeros((S, T, V))
        for s in range(S):
            for t in range(T):
                tt = T * rd + t
                b = 2.0 + 0.01 * tt if slope_sign[s] < 0 else 12.0 - 0.01 * tt
                z[s, t, :20] = b
                z[s, t, 20 + s] = 0.3
        out.append(z)
    return out


def test_ratchet_rounds_parity():
    """Budgets across rounds equal the oracle's: a falling confidence grows, a rising one never does."""
    S, T, V = 3, 64, 2048
    p = kvc.ratchet_params(max_steps=T)
    state = torch.zeros(kvc.kvc_ratchet_state_bytes(S, p), dtype=torch.uint8, device=DEV)
    budget = torch.zeros(S, dtype=torch.int32, device=DEV)
    kvc.kvc_ratchet_init(state, budget, S, p)
    orc = [opath.Ratchet() for _ in range(S)]
    seqs = _trend_logits(S, T, V, 8, slope_sign=[-1, +1, -1])
    for rd, z in enumerate(seqs):
        kvc.kvc_confidence_ratchet(z.to(DEV), state, budget, p)
        torch.cuda.synchronize()
        want = [orc[s].round(z[s].numpy().astype(np.float64)) for s in range(S)]
        assert budget.cpu().tolist() == want, f"round {rd}"
        st = kvc.ratchet_seq_states(state, S)
        for s in range(S):
            assert st[s].budget == want[s] and st[s].expansions == orc[s].expansions
            if not math.isnan(orc[s].last_slope):
                # fp32 confidences against fp64: the slopes agree to ~1e-8 absolute here
                assert abs(st[s].last_slope - orc[s].last_slope) <= 1e-6 + 1e-4 * abs(orc[s].last_slope)
    assert budget.cpu().tolist()[1] == 512


def test_ratchet_random_logits_budget_sequence():
    """N(0, 2) logits at the 128,256-token vocabulary for 6 rounds: budgets equal the oracle's unless the fitted
    slope is within fp32 noise of zero (then either decision is correct)."""
    S, T = 2, 64
    spec = synth.Spec(name="logits", seed=52, num_seqs=S, num_layers=1, num_q_heads=1, num_kv_heads=1, head_dim=64,
                      dtype="f32", ctx=[16] * S, budget=512)
    p = kvc.ratchet_params(max_steps=T)
    state = torch.zeros(kvc.kvc_ratchet_state_bytes(S, p), dtype=torch.uint8, device=DEV)
    budget = torch.zeros(S, dtype=torch.int32, device=DEV)
    kvc.kvc_ratchet_init(state, budget, S, p)
    orc = [opath.Ratchet() for _ in range(S)]
    for rd in range(6):
        z = torch.stack([synth.logits(spec, s, rd * T, T, device=DEV) for s in range(S)])
        kvc.kvc_confidence_ratchet(z, state, budget, p)
        torch.cuda.synchronize()
        zl = z.cpu().numpy().astype(np.float64)
        for s in range(S):
            b = orc[s].round(zl[s])
            if int(budget[s]) != b:
                assert abs(orc[s].last_slope) < 1e-5, f"round {rd} seq {s}: decisions differ at slope {orc[s].last_slope}"
                return   # the two trajectories legitimately part here


# ----------------------------------------------------------------------------- device-reported faults

def test_faults_are_reported_not_trapped():
    spec = small_spec(ctx=(600,), seed=61, queries="beacon_recent")
    w = H.build(spec)
    H.set_lse(w, H.oracle_lse(w))
    status = torch.zeros(2, dtype=torch.int32, device=DEV)
    scores = torch.zeros((spec.rows, spec.max_slots), device=DEV)
    bt = w.cache.block_table
    saved = bt[3, 2].item()
    bt[3, 2] = w.layout.num_pages + 1000           # a page id outside the pool
    kvc.kvc_score_from_lse(w.cache, w.queries, scores, 0, status)
    torch.cuda.synchronize()
    assert kvc.device_status(status)[:2] == (1, 3)
    status.zero_()
    kvc.kvc_score_from_lse(w.cache, w.queries, scores, kvc.KVC_SCORE_SIMT, status)
    torch.cuda.synchronize()
    assert kvc.device_status(status)[:2] == (1, 3)
    bt[3, 2] = saved
    # row length over capacity
    status.zero_()
    w.cache.row_len[5] = spec.max_slots + 1
    kvc.kvc_score_from_lse(w.cache, w.queries, scores, 0, status)
    torch.cuda.synchronize()
    assert kvc.device_status(status)[:2] == (2, 5)
    w.cache.row_len[5] = 600
    # non-finite LSE
    status.zero_()
    w.queries.lse[0, 0, 9, 3] = float("nan")
    kvc.kvc_score_from_lse(w.cache, w.queries, scores, 0, status)
    torch.cuda.synchronize()
    assert kvc.device_status(status)[0] == 3
    # kept count that disagrees with the mask
    status.zero_()
    keep = torch.ones((spec.rows, spec.max_slots), dtype=torch.uint8, device=DEV)
    kept = torch.full((spec.rows,), 10, dtype=torch.int32, device=DEV)
    z = torch.zeros((spec.rows, spec.max_slots), dtype=torch.int32, device=DEV)
    nm = torch.zeros(spec.rows, dtype=torch.int32, device=DEV)
    kvc.kvc_plan_slots(w.cache, keep, kept, z, z.clone(), nm, status)
    torch.cuda.synchronize()
    assert kvc.device_status(status)[0] == 4
    assert (nm == -1).all()                         # rejected rows: the compaction leaves them alone
    # host-side rejection enqueues nothing
    with pytest.raises(kvc.KvcError):
        kvc.kvc_lrfu_update(w.cache, scores, scores, -1.0)
