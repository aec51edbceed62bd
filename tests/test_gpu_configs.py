"""Configuration-level parity: whole eviction rounds (ratchet -> score -> LRFU -> select -> plan ->
compact) through ``EvictionRound``, beside the oracle run on the same seeded inputs.

Chained rounds compare each step with the tolerance fixed for it: scores 1e-6 + 1e-3 relative;
kept sets identical except entries whose oracle LRFU value lies within 1e-4 relative of the
oracle's budget-th value, or whose score lies within 1e-4 relative of the oracle's gate threshold
(the two places where fp32 against fp64 may legitimately flip a decision).  When the kept sets are
identical the compacted state (pools, block table, positions, labels, row lengths, freed list) must
equal the oracle's bit for bit.
"""
import numpy as np
import pytest
import torch

from agent_kv_cache_lse_b200 import kvc, synth
from agent_kv_cache_lse_b200.round import EvictionRound
from oracle import cache as ocache
from oracle import path as opath

from . import helpers as H

pytestmark = pytest.mark.gpu
DEV = "cuda"
HIT = float(np.float32(0.9))


def check_keep(gk, ok, ocrf, osc, ohits, B):
    """True when identical; otherwise every difference must sit in a tolerance band (asserted)."""
    diff = gk.astype(bool) != ok.astype(bool)
    if not diff.any():
        return True
    n = len(ok)
    kth = np.sort(ocrf)[::-1][min(B, n) - 1] if n and B > 0 else 0.0
    tau = osc[ohits].min() if ohits.any() else 0.0
    near = (np.abs(ocrf - kth) <= 1e-4 * abs(kth)) | (np.abs(osc - tau) <= 1e-4 * tau)
    assert near[diff].all(), f"{int((diff & ~near).sum())} kept-set differences outside the tolerance bands"
    return False


def snapshot(w):
    """Whole-cache host copy (small workloads only)."""
    c = w.cache
    return dict(k=c.k_pool.cpu().view(torch.int16 if c.k_pool.dtype == torch.bfloat16 else torch.int32).numpy(),
                v=c.v_pool.cpu().view(torch.int16 if c.v_pool.dtype == torch.bfloat16 else torch.int32).numpy(),
                kf=c.k_pool.cpu().to(torch.float64).numpy(), bt=c.block_table.cpu().numpy(),
                rl=c.row_len.cpu().numpy(), sp=c.slot_pos.cpu().numpy(), sl=c.slot_label.cpu().numpy())


def run_and_check(w, budgets, logits=None, rows=None):
    """One chained round on the GPU and on the oracle (for `rows`, default all); returns True when the kept
    sets were identical (then the compacted rows were also checked bit for bit)."""
    spec, geo, P = w.spec, w.geo, w.spec.page_size
    all_rows = rows is None
    rows = list(range(spec.rows)) if rows is None else rows
    snaps = H.snap_rows(w, rows)
    lse64 = H.oracle_lse(w, rows, snaps)
    if not all_rows:
        kvc.kvc_query_lse(w.cache, w.queries)      # the unsampled rows' LSE only feeds unchecked rows
        torch.cuda.synchronize()
    H.set_lse(w, lse64, None if all_rows else rows)
    lse32 = lse64.astype(np.float32)
    full0 = snapshot(w) if all_rows else None
    rl0 = w.cache.row_len.cpu().numpy()
    rnd = EvictionRound(w.cache)
    if logits is None:
        rnd.budget.copy_(torch.tensor(budgets, dtype=torch.int32))
    conf = None if logits is None else torch.zeros(logits.shape[:2], device=DEV)
    rnd.run(w.queries, logits, hit_mass=HIT, confidence_out=conf)
    torch.cuda.synchronize()
    assert rnd.device_status()[0] == 0, rnd.device_status()
    if logits is not None:
        orc_r = [opath.Ratchet() for _ in range(spec.num_seqs)]
        lg = logits.cpu().numpy().astype(np.float64)
        budgets = [orc_r[s].round(lg[s]) for s in range(spec.num_seqs)]
        assert rnd.budget.cpu().tolist() == budgets
        want = np.array([[opath.token_confidence(lg[s, t]) for t in range(lg.shape[1])] for s in range(lg.shape[0])])
        assert np.max(np.abs(conf.cpu().numpy() - want)) < 3e-5
    osc = H.oracle_scores(w, lse32, rows, snaps)
    gsc = rnd.scores.cpu().numpy() if all_rows else {r: rnd.scores[r].cpu().numpy() for r in rows}
    gkeep = rnd.keep.cpu().numpy() if all_rows else {r: rnd.keep[r].cpu().numpy() for r in rows}
    same, okeeps, ocrfs = True, {}, {}
    for r in rows:
        sn = snaps[r]
        n = sn.n
        s = geo.coords(r)[0]
        H.assert_scores_close(gsc[r][:n], osc[r], f"row {r}")
        ocrf = opath.lrfu_update(np.zeros(n), osc[r], sn.sp[:n], 0.5, HIT)
        ohit = opath.hit_gate(osc[r], sn.sp[:n], HIT)
        okeep = opath.select_budget(ocrf, sn.sp[:n], int(budgets[s]))
        okeeps[r], ocrfs[r] = okeep, ocrf
        same &= check_keep(gkeep[r][:n], okeep, ocrf, osc[r], ohit, int(budgets[s]))
    if not same:
        return False
    # compaction of each checked row, on its own pages, against the device state
    rl1 = w.cache.row_len.cpu().numpy()
    off = np.concatenate([[0], np.cumsum([-(-int(a) // P) - (-(-int(b) // P)) for a, b in zip(rl0, rl1)])])
    freed_dev = rnd.freed.cpu().numpy()
    for r in rows:
        sn = snaps[r]
        src, dst, m = opath.plan_slots(okeeps[r], sn.n)
        row = opath.PagedRow(block_table=np.arange(len(sn.pages)), n=sn.n, slot_pos=sn.sp.copy(),
                             slot_label=sn.sl.copy(), crf=None)
        k2, v2, new, freed_local = opath.compact_row(sn.kbits, sn.vbits, row, src, dst, m, P)
        kp = -(-m // P)
        bt1 = w.cache.block_table[r].cpu().numpy()
        assert int(rl1[r]) == m
        assert np.array_equal(bt1[:kp], sn.pages[:kp]) and np.all(bt1[kp:len(sn.pages)] == -1)
        pg = torch.from_numpy(sn.pages[:kp].astype(np.int64)).to(DEV)
        assert np.array_equal(H._bits(w.cache.k_pool[pg]).cpu().numpy(), k2[:kp])
        assert np.array_equal(H._bits(w.cache.v_pool[pg]).cpu().numpy(), v2[:kp])
        assert np.array_equal(w.cache.slot_pos[r].cpu().numpy(), new.slot_pos)
        assert np.array_equal(w.cache.slot_label[r].cpu().numpy(), new.slot_label)
        assert np.array_equal(freed_dev[off[r]:off[r + 1]], sn.pages[freed_local])
    if all_rows:
        # the entire pool: pages of no row, and every byte of every row, as the oracle's gather compaction
        plans = {r: opath.plan_slots(okeeps[r], snaps[r].n) for r in rows}
        k2, v2, *_ , fr = ocache.compact_cache(geo, full0["k"], full0["v"], full0["bt"], full0["rl"], full0["sp"],
                                                full0["sl"], None, plans)
        st1 = snapshot(w)
        assert np.array_equal(st1["k"], k2) and np.array_equal(st1["v"], v2)
        assert int(rnd.num_freed[0]) == len(fr) and np.array_equal(freed_dev[:len(fr)], fr)
    return True


@pytest.mark.parametrize("variant", [0, 1])
def test_tiny_round(variant):
    """1 seq, 4 q / 2 KV heads, D 64, fp32, 1,024 tokens in shuffled pages, 8 action queries, budget 256."""
    spec = synth.tiny(variant=variant)
    w = H.build(spec)
    assert run_and_check(w, [spec.budget])


@pytest.mark.parametrize("ctx", [4096 + 99, 32768])
def test_llama8b_layer_round(ctx):
    """32 q / 8 KV heads, D 128, bf16, 2% heavy hitters, action queries, budget 512; 32K is the bench workload,
    run in the bench's launch configuration (ratchet over 64 steps of 128,256-token logits first)."""
    spec = synth.llama8b_layer(ctx=ctx)
    w = H.build(spec)
    logits = torch.stack([synth.logits(spec, 0, 0, 64, device=DEV)])
    run_and_check(w, None, logits=logits)


def test_batch_round_small():
    """Batch-16 shape scaled down: 3 seqs of uneven length, 2 layers x 8 KV heads, shared fragmented pool."""
    spec = synth.batch16(num_seqs=3, num_layers=2, lo=1500, hi=3500)
    w = H.build(spec)
    logits = torch.stack([synth.logits(spec, s, 0, 64, device=DEV) for s in range(spec.num_seqs)])
    run_and_check(w, None, logits=logits)


def test_batch16_full_sampled():
    """Batch 16 x 32 layers x 8 KV heads at 8K-33K context (all rows scored on the GPU); the oracle checks
    four sampled rows end to end."""
    spec = synth.batch16()
    w = H.build(spec)
    logits = torch.stack([synth.logits(spec, s, 0, 64, device=DEV) for s in range(spec.num_seqs)])
    rows = [0, spec.row_id(5, 17, 3), spec.row_id(11, 31, 7), spec.rows - 1]
    run_and_check(w, None, logits=logits, rows=rows)


def test_streaming_rounds():
    """Streaming shape: beacon + recent queries (LSE computed by the library), 28 q / 4 KV heads, the LRFU state
    carried across rounds, 64 decoded tokens appended between compactions.  The oracle keeps its own state from
    the initial generated cache onward; the appended tokens go to pages no block table references (the same
    pages on both sides)."""
    spec = synth.streaming(num_seqs=2, ctx=2048)
    spec.spare_frac = 0.7
    spec.budget = 1800
    w = H.build(spec)
    geo, P, D = w.geo, spec.page_size, spec.head_dim
    rnd = EvictionRound(w.cache)
    rnd.budget.fill_(spec.budget)
    o = snapshot(w)                      # oracle state: the generated cache, before any kernel ran
    o["crf"] = np.zeros((spec.rows, spec.max_slots))
    in_use = set(int(x) for x in o["bt"][o["bt"] >= 0])
    free = [p for p in range(w.layout.num_pages) if p not in in_use]
    n_total = [2048] * spec.num_seqs
    for rd in range(10):
        qs = synth.streaming_queries(spec, n_total, device=DEV)
        q = kvc.QuerySet(qs.q, torch.zeros((spec.num_seqs, 1, spec.num_q_heads, qs.max_q), device=DEV),
                         qs.q_pos, qs.num_q)
        rnd.run(q, None, hit_mass=HIT, score_flags=kvc.KVC_SCORE_COMPUTE_LSE)
        torch.cuda.synchronize()
        assert rnd.device_status()[0] == 0
        hq = qs.q.cpu().to(torch.float64).numpy()
        qpos, numq = qs.q_pos.cpu().numpy(), qs.num_q.cpu().numpy()
        kf = torch.from_numpy(o["k"]).view(torch.bfloat16).to(torch.float64).numpy()
        lse_o = ocache.lse_cache(geo, kf, o["bt"], o["rl"], o["sp"], hq, qpos, numq, qs.max_q)
        glse = q.lse.cpu().numpy().astype(np.float64)
        assert np.max(np.abs(glse - lse_o)) < 5e-5, "the library's LSE pass against the oracle's"
        osc = ocache.score_cache(geo, kf, o["bt"], o["rl"], o["sp"], hq, lse_o.astype(np.float32), qpos, numq)
        crf_o, ohits = ocache.lrfu_cache(geo, osc, o["crf"], o["rl"], o["sp"], 0.5, HIT)
        okeep, _ = ocache.select_cache(geo, crf_o, o["rl"], o["sp"], o["sl"], [spec.budget] * spec.num_seqs)
        gsc, gkeep = rnd.scores.cpu().numpy(), rnd.keep.cpu().numpy()
        same = True
        for r in range(spec.rows):
            n = int(o["rl"][r])
            H.assert_scores_close(gsc[r, :n], osc[r, :n], f"round {rd} row {r}")
            same &= check_keep(gkeep[r, :n], okeep[r, :n], crf_o[r, :n], osc[r, :n], ohits[r, :n], spec.budget)
        if not same:
            return   # both sides are right; their states part here
        plans = ocache.plan_cache(geo, okeep, o["rl"])
        k2, v2, bt2, rl2, sp2, sl2, crf2, fr = ocache.compact_cache(geo, o["k"], o["v"], o["bt"], o["rl"], o["sp"],
                                                                    o["sl"], crf_o, plans)
        st1 = snapshot(w)
        for key, val in (("k", k2), ("v", v2), ("bt", bt2), ("rl", rl2), ("sp", sp2), ("sl", sl2)):
            assert np.array_equal(st1[key], val), f"round {rd}: {key}"
        gcrf = rnd.crf.cpu().numpy()
        for r in range(spec.rows):
            m = int(rl2[r])
            np.testing.assert_allclose(gcrf[r, :m], crf2[r, :m], rtol=2e-5, atol=1e-30)
        assert int(rnd.num_freed[0]) == len(fr)
        free.extend(int(x) for x in fr)
        # append 64 decoded tokens per row, to both states
        o = dict(k=k2, v=v2, bt=bt2, rl=rl2, sp=sp2, sl=sl2, crf=crf2)
        for r in range(spec.rows):
            s, l, h = geo.coords(r)
            m = int(o["rl"][r])
            pos = torch.arange(n_total[s], n_total[s] + 64)
            for slot in range(m, m + 64):
                if o["bt"][r, slot // P] < 0:
                    o["bt"][r, slot // P] = free.pop(0)
            slots = np.arange(m, m + 64)
            phys = o["bt"][r, slots // P].astype(np.int64) * P + slots % P
            kv = synth.key_values(spec, s, l, h, pos, "k")
            vv = synth.key_values(spec, s, l, h, pos, "v")
            o["k"].reshape(-1, D)[phys] = kv.view(torch.int16).numpy()
            o["v"].reshape(-1, D)[phys] = vv.view(torch.int16).numpy()
            w.cache.k_pool.view(-1, D)[torch.from_numpy(phys).to(DEV)] = kv.to(DEV)
            w.cache.v_pool.view(-1, D)[torch.from_numpy(phys).to(DEV)] = vv.to(DEV)
            o["sp"][r, m:m + 64] = pos.numpy()
            o["sl"][r, m:m + 64] = synth.LABEL_REASON
            o["rl"][r] = m + 64
            o["crf"][r, m:m + 64] = 0.0
            rnd.crf[r, m:m + 64] = 0.0
        w.cache.block_table.copy_(torch.from_numpy(o["bt"]))
        w.cache.row_len.copy_(torch.from_numpy(o["rl"]))
        w.cache.slot_pos.copy_(torch.from_numpy(o["sp"]))
        w.cache.slot_label.copy_(torch.from_numpy(o["sl"]))
        n_total = [n + 64 for n in n_total]


def _stress_cache(S, L, ctx, seed, device=DEV):
    spec = synth.stress(num_seqs=S, num_layers=L, ctx=ctx, seed=seed)
    layout = synth.make_layout(spec)
    g = torch.Generator(device=device).manual_seed(seed)
    pools = []
    for _ in range(2):
        pool = torch.empty((layout.num_pages, spec.page_size, spec.head_dim), dtype=torch.int16, device=device)
        flat = pool.view(-1)
        step = 1 << 28
        for a in range(0, flat.numel(), step):
            flat[a:a + step].random_(-32768, 32767, generator=g)
        pools.append(pool.view(torch.bfloat16))
    cache = kvc.Cache(pools[0], pools[1], layout.block_table.to(device), layout.row_len.to(device),
                      layout.slot_pos.to(device), layout.slot_label.to(device), S, L, spec.num_kv_heads)
    return spec, layout, cache


@pytest.mark.parametrize("size", ["small", "full"])
def test_stress_ties(size):
    """Stress shape: CRF quantised to k * 2^-10 (k uniform in 0..63), budget freeing 40% of each row's pages;
    selection with position tie-breaks, plan and compaction bit-exact against the oracle (full size: 64 seqs x
    16 layers x 8 KV heads x 33,000 tokens, ~140 GB of K+V, four sampled rows)."""
    S, L = (4, 2) if size == "small" else (64, 16)
    spec, layout, cache = _stress_cache(S, L, 1000 if size == "small" else 33000, seed=5)
    rows = list(range(spec.rows)) if size == "small" else [0, 1234, 5000, spec.rows - 1]
    n = spec.ctx[0]
    B = synth.stress_budget(n)
    P = spec.page_size
    ms = spec.max_slots
    crf = torch.empty((spec.rows, ms), dtype=torch.float32, device=DEV)
    idx = torch.arange(ms, device=DEV, dtype=torch.int64)
    for r0 in range(0, spec.rows, 256):
        rr = torch.arange(r0, min(spec.rows, r0 + 256), device=DEV, dtype=torch.int64)
        crf[r0:r0 + len(rr)] = synth.uniform_int(spec.seed, synth.S_TIE, rr[:, None] * ms + idx[None, :], 0,
                                                 63).to(torch.float32) * 2.0**-10
    bt0 = layout.block_table.numpy()
    sub_pages = {r: [int(p) for p in bt0[r, :-(-n // P)]] for r in rows}
    kbits = {r: cache.k_pool.view(torch.int16)[torch.tensor(sub_pages[r], device=DEV)].cpu().numpy() for r in rows}
    vbits = {r: cache.v_pool.view(torch.int16)[torch.tensor(sub_pages[r], device=DEV)].cpu().numpy() for r in rows}
    crf_h = {r: crf[r].cpu().numpy() for r in rows}
    budget = torch.full((S,), B, dtype=torch.int32, device=DEV)
    rnd = EvictionRound(cache)
    kvc.kvc_select_budget(cache, crf, budget, rnd.keep, rnd.kept, 0, rnd.status)
    kvc.kvc_plan_slots(cache, rnd.keep, rnd.kept, rnd.move_src, rnd.move_dst, rnd.num_moves, rnd.status)
    kvc.kvc_compact_pages(cache, rnd.move_src, rnd.move_dst, rnd.num_moves, rnd.kept, crf, rnd.freed, rnd.num_freed,
                          rnd.workspace, rnd.status)
    torch.cuda.synchronize()
    assert rnd.device_status()[0] == 0
    pages_before = -(-n // P)
    assert int(rnd.num_freed[0]) == spec.rows * (pages_before - (-(-B // P)))
    assert (pages_before - (-(-B // P))) == int(round(0.4 * pages_before))
    sp0, sl0 = layout.slot_pos.numpy(), layout.slot_label.numpy()
    for r in rows:
        keep = opath.select_budget(crf_h[r][:n].astype(np.float64), sp0[r, :n], B)
        assert np.array_equal(rnd.keep[r, :n].cpu().numpy().astype(bool), keep), f"row {r}"
        src, dst, m = opath.plan_slots(keep, n)
        local_bt = np.arange(len(sub_pages[r]))
        row = opath.PagedRow(block_table=local_bt, n=n, slot_pos=sp0[r].copy(), slot_label=sl0[r].copy(),
                             crf=crf_h[r].copy())
        k2, v2, new, freed = opath.compact_row(kbits[r], vbits[r], row, src, dst, m, P)
        kept_pages = -(-m // P)
        got_pages = cache.block_table[r, :kept_pages].cpu().numpy()
        assert np.array_equal(got_pages, np.array(sub_pages[r][:kept_pages]))
        gk = cache.k_pool.view(torch.int16)[torch.from_numpy(got_pages).to(DEV)].cpu().numpy()
        gv = cache.v_pool.view(torch.int16)[torch.from_numpy(got_pages).to(DEV)].cpu().numpy()
        assert np.array_equal(gk, k2[:kept_pages]) and np.array_equal(gv, v2[:kept_pages])
        assert np.array_equal(cache.slot_pos[r].cpu().numpy(), new.slot_pos)
        assert np.array_equal(crf[r].cpu().numpy(), new.crf)
        assert int(cache.row_len[r]) == m
        assert np.all(cache.block_table[r, kept_pages:].cpu().numpy() == -1)
    del rnd, crf, cache
    torch.cuda.empty_cache()
