"""Configuration-level parity: whole eviction rounds (ratchet -> score -> LRFU -> select -> plan ->
compact) through ``EvictionRound``, beside the oracle run on the same seeded inputs.

Chained rounds compare each step with the tolerance fixed for it: scores 1e-6 + 1e-3 relative;
kept sets identical except entries whose oracle LRFU value lies within 1e-4 relative of the
oracle's budget-th value, or whose score lies within 1e-4 relative of the oracle's gate threshold
(the two places where fp32 against fp64 may legitimately flip a decision).  The oracle then plans and
compacts with the GPU's keep mask, and the compacted state (pools, block table, positions, labels, row
lengths, freed list) must equal the oracle's bit for bit; multi-round runs carry the oracle's state
forward on the GPU's decisions wherever those sit in a tolerance band, so the two stay in lockstep.
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


def _orig_slots(src, dst, size):
    """Slot j after compaction holds the entry that was at orig[j] before it."""
    orig = np.arange(size)
    orig[np.asarray(dst, dtype=np.int64)] = np.asarray(src, dtype=np.int64)
    return orig


def check_crf(gcrf, ocrf, osc, ohits, orig, m, what):
    """CRF after compaction against the oracle's, entry by entry: within the score tolerance, except where the
    GPU's hit decision sits in the gate-threshold band (then the two differ by that entry's hit)."""
    want = ocrf[orig[:m]]
    tau = osc[ohits].min() if ohits.any() else 0.0
    band = np.abs(osc[orig[:m]] - tau) <= 1e-4 * tau
    bad = np.abs(gcrf[:m] - want) > 1e-6 + 1e-3 * np.abs(want)
    assert not (bad & ~band).any(), f"{what}: {int((bad & ~band).sum())} CRF values out of tolerance"
    return bad & band


def run_and_check(w, budgets, logits=None, rows=None):
    """One chained round on the GPU and on the oracle (for `rows`, default all).  Scores and kept sets are compared
    with their tolerances; then the oracle plans and compacts with the GPU's keep mask (identical to its own except
    inside the tolerance bands), and the compacted rows, the freed list and (for whole-cache runs) every byte of
    both pools must equal the GPU's bit for bit.  Returns the number of kept-set differences in the bands."""
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
    gkept = rnd.kept.cpu().numpy()
    gcrf_all = rnd.crf.cpu().numpy() if all_rows else {r: rnd.crf[r].cpu().numpy() for r in rows}
    in_band = 0
    for r in rows:
        sn = snaps[r]
        n = sn.n
        s = geo.coords(r)[0]
        H.assert_scores_close(gsc[r][:n], osc[r], f"row {r}")
        ocrf = opath.lrfu_update(np.zeros(n), osc[r], sn.sp[:n], 0.5, HIT)
        ohit = opath.hit_gate(osc[r], sn.sp[:n], HIT)
        okeep = opath.select_budget(ocrf, sn.sp[:n], int(budgets[s]))
        gk = gkeep[r][:n].astype(bool)
        if not check_keep(gk, okeep, ocrf, osc[r], ohit, int(budgets[s])):
            in_band += int((gk != okeep).sum())
        assert int(gk.sum()) == min(int(budgets[s]), n) == int(gkept[r])
        assert not gkeep[r][n:].any()
        # CRF moved by the compaction: the GPU's LRFU value of each surviving entry
        src, dst, m = opath.plan_slots(gk, n)
        check_crf(gcrf_all[r], ocrf, osc[r], ohit, _orig_slots(src, dst, n), m, f"row {r}")
    # compaction of each checked row on the GPU's keep mask, on its own pages, against the device state
    rl1 = w.cache.row_len.cpu().numpy()
    off = np.concatenate([[0], np.cumsum([-(-int(a) // P) - (-(-int(b) // P)) for a, b in zip(rl0, rl1)])])
    freed_dev = rnd.freed.cpu().numpy()
    for r in rows:
        sn = snaps[r]
        src, dst, m = opath.plan_slots(gkeep[r][:sn.n].astype(bool), sn.n)
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
        plans = {r: opath.plan_slots(gkeep[r][:snaps[r].n].astype(bool), snaps[r].n) for r in rows}
        k2, v2, *_ , fr = ocache.compact_cache(geo, full0["k"], full0["v"], full0["bt"], full0["rl"], full0["sp"],
                                                full0["sl"], None, plans)
        st1 = snapshot(w)
        assert np.array_equal(st1["k"], k2) and np.array_equal(st1["v"], v2)
        assert int(rnd.num_freed[0]) == len(fr) and np.array_equal(freed_dev[:len(fr)], fr)
    return in_band


@pytest.mark.parametrize("variant", [0, 1])
def test_tiny_round(variant):
    """1 seq, 4 q / 2 KV heads, D 64, fp32, 1,024 tokens in shuffled pages, 8 action queries, budget 256."""
    spec = synth.tiny(variant=variant)
    w = H.build(spec)
    assert run_and_check(w, [spec.budget]) == 0


@pytest.mark.parametrize("ctx", [4096 + 99, 32768])
def test_llama8b_layer_round(ctx):
    """32 q / 8 KV heads, D 128, bf16, 2% heavy hitters, action queries, budget 512; 32K is the bench workload,
    run in the bench's launch configuration (ratchet over 64 steps of 128,256-token logits first)."""
    spec = synth.llama8b_layer(ctx=ctx)
    w = H.build(spec)
    logits = torch.stack([synth.logits(spec, 0, 0, 64, device=DEV)])
    assert run_and_check(w, None, logits=logits) <= 2


def test_batch_round_small():
    """Batch-16 shape scaled down: 3 seqs of uneven length, 2 layers x 8 KV heads, shared fragmented pool."""
    spec = synth.batch16(num_seqs=3, num_layers=2, lo=1500, hi=3500)
    w = H.build(spec)
    logits = torch.stack([synth.logits(spec, s, 0, 64, device=DEV) for s in range(spec.num_seqs)])
    assert run_and_check(w, None, logits=logits) <= 2 * spec.rows


def test_batch16_full_sampled():
    """Batch 16 x 32 layers x 8 KV heads at 8K-33K context (all rows scored on the GPU); the oracle checks 32
    sampled rows end to end (every sequence at least once, the first and the last row among them)."""
    spec = synth.batch16()
    w = H.build(spec)
    logits = torch.stack([synth.logits(spec, s, 0, 64, device=DEV) for s in range(spec.num_seqs)])
    rng = np.random.default_rng(3)
    rows = {0, spec.rows - 1}
    rows |= {spec.row_id(s, int(rng.integers(spec.num_layers)), int(rng.integers(spec.num_kv_heads)))
             for s in range(spec.num_seqs)}
    while len(rows) < 32:
        rows.add(int(rng.integers(spec.rows)))
    assert run_and_check(w, None, logits=logits, rows=sorted(rows)) <= 2 * len(rows)


class RowState:
    """The oracle's own copy of one row: its logical pages (raw bits, local page order), positions, labels, CRF."""

    def __init__(self, kb, vb, sp, sl, n, max_slots):
        self.kb, self.vb, self.sp, self.sl, self.n = kb, vb, sp.astype(np.int64), sl.copy(), n
        self.crf = np.zeros(max_slots)


class FreeStack:
    """The free pages as a device stack (the library's append takes pages from its top; compaction's freed pages
    are pushed on it)."""

    def __init__(self, pages, capacity):
        self.pages = torch.full((capacity,), -1, dtype=torch.int32, device=DEV)
        self.pages[:len(pages)] = torch.tensor(pages, dtype=torch.int32, device=DEV)
        self.depth = torch.tensor([len(pages)], dtype=torch.int64, device=DEV)

    def push(self, freed, n):
        d = int(self.depth[0])
        self.pages[d:d + n] = freed[:n]
        self.depth += n


def append_tokens(w, rnd, n_total, stack, states, count=64):
    """Append `count` decoded tokens to every row through kvc_append_tokens (pages from the free stack), and the
    same tokens to the oracle's sampled rows; the values come from the seeded generator on both sides."""
    spec, geo, P, D = w.spec, w.geo, w.spec.page_size, w.spec.head_dim
    c = w.cache
    rl = c.row_len.cpu().numpy()
    kv = torch.empty((spec.rows, count, D), dtype=c.k_pool.dtype, device=DEV)
    vv = torch.empty_like(kv)
    new_pos = torch.empty((spec.num_seqs, count), dtype=torch.int32, device=DEV)
    for s in range(spec.num_seqs):
        new_pos[s] = torch.arange(n_total[s], n_total[s] + count, dtype=torch.int32, device=DEV)
    for r in range(spec.rows):
        s, l, h = geo.coords(r)
        pos = torch.arange(n_total[s], n_total[s] + count, dtype=torch.int64, device=DEV)
        kv[r] = synth.key_values(spec, s, l, h, pos, "k")
        vv[r] = synth.key_values(spec, s, l, h, pos, "v")
        if r in states:
            st = states[r]
            m = int(rl[r])
            slots = np.arange(m, m + count)
            need = (m + count + P - 1) // P
            if st.kb.shape[0] < need:
                extra = need - st.kb.shape[0]
                st.kb = np.concatenate([st.kb, np.zeros((extra, P, D), dtype=st.kb.dtype)])
                st.vb = np.concatenate([st.vb, np.zeros((extra, P, D), dtype=st.vb.dtype)])
            st.kb.reshape(-1, D)[slots] = H._bits(kv[r]).cpu().numpy()
            st.vb.reshape(-1, D)[slots] = H._bits(vv[r]).cpu().numpy()
            st.sp[slots] = pos.cpu().numpy()
            st.sl[slots] = synth.LABEL_REASON
            st.crf[slots] = 0.0
            st.n = m + count
    ws = torch.zeros(kvc.kvc_append_workspace_bytes(spec.rows) // 8, dtype=torch.int64, device=DEV)
    kvc.kvc_append_tokens(c, kv, vv, new_pos, synth.LABEL_REASON, rnd.crf, stack.pages, stack.depth, ws, rnd.status)
    torch.cuda.synchronize()
    assert rnd.device_status()[0] == 0, rnd.device_status()
    assert np.array_equal(c.row_len.cpu().numpy(), rl + count)
    for s in range(spec.num_seqs):
        n_total[s] += count


def streaming_lockstep(spec, rounds, sample):
    """Streaming rounds in lockstep with the oracle on the sampled rows: beacon + recent queries with the LSE
    computed by the library, the LRFU state carried across rounds, 64 decoded tokens appended after each
    compaction.  Every round compares the LSE, scores, kept set, CRF and the compacted row (pages bit for bit,
    positions, labels, freed pages); the oracle then carries on from the GPU's keep mask and, where a hit decision
    sits in the gate-threshold band, from the GPU's CRF value, so that its state follows the GPU's.  The decoded
    tokens go in through the library's append (pages from a free stack fed by each compaction's freed list)."""
    w = H.build(spec)
    geo, P, G = w.geo, spec.page_size, spec.group
    rnd = EvictionRound(w.cache)
    rnd.budget.fill_(spec.budget)
    snaps = H.snap_rows(w, sample)
    states = {r: RowState(snaps[r].kbits, snaps[r].vbits, snaps[r].sp, snaps[r].sl, snaps[r].n, spec.max_slots)
              for r in sample}
    bt0 = w.cache.block_table.cpu().numpy()
    in_use = set(int(x) for x in bt0[bt0 >= 0])
    stack = FreeStack([p for p in range(w.layout.num_pages) if p not in in_use], w.layout.num_pages)
    n_total = list(spec.ctx)
    band_total = 0
    for rd in range(rounds):
        bt_before = w.cache.block_table.cpu().numpy()
        rl_before = w.cache.row_len.cpu().numpy()
        qs = synth.streaming_queries(spec, n_total, device=DEV)
        q = kvc.QuerySet(qs.q, torch.zeros((spec.num_seqs, 1, spec.num_q_heads, qs.max_q), device=DEV),
                         qs.q_pos, qs.num_q)
        rnd.run(q, None, hit_mass=HIT, score_flags=kvc.KVC_SCORE_COMPUTE_LSE)
        torch.cuda.synchronize()
        assert rnd.device_status()[0] == 0, (rd, rnd.device_status())
        rl_after = w.cache.row_len.cpu().numpy()
        bt_after = w.cache.block_table.cpu().numpy()
        per_row = [-(-int(a) // P) - (-(-int(b) // P)) for a, b in zip(rl_before, rl_after)]
        off = np.concatenate([[0], np.cumsum(per_row)])
        nf = int(rnd.num_freed[0])
        assert nf == off[-1]
        freed_dev = rnd.freed[:nf].cpu().numpy()
        qpos = qs.q_pos.cpu().numpy()
        for r in sample:
            st = states[r]
            s, l, h = geo.coords(r)
            n = st.n
            assert int(rl_before[r]) == n
            what = f"round {rd} row {r}"
            kf = torch.from_numpy(st.kb.reshape(-1, spec.head_dim)[:n]).view(torch.bfloat16).to(torch.float64).numpy()
            qg = qs.q[s, l, :, h * G:(h + 1) * G].cpu().to(torch.float64).numpy()
            lse_o = opath.attention_lse(qg, kf, qpos[s], st.sp[:n])
            glse = q.lse[s, l, h * G:(h + 1) * G].cpu().numpy().astype(np.float64)
            assert np.max(np.abs(glse - lse_o)) < 5e-5, f"{what}: the library's LSE pass against the oracle's"
            osc = opath.scores_from_lse(qg, kf, qpos[s], st.sp[:n], lse_o.astype(np.float32).astype(np.float64))
            H.assert_scores_close(rnd.scores[r, :n].cpu().numpy(), osc, what)
            ohit = opath.hit_gate(osc, st.sp[:n], HIT)
            ocrf = opath.lrfu_update(st.crf[:n], osc, st.sp[:n], 0.5, HIT)
            okeep = opath.select_budget(ocrf, st.sp[:n], spec.budget)
            gk = rnd.keep[r, :n].cpu().numpy().astype(bool)
            if not check_keep(gk, okeep, ocrf, osc, ohit, spec.budget):
                band_total += int((gk != okeep).sum())
            # the oracle compacts on the GPU's keep mask
            src, dst, m = opath.plan_slots(gk, n)
            crf_full = st.crf.copy()
            crf_full[:n] = ocrf
            npg = -(-n // P)
            row = opath.PagedRow(block_table=np.arange(npg), n=n, slot_pos=st.sp.copy(), slot_label=st.sl.copy(),
                                 crf=crf_full)
            kb2, vb2, new, freed_local = opath.compact_row(st.kb[:npg], st.vb[:npg], row, src, dst, m, P)
            kp = -(-m // P)
            assert int(rl_after[r]) == m, what
            assert np.array_equal(bt_after[r, :kp], bt_before[r, :kp]) and np.all(bt_after[r, kp:npg] == -1), what
            pg = torch.from_numpy(bt_after[r, :kp].astype(np.int64)).to(DEV)
            assert np.array_equal(H._bits(w.cache.k_pool[pg]).cpu().numpy(), kb2[:kp]), what
            assert np.array_equal(H._bits(w.cache.v_pool[pg]).cpu().numpy(), vb2[:kp]), what
            assert np.array_equal(w.cache.slot_pos[r].cpu().numpy(), new.slot_pos.astype(np.int32)), what
            assert np.array_equal(w.cache.slot_label[r].cpu().numpy(), new.slot_label), what
            assert np.array_equal(freed_dev[off[r]:off[r + 1]], bt_before[r, freed_local]), what
            gcrf = rnd.crf[r].cpu().numpy().astype(np.float64)
            adopt = check_crf(gcrf, ocrf, osc, ohit, _orig_slots(src, dst, n), m, what)
            new.crf[:m][adopt] = gcrf[:m][adopt]
            st.kb, st.vb, st.sp, st.sl, st.crf, st.n = kb2[:kp], vb2[:kp], new.slot_pos, new.slot_label, new.crf, m
        stack.push(rnd.freed, nf)
        if rd + 1 < rounds:
            append_tokens(w, rnd, n_total, stack, states)
    return band_total


def test_streaming_rounds():
    """Streaming shape scaled down: 2 sequences x 2,048 tokens, 28 q / 4 KV heads, budget 1,800, 30 rounds, every
    row checked in lockstep."""
    spec = synth.streaming(num_seqs=2, ctx=2048)
    spec.spare_frac = 0.05
    spec.budget = 1800
    assert streaming_lockstep(spec, 30, list(range(spec.rows))) <= 30 * spec.rows


def test_streaming_rounds_full():
    """The streaming workload at size: 8 sequences x 32K tokens growing by 64 decoded tokens per round, 28 q / 4 KV
    heads, budget 30,000, 200 rounds; four sampled rows checked in lockstep every round."""
    spec = synth.streaming()
    sample = [0, spec.row_id(3, 0, 1), spec.row_id(5, 0, 2), spec.rows - 1]
    assert streaming_lockstep(spec, 200, sample) <= 200 * len(sample)


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


def test_stress_scored_round_sampled():
    """The stress shape through a whole scored round: 64 sequences x 33,000 tokens (partial last page) x 4 layers x
    8 KV heads, 32 q heads, action-token queries, a budget that frees 40% of every row's pages; all 2,048 rows are
    scored, gated, selected, planned and compacted on the GPU and eight sampled rows are checked end to end."""
    spec = synth.stress(num_seqs=64, num_layers=4, ctx=33000)
    spec.queries = "action"
    w = H.build(spec, fill="randn")
    B = synth.stress_budget(spec.ctx[0])
    rng = np.random.default_rng(8)
    rows = sorted({0, spec.rows - 1} | {int(x) for x in rng.choice(spec.rows, size=6, replace=False)})
    assert run_and_check(w, [B] * spec.num_seqs, rows=rows) <= 2 * len(rows)
    pages = -(-spec.ctx[0] // spec.page_size)
    assert pages - (-(-B // spec.page_size)) == int(round(0.4 * pages))
    del w
    torch.cuda.empty_cache()


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
