"""Parity of the step-aware ranking scores ("StepKV: Step-Aware KV Cache Compression for LLM Agents", abstract)
against the oracle, and of the top-budget selection run on them.

Tolerance: the blended scores within 1e-6 + 1e-3 |oracle| (the scores' bound; the kernel's step sums are
exact integer sums of the scores at a per-row fixed point of max|s| * 2^-39, the blend one fp32 FMA).
"""
import numpy as np
import pytest
import torch

from agent_kv_cache_lse_b200 import kvc, synth
from oracle import path as opath
from oracle import stepkv as osk

pytestmark = pytest.mark.gpu

DEV = "cuda"


def workload(ctx=(1500, 2817, 4000), L=2, Hkv=4, seed=51, permute=False, shorten=False, pad=3):
    spec = synth.Spec(name="stepkv", seed=seed, num_seqs=len(ctx), num_layers=L, num_q_heads=Hkv, num_kv_heads=Hkv,
                      head_dim=64, dtype="f32", ctx=list(ctx), budget=256)
    lay = synth.make_layout(spec)
    g = torch.Generator().manual_seed(seed)
    pos, rl = lay.slot_pos.clone(), lay.row_len.clone()
    for r in range(spec.rows):
        n = int(rl[r])
        if permute:
            pos[r, :n] = pos[r, :n][torch.randperm(n, generator=g)]
        if shorten and r % 3 == 1:
            rl[r] = n // 2
    starts = [synth.step_starts(spec, s) for s in range(spec.num_seqs)]
    ms = max(len(x) for x in starts) + pad
    st = torch.full((spec.num_seqs, ms), 2**31 - 1, dtype=torch.int32)
    for s, x in enumerate(starts):
        st[s, :len(x)] = x
    ns = torch.tensor([len(x) for x in starts], dtype=torch.int32)
    rng = np.random.default_rng(seed)
    sc = (np.exp(rng.standard_normal((spec.rows, spec.max_slots)) * 2) *
          (rng.random((spec.rows, spec.max_slots)) < 0.9)).astype(np.float32)
    dummy = torch.zeros((1, 16, 64), device=DEV)
    cache = kvc.Cache(dummy, dummy, lay.block_table.to(DEV), rl.to(DEV), pos.to(DEV), lay.slot_label.to(DEV),
                      spec.num_seqs, L, Hkv)
    return spec, cache, torch.from_numpy(sc).to(DEV), st.to(DEV), ns.to(DEV), sc, pos.numpy(), rl.numpy(), starts


def check(spec, out, sc, pos, rl, starts, beta, what):
    got = out.cpu().numpy()
    for r in range(spec.rows):
        s, _, _ = spec.row_coords(r)
        n = int(rl[r])
        want = osk.combined_scores(sc[r, :n].astype(np.float64), pos[r, :n], starts[s].numpy(), beta)
        err = np.abs(got[r, :n] - want)
        bad = err > 1e-6 + 1e-3 * np.abs(want)
        assert not bad.any(), f"{what} row {r}: {int(bad.sum())} values out of tolerance, max err {err.max()}"


@pytest.mark.parametrize("case", ["plain", "permuted_short", "beta03", "beta1", "long_rows", "wide_table",
                                  "long_wide_table"])
def test_step_scores_parity(case):
    """Rows up to 34,816 slots run the register-resident kernel; "long_rows" (40,000 slots) the three-pass one.
    Step tables of up to 64 columns keep one copy of the step sums per warp; the "wide" cases (90 columns) add
    into one shared copy instead."""
    beta = {"beta03": 0.3, "beta1": 1.0}.get(case, 0.5)
    ctx = (40000, 1200) if case.startswith("long") else (1500, 2817, 4000)
    spec, cache, s, st, ns, sc, pos, rl, starts = workload(ctx=ctx, permute=case in ("permuted_short", "long_rows",
                                                                                     "long_wide_table"),
                                                           shorten=case == "permuted_short",
                                                           pad=90 - 25 if "wide" in case else 3)
    out = torch.full_like(s, -5.0)
    status = torch.zeros(2, dtype=torch.int32, device=DEV)
    kvc.kvc_step_scores(cache, s, st, ns, out, beta, status)
    torch.cuda.synchronize()
    assert kvc.device_status(status)[0] == 0
    check(spec, out, sc, pos, rl, starts, beta, case)
    o = out.cpu().numpy()
    for r in range(spec.rows):
        assert np.all(o[r, int(rl[r]):] == -5.0), "slots beyond the row length must not be written"


def test_beta_zero_is_the_saliency_and_in_place_is_the_same():
    spec, cache, s, st, ns, sc, pos, rl, starts = workload(seed=52)
    out = torch.zeros_like(s)
    kvc.kvc_step_scores(cache, s, st, ns, out, 0.0)
    torch.cuda.synchronize()
    n = torch.tensor(rl)
    for r in range(spec.rows):
        assert torch.equal(out[r, :int(n[r])], s[r, :int(n[r])])
    a = torch.zeros_like(s)
    kvc.kvc_step_scores(cache, s, st, ns, a, 0.5)
    b = s.clone()
    kvc.kvc_step_scores(cache, b, st, ns, b, 0.5)           # in place
    c = torch.zeros_like(s)
    kvc.kvc_step_scores(cache, s, st, ns, c, 0.5)
    torch.cuda.synchronize()
    for r in range(spec.rows):
        m = int(n[r])
        assert torch.equal(a[r, :m], b[r, :m]) and torch.equal(a[r, :m], c[r, :m]), "results must repeat bit for bit"


def test_bad_step_tables_are_reported():
    spec, cache, s, st, ns, sc, pos, rl, starts = workload(ctx=(5000, 6000), L=1, Hkv=2, seed=53)
    assert int(ns[1]) >= 2, "the case needs two steps in sequence 1"
    out = torch.zeros_like(s)
    status = torch.zeros(2, dtype=torch.int32, device=DEV)
    st2 = st.clone()
    st2[1, 1] = st2[1, 0]                                   # not strictly ascending in sequence 1
    kvc.kvc_step_scores(cache, s, st2, ns, out, 0.5, status)
    torch.cuda.synchronize()
    code, row, _ = kvc.device_status(status)
    assert code == 8 and spec.row_coords(row)[0] == 1
    status.zero_()
    ns2 = ns.clone()
    ns2[0] = 0
    kvc.kvc_step_scores(cache, s, st, ns2, out, 0.5, status)
    torch.cuda.synchronize()
    code, row, _ = kvc.device_status(status)
    assert code == 8 and spec.row_coords(row)[0] == 0


def test_selection_on_step_scores_matches_the_oracle():
    """The blended scores rank the row through the same top-budget selection as the LRFU values."""
    spec, cache, s, st, ns, sc, pos, rl, starts = workload(seed=54, permute=True)
    out = torch.zeros_like(s)
    kvc.kvc_step_scores(cache, s, st, ns, out, 0.5)
    budget = torch.full((spec.num_seqs,), 700, dtype=torch.int32, device=DEV)
    keep = torch.zeros((spec.rows, spec.max_slots), dtype=torch.uint8, device=DEV)
    kept = torch.zeros(spec.rows, dtype=torch.int32, device=DEV)
    kvc.kvc_select_budget(cache, out, budget, keep, kept)
    torch.cuda.synchronize()
    o, k = out.cpu().numpy(), keep.cpu().numpy().astype(bool)
    for r in range(spec.rows):
        s_, _, _ = spec.row_coords(r)
        n = int(rl[r])
        want = osk.combined_scores(sc[r, :n].astype(np.float64), pos[r, :n], starts[s_].numpy(), 0.5)
        ok = opath.select_budget(want, pos[r, :n], 700)
        # identical except entries within 1e-4 relative of the oracle's budget-th value
        kth = np.sort(want)[::-1][min(700, n) - 1]
        near = np.abs(want - kth) <= 1e-4 * abs(kth)
        assert np.array_equal(k[r, :n] & ~near, ok & ~near), f"row {r}"
        assert int(kept[r]) == min(700, n)
        # and the GPU's own selection is exact on its own blended values
        assert np.array_equal(k[r, :n], opath.select_budget(o[r, :n].astype(np.float64), pos[r, :n], 700))


def test_step_scores_bench_workload_sampled_rows():
    """The workload bench.py --stepkv times: 16 sequences x 8 layers x 8 KV heads at 8K-33K (1,024 rows, the
    register-resident kernel), checked on sampled rows."""
    b = synth.batch16(num_layers=8)
    spec, cache, s, st, ns, sc, pos, rl, starts = workload(ctx=tuple(b.ctx), L=8, Hkv=8, seed=55)
    out = torch.zeros_like(s)
    status = torch.zeros(2, dtype=torch.int32, device=DEV)
    kvc.kvc_step_scores(cache, s, st, ns, out, 0.5, status)
    torch.cuda.synchronize()
    assert kvc.device_status(status)[0] == 0
    got = out.cpu().numpy()
    for r in (0, 255, 511, 800, 1023):
        s_, _, _ = spec.row_coords(r)
        n = int(rl[r])
        want = osk.combined_scores(sc[r, :n].astype(np.float64), pos[r, :n], starts[s_].numpy(), 0.5)
        err = np.abs(got[r, :n] - want)
        assert np.all(err <= 1e-6 + 1e-3 * np.abs(want)), f"row {r}: max err {err.max()}"
