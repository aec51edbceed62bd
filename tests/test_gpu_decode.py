"""Parity of the fused decode step (paged attention with the scores folded in; "ActKV Dissected",
Component 3) against the oracle's decode step on identical seeded inputs.

Tolerances (fp32 kernel against the fp64 oracle on the same bf16 or fp32 inputs): the output
within 2e-5 + 1e-4 |oracle| (a convex combination of value vectors of unit scale, fp32
products and sums over up to 32K keys); the LSE within 2e-5 absolute (fp32 logits and an fp32
sum of exponentials relative to the row maximum); the scores with the scoring pass's bound,
1e-6 + 1e-3 |oracle|.
"""
import numpy as np
import pytest
import torch

from agent_kv_cache_lse_b200 import kvc, synth
from oracle import decode as od

from . import helpers as H

pytestmark = pytest.mark.gpu

DEV = "cuda"


def spec_of(S=1, L=1, Hq=32, Hkv=8, D=128, ctx=(4096 + 99,), dtype="bf16", seed=31, heavy=0.02, P=16):
    return synth.Spec(name="decode", seed=seed, num_seqs=S, num_layers=L, num_q_heads=Hq, num_kv_heads=Hkv,
                      head_dim=D, dtype=dtype, ctx=list(ctx), budget=512, heavy_frac=heavy, page_size=P)


def decode_inputs(w, q_pos=None):
    """The step's query [S][L][Hq][D] (the first query of each sequence's set) and its positions."""
    q = w.queries.q[:, :, 0].contiguous()
    if q_pos is None:
        q_pos = list(w.spec.ctx)                  # the next token: every cached key is visible
    return q, torch.tensor(q_pos, dtype=torch.int32, device=DEV)


def row_kv(w, r):
    c, P = w.cache, w.spec.page_size
    n = int(c.row_len[r])
    pages = c.block_table[r, :-(-n // P)].to(torch.int64)
    k = c.k_pool[pages].reshape(-1, w.spec.head_dim)[:n].cpu().to(torch.float64).numpy()
    v = c.v_pool[pages].reshape(-1, w.spec.head_dim)[:n].cpu().to(torch.float64).numpy()
    return k, v, c.slot_pos[r, :n].cpu().numpy()


def oracle_rows(w, q, q_pos, rows):
    """{row: (out [G, D], lse [G], inc [n])} from the oracle, on host copies of the inputs."""
    G = w.spec.group
    qh = q.cpu().to(torch.float64).numpy()
    qp = q_pos.cpu().numpy()
    res = {}
    for r in rows:
        s, l, h = w.spec.row_coords(r)
        k, v, pos = row_kv(w, r)
        qg = qh[s, l, h * G:(h + 1) * G]
        if k.shape[0] == 0:
            res[r] = (np.zeros_like(qg), np.full(G, -np.inf), np.zeros(0))
        else:
            res[r] = od.decode_step(qg, k, v, int(qp[s]), pos)
    return res


def run(w, q, q_pos, scores=None, flags=0):
    S, L, Hq, D = q.shape
    out = torch.full((S, L, Hq, D), 7.0, device=DEV)
    lse = torch.full((S, L, Hq), 7.0, device=DEV)
    status = torch.zeros(2, dtype=torch.int32, device=DEV)
    kvc.kvc_decode_attention(w.cache, q, q_pos, out, lse, scores, flags, status)
    torch.cuda.synchronize()
    return out, lse, status


def check(w, q, q_pos, out, lse, scores, rows, what):
    G = w.spec.group
    orc = oracle_rows(w, q, q_pos, rows)
    o, ls = out.cpu().numpy(), lse.cpu().numpy()
    sc = scores.cpu().numpy() if scores is not None else None
    for r in rows:
        s, l, h = w.spec.row_coords(r)
        eo, el, ei = orc[r]
        go, gl = o[s, l, h * G:(h + 1) * G], ls[s, l, h * G:(h + 1) * G]
        fin = np.isfinite(el)
        assert np.array_equal(np.isfinite(gl), fin), f"{what} row {r}: empty heads differ"
        assert np.all(np.abs(gl[fin] - el[fin]) <= 2e-5), f"{what} row {r}: lse {gl} vs {el}"
        err = np.abs(go - eo)
        assert np.all(err <= 2e-5 + 1e-4 * np.abs(eo)), f"{what} row {r}: output max err {err.max()}"
        if sc is not None:
            H.assert_scores_close(sc[r, :len(ei)], ei, f"{what} row {r}")


CASES = {
    "llama8b_shape_ragged": dict(),
    "multi_seq_layer": dict(S=3, L=2, ctx=(1500, 2817, 4000), seed=32),
    "gqa7": dict(Hq=28, Hkv=4, ctx=(2100,), seed=33),
    "gqa1_f32_d64": dict(Hq=4, Hkv=4, D=64, dtype="f32", ctx=(3000,), seed=34),
    "gqa8_d64": dict(Hq=16, Hkv=2, D=64, ctx=(2500,), seed=35),
    "gqa4_d64": dict(Hq=8, Hkv=2, D=64, ctx=(2222, 999), S=2, seed=46),
    "gqa3": dict(Hq=24, Hkv=8, ctx=(1800,), seed=47),
    "gqa8_d128": dict(Hq=64, Hkv=8, ctx=(3001, 1234), S=2, seed=49),
    # 8-token pages: 8-slot chunks, so the dot products run on the FMA pipes with the logits in TMEM (G = 4)
    # and in shared memory (G = 8)
    "pages8_gqa4": dict(ctx=(2500, 777), S=2, seed=50, P=8),
    # one and two query heads per KV head on the tensor-core chunks
    "mha_bf16": dict(Hq=8, Hkv=8, ctx=(2600,), seed=53),
    "gqa2_bf16": dict(Hq=16, Hkv=8, ctx=(1500, 2222), S=2, seed=54),
    "mha_bf16_d64": dict(Hq=4, Hkv=4, D=64, ctx=(3100,), seed=55),
    "pages8_gqa8": dict(Hq=64, Hkv=8, ctx=(1900,), seed=51, P=8),
    # 12-token pages: 12-slot chunks (not a power of two)
    "pages12_gqa4": dict(ctx=(2000,), seed=52, P=12),
    "gqa2_f32": dict(Hq=4, Hkv=2, dtype="f32", ctx=(1111,), seed=36),
    "short_rows": dict(S=2, ctx=(17, 300), seed=37),
}


@pytest.mark.parametrize("case", list(CASES), ids=list(CASES))
def test_decode_parity(case):
    w = H.build(spec_of(**CASES[case]))
    q, q_pos = decode_inputs(w)
    scores = torch.full((w.spec.rows, w.spec.max_slots), -7.0, device=DEV)
    out, lse, status = run(w, q, q_pos, scores)
    assert kvc.device_status(status)[0] == 0
    check(w, q, q_pos, out, lse, scores, range(w.spec.rows), case)
    rl = w.layout.row_len.numpy()
    got = scores.cpu().numpy()
    for r in range(w.spec.rows):
        assert np.all(got[r, rl[r]:] == -7.0), "slots beyond the row length must not be written"


def test_decode_causal_mask_and_permuted_slots():
    """A query in the middle of the context sees only the slots at or before it, wherever they sit in the row
    (after a compaction the slot order is not position order)."""
    w = H.build(spec_of(S=2, ctx=(3000, 2000), seed=38))
    g = torch.Generator().manual_seed(5)
    for r in range(w.spec.rows):
        n = int(w.cache.row_len[r])
        perm = torch.randperm(n, generator=g).to(torch.int32)
        w.cache.slot_pos[r, :n] = w.cache.slot_pos[r, :n][perm.to(DEV).long()]
    q, q_pos = decode_inputs(w, q_pos=[1234, 17])
    scores = torch.zeros((w.spec.rows, w.spec.max_slots), device=DEV)
    out, lse, status = run(w, q, q_pos, scores)
    assert kvc.device_status(status)[0] == 0
    check(w, q, q_pos, out, lse, scores, range(w.spec.rows), "mid-context")
    # hidden slots get exactly zero
    sp = w.cache.slot_pos.cpu().numpy()
    got = scores.cpu().numpy()
    for r in range(w.spec.rows):
        s, _, _ = w.spec.row_coords(r)
        n = int(w.cache.row_len[r])
        assert np.all(got[r, :n][sp[r, :n] > int(q_pos[s])] == 0.0)


def test_decode_no_visible_key_and_empty_row():
    """A query before every cached key and an empty row: lse -inf, output zeros, scores zero."""
    w = H.build(spec_of(S=2, ctx=(500, 600), seed=39))
    w.cache.slot_pos[:, :].add_(10)
    w.cache.row_len[w.spec.row_id(1, 0, 3)] = 0
    q, q_pos = decode_inputs(w, q_pos=[5, 10**6])
    scores = torch.full((w.spec.rows, w.spec.max_slots), 3.0, device=DEV)
    out, lse, status = run(w, q, q_pos, scores)
    assert kvc.device_status(status)[0] == 0
    G = w.spec.group
    assert torch.all(torch.isneginf(lse[0])) and torch.all(out[0] == 0)
    assert torch.all(scores[:w.spec.num_kv_heads, :500] == 0)
    h = 3
    assert torch.all(torch.isneginf(lse[1, 0, h * G:(h + 1) * G])) and torch.all(out[1, 0, h * G:(h + 1) * G] == 0)
    assert torch.all(scores[w.spec.row_id(1, 0, 3)] == 3.0)
    check(w, q, q_pos, out, lse, scores, range(w.spec.rows), "empty")


def test_decode_accumulate_deterministic_and_attention_only():
    w = H.build(spec_of(ctx=(2500,), seed=40))
    q, q_pos = decode_inputs(w)
    s1 = torch.zeros((w.spec.rows, w.spec.max_slots), device=DEV)
    o1, l1, _ = run(w, q, q_pos, s1)
    s2 = s1.clone()
    o2, l2, _ = run(w, q, q_pos, s2, kvc.KVC_SCORE_ACCUMULATE)
    torch.testing.assert_close(s2, 2 * s1, rtol=1e-6, atol=0)
    assert torch.equal(o1, o2) and torch.equal(l1, l2), "results must repeat bit for bit"
    o3, l3, st = run(w, q, q_pos, None)
    assert kvc.device_status(st)[0] == 0
    assert torch.equal(o1, o3) and torch.equal(l1, l3)


def test_decode_reports_bad_page():
    w = H.build(spec_of(ctx=(700,), seed=41))
    w.cache.block_table[2, 3] = -1
    q, q_pos = decode_inputs(w)
    _, _, status = run(w, q, q_pos, None)
    code, row, _ = kvc.device_status(status)
    assert (code, row) == (1, 2)


def test_decode_host_validation():
    w = H.build(spec_of(ctx=(300,), seed=42))
    q, q_pos = decode_inputs(w)
    out = torch.zeros(q.shape, device=DEV)
    lse = torch.zeros(q.shape[:3], device=DEV)
    with pytest.raises(kvc.KvcError, match="unknown flags"):
        kvc.kvc_decode_attention(w.cache, q, q_pos, out, lse, None, 2)
    q9 = torch.zeros((1, 1, 72, 128), dtype=q.dtype, device=DEV)   # 9 query heads per KV head
    with pytest.raises(kvc.KvcError, match="at most 8"):
        kvc.kvc_decode_attention(w.cache, q9, q_pos, torch.zeros(q9.shape, device=DEV),
                                 torch.zeros(q9.shape[:3], device=DEV), None, 0)


def test_decode_unaligned_scores_keep_logits_in_shared_memory():
    """Scores that do not start on a 16-byte boundary cannot ride in the stages' 16-byte copies, so the kernel
    keeps the logits in shared memory instead of TMEM (and forms the dot products on the FMA pipes, not the
    tensor cores): both layouts match the oracle, and each other within the same bounds."""
    w = H.build(spec_of(ctx=(3001,), seed=45))
    q, q_pos = decode_inputs(w)
    R, M = w.spec.rows, w.spec.max_slots
    base = torch.full((R * M + 1,), -7.0, device=DEV)
    shifted = base[1:].view(R, M)
    assert shifted.data_ptr() % 16 != 0
    out, lse, status = run(w, q, q_pos, shifted)
    assert kvc.device_status(status)[0] == 0
    check(w, q, q_pos, out, lse, shifted, range(R), "unaligned scores")
    assert torch.all(shifted[:, 3001:] == -7.0) and base[0] == -7.0
    aligned = torch.full((R, M), -7.0, device=DEV)
    out2, lse2, _ = run(w, q, q_pos, aligned)
    check(w, q, q_pos, out2, lse2, aligned, range(R), "aligned scores")
    torch.testing.assert_close(out, out2, rtol=2e-4, atol=4e-5)
    torch.testing.assert_close(lse, lse2, rtol=0, atol=4e-5)
    torch.testing.assert_close(aligned, shifted, rtol=2e-3, atol=2e-6)


def test_decode_unaligned_query_takes_the_simt_chunks():
    """A query that does not start on a 4-byte boundary cannot feed the tensor-core chunks (their query fragments are
    bf16 pairs): the kernel forms the dot products on the FMA pipes instead; both match the oracle."""
    w = H.build(spec_of(S=2, ctx=(1700, 2900), seed=48))
    q, q_pos = decode_inputs(w)
    base = torch.empty(q.numel() + 1, dtype=q.dtype, device=DEV)
    qs = base[1:].view(q.shape)
    qs.copy_(q)
    assert qs.data_ptr() % 4 != 0
    R, M = w.spec.rows, w.spec.max_slots
    scores = torch.full((R, M), -7.0, device=DEV)
    out, lse, status = run(w, qs, q_pos, scores)
    assert kvc.device_status(status)[0] == 0
    check(w, q, q_pos, out, lse, scores, range(R), "unaligned query")
    s2 = torch.full((R, M), -7.0, device=DEV)
    out2, lse2, _ = run(w, q, q_pos, s2)
    torch.testing.assert_close(out, out2, rtol=2e-4, atol=4e-5)
    torch.testing.assert_close(lse, lse2, rtol=0, atol=4e-5)
    torch.testing.assert_close(scores, s2, rtol=2e-3, atol=2e-6)


def test_decode_long_row_many_chunks_per_warp():
    """A 90,000-slot row (one query head per KV head, the longest the logits buffer takes at this width): each
    warp streams about 88 chunks, so its page ids come in three batches of 32."""
    w = H.build(spec_of(Hq=1, Hkv=1, ctx=(90000,), seed=44, heavy=0.01))
    q, q_pos = decode_inputs(w, q_pos=[70000])
    scores = torch.zeros((w.spec.rows, w.spec.max_slots), device=DEV)
    out, lse, status = run(w, q, q_pos, scores)
    assert kvc.device_status(status)[0] == 0
    check(w, q, q_pos, out, lse, scores, [0], "long row")


def test_decode_full_size_sampled_rows():
    """The Llama-3-8B layer at 32K context, in the launch configuration the benchmark times
    (all 32 layers), checked on sampled rows."""
    spec = synth.Spec(name="decode_llama8b_32k", seed=43, num_seqs=1, num_layers=32, num_q_heads=32, num_kv_heads=8,
                      head_dim=128, dtype="bf16", ctx=[32768], budget=512, heavy_frac=0.02)
    w = H.build(spec)
    q, q_pos = decode_inputs(w)
    scores = torch.zeros((spec.rows, spec.max_slots), device=DEV)
    out, lse, status = run(w, q, q_pos, scores)
    assert kvc.device_status(status)[0] == 0
    check(w, q, q_pos, out, lse, scores, [0, 77, 130, 255], "llama8b 32k")
    # every row's scores sum to its group size (the probabilities of each head sum to one)
    sums = scores.sum(dim=1).cpu().numpy()
    assert np.all(np.abs(sums - spec.group) <= 1e-3 * spec.group)


def test_decode_bench_workload_sampled_rows():
    """The workload and launch configuration bench.py --decode times: one layer of the batch of 16 sequences
    (context 8K-33K, 128 rows), checked on sampled rows."""
    spec = synth.batch16(num_layers=1)
    w = H.build(spec)
    q, q_pos = decode_inputs(w)
    scores = torch.zeros((spec.rows, spec.max_slots), device=DEV)
    out, lse, status = run(w, q, q_pos, scores, kvc.KVC_SCORE_ACCUMULATE)
    assert kvc.device_status(status)[0] == 0
    check(w, q, q_pos, out, lse, scores, [0, 37, 64, 101, 127], "batch16 layer")
