"""CPU-only checks of the C-ABI library and the host logic (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

from agent_kv_cache_lse_b200 import kvc, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    with open(os.path.join(ROOT, "include", "kvc.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(kvc_\w+)\s*\(", text, re.M)))


def test_library_exports_every_declared_entry_point():
    L = kvc.lib()
    names = declared_entry_points()
    assert {"kvc_score_from_lse", "kvc_lrfu_update", "kvc_select_budget", "kvc_plan_slots", "kvc_compact_pages",
            "kvc_confidence_ratchet"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/kvc.h but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", kvc.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (kvc_\w+)", out))
    assert set(names) == exported, f"exports differ from the header: {set(names) ^ exported}"
    assert set(kvc.EXPORTS) == set(names)


def test_noalloc_row_limit_matches_header():
    """The binding's copy of KVC_NOALLOC_MAX_ROWS is the header's value (the GPU test builds its over-limit case
    from the binding's copy)."""
    with open(os.path.join(ROOT, "include", "kvc.h")) as f:
        m = re.search(r"#define\s+KVC_NOALLOC_MAX_ROWS\s+(\d+)", f.read())
    assert m and int(m.group(1)) == kvc.NOALLOC_MAX_ROWS


def test_struct_layouts_match_header_sizes():
    # kvc_cache: 2 pointers + int64 + 4 int32 + 4 pointers + 4 int32 (with padding) on LP64
    assert ctypes.sizeof(kvc.KvcCache) == 2 * 8 + 8 + 4 * 4 + 4 * 8 + 4 * 4
    assert ctypes.sizeof(kvc.KvcQueries) == 4 * 8 + 2 * 4
    assert ctypes.sizeof(kvc.KvcRatchetParams) == 10 * 4
    assert ctypes.sizeof(kvc.KvcRatchetSeqState) == 3 * 8 + 6 * 8 + 4 * 4


def test_host_validation_without_gpu():
    L = kvc.lib()
    assert L.kvc_score_from_lse(None, None, None, 0, None, None) == kvc.KVC_ERR_INVALID_ARGUMENT
    assert b"NULL" in L.kvc_last_error()
    c = kvc.KvcCache()
    c.num_seqs, c.num_layers, c.num_kv_heads = 1, 1, 1
    c.page_size, c.max_pages_per_row, c.head_dim, c.dtype = 16, 4, 96, kvc.KVC_BF16
    c.block_table = c.row_len = c.slot_pos = 16
    assert L.kvc_select_budget(ctypes.byref(c), 16, 16, 0, 16, 16, None, None) == kvc.KVC_ERR_UNSUPPORTED
    c.head_dim = 128
    assert L.kvc_lrfu_update(ctypes.byref(c), 16, 16, ctypes.c_float(-1.0), ctypes.c_float(0.9), 1, 0, None,
                             None) == kvc.KVC_ERR_INVALID_ARGUMENT
    assert L.kvc_compact_pages(ctypes.byref(c), 16, 16, 16, 16, None, 16, 4, 16, 16, 0, None,
                               None) == kvc.KVC_ERR_INVALID_ARGUMENT   # pools missing
    p = kvc.ratchet_params()
    assert kvc.kvc_ratchet_state_bytes(16, p) > 16 * ctypes.sizeof(kvc.KvcRatchetSeqState)
    bad = kvc.ratchet_params(top_k=0)
    assert kvc.kvc_ratchet_state_bytes(16, bad) == 0
    assert kvc.kvc_compact_workspace_bytes(10) == 11 * 8
    assert L.kvc_status_string(2) == b"unsupported"


def test_generator_is_chunking_independent():
    spec = synth.llama8b_layer(ctx=1024)
    pos = torch.arange(0, 1024)
    whole = synth.key_values(spec, 0, 0, 3, pos)
    parts = torch.cat([synth.key_values(spec, 0, 0, 3, pos[a:a + 100]) for a in range(0, 1024, 100)])
    assert torch.equal(whole.view(torch.int16), parts.view(torch.int16))
    x = synth.normal(7, synth.S_Q, torch.arange(200000))
    assert abs(float(x.mean())) < 0.01 and abs(float(x.std()) - 1.0) < 0.01


def test_segment_trace_shape():
    """Observation / reasoning / action segments in the ranges given, observation first; actions ~1-2%."""
    spec = synth.llama8b_layer()
    lab = synth.segment_labels(spec, 0, 32768).numpy()
    assert lab[0] == synth.LABEL_OBS
    runs = np.split(lab, np.flatnonzero(np.diff(lab)) + 1)
    for run in runs[:-1]:
        lo, hi = spec.seg_ranges[int(run[0])]
        assert lo <= len(run) <= hi
    share = float((lab == synth.LABEL_ACTION).mean())
    assert 0.005 < share < 0.03


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "agent_kv_cache_lse_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                with open(os.path.join(dirpath, f)) as fh:
                    src = fh.read()
                assert not re.search(r"^\s*(from|import)\s+oracle\b", src, re.M), f"{f} imports the oracle"


def test_layout_block_tables_are_disjoint():
    spec = synth.batch16(num_seqs=3, num_layers=2, lo=300, hi=900)
    lay = synth.make_layout(spec)
    bt = lay.block_table.numpy()
    used = bt[bt >= 0]
    assert len(np.unique(used)) == len(used)
    assert used.max() < lay.num_pages
    for r in range(spec.rows):
        assert (bt[r] >= 0).sum() == -(-int(lay.row_len[r]) // 16)


def test_bench_traffic_follows_kernel_source(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed ncu summary only while the kernel source hash matches."""
    import hashlib
    import bench
    t = bench.profiled_traffic()
    assert t is None or t > 0
    src = tmp_path / "k.cu"
    src.write_text("x")
    prof = tmp_path / "p.md"
    prof.write_text(f"source: {src}\nsource_sha256: {'0' * 64}\ndram_bytes_per_launch: 5\n")
    monkeypatch.setattr(bench, "SCORE_PROFILE", str(prof))
    assert bench.profiled_traffic() is None
    prof.write_text(f"source: {src}\nsource_sha256: {hashlib.sha256(b'x').hexdigest()}\ndram_bytes_per_launch: 5\n")
    assert bench.profiled_traffic() == 5
    assert bench.profiled_traffic(str(prof)) == 5
    d = bench.profiled_traffic(bench.DECODE_PROFILE)
    assert d is None or d > 0


def test_decode_host_validation_without_gpu():
    """kvc_decode_attention refuses bad arguments, and rows whose logits cannot fit a cluster, before any launch
    (the fake pointers are never dereferenced)."""
    L = kvc.lib()
    c = kvc.KvcCache()
    c.num_seqs, c.num_layers, c.num_kv_heads = 1, 1, 1
    c.page_size, c.max_pages_per_row, c.head_dim, c.dtype = 16, 4, 128, kvc.KVC_BF16
    c.block_table = c.row_len = c.slot_pos = 256
    c.k_pool = c.v_pool = 256
    c.num_pages = 4
    f = ctypes.c_void_p(256)
    call = lambda q=f, hq=4, flags=0: L.kvc_decode_attention(ctypes.byref(c), q, f, hq, f, f, None, flags, None, None)
    assert call(q=None) == kvc.KVC_ERR_INVALID_ARGUMENT
    assert call(flags=2) == kvc.KVC_ERR_INVALID_ARGUMENT
    assert call(hq=0) == kvc.KVC_ERR_INVALID_ARGUMENT
    assert call(hq=9) == kvc.KVC_ERR_UNSUPPORTED            # 9 query heads per KV head
    c.max_pages_per_row = 10000                             # 160,000 slots: logits beyond a cluster's memory
    assert call() == kvc.KVC_ERR_UNSUPPORTED
    assert b"logits" in L.kvc_last_error()


@pytest.mark.skipif(torch.cuda.is_available(), reason="a supported size would launch the kernel on fake pointers")
@pytest.mark.parametrize("group,limit", [(1, 215040), (2, 143360), (4, 82736), (8, 42320)])
def test_decode_row_limit_matches_the_header(group, limit):
    """bf16, head_dim 128, 16-slot pages: the longest row the decode entry point takes, as the header states it.
    Without a GPU a supported size gets as far as the launch and fails there (KVC_ERR_CUDA); one page more is
    refused on the host (KVC_ERR_UNSUPPORTED)."""
    L = kvc.lib()
    c = kvc.KvcCache()
    c.num_seqs, c.num_layers, c.num_kv_heads = 1, 1, 8
    c.page_size, c.head_dim, c.dtype = 16, 128, kvc.KVC_BF16
    c.block_table = c.row_len = c.slot_pos = 256
    c.k_pool = c.v_pool = 256
    c.num_pages = 4
    f = ctypes.c_void_p(256)
    for pages, want in ((limit // 16, kvc.KVC_ERR_CUDA), (limit // 16 + 1, kvc.KVC_ERR_UNSUPPORTED)):
        c.max_pages_per_row = pages
        assert L.kvc_decode_attention(ctypes.byref(c), f, f, 8 * group, f, f, f, 0, None, None) == want, pages


def test_step_scores_host_validation_without_gpu():
    """kvc_step_scores refuses bad arguments before any launch (fake pointers are never dereferenced)."""
    L = kvc.lib()
    c = kvc.KvcCache()
    c.num_seqs, c.num_layers, c.num_kv_heads = 1, 1, 1
    c.page_size, c.max_pages_per_row, c.head_dim, c.dtype = 16, 4, 128, kvc.KVC_BF16
    c.block_table = c.row_len = c.slot_pos = 256
    f = ctypes.c_void_p(256)
    call = lambda sc=f, ms=8, beta=0.5: L.kvc_step_scores(ctypes.byref(c), sc, f, f, ms, ctypes.c_float(beta), f,
                                                          None, None)
    assert call(sc=None) == kvc.KVC_ERR_INVALID_ARGUMENT
    assert call(ms=0) == kvc.KVC_ERR_UNSUPPORTED and call(ms=4097) == kvc.KVC_ERR_UNSUPPORTED
    assert call(beta=1.5) == kvc.KVC_ERR_INVALID_ARGUMENT and call(beta=float("nan")) == kvc.KVC_ERR_INVALID_ARGUMENT


def test_step_starts_follow_reasoning_segments():
    spec = synth.llama8b_layer()
    st = synth.step_starts(spec, 0).numpy()
    lab = synth.segment_labels(spec, 0, spec.ctx[0]).numpy()
    assert st[0] == 0 and np.all(np.diff(st) > 0)
    assert np.all(lab[st[1:]] == synth.LABEL_REASON) and np.all(lab[st[1:] - 1] != synth.LABEL_REASON)
    assert len(st) - 1 == int(((lab[1:] == synth.LABEL_REASON) & (lab[:-1] != synth.LABEL_REASON)).sum())


def test_binding_checks_shapes_and_dtypes():
    """The Python binding refuses mismatched tensors before the C call (CPU tensors: nothing reaches a device)."""
    S, L, Hkv, P, D, mp = 2, 1, 2, 16, 64, 4
    rows = S * L * Hkv
    cache = kvc.Cache(torch.zeros((8, P, D), dtype=torch.bfloat16), torch.zeros((8, P, D), dtype=torch.bfloat16),
                      torch.zeros((rows, mp), dtype=torch.int32), torch.zeros(rows, dtype=torch.int32),
                      torch.zeros((rows, mp * P), dtype=torch.int32), None, S, L, Hkv)
    q = torch.zeros((S, L, 4, D), dtype=torch.bfloat16)
    qp = torch.zeros(S, dtype=torch.int32)
    out, lse = torch.zeros((S, L, 4, D)), torch.zeros((S, L, 4))
    with pytest.raises(kvc.KvcError, match="q: dtype"):
        kvc.kvc_decode_attention(cache, q.float(), qp, out, lse)
    with pytest.raises(kvc.KvcError, match="out: shape"):
        kvc.kvc_decode_attention(cache, q, qp, out[:, :, :2], lse)
    with pytest.raises(kvc.KvcError, match="scores: shape"):
        kvc.kvc_decode_attention(cache, q, qp, out, lse, torch.zeros((rows, 5)))
    with pytest.raises(kvc.KvcError, match="q_pos: dtype"):
        kvc.kvc_decode_attention(cache, q, qp.long(), out, lse)
    sc = torch.zeros((rows, mp * P))
    st, ns = torch.zeros((S, 3), dtype=torch.int32), torch.ones(S, dtype=torch.int32)
    with pytest.raises(kvc.KvcError, match="step_start: shape"):
        kvc.kvc_step_scores(cache, sc, st[:1], ns, sc)
    with pytest.raises(kvc.KvcError, match="out must be contiguous"):
        kvc.kvc_step_scores(cache, sc, st, ns, torch.zeros((mp * P, rows)).t())


def test_beacon_update_host_validation():
    """Bad sizes are refused before anything reaches the device (fake pointers are never dereferenced)."""
    from agent_kv_cache_lse_b200 import kvc
    L = kvc.lib()
    fake = ctypes.c_void_p(256)
    call = lambda **kw: L.kvc_beacon_update(kw.get("q", fake), fake, kw.get("S", 1), 1, 1, kw.get("D", 128),
                                            kw.get("mq", 8), kw.get("dt", 1), fake, fake, kw.get("B", 4),
                                            kw.get("out", None), kw.get("omq", 0), None, None)
    assert call(q=None) == 1                       # KVC_ERR_INVALID_ARGUMENT
    assert call(B=0) == 2 and call(B=65) == 2      # KVC_ERR_UNSUPPORTED
    assert call(D=300) == 2 and call(mq=70000) == 2 and call(dt=7) == 2
    assert call(S=0) == 1
    assert call(out=fake, omq=2) == 1              # output rows fewer than beacons
