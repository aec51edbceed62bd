"""Benchmark of the eviction/compaction hot path on B200.

One step = one full eviction round (confidence ratchet -> score from LSE -> LRFU -> top-budget
select -> slot plan -> in-place compaction) over the Llama-3-8B-shaped single layer at 32K
context (32 q / 8 KV heads, head_dim 128, bf16, 16-token pages, ~608 action-token queries,
budget 512, 64 decode steps of 128,256-token logits for the ratchet).  Inputs are seeded
synthetic data resident in HBM; the compacted state is restored and L2 is flushed (a 256 MB
write) outside the timed region before every step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  N > 1 runs one independent replica per GPU (weak scaling:
the path shards by sequence and needs no collective).

Separate single-GPU lines for the entry points beside the round, each with its own workload,
metric and roofline:
  --decode   one decode step of paged attention with the scores folded in (kvc_decode_attention),
             one layer of the batch of 16 sequences at 8K-33K;
  --stepkv   step-aware ranking scores (kvc_step_scores), 16 sequences x 8 layers x 8 KV heads;
  --beacon   beacon-query maintenance (kvc_beacon_update), the streaming shape.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KV entries scored+compacted/sec at 32K ctx"
UNIT = "entries/s"
WORKLOAD = ("Llama-3-8B-shaped single layer: 32 q / 8 KV heads, head_dim 128, bf16 K/V ~N(0,1) with 2% "
            "heavy-hitter keys (x4), 32,768 tokens in 16-token pages (shuffled pool), observation/reasoning/"
            "action segments, all action tokens as queries, budget 512, ratchet over 64 steps x 128,256 logits")


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def algorithmic_work(spec, layout, queries):
    """FLOP of the QK^T contraction over visible (key, query-head) pairs, exps, and bytes of one round."""
    P, D = spec.page_size, spec.head_dim
    G = spec.group
    flops = exps = 0
    qpos = queries.q_pos.cpu().numpy()
    numq = queries.num_q.cpu().numpy()
    sp = layout.slot_pos
    entries = 0
    per_seq = {}
    ident = torch.arange(sp.shape[1], dtype=sp.dtype)
    for r in range(spec.rows):
        s, _, _ = spec.row_coords(r)
        n = int(layout.row_len[r])
        entries += n
        row_pos = sp[r, :n]
        # rows of a fresh layout hold token i in slot i: their visible pairs depend on the sequence only
        fresh = bool(torch.equal(row_pos, ident[:n]))
        key = (s, n) if fresh else None
        if key is not None and key in per_seq:
            vis_sum = per_seq[key]
        else:
            qp = np.sort(qpos[s, :numq[s]])
            vis_sum = int((G * (len(qp) - np.searchsorted(qp, row_pos.numpy(), side="left"))).sum())
            if key is not None:
                per_seq[key] = vis_sum
        flops += 2 * D * vis_sum
        exps += vis_sum
    esize = 2 if spec.dtype == "bf16" else 4
    nq_total = int(numq.sum())
    kv_bytes = entries * D * esize                                  # K read once by scoring
    meta = entries * (4 + 4 + 4 + 4 + 1 + 1)                        # scores w/r, crf r/w, pos r, keep w
    q_bytes = nq_total * spec.num_layers * spec.num_q_heads * (D * esize + 4)
    logits = spec.num_seqs * spec.logits_steps * spec.vocab * 4
    return dict(entries=entries, flops=flops, exps=exps, kv_bytes=kv_bytes, meta_bytes=meta, q_bytes=q_bytes,
                logits_bytes=logits)


class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML (the source nvidia-smi reads) every 2 ms in a
    thread while the timed region runs (nvidia-smi's own loop is too coarse for a region this short)."""

    REASONS = [("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap")]

    def __init__(self, torch_index):
        self.torch_index = torch_index
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = None
        self._thread = None
        self.err = None

    def _handle(self, nv):
        uuid = None
        try:
            uuid = str(torch.cuda.get_device_properties(self.torch_index).uuid)
        except Exception:
            pass
        n = nv.nvmlDeviceGetCount()
        for i in range(n):
            h = nv.nvmlDeviceGetHandleByIndex(i)
            u = nv.nvmlDeviceGetUUID(h)
            u = u.decode() if isinstance(u, bytes) else u
            if uuid and u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                return h
        vis = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip().isdigit()]
        return nv.nvmlDeviceGetHandleByIndex(int(vis[self.torch_index]) if self.torch_index < len(vis) else self.torch_index)

    def start(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception as e:  # no NVML: report no clocks rather than guess
            self.err = repr(e)
            return
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    self.samples.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                    bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    for name, attr in self.REASONS:
                        if bits & getattr(nv, attr):
                            self.reasons.add(name)
                except Exception as e:
                    self.err = repr(e)
                time.sleep(0.002)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return {"error": self.err} if self.err else None
        self._stop.set()
        self._thread.join()
        if not self.samples:
            return {"error": self.err or "no samples"}
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "source": "NVML every 2 ms during the timed steps"}


def reduce_over_ranks(total_ms: float, entries: int, device):
    """Whole-job timing across replicas: the slowest rank's device time and the entries of all ranks."""
    t = torch.tensor([total_ms], dtype=torch.float64, device=device)
    e = torch.tensor([entries], dtype=torch.int64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    torch.distributed.all_reduce(e, op=torch.distributed.ReduceOp.SUM)
    return float(t.item()), int(e.item())


def build_workload(device):
    from agent_kv_cache_lse_b200 import kvc, synth
    spec = synth.llama8b_layer()
    layout = synth.make_layout(spec)
    kp = synth.fill_pool(spec, layout, "k", device)
    vp = synth.fill_pool(spec, layout, "v", device)
    qs = synth.make_queries(spec, device)
    lse = torch.zeros((1, 1, spec.num_q_heads, qs.max_q), dtype=torch.float32, device=device)
    cache = kvc.Cache(kp, vp, layout.block_table.to(device), layout.row_len.to(device), layout.slot_pos.to(device),
                      layout.slot_label.to(device), 1, 1, spec.num_kv_heads)
    queries = kvc.QuerySet(qs.q, lse, qs.q_pos.to(device), qs.num_q.to(device))
    # the attention kernel's LSE byproduct, produced here by the library's own LSE pass (setup, untimed)
    kvc.kvc_query_lse(cache, queries)
    logits = torch.stack([synth.logits(spec, 0, 0, spec.logits_steps, device=device)])
    torch.cuda.synchronize()
    return spec, layout, cache, queries, logits


def run_ours(args, rank, world, device):
    from agent_kv_cache_lse_b200 import kvc
    from agent_kv_cache_lse_b200.round import EvictionRound
    hbm, tf_burst, tf_sus, peak_kind = peaks()
    spec, layout, cache, queries, logits = build_workload(device)
    work = algorithmic_work(spec, layout, queries)
    rnd = EvictionRound(cache)
    mutable = [cache.k_pool, cache.v_pool, cache.block_table, cache.row_len, cache.slot_pos, cache.slot_label,
               rnd.crf]
    pristine = [t.clone() for t in mutable]
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    def restore():
        for t, p in zip(mutable, pristine):
            t.copy_(p)
        rnd.reset_ratchet()
        flush.fill_(1.0)

    side = torch.cuda.Stream(device=device)
    fork, join = torch.cuda.Event(), torch.cuda.Event()

    def step(e=None):
        # score, then the ratchet (side stream) beside the LRFU update, then select + plan (one launch), compact
        main = torch.cuda.current_stream()
        if e is not None:
            e[0].record(main)
        kvc.kvc_score_from_lse(cache, queries, rnd.scores, 0, rnd.status, main)
        if e is not None:
            e[1].record(main)
        # the LRFU update is enqueued first so that its clusters take their SMs before the ratchet's CTAs spread
        fork.record(main)
        kvc.kvc_lrfu_update(cache, rnd.scores, rnd.crf, 0.5, 0.9, 1, 0, rnd.status, main)
        side.wait_event(fork)
        kvc.kvc_confidence_ratchet(logits, rnd.state, rnd.budget, rnd.params, None, rnd.status, side)
        if e is not None:
            e[2].record(side)
        join.record(side)
        main.wait_event(join)
        kvc.kvc_select_plan(cache, rnd.crf, rnd.budget, rnd.keep, rnd.kept, rnd.move_src, rnd.move_dst,
                            rnd.num_moves, 0, rnd.status, main)
        kvc.kvc_compact_pages(cache, rnd.move_src, rnd.move_dst, rnd.num_moves, rnd.kept, rnd.crf, rnd.freed,
                              rnd.num_freed, rnd.workspace, rnd.status, main)
        if e is not None:
            e[3].record(main)

    for _ in range(args.warmup):
        restore()
        step()
    torch.cuda.synchronize()
    code = rnd.device_status()[0]
    if code != 0:
        raise RuntimeError(f"device status {rnd.device_status()} during warm-up")

    # the round as one CUDA graph (five calls, seven kernels, the ratchet on a parallel branch), with timing
    # events captured as nodes
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
    graph = None
    if not args.no_graph:
        restore()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step(ev)
        for _ in range(2):      # replay warm-up
            restore()
            graph.replay()
        torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    step_ms, score_ms, ratchet_ms = [], [], []
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]

    clocks = ClockSampler(torch.cuda.current_device())
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for k in range(args.steps):
        restore()
        if graph is not None:
            graph.replay()
            ev[3].synchronize()
            step_ms.append(ev[0].elapsed_time(ev[3]))
            score_ms.append(ev[0].elapsed_time(ev[1]))
            ratchet_ms.append(ev[1].elapsed_time(ev[2]))
        else:
            step(evs[k])
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    if graph is None:
        step_ms = [evs[k][0].elapsed_time(evs[k][3]) for k in range(args.steps)]
        score_ms = [evs[k][0].elapsed_time(evs[k][1]) for k in range(args.steps)]
        ratchet_ms = [evs[k][1].elapsed_time(evs[k][2]) for k in range(args.steps)]
    total_ms = float(sum(step_ms))
    entries_all = work["entries"] * world
    if world > 1:
        total_ms, entries_all = reduce_over_ranks(total_ms, work["entries"], device)
    assert rnd.device_status()[0] == 0

    # end to end through the same public calls with host buffers: H2D inputs, path, D2H results
    e2e = None
    if rank == 0:
        e2e = run_e2e(args, spec, cache, queries, logits, rnd, pristine, device)

    cpu = cpu_baseline("llama8b", [0, 2, 5, 7], 8, spec.budget) if (rank == 0 and world == 1 and not args.no_cpu) else None
    if rank != 0:
        return None
    ms_step = total_ms / args.steps
    value = entries_all / (total_ms / 1e3 / args.steps)
    score_avg = float(np.mean(score_ms))
    achieved = work["flops"] / (score_avg / 1e3) / 1e12
    bytes_step = work["kv_bytes"] + work["meta_bytes"] + work["q_bytes"] + work["logits_bytes"]
    t_roof = max(work["flops"] / (tf_burst * 1e12), bytes_step / (hbm * 1e9))
    sm_mhz = (clk or {}).get("sm_mhz", 1965.0)
    exp_ceiling = 16 * 148 * sm_mhz * 1e6
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "ms_per_step_p10_p50_p90": [float(np.percentile(step_ms, q)) for q in (10, 50, 90)],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded counter-based generator; shapes of the agent-trace workload)",
        "config": {"workload": WORKLOAD, "entries_per_step": work["entries"], "rows": spec.rows,
                   "queries": int(queries.num_q.sum()), "budget": spec.budget, "seq_len": 32768,
                   "parallelism": f"replicas x{world}", "l2": "flushed (256 MB write) before every step"},
        "roofline": {"kernel": "score_tc_kernel (kvc_score_from_lse)", "bound": "tensor", "achieved": achieved,
                     "peak": tf_burst, "unit": "TFLOP/s", "frac": achieved / tf_burst, "traffic": profiled_traffic(),
                     "traffic_unit": "bytes per launch (ncu dram read + write)",
                     "peak_source": f"{peak_kind} bf16 dense (burst)", "flops_per_launch": work["flops"],
                     "ms_per_launch": score_avg,
                     "exp_rate_per_s": work["exps"] / (score_avg / 1e3),
                     "exp_frac_of_mufu": work["exps"] / (score_avg / 1e3) / exp_ceiling},
        "step_roofline": {"t_roof_us": t_roof * 1e6, "t_step_us": ms_step * 1e3, "frac": t_roof / (ms_step / 1e3),
                          "bytes_per_step": bytes_step, "flops_per_step": work["flops"], "hbm_peak_gbs": hbm},
        "breakdown_ms": {"score": score_avg, "ratchet (beside the LRFU update)": float(np.mean(ratchet_ms)),
                         "after score: ratchet | lrfu, then select+plan+compact":
                             float(np.mean(step_ms) - np.mean(score_ms))},
        "gpu_launches": EvictionRound_KERNELS * args.steps,
        "launch": "CUDA graph of the round" if graph is not None else "direct C-ABI calls",
        "e2e": e2e,
        "cpu_baseline": cpu,
        "clocks": clk,
    }
    return line


EvictionRound_KERNELS = 7   # score, LRFU, confidence, budget update, select + plan, compaction moves, freed pages

SCORE_PROFILE = os.path.join(ROOT, "profiles", "score_tc_llama8b_32k.md")
DECODE_PROFILE = os.path.join(ROOT, "profiles", "decode_kernel_batch16_layer.md")
STEPKV_PROFILE = os.path.join(ROOT, "profiles", "step_scores_batch16_8layers.md")


def profiled_traffic(profile=None):
    """DRAM bytes per launch of a kernel from its committed ncu summary (the scoring kernel's by default), or
    None when the kernel source has changed since those counters were taken (the summary records the source's
    sha256)."""
    profile = profile or SCORE_PROFILE
    try:
        fields = {}
        with open(profile) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, _, v = line.partition(":")
                    fields[k.strip()] = v.strip()
        src = os.path.join(ROOT, fields["source"])
        with open(src, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
        if digest != fields["source_sha256"]:
            return None
        return int(fields["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def run_e2e(args, spec, cache, queries, logits, rnd, pristine, device):
    from agent_kv_cache_lse_b200 import kvc
    from agent_kv_cache_lse_b200.round import EvictionRound
    # host (pinned) copies of every input of a round
    h_in = {
        "k": pristine[0].cpu().pin_memory(), "v": pristine[1].cpu().pin_memory(),
        "bt": pristine[2].cpu().pin_memory(), "rl": pristine[3].cpu().pin_memory(),
        "sp": pristine[4].cpu().pin_memory(), "sl": pristine[5].cpu().pin_memory(),
        "q": queries.q.cpu().pin_memory(), "lse": queries.lse.cpu().pin_memory(),
        "qpos": queries.q_pos.cpu().pin_memory(), "numq": queries.num_q.cpu().pin_memory(),
        "logits": logits.cpu().pin_memory(),
    }
    # two device sets (inputs, round state, outputs) and two host output sets, so that round k + 1's inputs
    # cross PCIe while round k computes and its results come back (the link carries both directions at once)
    sets = []
    for _ in range(2):
        d = {k: torch.empty_like(v, device=device) for k, v in h_in.items()}
        c2 = kvc.Cache(d["k"], d["v"], d["bt"], d["rl"], d["sp"], d["sl"], 1, 1, spec.num_kv_heads)
        q2 = kvc.QuerySet(d["q"], d["lse"], d["qpos"], d["numq"])
        r2 = EvictionRound(c2)
        outs = {"k": d["k"], "v": d["v"], "bt": d["bt"], "rl": d["rl"], "sp": d["sp"], "sl": d["sl"], "crf": r2.crf,
                "freed": r2.freed, "num_freed": r2.num_freed, "budget": r2.budget}
        h_out = {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in outs.items()}
        sets.append((d, q2, r2, outs, h_out))
    h2d = sum(v.numel() * v.element_size() for v in h_in.values())
    d2h = sum(v.numel() * v.element_size() for v in sets[0][3].values())
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # set i's inputs have landed
    ev_done = [torch.cuda.Event() for _ in range(2)]  # set i's round has finished
    ev_out = [torch.cuda.Event() for _ in range(2)]   # set i's results are on the host (the set is free again)

    def one(k):
        i = k % 2
        d, q2, r2, outs, h_out = sets[i]
        s_in.wait_event(ev_out[i])
        with torch.cuda.stream(s_in):
            for key, v in h_in.items():
                d[key].copy_(v, non_blocking=True)
        ev_in[i].record(s_in)
        comp.wait_event(ev_in[i])
        r2.crf.zero_()
        r2.reset_ratchet(comp)
        r2.run(q2, d["logits"], stream=comp)
        ev_done[i].record(comp)
        s_out.wait_event(ev_done[i])
        with torch.cuda.stream(s_out):
            for key, v in outs.items():
                h_out[key].copy_(v, non_blocking=True)
        ev_out[i].record(s_out)

    for k in range(max(2, args.warmup)):
        one(k)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    s_in.wait_event(e0)
    for k in range(args.steps):
        one(k)
    comp.wait_event(ev_out[0])
    comp.wait_event(ev_out[1])
    e1.record(comp)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    entries = int(h_in["rl"].sum())
    return {"value": entries / (ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": ms, "pipeline": "each round copies its inputs in and its results out; two buffer sets "
                                          "let round k + 1's inputs and round k's results cross PCIe together"}


def oracle_row_inputs(spec, r, ratchet_steps):
    """Host inputs of one sampled row of a freshly laid-out workload, drawn from the seeded generator (no device
    involved): the row's keys and values (slot i holds token i), its group's query set with the LSE (oracle,
    prepared untimed), its labels, and `ratchet_steps` decode steps of logits of its sequence."""
    from agent_kv_cache_lse_b200 import synth
    from oracle import path as opath
    P, G = spec.page_size, spec.group
    s, l, h = spec.row_coords(r)
    n = spec.ctx[s]
    pos = torch.arange(n, dtype=torch.int64)
    k = synth.key_values(spec, s, l, h, pos, "k")
    v = synth.key_values(spec, s, l, h, pos, "v")
    npg = -(-n // P)
    kb = torch.zeros((npg * P, spec.head_dim), dtype=k.dtype)
    vb = torch.zeros_like(kb)
    kb[:n], vb[:n] = k, v
    kf = k.to(torch.float64).numpy()
    qp = synth.query_positions(spec, s)
    nq = len(qp)
    if spec.queries == "beacon_recent":
        qs = synth.streaming_queries(spec, list(spec.ctx), "cpu")
        q = qs.q[s, l, :nq, h * G:(h + 1) * G].to(torch.float64).numpy()
    else:
        q = synth.query_vectors(spec, s, l, nq)[:, h * G:(h + 1) * G].to(torch.float64).numpy()
    qp = qp.numpy()
    lse = opath.attention_lse(q, kf, qp, pos.numpy()).astype(np.float32).astype(np.float64)
    labels = (synth.segment_labels(spec, s, n) if spec.queries == "action"
              else torch.full((n,), synth.LABEL_REASON, dtype=torch.uint8)).numpy()
    logits = synth.logits(spec, s, 0, ratchet_steps).numpy().astype(np.float64) if ratchet_steps else None
    return dict(n=n, kf=kf, kb=kb.view(npg, P, -1).view(torch.int16).numpy(),
                vb=vb.view(npg, P, -1).view(torch.int16).numpy(), q=q, qp=qp, lse=lse, pos=pos.numpy(),
                labels=labels, logits=logits)


def oracle_row_path(spec, x, budget):
    """The oracle's path on one prepared row: scored, gated, selected, planned and compacted, plus the decode
    steps of the confidence monitor it carries.  Returns the entries processed."""
    from oracle import path as opath
    n, pos = x["n"], x["pos"]
    s = opath.scores_from_lse(x["q"], x["kf"], x["qp"], pos, x["lse"])
    crf = opath.lrfu_update(np.zeros(n), s, pos, 0.5, 0.9)
    keep = opath.select_budget(crf, pos, budget)
    src, dst, m = opath.plan_slots(keep, n)
    row = opath.PagedRow(block_table=np.arange(x["kb"].shape[0]), n=n, slot_pos=pos.copy(),
                         slot_label=x["labels"].copy(), crf=crf)
    opath.compact_row(x["kb"], x["vb"], row, src, dst, m, spec.page_size)
    if x["logits"] is not None:
        opath.Ratchet().round(x["logits"])
    return n


def _oracle_worker(job):
    """One sampled row in a spawned worker process limited to one BLAS thread: inputs prepared untimed, then the
    oracle's path timed.  Returns (entries, seconds)."""
    config, r, steps, budget = job
    from threadpoolctl import threadpool_limits
    with threadpool_limits(1):
        spec = config_spec(config)
        x = oracle_row_inputs(spec, r, steps)
        t0 = time.perf_counter()
        e = oracle_row_path(spec, x, budget)
        return e, time.perf_counter() - t0


def _oracle_prepare_worker(job):
    config, r, steps, budget = job
    from threadpoolctl import threadpool_limits
    with threadpool_limits(1):
        spec = config_spec(config)
        return oracle_row_inputs(spec, r, steps)


def _oracle_timed_worker(args):
    config, x, budget = args
    from threadpoolctl import threadpool_limits
    with threadpool_limits(1):
        spec = config_spec(config)
        t0 = time.perf_counter()
        e = oracle_row_path(spec, x, budget)
        return e, time.perf_counter() - t0


def cpu_baseline(config, rows, ratchet_steps, budget):
    """The oracle on the host cores over a bounded sample of the workload's rows, as two figures: one process with
    one thread running the sampled rows one after another, and a pool of one-thread processes (one per core,
    started with spawn) running them side by side.  Inputs (including the LSE) are prepared untimed."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    cores = len(os.sched_getaffinity(0))
    jobs = [(config, r, ratchet_steps, budget) for r in rows]
    nproc = min(cores, len(jobs))
    # spawned workers (never forked from a process that holds a CUDA context); a dead worker raises here
    with ProcessPoolExecutor(max_workers=nproc, mp_context=mp.get_context("spawn")) as pool:
        inputs = list(pool.map(_oracle_prepare_worker, jobs))
        # one thread: the rows one after another, each in a one-thread worker
        single = [pool.submit(_oracle_timed_worker, (config, x, budget)).result() for x in inputs]
        t0 = time.perf_counter()
        par = list(pool.map(_oracle_timed_worker, [(config, x, budget) for x in inputs]))
        t_par = time.perf_counter() - t0
    entries = sum(e for e, _ in single)
    t_single = sum(t for _, t in single)
    return {"value": entries / t_par, "unit": UNIT, "cores": nproc, "kind": "oracle",
            "one_thread": {"value": entries / t_single, "unit": UNIT, "cores": 1, "seconds": t_single},
            "sample": f"{len(rows)} of {config_spec(config).rows} rows ({entries} entries) through score/LRFU/select/"
                      f"plan/compact plus {ratchet_steps} ratchet decode steps per row (the rows' share of the "
                      f"round's monitor work), numpy fp64; value = the rows in parallel over {nproc} "
                      f"one-thread processes ({t_par:.1f} s wall), one_thread = one after another, one thread "
                      f"({t_single:.1f} s); inputs and LSE prepared untimed",
            "seconds": t_par, "host_cores": cores}


def config_spec(config, seqs=None, layers=None):
    """The workload of a bench configuration (seeded; the same spec on the GPU side and in the oracle's sample).
    seqs / layers shrink batch16 and stress to fewer sequences or layers of the same rows (a case small enough
    for an ncu capture)."""
    from agent_kv_cache_lse_b200 import synth
    size = {k: v for k, v in (("num_seqs", seqs), ("num_layers", layers)) if v is not None}
    if config == "llama8b":
        return synth.llama8b_layer()
    if config == "batch16":
        return synth.batch16(**size)
    if config == "stress":
        return synth.stress(**size)
    if config == "streaming":
        return synth.streaming()
    raise ValueError(config)


def run_reference(args, rank, world):
    """The oracle as the reference arm: each step is one row of the workload through the whole path plus
    8 of the 64 ratchet steps (its share), on the host cores."""
    if rank != 0:
        return None
    spec = config_spec("llama8b")
    x = oracle_row_inputs(spec, 0, 8)
    for _ in range(args.warmup):
        oracle_row_path(spec, x, spec.budget)
    t0 = time.perf_counter()
    entries = 0
    for _ in range(args.steps):
        entries += oracle_row_path(spec, x, spec.budget)
    dt = time.perf_counter() - t0
    value = entries / dt
    cores = len(os.sched_getaffinity(0))
    sample = f"1 of {spec.rows} rows (32,768 entries) + 8 of 64 ratchet steps per step, numpy fp64 in one process"
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def randn_pool(spec, layout, seed, device):
    """A pool of N(0, 1) values from torch's seeded generator in the spec dtype (the same values on every call)."""
    from agent_kv_cache_lse_b200 import synth
    g = torch.Generator(device=device).manual_seed(seed)
    pool = torch.empty((layout.num_pages, spec.page_size, spec.head_dim), dtype=synth.torch_dtype(spec), device=device)
    return refill_randn(pool, g, seed)


def refill_randn(pool, g, seed):
    g.manual_seed(seed)
    flat = pool.view(-1)
    step = 1 << 28
    for a in range(0, flat.numel(), step):
        b = min(flat.numel(), a + step)
        flat[a:b] = torch.randn(b - a, generator=g, device=pool.device, dtype=torch.float32).to(pool.dtype)
    return pool


CONFIG_TEXT = {
    "batch16": ("Batch of 16 sequences, context uniform in 8K-33K (seeded), 32 layers x 8 KV heads (32 q heads), "
                "head_dim 128, bf16 K/V ~N(0,1), 16-token pages in a shuffled pool with 5% spare pages, action-token "
                "queries, budget from the confidence ratchet (512 start, x1.75, cap 30,000) over 64 steps x 128,256 "
                "logits ~N(0, 2^2) per sequence"),
    "stress": ("Stress: 64 sequences x 33,000 tokens (partial last page) x 16 layers x 8 KV heads (32 q heads), "
               "head_dim 128, bf16 K/V ~N(0,1) (~138 GB of K+V; the 32-layer model runs as two such halves), "
               "shuffled pool, action-token queries, budget freeing 40% of every row's pages"),
}


def run_config(args, device):
    """One eviction round on the batch-16 or the stress workload: entries scored and compacted per second, with
    the round's roofline and the oracle on a sample of rows.  batch16 restores its pools from a copy, stress
    regenerates them (no room for a copy) outside the timed region."""
    from agent_kv_cache_lse_b200 import kvc, synth
    from agent_kv_cache_lse_b200.round import EvictionRound
    hbm, tf_burst, tf_sus, peak_kind = peaks()
    name = args.config
    spec = config_spec(name, args.seqs, args.layers)
    layout = synth.make_layout(spec)
    stress = name == "stress"
    if stress:
        gk = torch.Generator(device=device)
        gv = torch.Generator(device=device)
        kp = randn_pool(spec, layout, 51, device)
        vp = randn_pool(spec, layout, 52, device)
    else:
        kp = synth.fill_pool(spec, layout, "k", device)
        vp = synth.fill_pool(spec, layout, "v", device)
    qs = synth.make_queries(spec, device)
    lse = torch.zeros((spec.num_seqs, spec.num_layers, spec.num_q_heads, qs.max_q), dtype=torch.float32,
                      device=device)
    cache = kvc.Cache(kp, vp, layout.block_table.to(device), layout.row_len.to(device), layout.slot_pos.to(device),
                      layout.slot_label.to(device), spec.num_seqs, spec.num_layers, spec.num_kv_heads)
    queries = kvc.QuerySet(qs.q, lse, qs.q_pos.to(device), qs.num_q.to(device))
    kvc.kvc_query_lse(cache, queries)           # the attention kernel's LSE byproduct (setup, untimed)
    logits = None
    budget = spec.budget
    if stress:
        budget = synth.stress_budget(spec.ctx[0])
    else:
        logits = torch.stack([synth.logits(spec, s_, 0, spec.logits_steps, device=device)
                              for s_ in range(spec.num_seqs)])
    torch.cuda.synchronize()
    work = algorithmic_work(spec, layout, queries)
    rnd = EvictionRound(cache)
    meta = [cache.block_table, cache.row_len, cache.slot_pos, cache.slot_label]
    pristine = [t.clone() for t in meta] + ([] if stress else [kp.clone(), vp.clone()])
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)

    def restore():
        for t, p_ in zip(meta, pristine):
            t.copy_(p_)
        if stress:
            refill_randn(kp, gk, 51)
            refill_randn(vp, gv, 52)
        else:
            kp.copy_(pristine[4])
            vp.copy_(pristine[5])
        rnd.crf.zero_()
        rnd.reset_ratchet()
        rnd.budget.fill_(budget if stress else spec.budget)
        flush.fill_(1.0)

    def step(e):
        main = torch.cuda.current_stream()
        e[0].record(main)
        kvc.kvc_score_from_lse(cache, queries, rnd.scores, 0, rnd.status, main)
        e[1].record(main)
        rnd.run_after_scores(logits, 0.5, 0.9, main)
        e[2].record(main)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.warmup + args.steps)]
    for k in range(args.warmup):
        restore()
        step(ev[k])
    torch.cuda.synchronize()
    if rnd.device_status()[0] != 0:
        raise RuntimeError(f"device status {rnd.device_status()} during warm-up")
    clocks = ClockSampler(torch.cuda.current_device())
    step_ms, score_ms = [], []
    for k in range(args.warmup, args.warmup + args.steps):
        restore()
        torch.cuda.synchronize()
        if k == args.warmup:
            clocks.start()
        step(ev[k])
        torch.cuda.synchronize()
        step_ms.append(ev[k][0].elapsed_time(ev[k][2]))
        score_ms.append(ev[k][0].elapsed_time(ev[k][1]))
    clk = clocks.stop()
    assert rnd.device_status()[0] == 0, rnd.device_status()
    ms_step = float(np.mean(step_ms))
    score_avg = float(np.mean(score_ms))
    achieved = work["flops"] / (score_avg / 1e3) / 1e12
    bytes_step = work["kv_bytes"] + work["meta_bytes"] + work["q_bytes"] + (0 if stress else work["logits_bytes"])
    t_roof = max(work["flops"] / (tf_burst * 1e12), bytes_step / (hbm * 1e9))
    rng = np.random.default_rng(17)
    sample = sorted(int(x) for x in rng.choice(spec.rows, size=8, replace=False))
    steps_share = 0 if stress else max(1, round(spec.logits_steps * spec.num_seqs / spec.rows))
    del pristine
    reduced = args.seqs is not None or args.layers is not None  # a smaller case: no oracle leg
    cpu = None if args.no_cpu or reduced else cpu_baseline(name, sample, steps_share, budget)
    return {
        "metric": f"KV entries scored+compacted/sec ({name} workload)", "value": work["entries"] / (ms_step / 1e3),
        "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "ms_per_step_p10_p50_p90": [float(np.percentile(step_ms, q)) for q in (10, 50, 90)],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; " + ("torch N(0,1) pools" if stress else "counter-based generator") + ")",
        "config": {"workload": CONFIG_TEXT[name] if args.seqs is None and args.layers is None else
                   f"{CONFIG_TEXT[name]}, reduced to {spec.num_seqs} sequences x {spec.num_layers} layers",
                   "entries_per_step": work["entries"], "rows": spec.rows,
                   "queries": int(queries.num_q.sum()), "budget": "ratchet" if logits is not None else budget,
                   "l2": "flushed (256 MB write) before every step; inputs far larger than L2"},
        "roofline": {"kernel": "score_tc_kernel (kvc_score_from_lse)", "bound": "tensor", "achieved": achieved,
                     "peak": tf_sus, "unit": "TFLOP/s", "frac": achieved / tf_sus, "traffic": None,
                     "peak_source": f"{peak_kind} bf16 dense (sustained: a kernel of milliseconds)",
                     "flops_per_launch": work["flops"], "ms_per_launch": score_avg},
        "step_roofline": {"t_roof_us": t_roof * 1e6, "t_step_us": ms_step * 1e3, "frac": t_roof / (ms_step / 1e3),
                          "bytes_per_step": bytes_step, "flops_per_step": work["flops"], "hbm_peak_gbs": hbm,
                          "tensor_peak_tflops": tf_burst},
        "breakdown_ms": {"score": score_avg, "after score": ms_step - score_avg},
        "gpu_launches": (EvictionRound_KERNELS if logits is not None else 5) * args.steps,
        "launch": "direct C-ABI calls", "e2e": None,
        "e2e_note": "not measured: a host round trip of the whole pool per step is not how this path is used",
        "cpu_baseline": cpu, "clocks": clk,
    }


def append_decoded(spec, cache, crf, n_total, free, count=64):
    """Untimed bookkeeping between streaming rounds: `count` decoded tokens per row (seeded K/V at the next
    positions) go into the row's next slots, taking pages from the free list in order when the row needs one."""
    from agent_kv_cache_lse_b200 import synth
    P, D = spec.page_size, spec.head_dim
    dev = cache.k_pool.device
    bt = cache.block_table.cpu().numpy()
    rl = cache.row_len.cpu().numpy()
    phys, kv, vv, rows_idx, slots_all, pos_all = [], [], [], [], [], []
    for r in range(spec.rows):
        s, l, h = spec.row_coords(r)
        m = int(rl[r])
        for p in range(m // P, (m + count - 1) // P + 1):
            if bt[r, p] < 0:
                bt[r, p] = free.pop(0)
        slots = np.arange(m, m + count)
        pos = torch.arange(n_total[s], n_total[s] + count, dtype=torch.int64, device=dev)
        phys.append(bt[r, slots // P].astype(np.int64) * P + slots % P)
        kv.append(synth.key_values(spec, s, l, h, pos, "k"))
        vv.append(synth.key_values(spec, s, l, h, pos, "v"))
        rows_idx.append(np.full(count, r))
        slots_all.append(slots)
        pos_all.append(np.arange(n_total[s], n_total[s] + count))
    ph = torch.from_numpy(np.concatenate(phys)).to(dev)
    cache.k_pool.view(-1, D)[ph] = torch.cat(kv)
    cache.v_pool.view(-1, D)[ph] = torch.cat(vv)
    ri = torch.from_numpy(np.concatenate(rows_idx)).to(dev)
    si = torch.from_numpy(np.concatenate(slots_all)).to(dev)
    cache.slot_pos[ri, si] = torch.from_numpy(np.concatenate(pos_all).astype(np.int32)).to(dev)
    cache.slot_label[ri, si] = synth.LABEL_REASON
    crf[ri, si] = 0.0
    cache.block_table.copy_(torch.from_numpy(bt))
    cache.row_len.copy_(torch.from_numpy(rl + count))
    for s in range(spec.num_seqs):
        n_total[s] += count


def run_streaming(args, device):
    """Streaming rounds: 8 sequences x 32K context, 28 q / 4 KV heads, one layer; each round scores the cache
    with 16 beacon + 32 recent queries (the library's LSE pass for them timed inside the round), folds the hits into
    the carried LRFU values, keeps the top 30,000 per row, plans and compacts; 64 decoded tokens per row are
    appended between rounds (untimed).  Entries per second over `--rounds` rounds."""
    from agent_kv_cache_lse_b200 import kvc, synth
    from agent_kv_cache_lse_b200.round import EvictionRound
    hbm, tf_burst, tf_sus, peak_kind = peaks()
    spec = config_spec("streaming")
    layout = synth.make_layout(spec)
    kp = synth.fill_pool(spec, layout, "k", device)
    vp = synth.fill_pool(spec, layout, "v", device)
    cache = kvc.Cache(kp, vp, layout.block_table.to(device), layout.row_len.to(device), layout.slot_pos.to(device),
                      layout.slot_label.to(device), spec.num_seqs, spec.num_layers, spec.num_kv_heads)
    rnd = EvictionRound(cache)
    mutable = [kp, vp, cache.block_table, cache.row_len, cache.slot_pos, cache.slot_label, rnd.crf]
    pristine = [t.clone() for t in mutable]
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    D, G = spec.head_dim, spec.group

    # The round's calls (LSE pass + scores, LRFU + select, plan, compaction) as one CUDA graph over persistent
    # query buffers, with timing events captured as nodes: every round replays it after the round's queries
    # are copied in (the query count, the pools and every other pointer stay fixed from round to round).
    g = {}

    def round_calls(q, e):
        main = torch.cuda.current_stream()
        e[0].record(main)
        kvc.kvc_score_from_lse(cache, q, rnd.scores, kvc.KVC_SCORE_COMPUTE_LSE, rnd.status, main)
        e[1].record(main)
        rnd.run_after_scores(None, 0.5, 0.9, main)
        e[2].record(main)

    def stream_rounds(rounds, timed):
        for t, p_ in zip(mutable, pristine):
            t.copy_(p_)
        rnd.budget.fill_(spec.budget)
        bt0 = cache.block_table.cpu().numpy()
        used = set(int(x) for x in bt0[bt0 >= 0])
        free = [p for p in range(layout.num_pages) if p not in used]
        n_total = list(spec.ctx)
        out = []
        for rd in range(rounds):
            qs = synth.streaming_queries(spec, n_total, device=device)
            if "q" not in g:
                g["bufs"] = (qs.q.clone(), torch.empty((spec.num_seqs, 1, spec.num_q_heads, qs.max_q), device=device),
                             qs.q_pos.clone(), qs.num_q.clone())
                g["q"] = kvc.QuerySet(*g["bufs"])
                g["max_q"] = qs.max_q
            assert qs.max_q == g["max_q"]
            g["bufs"][0].copy_(qs.q)
            g["bufs"][2].copy_(qs.q_pos)
            g["bufs"][3].copy_(qs.num_q)
            entries = int(cache.row_len.sum())
            work = None
            if timed:
                work = (entries, streaming_work(spec, cache, qs))
            if args.no_graph or "warm" not in g:   # the first round runs the calls directly (one-time host set-up)
                g["warm"] = True
                flush.fill_(1.0)
                e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                round_calls(g["q"], e)
            else:
                if "graph" not in g:
                    torch.cuda.synchronize()
                    g["ev"] = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
                    g["graph"] = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g["graph"]):
                        round_calls(g["q"], g["ev"])
                flush.fill_(1.0)
                g["graph"].replay()
                e = g["ev"]
            torch.cuda.synchronize()
            out.append((e[0].elapsed_time(e[2]), e[0].elapsed_time(e[1]), work))
            free.extend(int(x) for x in rnd.freed[:int(rnd.num_freed[0])].cpu().tolist())
            append_decoded(spec, cache, rnd.crf, n_total, free)
        return out

    stream_rounds(max(1, args.warmup), False)
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    res = stream_rounds(args.rounds, True)
    clk = clocks.stop()
    assert rnd.device_status()[0] == 0, rnd.device_status()
    step_ms = [r[0] for r in res]
    score_ms = [r[1] for r in res]
    entries = sum(r[2][0] for r in res)
    flops = sum(r[2][1] for r in res)
    total_ms = float(sum(step_ms))
    achieved = flops / (sum(score_ms) / 1e3) / 1e12
    bytes_round = [r[2][0] * (D * 2 + 18) for r in res]
    t_roof = sum(max(r[2][1] / (tf_burst * 1e12), b / (hbm * 1e9)) for r, b in zip(res, bytes_round))
    cpu = None if args.no_cpu else cpu_baseline("streaming", [0, 9, 18, 31], 0, spec.budget)
    return {
        "metric": "KV entries scored+compacted/sec (streaming workload)", "value": entries / (total_ms / 1e3),
        "unit": UNIT, "n_gpus": 1, "steps": args.rounds, "warmup": args.warmup, "ms_per_step": total_ms / args.rounds,
        "ms_per_step_p10_p50_p90": [float(np.percentile(step_ms, q)) for q in (10, 50, 90)],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded counter-based generator)",
        "config": {"workload": "Streaming: 8 sequences x 32K context growing by 64 decoded tokens per round, 1 layer, "
                               "28 q / 4 KV heads, head_dim 128, bf16; 16 beacon + 32 recent queries per round with "
                               "their LSE computed in the round; LRFU carried across rounds; budget 30,000",
                   "rounds": args.rounds, "entries_total": entries, "total_ms": total_ms,
                   "l2": "flushed (256 MB write) before every round"},
        "roofline": {"kernel": "score_tc_kernel + LSE pass (kvc_score_from_lse with KVC_SCORE_COMPUTE_LSE)",
                     "bound": "tensor", "achieved": achieved, "peak": tf_burst, "unit": "TFLOP/s",
                     "frac": achieved / tf_burst, "traffic": None,
                     "peak_source": f"{peak_kind} bf16 dense (burst)",
                     "note": "FLOP counts the scoring contraction only; the LSE pass over the same pairs is extra work"},
        "step_roofline": {"t_roof_us_total": t_roof * 1e6, "t_us_total": total_ms * 1e3, "frac": t_roof / (total_ms / 1e3)},
        "breakdown_ms": {"score incl. LSE pass": float(np.mean(score_ms)),
                         "after score": float(np.mean(step_ms) - np.mean(score_ms))},
        "gpu_launches": 6 * args.rounds,
        "launch": "direct C-ABI calls" if args.no_graph else "CUDA graph of the round, replayed every round",
        "e2e": None, "e2e_note": "not measured for this line", "cpu_baseline": cpu, "clocks": clk,
    }


def run_kvstreams(args, device):
    """KV-streams ("KV-streams for Efficient Compaction in Agentic Reinforcement Learning", abstract): the
    streaming workload's compacted cache carried across rollouts instead of flushed and prefilled again.  Each
    round (timed): score with the beacon LSE pass -> LRFU + select -> plan -> compact -> the round's 64 decoded
    tokens per row appended into freed pages (kvc_append_tokens, pages from a stack fed by the freed lists).  At
    every rollout boundary the carried cache simply continues; a flush-and-re-prefill baseline would instead
    rebuild every row from its whole context, so the line reports the prefill tokens that avoids and the
    measured time this library needs to write those rows' K/V back into the pool through the same append path
    (the memory-traffic part of a re-prefill; the model forward it would also need is outside this library)."""
    from agent_kv_cache_lse_b200 import kvc, synth
    from agent_kv_cache_lse_b200.round import EvictionRound
    spec = config_spec("streaming")
    rollouts, per = args.rollouts, args.rounds // max(1, args.rollouts)
    layout = synth.make_layout(spec)
    kp = synth.fill_pool(spec, layout, "k", device)
    vp = synth.fill_pool(spec, layout, "v", device)
    cache = kvc.Cache(kp, vp, layout.block_table.to(device), layout.row_len.to(device), layout.slot_pos.to(device),
                      layout.slot_label.to(device), spec.num_seqs, spec.num_layers, spec.num_kv_heads)
    rnd = EvictionRound(cache)
    rnd.budget.fill_(spec.budget)
    P, D, count = spec.page_size, spec.head_dim, 64
    bt0 = layout.block_table.numpy()
    used = set(int(x) for x in bt0[bt0 >= 0])
    free0 = [p for p in range(layout.num_pages) if p not in used]
    stack = torch.full((layout.num_pages,), -1, dtype=torch.int32, device=device)
    stack[:len(free0)] = torch.tensor(free0, dtype=torch.int32, device=device)
    depth = torch.tensor([len(free0)], dtype=torch.int64, device=device)
    ws = torch.zeros(kvc.kvc_append_workspace_bytes(spec.rows) // 8, dtype=torch.int64, device=device)
    k_new = torch.empty((spec.rows, count, D), dtype=kp.dtype, device=device)
    v_new = torch.empty_like(k_new)
    new_pos = torch.empty((spec.num_seqs, count), dtype=torch.int32, device=device)
    n_total = list(spec.ctx)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)

    def draw(n_tot):
        for s_ in range(spec.num_seqs):
            new_pos[s_] = torch.arange(n_tot[s_], n_tot[s_] + count, dtype=torch.int32, device=device)
        for r in range(spec.rows):
            s_, l, h = spec.row_coords(r)
            pos = torch.arange(n_tot[s_], n_tot[s_] + count, dtype=torch.int64, device=device)
            k_new[r] = synth.key_values(spec, s_, l, h, pos, "k")
            v_new[r] = synth.key_values(spec, s_, l, h, pos, "v")

    round_ms, entries_total, avoided = [], 0, 0
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    for ro in range(rollouts):
        for rd in range(per):
            qs = synth.streaming_queries(spec, n_total, device=device)
            q = kvc.QuerySet(qs.q, torch.empty((spec.num_seqs, 1, spec.num_q_heads, qs.max_q), device=device),
                             qs.q_pos, qs.num_q)
            draw(n_total)
            entries_total += int(cache.row_len.sum())
            flush.fill_(1.0)
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            main = torch.cuda.current_stream()
            e[0].record(main)
            kvc.kvc_score_from_lse(cache, q, rnd.scores, kvc.KVC_SCORE_COMPUTE_LSE, rnd.status, main)
            rnd.run_after_scores(None, 0.5, 0.9, main)
            e[1].record(main)
            nf = int(rnd.num_freed[0])          # the freed pages go on the stack (host bookkeeping, untimed)
            d = int(depth[0])
            stack[d:d + nf] = rnd.freed[:nf]
            depth += nf
            e[2].record(main)
            kvc.kvc_append_tokens(cache, k_new, v_new, new_pos, synth.LABEL_REASON, rnd.crf, stack, depth, ws,
                                  rnd.status, main)
            e[3].record(main)
            torch.cuda.synchronize()
            round_ms.append(e[0].elapsed_time(e[1]) + e[2].elapsed_time(e[3]))
            for s_ in range(spec.num_seqs):
                n_total[s_] += count
        # rollout boundary: a flush would re-prefill every sequence's whole context in every layer and KV head
        avoided += sum(n_total[spec.row_coords(r)[0]] for r in range(spec.rows))
    clk = clocks.stop()
    assert rnd.device_status()[0] == 0, rnd.device_status()
    # the re-prefill's cache writes: every row rebuilt from empty through the append path, timed for as many
    # tokens per row as the pool holds and scaled to the whole context (the writes are linear in the tokens)
    ctx = max(n_total)
    rebuild_tokens = min(ctx, spec.max_slots, (layout.num_pages // spec.rows) * P)
    kbig = torch.empty((spec.rows, rebuild_tokens, D), dtype=kp.dtype, device=device)
    kbig.normal_()
    posbig = torch.arange(rebuild_tokens, dtype=torch.int32, device=device).repeat(spec.num_seqs, 1).contiguous()
    times = []
    for _ in range(3):
        cache.row_len.zero_()
        cache.block_table.fill_(-1)
        stack[:layout.num_pages] = torch.arange(layout.num_pages, dtype=torch.int32, device=device)
        depth.fill_(layout.num_pages)
        flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        kvc.kvc_append_tokens(cache, kbig, kbig, posbig, synth.LABEL_REASON, None, stack, depth, ws, rnd.status)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    assert rnd.device_status()[0] == 0, rnd.device_status()
    rebuild_ms = float(np.median(times)) * ctx / rebuild_tokens
    total_ms = float(sum(round_ms))
    return {
        "metric": "KV entries scored+compacted/sec with the cache carried across rollouts (KV-streams)",
        "value": entries_total / (total_ms / 1e3), "unit": UNIT, "n_gpus": 1, "steps": len(round_ms),
        "warmup": 0, "ms_per_step": total_ms / len(round_ms),
        "ms_per_step_p10_p50_p90": [float(np.percentile(round_ms, q)) for q in (10, 50, 90)],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded counter-based generator)",
        "config": {"workload": f"streaming shape (8 sequences, 32K context, 28 q / 4 KV heads, budget 30,000), "
                               f"{rollouts} rollouts x {per} rounds, 64 decoded tokens per row appended each round",
                   "l2": "flushed (256 MB write) before every round"},
        "kv_streams": {"prefill_entries_avoided": avoided, "rollout_boundaries": rollouts,
                       "context_tokens_at_end": ctx,
                       "rebuild_ms_per_boundary": rebuild_ms,
                       "rebuild_note": "time to write every row's whole context back into the pool through "
                                       "kvc_append_tokens (the cache-write part of a re-prefill, no model forward), "
                                       "timed on as many tokens per row as the pool holds and scaled to the context",
                       "carried_state_check": "tests/test_gpu_configs.py::test_streaming_rounds_full (200 rounds in "
                                              "lockstep with the oracle, appends through the same kernel)"},
        "gpu_launches": 9 * len(round_ms), "launch": "direct C-ABI calls", "e2e": None,
        "e2e_note": "not measured for this line", "cpu_baseline": None, "clocks": clk,
    }


def streaming_work(spec, cache, qs):
    """QK^T FLOP over the visible pairs of one streaming round (beacons see every key; recent queries are causal)."""
    qpos = qs.q_pos.cpu().numpy()
    sp = cache.slot_pos.cpu().numpy()
    rl = cache.row_len.cpu().numpy()
    G, D = spec.group, spec.head_dim
    vis = 0
    for r in range(spec.rows):
        s, _, _ = spec.row_coords(r)
        qp = np.sort(qpos[s].astype(np.int64))
        vis += int((G * (len(qp) - np.searchsorted(qp, sp[r, :rl[r]], side="left"))).sum())
    return 2 * D * vis


def run_beacon(args, device):
    """Beacon-query maintenance on the streaming shape (8 sequences, 1 layer, 28 query heads, head_dim 128,
    16 beacons per group, 64 new queries per group per round): rounds per second of kvc_beacon_update, with
    the L2 cache flushed before every timed call; a separate line, not the eviction round."""
    from agent_kv_cache_lse_b200 import kvc
    S, L, Hq, D, B, m = 8, 1, 28, 128, 16, 64
    gen = torch.Generator(device=device).manual_seed(4)
    q = torch.randn((S, L, m, Hq, D), generator=gen, device=device).to(torch.bfloat16)
    num_q = torch.full((S,), m, dtype=torch.int32, device=device)
    beacons = torch.zeros((S, L, Hq, B, D), device=device)
    counts = torch.zeros((S, L, Hq, B), dtype=torch.int32, device=device)
    out = torch.zeros((S, L, B + 32, Hq, D), dtype=torch.bfloat16, device=device)
    st = torch.zeros(2, dtype=torch.int32, device=device)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    for _ in range(max(3, args.warmup)):
        kvc.kvc_beacon_update(q, num_q, beacons, counts, out, st)
    torch.cuda.synchronize()
    ts = []
    for _ in range(args.steps):
        flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        kvc.kvc_beacon_update(q, num_q, beacons, counts, out, st)
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    assert int(st[0]) == 0
    ms = float(np.median(ts))
    groups = S * L * Hq
    algo = (S * L * m * Hq * D * 2) + groups * B * D * 4 * 2 + groups * B * 4 * 2 + S * L * B * Hq * D * 2
    hbm, _, _, kind = peaks()
    achieved = algo / (ms / 1e3) / 1e9
    return {"metric": "beacon queries folded per second (streaming shape)", "value": groups * m / (ms / 1e3),
            "unit": "queries/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "dtype": "bf16 queries, fp32 beacons", "data": "synthetic",
            "config": {"workload": "beacon maintenance: 8 seqs x 1 layer x 28 q heads, head_dim 128, 16 beacons, "
                                   "64 new queries per group", "l2": "flushed (256 MB write) before every call"},
            "roofline": {"kernel": "beacon_kernel (kvc_beacon_update)", "bound": "hbm", "achieved": achieved,
                         "peak": hbm, "unit": "GB/s", "frac": achieved / hbm, "traffic": None,
                         "peak_source": f"{kind} HBM copy", "bytes_per_launch": algo},
            "gpu_launches": args.steps}


def decode_workload(spec, device):
    """Cache of a decode workload and the step's query (the first query of each sequence's set) at the next
    position, so that every cached key is visible."""
    from agent_kv_cache_lse_b200 import kvc, synth
    layout = synth.make_layout(spec)
    kp = synth.fill_pool(spec, layout, "k", device)
    vp = synth.fill_pool(spec, layout, "v", device)
    qs = synth.make_queries(spec, device)
    cache = kvc.Cache(kp, vp, layout.block_table.to(device), layout.row_len.to(device), layout.slot_pos.to(device),
                      layout.slot_label.to(device), spec.num_seqs, spec.num_layers, spec.num_kv_heads)
    q = qs.q[:, :, 0].contiguous()
    q_pos = torch.tensor(list(spec.ctx), dtype=torch.int32, device=device)
    return cache, q, q_pos, int(layout.row_len.sum())


def time_decode(args, spec, device, flush):
    from agent_kv_cache_lse_b200 import kvc
    cache, q, q_pos, entries = decode_workload(spec, device)
    S, L, Hq, D = q.shape
    out = torch.empty((S, L, Hq, D), device=device)
    lse = torch.empty((S, L, Hq), device=device)
    scores = torch.zeros((spec.rows, spec.max_slots), device=device)
    st = torch.zeros(2, dtype=torch.int32, device=device)
    for _ in range(max(3, args.warmup)):
        kvc.kvc_decode_attention(cache, q, q_pos, out, lse, scores, kvc.KVC_SCORE_ACCUMULATE, st)
    torch.cuda.synchronize()
    ts = []
    for _ in range(args.steps):
        flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        kvc.kvc_decode_attention(cache, q, q_pos, out, lse, scores, kvc.KVC_SCORE_ACCUMULATE, st)
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    assert int(st[0]) == 0, kvc.device_status(st)
    elem = 2 if spec.dtype == "bf16" else 4
    # per visible entry: K and V rows, its slot position, and the score's read-modify-write; per query head:
    # the query, the output row and the LSE; per row: its length and block-table row
    algo = (entries * (2 * D * elem + 4 + 8) + S * L * Hq * (D * elem + D * 4 + 4)
            + spec.rows * (4 + spec.max_pages_per_row * 4))
    ms = float(np.median(ts))
    del cache
    return ms, entries, algo, ts


def run_decode(args, device):
    """One decode step of paged attention with the scores folded in (kvc_decode_attention, accumulating into the
    round's scores): KV entries attended and scored per second for one layer of the batch of 16 sequences
    (context 8K-33K, 32 q / 8 KV heads, head_dim 128, bf16), L2 flushed before every call; the single Llama-3-8B
    layer at 32K is timed beside it.  A separate line, not the eviction round."""
    from agent_kv_cache_lse_b200 import synth
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    hbm, _, _, kind = peaks()
    ms, entries, algo, ts = time_decode(args, synth.batch16(num_layers=1), device, flush)
    ms1, entries1, algo1, _ = time_decode(args, synth.llama8b_layer(), device, flush)
    # the same layer of the batch of 16 with 64 query heads (G = 8, the shape of the larger Llama-3 models)
    g8 = dataclasses.replace(synth.batch16(num_layers=1), name="batch16_L1_g8", num_q_heads=64)
    ms8, entries8, algo8, _ = time_decode(args, g8, device, flush)
    achieved = algo / (ms / 1e3) / 1e9
    p10, p50, p90 = (float(x) for x in np.percentile(ts, [10, 50, 90]))
    return {"metric": "KV entries attended+scored/sec (fused decode step)", "value": entries / (ms / 1e3),
            "unit": "entries/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "ms_per_step_p10_p50_p90": [p10, p50, p90], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 K/V/Q, fp32 accumulate", "data": "synthetic",
            "config": {"workload": "decode step, one layer of the batch of 16 sequences (context 8K-33K, "
                                   f"{entries} cached entries), 32 q / 8 KV heads, head_dim 128, bf16, 16-token pages",
                       "l2": "flushed (256 MB write) before every call"},
            "group8": {"shape": "the same layer with 64 q / 8 KV heads (G = 8)", "entries": entries8, "ms": ms8,
                       "entries_per_s": entries8 / (ms8 / 1e3), "achieved_gbs": algo8 / (ms8 / 1e3) / 1e9,
                       "frac": algo8 / (ms8 / 1e3) / 1e9 / hbm},
            "single_layer_32k": {"entries": entries1, "ms": ms1, "entries_per_s": entries1 / (ms1 / 1e3),
                                 "achieved_gbs": algo1 / (ms1 / 1e3) / 1e9},
            "roofline": {"kernel": "decode_kernel (kvc_decode_attention)", "bound": "hbm", "achieved": achieved,
                         "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                         "traffic": profiled_traffic(DECODE_PROFILE),
                         "peak_source": f"{kind} HBM copy", "bytes_per_launch": algo},
            "gpu_launches": args.steps}


def run_stepkv(args, device):
    """Step-aware ranking scores (kvc_step_scores, beta 0.5) on the batch of 16 sequences x 8 layers x 8 KV heads
    (context 8K-33K, step starts where reasoning segments begin): entries ranked per second, L2 flushed before
    every call.  A separate line, not the eviction round."""
    from agent_kv_cache_lse_b200 import kvc, synth
    spec = synth.batch16(num_layers=8)
    lay = synth.make_layout(spec)
    starts = [synth.step_starts(spec, s) for s in range(spec.num_seqs)]
    ms = max(len(x) for x in starts)
    st = torch.full((spec.num_seqs, ms), 2**31 - 1, dtype=torch.int32)
    for i, x in enumerate(starts):
        st[i, :len(x)] = x
    ns = torch.tensor([len(x) for x in starts], dtype=torch.int32, device=device)
    st = st.to(device)
    dummy = torch.zeros((1, 16, spec.head_dim), dtype=torch.bfloat16, device=device)
    cache = kvc.Cache(dummy, dummy, lay.block_table.to(device), lay.row_len.to(device), lay.slot_pos.to(device),
                      lay.slot_label.to(device), spec.num_seqs, spec.num_layers, spec.num_kv_heads)
    gen = torch.Generator(device=device).manual_seed(5)
    scores = torch.rand((spec.rows, spec.max_slots), generator=gen, device=device)
    out = torch.empty_like(scores)
    stt = torch.zeros(2, dtype=torch.int32, device=device)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    for _ in range(max(3, args.warmup)):
        kvc.kvc_step_scores(cache, scores, st, ns, out, 0.5, stt)
    torch.cuda.synchronize()
    ts = []
    for _ in range(args.steps):
        flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        kvc.kvc_step_scores(cache, scores, st, ns, out, 0.5, stt)
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    assert int(stt[0]) == 0, kvc.device_status(stt)
    entries = int(lay.row_len.sum())
    algo = entries * 12 + spec.rows * 4 + spec.num_seqs * (ms + 1) * 4   # scores r, positions r, blend w
    ms_ = float(np.median(ts))
    hbm, _, _, kind = peaks()
    achieved = algo / (ms_ / 1e3) / 1e9
    return {"metric": "KV entries ranked/sec (step-aware scores)", "value": entries / (ms_ / 1e3), "unit": "entries/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"step-aware scores, batch of 16 sequences x 8 layers x 8 KV heads, context 8K-33K "
                                   f"({entries} entries), {ms} steps at most per sequence, beta 0.5",
                       "l2": "flushed (256 MB write) before every call"},
            "roofline": {"kernel": "step_scores_reg_kernel (kvc_step_scores)", "bound": "hbm", "achieved": achieved,
                         "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                         "traffic": profiled_traffic(STEPKV_PROFILE),
                         "peak_source": f"{kind} HBM copy", "bytes_per_launch": algo},
            "gpu_launches": args.steps}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-baseline leg")
    ap.add_argument("--no-graph", action="store_true", help="launch the round's five calls directly instead of a CUDA graph")
    ap.add_argument("--beacon", action="store_true", help="time beacon-query maintenance instead of the round")
    ap.add_argument("--decode", action="store_true", help="time the fused decode step instead of the round")
    ap.add_argument("--stepkv", action="store_true", help="time the step-aware ranking scores instead of the round")
    ap.add_argument("--config", default="llama8b", choices=["llama8b", "batch16", "stress", "streaming"],
                    help="workload of the round (llama8b is the headline line)")
    ap.add_argument("--rounds", type=int, default=200, help="rounds of the streaming workload")
    ap.add_argument("--seqs", type=int, default=None, help="batch16 / stress: fewer sequences (a smaller case)")
    ap.add_argument("--layers", type=int, default=None, help="batch16 / stress: fewer layers (a smaller case)")
    ap.add_argument("--kvstreams", action="store_true", help="the streaming workload carried across rollouts")
    ap.add_argument("--rollouts", type=int, default=5, help="rollouts of the --kvstreams line")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", rank)))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", torch.cuda.current_device())
    from agent_kv_cache_lse_b200 import kvc
    kvc.lib()   # raises if the CUDA library is missing
    if args.beacon:
        line = run_beacon(args, device)
    elif args.decode:
        line = run_decode(args, device)
    elif args.stepkv:
        line = run_stepkv(args, device)
    elif args.kvstreams:
        line = run_kvstreams(args, device)
    elif args.config in ("batch16", "stress"):
        line = run_config(args, device)
    elif args.config == "streaming":
        line = run_streaming(args, device)
    else:
        line = run_ours(args, rank, world, device)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
