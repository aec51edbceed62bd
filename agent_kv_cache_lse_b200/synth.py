"""Seeded synthetic inputs for the eviction/compaction path.

Every value drawn here is a pure function of ``(seed, stream, counter)``: the
same element comes out bit for bit on the CPU or on a CUDA device, in any
chunking.  That lets the CPU oracle regenerate any sampled row of a workload
that lives on the GPU without reading it back from the device.

* Hash: the 32-bit finaliser of MurmurHash3 (Austin Appleby, public domain),
  applied twice to fold a 64-bit counter into a stream key.  All products are
  formed from 16-bit halves so no int64 product ever overflows.
* Normals: Irwin-Hall sum of four 16-bit uniforms, centred and scaled once in
  fp32 (the integer sum is exact in fp32, the single multiply is correctly
  rounded on every IEEE device), then rounded to bf16 by round-to-nearest-even
  when the workload is bf16.

The workloads follow the agent-trace shapes of the ActKV write-up ("ActKV
Dissected", Summary and introduction: ~31-33K-token ReAct trajectories whose
observation and reasoning segments hold >99% of entries and actions <1%) and
the five configurations the path is measured on.  This module holds none of
the method's arithmetic: it only draws inputs and lays them out in a paged pool.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

M32 = 0xFFFFFFFF

# stream ids: one per kind of drawn quantity
S_K, S_V, S_Q, S_SEG, S_HEAVY, S_PAGES, S_LOGITS, S_BEACON, S_RECENT, S_CTX, S_BUDGET, S_TIE = range(1, 13)

# counter field widths: seq | layer | head | pos-or-index | dim
_W_LAYER, _W_HEAD, _W_POS, _W_DIM = 8, 8, 20, 8


def _mul32(h: torch.Tensor, c: int) -> torch.Tensor:
    """(h * c) mod 2**32 for h in [0, 2**32) without int64 overflow."""
    c_lo, c_hi = c & 0xFFFF, c >> 16
    h_lo, h_hi = h & 0xFFFF, h >> 16
    mid = (h_lo * c_hi + h_hi * c_lo) & 0xFFFF
    return (h_lo * c_lo + (mid << 16)) & M32


def _fmix32(h: torch.Tensor) -> torch.Tensor:
    h = h ^ (h >> 16)
    h = _mul32(h, 0x85EBCA6B)
    h = h ^ (h >> 13)
    h = _mul32(h, 0xC2B2AE35)
    h = h ^ (h >> 16)
    return h


def _fmix32_int(h: int) -> int:
    h &= M32
    h ^= h >> 16
    h = (h * 0x85EBCA6B) & M32
    h ^= h >> 13
    h = (h * 0xC2B2AE35) & M32
    h ^= h >> 16
    return h


def stream_key(seed: int, stream: int) -> int:
    return _fmix32_int((seed * 0x9E3779B1 + stream * 0x85EBCA77 + 0x165667B1) & M32)


def hash_u32(seed: int, stream: int, idx: torch.Tensor) -> torch.Tensor:
    """32-bit hash of a non-negative int64 counter tensor (values in [0, 2**32))."""
    idx = idx.to(torch.int64)
    key = stream_key(seed, stream)
    hi = _fmix32((idx >> 32) ^ key)
    return _fmix32((idx & M32) ^ hi)


def uniform_int(seed: int, stream: int, idx: torch.Tensor, lo: int, hi: int) -> torch.Tensor:
    """Integers in [lo, hi] (inclusive)."""
    return lo + hash_u32(seed, stream, idx) % (hi - lo + 1)


def bernoulli(seed: int, stream: int, idx: torch.Tensor, p: float) -> torch.Tensor:
    return hash_u32(seed, stream, idx) < int(round(p * 2.0**32))


_IH_SCALE = torch.tensor(math.sqrt(3.0) / 65536.0, dtype=torch.float32).item()


def normal(seed: int, stream: int, idx: torch.Tensor, sigma: float = 1.0) -> torch.Tensor:
    """Approximately N(0, sigma^2) fp32 values (Irwin-Hall of four 16-bit uniforms)."""
    idx = idx.to(torch.int64)
    a = hash_u32(seed, stream, 2 * idx)
    b = hash_u32(seed, stream, 2 * idx + 1)
    s = (a & 0xFFFF) + (a >> 16) + (b & 0xFFFF) + (b >> 16) - 2 * 65535
    x = s.to(torch.float32) * torch.tensor(_IH_SCALE, dtype=torch.float32, device=idx.device)
    if sigma != 1.0:
        x = x * torch.tensor(sigma, dtype=torch.float32, device=idx.device)
    return x


def counter(seq, layer, head, pos, dim):
    """Composite counter; each argument is an int or a broadcastable int64 tensor."""
    c = seq
    c = c * (1 << _W_LAYER) + layer
    c = c * (1 << _W_HEAD) + head
    c = c * (1 << _W_POS) + pos
    c = c * (1 << _W_DIM) + dim
    return c


# ----------------------------------------------------------------------------
# workload specifications
# ----------------------------------------------------------------------------

LABEL_OBS, LABEL_REASON, LABEL_ACTION = 0, 1, 2


@dataclasses.dataclass
class Spec:
    """One synthetic workload of the path (sizes, shapes and draws)."""

    name: str
    seed: int
    num_seqs: int
    num_layers: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str                      # "f32" or "bf16"
    ctx: Sequence[int]              # context length of each sequence
    budget: int
    page_size: int = 16
    heavy_frac: float = 0.0         # share of keys whose vector is scaled by heavy_scale
    heavy_scale: float = 4.0
    spare_frac: float = 0.0         # extra free pages in the pool
    shuffle_pages: bool = True      # fragmented pool (pages in random physical order)
    queries: str = "action"         # "action" | "fixed" | "beacon_recent"
    fixed_q_pos: Sequence[int] = ()
    seg_ranges: Sequence[Sequence[int]] = ((200, 1500), (100, 800), (8, 40))
    num_beacons: int = 16
    num_recent: int = 32
    extra_slots: int = 0            # headroom pages per row (for appends between rounds)
    logits_steps: int = 64
    vocab: int = 128256
    logits_sigma: float = 2.0

    @property
    def rows(self) -> int:
        return self.num_seqs * self.num_layers * self.num_kv_heads

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def row_id(self, s: int, l: int, h: int) -> int:
        return (s * self.num_layers + l) * self.num_kv_heads + h

    def row_coords(self, r: int):
        h = r % self.num_kv_heads
        sl = r // self.num_kv_heads
        return sl // self.num_layers, sl % self.num_layers, h

    @property
    def max_pages_per_row(self) -> int:
        return -(-max(self.ctx) // self.page_size) + self.extra_slots // self.page_size

    @property
    def max_slots(self) -> int:
        return self.max_pages_per_row * self.page_size


def tiny(seed: int = 1, variant: int = 0) -> Spec:
    """1 seq, 1 layer, 4 q / 2 KV heads, D 64, fp32, 1,024 tokens, 8 action queries."""
    qpos = list(range(1016, 1024)) if variant == 0 else list(range(504, 512))
    return Spec(name="tiny" if variant == 0 else "tiny_mid", seed=seed, num_seqs=1, num_layers=1,
                num_q_heads=4, num_kv_heads=2, head_dim=64, dtype="f32", ctx=[1024], budget=256,
                queries="fixed", fixed_q_pos=qpos)


def llama8b_layer(seed: int = 2, ctx: int = 32768) -> Spec:
    """One Llama-3-8B-shaped layer at 32K context (32 q / 8 KV heads, D 128, bf16)."""
    return Spec(name=f"llama8b_layer_{ctx}", seed=seed, num_seqs=1, num_layers=1, num_q_heads=32,
                num_kv_heads=8, head_dim=128, dtype="bf16", ctx=[ctx], budget=512, heavy_frac=0.02)


def batch16(seed: int = 3, num_seqs: int = 16, num_layers: int = 32, lo: int = 8192, hi: int = 33792) -> Spec:
    ctx = uniform_int(seed, S_CTX, torch.arange(num_seqs), lo, hi).tolist()
    return Spec(name=f"batch{num_seqs}_L{num_layers}", seed=seed, num_seqs=num_seqs, num_layers=num_layers,
                num_q_heads=32, num_kv_heads=8, head_dim=128, dtype="bf16", ctx=ctx, budget=512,
                spare_frac=0.05)


def streaming(seed: int = 4, num_seqs: int = 8, ctx: int = 32768) -> Spec:
    return Spec(name=f"streaming_b{num_seqs}", seed=seed, num_seqs=num_seqs, num_layers=1, num_q_heads=28,
                num_kv_heads=4, head_dim=128, dtype="bf16", ctx=[ctx] * num_seqs, budget=30000,
                queries="beacon_recent", extra_slots=64 * 4)


def stress(seed: int = 5, num_seqs: int = 64, num_layers: int = 16, ctx: int = 33000) -> Spec:
    return Spec(name=f"stress_b{num_seqs}_L{num_layers}", seed=seed, num_seqs=num_seqs, num_layers=num_layers,
                num_q_heads=32, num_kv_heads=8, head_dim=128, dtype="bf16", ctx=[ctx] * num_seqs, budget=0)


def stress_budget(n: int, page: int = 16, frac: float = 0.4) -> int:
    """Budget whose compaction frees round(frac * pages) of a row's pages."""
    pages = -(-n // page)
    keep_pages = pages - int(round(frac * pages))
    return keep_pages * page


# ----------------------------------------------------------------------------
# segments and query sets
# ----------------------------------------------------------------------------

def segment_labels(spec: Spec, s: int, n: int) -> torch.Tensor:
    """Per-token labels of sequence s: observation, reasoning, action segments repeating, observation first."""
    labels = torch.empty(n, dtype=torch.uint8)
    pos, k = 0, 0
    while pos < n:
        kind = k % 3
        lo, hi = spec.seg_ranges[kind]
        ln = int(uniform_int(spec.seed, S_SEG, torch.tensor([s * 100000 + k]), lo, hi)[0])
        labels[pos:pos + ln] = kind
        pos += ln
        k += 1
    return labels


def query_positions(spec: Spec, s: int) -> torch.Tensor:
    """Token positions of the query set of sequence s (ascending); beacons carry INT32_MAX."""
    if spec.queries == "fixed":
        return torch.tensor(list(spec.fixed_q_pos), dtype=torch.int32)
    if spec.queries == "action":
        lab = segment_labels(spec, s, spec.ctx[s])
        return torch.nonzero(lab == LABEL_ACTION).flatten().to(torch.int32)
    if spec.queries == "beacon_recent":
        n = spec.ctx[s]
        beacons = torch.full((spec.num_beacons,), 2**31 - 1, dtype=torch.int32)
        recent = torch.arange(n - spec.num_recent, n, dtype=torch.int32)
        return torch.cat([beacons, recent])
    raise ValueError(spec.queries)


def step_starts(spec: Spec, s: int) -> torch.Tensor:
    """Start positions of the reasoning steps of sequence s: 0, then every position where a reasoning
    segment begins (input construction for step-aware ranking; a ReAct step = thought, action, observation)."""
    lab = segment_labels(spec, s, spec.ctx[s])
    begin = torch.nonzero((lab[1:] == LABEL_REASON) & (lab[:-1] != LABEL_REASON)).flatten() + 1
    return torch.cat([torch.zeros(1, dtype=torch.int64), begin]).to(torch.int32)


# ----------------------------------------------------------------------------
# paged layout and pools
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Layout:
    num_pages: int
    block_table: torch.Tensor   # [rows, max_pages] int32, -1 = none
    row_len: torch.Tensor       # [rows] int32
    slot_pos: torch.Tensor      # [rows, max_slots] int32
    slot_label: torch.Tensor    # [rows, max_slots] uint8


def make_layout(spec: Spec) -> Layout:
    """Block table (fragmented pool), row lengths, slot positions and labels (CPU tensors)."""
    P = spec.page_size
    rows, mp = spec.rows, spec.max_pages_per_row
    row_len = torch.empty(rows, dtype=torch.int32)
    pages_needed = torch.empty(rows, dtype=torch.int64)
    for r in range(rows):
        s, _, _ = spec.row_coords(r)
        row_len[r] = spec.ctx[s]
        pages_needed[r] = -(-spec.ctx[s] // P)
    used = int(pages_needed.sum())
    num_pages = used + int(math.ceil(spec.spare_frac * used))
    if spec.shuffle_pages:
        keys = hash_u32(spec.seed, S_PAGES, torch.arange(num_pages)) * (1 << 32) + torch.arange(num_pages)
        perm = torch.argsort(keys).to(torch.int32)
    else:
        perm = torch.arange(num_pages, dtype=torch.int32)
    bt = torch.full((rows, mp), -1, dtype=torch.int32)
    lp = torch.arange(mp, dtype=torch.int64)
    starts = torch.cumsum(pages_needed, 0) - pages_needed
    for r in range(rows):
        k = int(pages_needed[r])
        bt[r, :k] = perm[int(starts[r]):int(starts[r]) + k]
    slot_pos = torch.arange(spec.max_slots, dtype=torch.int32).repeat(rows, 1)
    slot_label = torch.zeros((rows, spec.max_slots), dtype=torch.uint8)
    for s in range(spec.num_seqs):
        lab = segment_labels(spec, s, spec.ctx[s]) if spec.queries == "action" else \
            torch.full((spec.ctx[s],), LABEL_REASON, dtype=torch.uint8)
        for l in range(spec.num_layers):
            for h in range(spec.num_kv_heads):
                slot_label[spec.row_id(s, l, h), :spec.ctx[s]] = lab
    return Layout(num_pages=num_pages, block_table=bt, row_len=row_len, slot_pos=slot_pos, slot_label=slot_label)


def torch_dtype(spec: Spec):
    return torch.float32 if spec.dtype == "f32" else torch.bfloat16


def key_values(spec: Spec, s: int, l: int, h: int, pos: torch.Tensor, which: str = "k") -> torch.Tensor:
    """K (or V) vectors of (seq s, layer l, KV head h) at token positions pos: [len(pos), D] in the spec dtype."""
    dev = pos.device
    d = torch.arange(spec.head_dim, device=dev, dtype=torch.int64)
    c = counter(s, l, h, pos.to(torch.int64)[:, None], d[None, :])
    x = normal(spec.seed, S_K if which == "k" else S_V, c)
    if which == "k" and spec.heavy_frac > 0:
        hv = bernoulli(spec.seed, S_HEAVY, counter(s, l, h, pos.to(torch.int64), 0), spec.heavy_frac)
        x = torch.where(hv[:, None], x * torch.tensor(spec.heavy_scale, dtype=torch.float32, device=dev), x)
    return x.to(torch_dtype(spec))


def fill_pool(spec: Spec, layout: Layout, which: str = "k", device="cpu", chunk_tokens: int = 1 << 20) -> torch.Tensor:
    """Paged pool [num_pages, page_size, D] holding K (or V) of every row at its block-table pages."""
    P, D = spec.page_size, spec.head_dim
    pool = torch.zeros((layout.num_pages, P, D), dtype=torch_dtype(spec), device=device)
    flat = pool.view(-1, D)
    bt = layout.block_table.to(device)
    for r in range(spec.rows):
        s, l, h = spec.row_coords(r)
        n = int(layout.row_len[r])
        for a in range(0, n, chunk_tokens):
            b = min(n, a + chunk_tokens)
            slots = torch.arange(a, b, device=device, dtype=torch.int64)
            pos = layout.slot_pos[r, a:b].to(device=device, dtype=torch.int64)
            phys = bt[r, slots // P].to(torch.int64) * P + slots % P
            flat[phys] = key_values(spec, s, l, h, pos, which)
    return pool


@dataclasses.dataclass
class Queries:
    q: torch.Tensor        # [S, L, max_q, Hq, D]
    q_pos: torch.Tensor    # [S, max_q] int32 (INT32_MAX = beacon, no causal mask)
    num_q: torch.Tensor    # [S] int32
    max_q: int


def make_queries(spec: Spec, device="cpu") -> Queries:
    """Query vectors and positions; action/fixed queries use the query index as counter field."""
    pos_list = [query_positions(spec, s) for s in range(spec.num_seqs)]
    max_q = max(1, max(len(p) for p in pos_list))
    S, L, Hq, D = spec.num_seqs, spec.num_layers, spec.num_q_heads, spec.head_dim
    q = torch.zeros((S, L, max_q, Hq, D), dtype=torch_dtype(spec), device=device)
    q_pos = torch.full((S, max_q), -1, dtype=torch.int32)
    num_q = torch.zeros(S, dtype=torch.int32)
    for s in range(S):
        nq = len(pos_list[s])
        q_pos[s, :nq] = pos_list[s]
        num_q[s] = nq
        for l in range(L):
            q[s, l, :nq] = query_vectors(spec, s, l, nq, device)
    return Queries(q=q, q_pos=q_pos.to(device), num_q=num_q.to(device), max_q=max_q)


def query_vectors(spec: Spec, s: int, l: int, nq: int, device="cpu") -> torch.Tensor:
    """Query vectors [nq, Hq, D] of sequence s, layer l (action/fixed query sets: the query index is the
    counter field), in the spec dtype; what make_queries places at q[s, l, :nq]."""
    j = torch.arange(nq, device=device, dtype=torch.int64)
    hh = torch.arange(spec.num_q_heads, device=device, dtype=torch.int64)
    d = torch.arange(spec.head_dim, device=device, dtype=torch.int64)
    c = counter(s, l, hh[None, :, None], j[:, None, None], d[None, None, :])
    return normal(spec.seed, S_Q, c).to(torch_dtype(spec))


def logits(spec: Spec, s: int, step0: int, steps: int, device="cpu") -> torch.Tensor:
    """Decode-step logits of sequence s for global steps [step0, step0+steps): [steps, vocab] fp32."""
    t = torch.arange(step0, step0 + steps, device=device, dtype=torch.int64)
    v = torch.arange(spec.vocab, device=device, dtype=torch.int64)
    c = (s * (1 << 24) + t[:, None]) * (1 << 20) + v[None, :]
    return normal(spec.seed, S_LOGITS, c, sigma=spec.logits_sigma)


def streaming_queries(spec: Spec, n_total: Sequence[int], device="cpu") -> Queries:
    """Beacon plus recent query set at the current decode position of each sequence.

    Beacons (INT32_MAX position, unmasked) are fixed per (seq, layer, q head, index);
    the recent queries are the last `num_recent` decoded tokens, drawn by position.
    """
    S, L, Hq, D = spec.num_seqs, spec.num_layers, spec.num_q_heads, spec.head_dim
    nb, nr = spec.num_beacons, spec.num_recent
    max_q = nb + nr
    q = torch.zeros((S, L, max_q, Hq, D), dtype=torch_dtype(spec), device=device)
    q_pos = torch.full((S, max_q), 2**31 - 1, dtype=torch.int32)
    hh = torch.arange(Hq, device=device, dtype=torch.int64)
    d = torch.arange(D, device=device, dtype=torch.int64)
    for s in range(S):
        n = int(n_total[s])
        rec = torch.arange(n - nr, n, dtype=torch.int64)
        q_pos[s, nb:] = rec.to(torch.int32)
        for l in range(L):
            jb = torch.arange(nb, device=device, dtype=torch.int64)
            cb = counter(s, l, hh[None, :, None], jb[:, None, None], d[None, None, :])
            q[s, l, :nb] = normal(spec.seed, S_BEACON, cb).to(torch_dtype(spec))
            cr = counter(s, l, hh[None, :, None], rec.to(device)[:, None, None], d[None, None, :])
            q[s, l, nb:] = normal(spec.seed, S_RECENT, cr).to(torch_dtype(spec))
    num_q = torch.full((S,), max_q, dtype=torch.int32)
    return Queries(q=q, q_pos=q_pos.to(device), num_q=num_q.to(device), max_q=max_q)
