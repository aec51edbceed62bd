"""Thin ctypes binding of libkvc (the C ABI declared in include/kvc.h).

Argument marshalling only: every function here packs torch tensors (device memory
owned by the caller) into the C structures and calls the entry point of the same
name.  No step of the path runs in Python.  The library is loaded from this
package directory on first use; if it is missing the import of a function raises
instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvc.so")

KVC_OK, KVC_ERR_INVALID_ARGUMENT, KVC_ERR_UNSUPPORTED, KVC_ERR_CUDA, KVC_ERR_DEVICE_FAULT, KVC_ERR_TIMEOUT = range(6)
KVC_F32, KVC_BF16 = 0, 1
KVC_SCORE_ACCUMULATE, KVC_SCORE_COMPUTE_LSE, KVC_SCORE_SIMT = 1, 2, 4
KVC_HIT_BINARY = 1
DEV_CODES = {0: "ok", 1: "bad page", 2: "bad length", 3: "non-finite value", 4: "kept mismatch",
             5: "freed list overflow", 6: "bad move", 7: "timeout", 8: "bad step table"}

EXPORTS = ["kvc_status_string", "kvc_last_error", "kvc_version", "kvc_query_lse", "kvc_score_from_lse",
           "kvc_lrfu_update", "kvc_select_budget", "kvc_plan_slots", "kvc_compact_workspace_bytes",
           "kvc_compact_pages", "kvc_compact_pages_noalloc", "kvc_ratchet_state_bytes", "kvc_ratchet_init",
           "kvc_confidence_ratchet", "kvc_beacon_update", "kvc_lrfu_select", "kvc_decode_attention",
           "kvc_step_scores", "kvc_append_workspace_bytes", "kvc_append_tokens", "kvc_select_plan"]


class KvcCache(ctypes.Structure):
    _fields_ = [("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p), ("num_pages", ctypes.c_int64),
                ("page_size", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("max_pages_per_row", ctypes.c_int32), ("block_table", ctypes.c_void_p),
                ("row_len", ctypes.c_void_p), ("slot_pos", ctypes.c_void_p), ("slot_label", ctypes.c_void_p),
                ("num_seqs", ctypes.c_int32), ("num_layers", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class KvcQueries(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("q_pos", ctypes.c_void_p),
                ("num_q", ctypes.c_void_p), ("max_q", ctypes.c_int32), ("num_q_heads", ctypes.c_int32)]


class KvcRatchetParams(ctypes.Structure):
    _fields_ = [("top_k", ctypes.c_int32), ("window", ctypes.c_int32), ("stride", ctypes.c_int32),
                ("grow_num", ctypes.c_int32), ("grow_den", ctypes.c_int32), ("init_budget", ctypes.c_int32),
                ("cap", ctypes.c_int32), ("min_points", ctypes.c_int32), ("max_steps", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class KvcRatchetSeqState(ctypes.Structure):
    _fields_ = [("steps_seen", ctypes.c_int64), ("last_expand_step", ctypes.c_int64),
                ("next_window", ctypes.c_int64), ("fit_n", ctypes.c_double), ("fit_sx", ctypes.c_double),
                ("fit_sy", ctypes.c_double), ("fit_sxy", ctypes.c_double), ("fit_sxx", ctypes.c_double),
                ("last_slope", ctypes.c_double), ("budget", ctypes.c_int32), ("expansions", ctypes.c_int32),
                ("last_points", ctypes.c_int32), ("reserved", ctypes.c_int32)]


def ratchet_params(top_k=20, window=64, stride=8, grow_num=7, grow_den=4, init_budget=512, cap=30000,
                   min_points=2, max_steps=64) -> KvcRatchetParams:
    return KvcRatchetParams(top_k, window, stride, grow_num, grow_den, init_budget, cap, min_points, max_steps, 0)


class KvcError(RuntimeError):
    pass


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libkvc.so from the package directory (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise KvcError(f"{LIB_PATH} is missing: build it with agent_kv_cache_lse_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, u32, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_float
        pc, pq, pr = ctypes.POINTER(KvcCache), ctypes.POINTER(KvcQueries), ctypes.POINTER(KvcRatchetParams)
        sig = {
            "kvc_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "kvc_last_error": (ctypes.c_char_p, []),
            "kvc_version": (i32, []),
            "kvc_query_lse": (ctypes.c_int, [pc, pq, vp, vp]),
            "kvc_score_from_lse": (ctypes.c_int, [pc, pq, vp, u32, vp, vp]),
            "kvc_lrfu_update": (ctypes.c_int, [pc, vp, vp, f32, f32, i32, u32, vp, vp]),
            "kvc_select_budget": (ctypes.c_int, [pc, vp, vp, u32, vp, vp, vp, vp]),
            "kvc_lrfu_select": (ctypes.c_int, [pc, vp, vp, f32, f32, i32, u32, vp, u32, vp, vp, vp, vp]),
            "kvc_plan_slots": (ctypes.c_int, [pc, vp, vp, vp, vp, vp, vp, vp]),
            "kvc_select_plan": (ctypes.c_int, [pc, vp, vp, u32, vp, vp, vp, vp, vp, vp, vp]),
            "kvc_compact_workspace_bytes": (ctypes.c_size_t, [i32]),
            "kvc_compact_pages": (ctypes.c_int, [pc, vp, vp, vp, vp, vp, vp, i64, vp, vp, ctypes.c_size_t, vp, vp]),
            "kvc_compact_pages_noalloc": (ctypes.c_int, [pc, vp, vp, vp, vp, vp, vp, i64, vp, vp, vp]),
            "kvc_ratchet_state_bytes": (ctypes.c_size_t, [i32, pr]),
            "kvc_ratchet_init": (ctypes.c_int, [vp, vp, i32, pr, vp]),
            "kvc_confidence_ratchet": (ctypes.c_int, [vp, i32, i32, i32, vp, vp, vp, pr, vp, vp]),
            "kvc_beacon_update": (ctypes.c_int, [vp, vp, i32, i32, i32, i32, i32, ctypes.c_int, vp, vp, i32, vp, i32,
                                                 vp, vp]),
            "kvc_decode_attention": (ctypes.c_int, [pc, vp, vp, i32, vp, vp, vp, u32, vp, vp]),
            "kvc_step_scores": (ctypes.c_int, [pc, vp, vp, vp, i32, f32, vp, vp, vp]),
            "kvc_append_workspace_bytes": (ctypes.c_size_t, [i32]),
            "kvc_append_tokens": (ctypes.c_int, [pc, vp, vp, vp, i32, ctypes.c_uint8, vp, vp, vp, vp, ctypes.c_size_t,
                                                 vp, vp]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, what: str):
    if status != KVC_OK:
        L = lib()
        raise KvcError(f"{what}: {L.kvc_status_string(status).decode()}: {L.kvc_last_error().decode()}")


def _expect(t: torch.Tensor, name: str, shape, dtype):
    """Raise KvcError unless t is a contiguous tensor of the given dtype and shape (None = any extent)."""
    if t.dtype != dtype:
        raise KvcError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.dim() != len(shape) or any(e is not None and t.shape[i] != e for i, e in enumerate(shape)):
        raise KvcError(f"{name}: shape {tuple(t.shape)}, expected {tuple('*' if e is None else e for e in shape)}")
    if not t.is_contiguous():
        raise KvcError(f"{name} must be contiguous")


@dataclass
class Cache:
    """Device tensors of a paged cache (see kvc_cache in include/kvc.h)."""
    k_pool: torch.Tensor        # [num_pages, page_size, D]
    v_pool: torch.Tensor
    block_table: torch.Tensor   # [rows, max_pages] int32
    row_len: torch.Tensor       # [rows] int32
    slot_pos: torch.Tensor      # [rows, max_slots] int32
    slot_label: Optional[torch.Tensor]  # [rows, max_slots] uint8
    num_seqs: int
    num_layers: int
    num_kv_heads: int

    @property
    def rows(self) -> int:
        return self.num_seqs * self.num_layers * self.num_kv_heads

    @property
    def page_size(self) -> int:
        return self.k_pool.shape[1]

    @property
    def max_slots(self) -> int:
        return self.block_table.shape[1] * self.page_size

    def struct(self) -> KvcCache:
        dt = {torch.float32: KVC_F32, torch.bfloat16: KVC_BF16}[self.k_pool.dtype]
        return KvcCache(self.k_pool.data_ptr(), self.v_pool.data_ptr(), self.k_pool.shape[0], self.k_pool.shape[1],
                        self.k_pool.shape[2], dt, self.block_table.shape[1], self.block_table.data_ptr(),
                        self.row_len.data_ptr(), self.slot_pos.data_ptr(),
                        None if self.slot_label is None else self.slot_label.data_ptr(),
                        self.num_seqs, self.num_layers, self.num_kv_heads, 0)


@dataclass
class QuerySet:
    """Device tensors of a query set (see kvc_queries in include/kvc.h)."""
    q: torch.Tensor       # [S, L, max_q, Hq, D]
    lse: torch.Tensor     # [S, L, Hq, max_q] fp32
    q_pos: torch.Tensor   # [S, max_q] int32
    num_q: torch.Tensor   # [S] int32

    def struct(self) -> KvcQueries:
        return KvcQueries(self.q.data_ptr(), self.lse.data_ptr(), self.q_pos.data_ptr(), self.num_q.data_ptr(),
                          self.q.shape[2], self.q.shape[3])


def kvc_query_lse(cache: Cache, queries: QuerySet, d_status=None, stream=None):
    cs, qs = cache.struct(), queries.struct()
    _check(lib().kvc_query_lse(ctypes.byref(cs), ctypes.byref(qs), _ptr(d_status), _stream(stream)), "kvc_query_lse")


def kvc_score_from_lse(cache: Cache, queries: QuerySet, scores: torch.Tensor, flags: int = 0, d_status=None,
                       stream=None):
    cs, qs = cache.struct(), queries.struct()
    _check(lib().kvc_score_from_lse(ctypes.byref(cs), ctypes.byref(qs), _ptr(scores), flags, _ptr(d_status),
                                    _stream(stream)), "kvc_score_from_lse")


def kvc_lrfu_update(cache: Cache, scores: torch.Tensor, crf: torch.Tensor, lam: float = 0.5, hit_mass: float = 0.9,
                    dt_rounds: int = 1, flags: int = 0, d_status=None, stream=None):
    cs = cache.struct()
    _check(lib().kvc_lrfu_update(ctypes.byref(cs), _ptr(scores), _ptr(crf), lam, hit_mass, dt_rounds, flags,
                                 _ptr(d_status), _stream(stream)), "kvc_lrfu_update")


def kvc_select_budget(cache: Cache, crf: torch.Tensor, budget: torch.Tensor, keep: torch.Tensor, kept: torch.Tensor,
                      protect_label_mask: int = 0, d_status=None, stream=None):
    cs = cache.struct()
    _check(lib().kvc_select_budget(ctypes.byref(cs), _ptr(crf), _ptr(budget), protect_label_mask, _ptr(keep),
                                   _ptr(kept), _ptr(d_status), _stream(stream)), "kvc_select_budget")


def kvc_lrfu_select(cache: Cache, scores: torch.Tensor, crf: torch.Tensor, budget: torch.Tensor, keep: torch.Tensor,
                    kept: torch.Tensor, lam: float = 0.5, hit_mass: float = 0.9, dt_rounds: int = 1, flags: int = 0,
                    protect_label_mask: int = 0, d_status=None, stream=None):
    """kvc_lrfu_update followed by kvc_select_budget, in one launch."""
    cs = cache.struct()
    _check(lib().kvc_lrfu_select(ctypes.byref(cs), _ptr(scores), _ptr(crf), lam, hit_mass, dt_rounds, flags,
                                 _ptr(budget), protect_label_mask, _ptr(keep), _ptr(kept), _ptr(d_status),
                                 _stream(stream)),
           "kvc_lrfu_select")


def kvc_plan_slots(cache: Cache, keep: torch.Tensor, kept: torch.Tensor, move_src: torch.Tensor,
                   move_dst: torch.Tensor, num_moves: torch.Tensor, d_status=None, stream=None):
    cs = cache.struct()
    _check(lib().kvc_plan_slots(ctypes.byref(cs), _ptr(keep), _ptr(kept), _ptr(move_src), _ptr(move_dst),
                                _ptr(num_moves), _ptr(d_status), _stream(stream)), "kvc_plan_slots")


def kvc_select_plan(cache: Cache, crf: torch.Tensor, budget: torch.Tensor, keep: torch.Tensor, kept: torch.Tensor,
                    move_src: torch.Tensor, move_dst: torch.Tensor, num_moves: torch.Tensor,
                    protect_label_mask: int = 0, d_status=None, stream=None):
    """kvc_select_budget followed by kvc_plan_slots, in one launch."""
    cs = cache.struct()
    _check(lib().kvc_select_plan(ctypes.byref(cs), _ptr(crf), _ptr(budget), protect_label_mask, _ptr(keep), _ptr(kept),
                                 _ptr(move_src), _ptr(move_dst), _ptr(num_moves), _ptr(d_status), _stream(stream)),
           "kvc_select_plan")


def kvc_compact_workspace_bytes(rows: int) -> int:
    return int(lib().kvc_compact_workspace_bytes(rows))


def kvc_compact_pages(cache: Cache, move_src, move_dst, num_moves, new_len, crf: Optional[torch.Tensor],
                      freed: torch.Tensor, num_freed: torch.Tensor, workspace: torch.Tensor, d_status=None,
                      stream=None):
    cs = cache.struct()
    _check(lib().kvc_compact_pages(ctypes.byref(cs), _ptr(move_src), _ptr(move_dst), _ptr(num_moves), _ptr(new_len),
                                   _ptr(crf), _ptr(freed), freed.numel(), _ptr(num_freed), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _ptr(d_status), _stream(stream)),
           "kvc_compact_pages")


def kvc_compact_pages_noalloc(cache: Cache, move_src, move_dst, num_moves, new_len, crf: Optional[torch.Tensor],
                              freed: torch.Tensor, num_freed: torch.Tensor, d_status=None, stream=None):
    """kvc_compact_pages with the library's built-in workspace, for callers that cannot allocate device memory
    (e.g. when the KV pool owns all free memory, or behind a foreign-function boundary).  At most KVC_NOALLOC_MAX_ROWS
    rows; calls that overlap on the GPU share the workspace and must be serialised."""
    cs = cache.struct()
    _check(lib().kvc_compact_pages_noalloc(ctypes.byref(cs), _ptr(move_src), _ptr(move_dst), _ptr(num_moves),
                                           _ptr(new_len), _ptr(crf), _ptr(freed), freed.numel(), _ptr(num_freed),
                                           _ptr(d_status), _stream(stream)),
           "kvc_compact_pages_noalloc")


NOALLOC_MAX_ROWS = 16384


def kvc_append_workspace_bytes(rows: int) -> int:
    return int(lib().kvc_append_workspace_bytes(rows))


def kvc_append_tokens(cache: Cache, k_new: torch.Tensor, v_new: torch.Tensor, new_pos: torch.Tensor, label: int,
                      crf: Optional[torch.Tensor], free_pages: torch.Tensor, free_count: torch.Tensor,
                      workspace: torch.Tensor, d_status=None, stream=None):
    """Append k_new/v_new [rows][count][D] at each row's end, pages from the free_pages stack (depth free_count)."""
    count = k_new.shape[1]
    _expect(k_new, "k_new", (cache.rows, count, cache.k_pool.shape[-1]), cache.k_pool.dtype)
    _expect(v_new, "v_new", (cache.rows, count, cache.k_pool.shape[-1]), cache.k_pool.dtype)
    _expect(new_pos, "new_pos", (cache.num_seqs, count), torch.int32)
    if crf is not None:
        _expect(crf, "crf", (cache.rows, cache.max_slots), torch.float32)
    cs = cache.struct()
    _check(lib().kvc_append_tokens(ctypes.byref(cs), _ptr(k_new), _ptr(v_new), _ptr(new_pos), count, label, _ptr(crf),
                                   _ptr(free_pages), _ptr(free_count), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _ptr(d_status), _stream(stream)),
           "kvc_append_tokens")


def kvc_ratchet_state_bytes(num_seqs: int, params: KvcRatchetParams) -> int:
    return int(lib().kvc_ratchet_state_bytes(num_seqs, ctypes.byref(params)))


def kvc_ratchet_init(state: torch.Tensor, budget: torch.Tensor, num_seqs: int, params: KvcRatchetParams,
                     stream=None):
    _check(lib().kvc_ratchet_init(_ptr(state), _ptr(budget), num_seqs, ctypes.byref(params), _stream(stream)),
           "kvc_ratchet_init")


def kvc_confidence_ratchet(logits: torch.Tensor, state: torch.Tensor, budget: torch.Tensor,
                           params: KvcRatchetParams, confidence_out: Optional[torch.Tensor] = None, d_status=None,
                           stream=None):
    S, T, V = logits.shape
    _check(lib().kvc_confidence_ratchet(_ptr(logits), S, T, V, _ptr(state), _ptr(budget), _ptr(confidence_out),
                                        ctypes.byref(params), _ptr(d_status), _stream(stream)),
           "kvc_confidence_ratchet")


def kvc_beacon_update(q: torch.Tensor, num_q: torch.Tensor, beacons: torch.Tensor, counts: torch.Tensor,
                      beacon_q: Optional[torch.Tensor] = None, d_status=None, stream=None):
    """q: [S][L][max_q][Hq][D] (bf16 or fp32); beacons: [S][L][Hq][B][D] fp32; counts: [S][L][Hq][B] int32;
    beacon_q: optional [S][L][out_max_q][Hq][D] in q's dtype (rows 0..B-1 receive the beacons)."""
    S, L, max_q, Hq, D = q.shape
    B = beacons.shape[3]
    dt = 1 if q.dtype == torch.bfloat16 else 0
    out_max_q = beacon_q.shape[2] if beacon_q is not None else 0
    _check(lib().kvc_beacon_update(_ptr(q), _ptr(num_q), S, L, Hq, D, max_q, dt, _ptr(beacons), _ptr(counts), B,
                                   _ptr(beacon_q), out_max_q, _ptr(d_status), _stream(stream)),
           "kvc_beacon_update")


def kvc_decode_attention(cache: Cache, q: torch.Tensor, q_pos: torch.Tensor, out: torch.Tensor, lse: torch.Tensor,
                         scores: Optional[torch.Tensor] = None, flags: int = 0, d_status=None, stream=None):
    """One decode step with the scores folded in.  q: [S][L][Hq][D] in the cache dtype; q_pos: [S] int32;
    out: [S][L][Hq][D] fp32; lse: [S][L][Hq] fp32; scores: optional [rows][max_slots] fp32
    (KVC_SCORE_ACCUMULATE adds into it).  Shapes and dtypes, which the C ABI cannot see, are checked here."""
    S, L, D = cache.num_seqs, cache.num_layers, cache.k_pool.shape[2]
    _expect(q, "q", (S, L, None, D), cache.k_pool.dtype)
    Hq = q.shape[2]
    _expect(q_pos, "q_pos", (S,), torch.int32)
    _expect(out, "out", (S, L, Hq, D), torch.float32)
    _expect(lse, "lse", (S, L, Hq), torch.float32)
    if scores is not None:
        _expect(scores, "scores", (cache.rows, cache.max_slots), torch.float32)
    cs = cache.struct()
    _check(lib().kvc_decode_attention(ctypes.byref(cs), _ptr(q), _ptr(q_pos), q.shape[2], _ptr(out), _ptr(lse),
                                      _ptr(scores), flags, _ptr(d_status), _stream(stream)),
           "kvc_decode_attention")


def kvc_step_scores(cache: Cache, scores: torch.Tensor, step_start: torch.Tensor, num_steps: torch.Tensor,
                    out: torch.Tensor, beta: float = 0.5, d_status=None, stream=None):
    """Step-aware ranking scores: (1 - beta) * s + beta * (mean score of the entry's step).  step_start:
    [S][max_steps] int32 ascending from 0; num_steps: [S] int32; out: [rows][max_slots] fp32 (may be scores)."""
    _expect(scores, "scores", (cache.rows, cache.max_slots), torch.float32)
    _expect(out, "out", (cache.rows, cache.max_slots), torch.float32)
    _expect(step_start, "step_start", (cache.num_seqs, None), torch.int32)
    _expect(num_steps, "num_steps", (cache.num_seqs,), torch.int32)
    cs = cache.struct()
    _check(lib().kvc_step_scores(ctypes.byref(cs), _ptr(scores), _ptr(step_start), _ptr(num_steps),
                                 step_start.shape[1], beta, _ptr(out), _ptr(d_status), _stream(stream)),
           "kvc_step_scores")


def ratchet_seq_states(state: torch.Tensor, num_seqs: int):
    """Host copy of the per-sequence ratchet records at the head of a state buffer."""
    raw = state[: num_seqs * ctypes.sizeof(KvcRatchetSeqState)].cpu().numpy().tobytes()
    n = ctypes.sizeof(KvcRatchetSeqState)
    return [KvcRatchetSeqState.from_buffer_copy(raw[i * n:(i + 1) * n]) for i in range(num_seqs)]


def device_status(d_status: torch.Tensor):
    """(code, row, name) of a d_status pair after a sync."""
    code, row = (int(x) for x in d_status.cpu().tolist())
    return code, row, DEV_CODES.get(code, "unknown")
