"""fp64 CPU oracle for the speculative-decoding attention / acceptance path.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline leg may
use this package; the product path never does.  It is independent of the CUDA library: it
imports nothing from it and shares no code with it, only the bytes of the seeded inputs.

The arithmetic lives in ``sd_oracle.c`` (plain C, double precision, one definition per
routine); this module only marshals numpy arrays through ctypes.  Arrays are host numpy arrays:
bf16 tensors are passed as uint16 bit patterns, fp32 tensors as float32.

Parity pins: every routine is pinned by the ``-m "not gpu"`` tests in ``tests/test_oracle_*``
(closed forms, invariants, brute force and library special cases).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

from . import build as _build

_LIB = None

F32 = "f32"
BF16 = "bf16"
_DT = {F32: 0, BF16: 1}


class _Cache(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("h_kv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("stride_b", ctypes.c_int64), ("stride_h", ctypes.c_int64),
                ("stride_pos", ctypes.c_int64), ("block_table", ctypes.c_void_p),
                ("max_pages", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("kv_len", ctypes.c_void_p)]


class _Query(ctypes.Structure):
    _fields_ = [("h_q", ctypes.c_int32), ("softmax_scale", ctypes.c_double),
                ("q_start", ctypes.c_void_p)]


def configure(handle):
    """Declare the C signatures on a loaded oracle library handle and return it."""
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    for name in ("orc_verify_attention", "orc_decode_attention"):
        getattr(handle, name).argtypes = [vp, vp, vp, i32, vp]
    handle.orc_text_anchored_attention.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp]
    handle.orc_sparse_attention.argtypes = [vp, vp, vp, i32, vp, i32, vp, vp]
    handle.orc_topk_select.argtypes = [vp, vp, vp, i32, vp, vp, i32, vp, vp]
    handle.orc_topk_scores.argtypes = [vp, vp, vp, i32, vp, vp, i64, vp]
    handle.orc_topk_attention_scores.argtypes = [vp, vp, vp, i32, vp, vp, i64, vp]
    handle.orc_topk_select_attention.argtypes = [vp, vp, vp, i32, vp, vp, i32, vp, vp]
    handle.orc_hsr_project.argtypes = [vp, vp, i32, i32, vp, vp, vp]
    handle.orc_accept_greedy.argtypes = [vp, vp, vp, i32, i32, vp, vp, i32]
    handle.orc_accept_sample.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, vp, vp, i32, vp, vp]
    handle.orc_rmsnorm_rows.argtypes = [vp, i32, i32, vp, ctypes.c_double, vp]
    handle.orc_rope_rows.argtypes = [vp, i32, i32, vp, ctypes.c_double]
    handle.orc_draft_layer.argtypes = [vp, vp, vp, i32, vp, i32, vp, vp]
    handle.orc_set_threads.argtypes = [i32]
    for name in ("orc_verify_attention", "orc_decode_attention", "orc_text_anchored_attention",
                 "orc_sparse_attention", "orc_topk_select", "orc_topk_scores",
                 "orc_topk_attention_scores", "orc_topk_select_attention",
                 "orc_hsr_project", "orc_accept_greedy", "orc_accept_sample",
                 "orc_rmsnorm_rows", "orc_rope_rows", "orc_draft_layer", "orc_set_threads"):
        getattr(handle, name).restype = ctypes.c_int
    return handle


def lib():
    global _LIB
    if _LIB is None:
        _LIB = configure(ctypes.CDLL(_build.build()))
    return _LIB


def set_threads(n: int) -> int:
    """Set the OpenMP thread count (n <= 0 keeps it); returns the count in use."""
    return int(lib().orc_set_threads(int(n)))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype=None):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=dtype)


class Cache:
    """Host-side description of a KV cache for the oracle (keeps its arrays alive)."""

    def __init__(self, dtype: str, k: np.ndarray, v: np.ndarray, kv_len, h_kv: int,
                 head_dim: int, block_table: Optional[np.ndarray] = None,
                 page_size: int = 0):
        self.dtype = dtype
        st = np.uint16 if dtype == BF16 else np.float32
        self.k = _c(k, st)
        self.v = _c(v, st)
        self.kv_len = _c(kv_len, np.int32)
        self.h_kv, self.head_dim = int(h_kv), int(head_dim)
        self.block_table = _c(block_table, np.int32)
        self.page_size = int(page_size)
        c = _Cache()
        c.dtype, c.h_kv, c.head_dim, c.page_size = _DT[dtype], self.h_kv, self.head_dim, self.page_size
        c.k, c.v = self.k.ctypes.data, self.v.ctypes.data
        if self.page_size == 0:
            # contiguous [batch][h_kv][l_cap][d]
            _, hk, l_cap, d = self.k.shape
            c.stride_b, c.stride_h, c.stride_pos = hk * l_cap * d, l_cap * d, d
            c.block_table, c.max_pages, c.num_pages = None, 0, 0
        else:
            c.stride_b = c.stride_h = c.stride_pos = 0
            c.block_table = self.block_table.ctypes.data
            c.max_pages = self.block_table.shape[1]
            c.num_pages = self.k.shape[0]
        c.kv_len = self.kv_len.ctypes.data
        self.struct = c


def _query(h_q, q_start, scale):
    qs = _c(q_start, np.int32)
    s = _Query()
    s.h_q, s.softmax_scale, s.q_start = int(h_q), float(scale), qs.ctypes.data
    return s, qs


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: invalid arguments (oracle status {rc})")


def verify_attention(h_q: int, q: np.ndarray, q_start, cache: Cache, scale: float = 0.0):
    """Dense verification attention; returns float64 [rows][h_q][d]."""
    qs, keep = _query(h_q, q_start, scale)
    qd = _c(q)
    out = np.zeros((int(keep[-1]), h_q, cache.head_dim), dtype=np.float64)
    rc = lib().orc_verify_attention(ctypes.byref(qs), _ptr(qd), ctypes.byref(cache.struct),
                                    len(keep) - 1, _ptr(out))
    _check(rc, "verify_attention")
    return out


def decode_attention(h_q: int, q: np.ndarray, cache: Cache, scale: float = 0.0):
    """Single-token decode (one row per sequence); returns float64 [batch][h_q][d]."""
    batch = cache.kv_len.shape[0]
    qs, _ = _query(h_q, np.arange(batch + 1), scale)
    qd = _c(q)
    out = np.zeros((batch, h_q, cache.head_dim), dtype=np.float64)
    rc = lib().orc_decode_attention(ctypes.byref(qs), _ptr(qd), ctypes.byref(cache.struct),
                                    batch, _ptr(out))
    _check(rc, "decode_attention")
    return out


def text_anchored_attention(h_q, q, q_start, cache: Cache, vis_begin, vis_end, window,
                            scale: float = 0.0):
    qs, keep = _query(h_q, q_start, scale)
    qd = _c(q)
    vb, ve, w = _c(vis_begin, np.int32), _c(vis_end, np.int32), _c(window, np.int32)
    out = np.zeros((int(keep[-1]), h_q, cache.head_dim), dtype=np.float64)
    rc = lib().orc_text_anchored_attention(ctypes.byref(qs), _ptr(qd), ctypes.byref(cache.struct),
                                           len(keep) - 1, _ptr(vb), _ptr(ve), _ptr(w), _ptr(out))
    _check(rc, "text_anchored_attention")
    return out


def sparse_attention(h_q, q, q_start, cache: Cache, idx, tail_begin, scale: float = 0.0):
    """idx: [batch][h_kv][k] int32 (negative entries are padding)."""
    qs, keep = _query(h_q, q_start, scale)
    qd = _c(q)
    ix = _c(idx, np.int32)
    tb = _c(tail_begin, np.int32)
    out = np.zeros((int(keep[-1]), h_q, cache.head_dim), dtype=np.float64)
    rc = lib().orc_sparse_attention(ctypes.byref(qs), _ptr(qd), ctypes.byref(cache.struct),
                                    len(keep) - 1, _ptr(ix), ix.shape[-1], _ptr(tb), _ptr(out))
    _check(rc, "sparse_attention")
    return out


def topk_select(h_q, q, q_start, cache: Cache, cand_begin, cand_end, k: int):
    """Returns (idx [batch][h_kv][k] int32 ascending, -1 padded; gap [batch][h_kv] float64)."""
    qs, keep = _query(h_q, q_start, 0.0)
    qd = _c(q)
    batch = len(keep) - 1
    cb, ce = _c(cand_begin, np.int32), _c(cand_end, np.int32)
    idx = np.full((batch, cache.h_kv, k), -1, dtype=np.int32)
    gap = np.zeros((batch, cache.h_kv), dtype=np.float64)
    rc = lib().orc_topk_select(ctypes.byref(qs), _ptr(qd), ctypes.byref(cache.struct), batch,
                               _ptr(cb), _ptr(ce), int(k), _ptr(idx), _ptr(gap))
    _check(rc, "topk_select")
    return idx, gap


def topk_scores(h_q, q, q_start, cache: Cache, cand_begin, cand_end):
    """Scores of every candidate: float64 [batch][h_kv][max candidates] (NaN where unused)."""
    qs, keep = _query(h_q, q_start, 0.0)
    qd = _c(q)
    batch = len(keep) - 1
    cb, ce = _c(cand_begin, np.int32), _c(cand_end, np.int32)
    width = int(max(1, (ce - cb).max()))
    sc = np.full((batch, cache.h_kv, width), np.nan, dtype=np.float64)
    rc = lib().orc_topk_scores(ctypes.byref(qs), _ptr(qd), ctypes.byref(cache.struct), batch,
                               _ptr(cb), _ptr(ce), width, _ptr(sc))
    _check(rc, "topk_scores")
    return sc


def topk_attention_scores(h_q, q, q_start, cache: Cache, cand_begin, cand_end,
                          scale: float = 0.0):
    """Mean attention weight that the text query rows of every sequence (the last rows of its
    cache, causal) give each candidate, averaged over rows and the KV head's query heads:
    float64 [batch][h_kv][max candidates] (NaN where unused)."""
    qs, keep = _query(h_q, q_start, scale)
    qd = _c(q)
    batch = len(keep) - 1
    cb, ce = _c(cand_begin, np.int32), _c(cand_end, np.int32)
    width = int(max(1, (ce - cb).max()))
    sc = np.full((batch, cache.h_kv, width), np.nan, dtype=np.float64)
    rc = lib().orc_topk_attention_scores(ctypes.byref(qs), _ptr(qd), ctypes.byref(cache.struct),
                                         batch, _ptr(cb), _ptr(ce), width, _ptr(sc))
    _check(rc, "topk_attention_scores")
    return sc


def topk_select_attention(h_q, q, q_start, cache: Cache, cand_begin, cand_end, k: int,
                          scale: float = 0.0):
    """Top-K by mean text attention.  Returns (idx [batch][h_kv][k] int32 ascending, -1 padded;
    gap [batch][h_kv] float64: (score_k - score_k+1) / score_1)."""
    qs, keep = _query(h_q, q_start, scale)
    qd = _c(q)
    batch = len(keep) - 1
    cb, ce = _c(cand_begin, np.int32), _c(cand_end, np.int32)
    idx = np.full((batch, cache.h_kv, k), -1, dtype=np.int32)
    gap = np.zeros((batch, cache.h_kv), dtype=np.float64)
    rc = lib().orc_topk_select_attention(ctypes.byref(qs), _ptr(qd), ctypes.byref(cache.struct),
                                         batch, _ptr(cb), _ptr(ce), int(k), _ptr(idx), _ptr(gap))
    _check(rc, "topk_select_attention")
    return idx, gap


def hsr_project(emb, hid, weight, bias=None):
    """y = W [e ; h] (+ b) in float64; emb/hid [n][D], weight [D][2D], bias [D] (bf16 bits)."""
    e, h, w = _c(emb, np.uint16), _c(hid, np.uint16), _c(weight, np.uint16)
    b = _c(bias, np.uint16)
    n, D = e.shape
    y = np.zeros((n, D), dtype=np.float64)
    rc = lib().orc_hsr_project(_ptr(e), _ptr(h), n, D, _ptr(w), _ptr(b), _ptr(y))
    _check(rc, "hsr_project")
    return y


def rmsnorm(x, gamma, eps: float):
    """Row-wise RMSNorm of float64 x [rows][n] with bf16 gamma [n]; returns float64."""
    xx = _c(np.atleast_2d(x), np.float64)
    gm = _c(gamma, np.uint16)
    y = np.zeros_like(xx)
    _check(lib().orc_rmsnorm_rows(_ptr(xx), xx.shape[0], xx.shape[1], _ptr(gm), float(eps),
                                  _ptr(y)), "rmsnorm")
    return y


def rope(v, pos, theta: float):
    """Rotary embedding (rotate-half pairs) of float64 rows v [rows][d] at positions pos [rows];
    returns a new float64 array."""
    vv = np.array(np.atleast_2d(v), dtype=np.float64, order="C")
    pp = _c(pos, np.float64)
    _check(lib().orc_rope_rows(_ptr(vv), vv.shape[0], vv.shape[1], _ptr(pp), float(theta)),
           "rope")
    return vv


class _DraftWeights(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("h_q", ctypes.c_int32), ("h_kv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("rms_eps", ctypes.c_double), ("rope_theta", ctypes.c_double),
                ("w_hsr", ctypes.c_void_p), ("ln1", ctypes.c_void_p), ("w_qkv", ctypes.c_void_p),
                ("b_qkv", ctypes.c_void_p), ("w_o", ctypes.c_void_p), ("ln2", ctypes.c_void_p),
                ("w_gate_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p)]


def draft_layer(wt, emb, hid, k_cache, v_cache, kv_len: int, window: int):
    """One draft layer for the rows of emb / hid [n][D] (bf16 bits), the last n positions of a
    one-sequence cache k_cache / v_cache [1][h_kv][cap][d] (bf16 bits, copied: the rows' k and v
    are written into the copies).  wt: an object with the fields of the weights (bf16 bits) and
    shapes.  Returns (y [n][D] float64, k copy, v copy, inter dict of x, q, o, x2)."""
    n, D = emb.shape
    k = np.array(k_cache, dtype=np.uint16, order="C")
    v = np.array(v_cache, dtype=np.uint16, order="C")
    cache = Cache(BF16, k, v, [kv_len], wt.h_kv, wt.head_dim)
    keep = {name: _c(getattr(wt, name), np.uint16) if getattr(wt, name) is not None else None
            for name in ("w_hsr", "ln1", "w_qkv", "b_qkv", "w_o", "ln2", "w_gate_up", "w_down")}
    s = _DraftWeights()
    s.d_model, s.h_q, s.h_kv, s.head_dim, s.d_ff = D, wt.h_q, wt.h_kv, wt.head_dim, wt.d_ff
    s.rms_eps, s.rope_theta = float(wt.rms_eps), float(wt.rope_theta)
    for name, arr in keep.items():
        setattr(s, name, None if arr is None else arr.ctypes.data)
    e, h = _c(emb, np.uint16), _c(hid, np.uint16)
    y = np.zeros((n, D), dtype=np.float64)
    hd = wt.h_q * wt.head_dim
    inter = np.zeros((n, 2 * D + 2 * hd), dtype=np.float64)
    rc = lib().orc_draft_layer(ctypes.byref(s), _ptr(e), _ptr(h), n, ctypes.byref(cache.struct),
                               int(window), _ptr(y), _ptr(inter))
    _check(rc, "draft_layer")
    parts = {"x": inter[:, :D], "q": inter[:, D:D + hd], "o": inter[:, D + hd:D + 2 * hd],
             "x2": inter[:, D + 2 * hd:]}
    return y, cache.k, cache.v, parts


def accept_greedy(tgt, draft_tokens, gamma, vocab: int, out_stride: Optional[int] = None):
    g = _c(gamma, np.int32)
    stride = int(out_stride if out_stride is not None else g.max() + 1)
    t, d = _c(tgt, np.float32), _c(draft_tokens, np.int32)
    n_acc = np.zeros(g.shape[0], dtype=np.int32)
    out = np.full((g.shape[0], stride), -1, dtype=np.int32)
    rc = lib().orc_accept_greedy(_ptr(t), _ptr(d), _ptr(g), g.shape[0], int(vocab), _ptr(n_acc),
                                 _ptr(out), stride)
    _check(rc, "accept_greedy")
    return n_acc, out


def accept_sample(tgt, drf, draft_tokens, u, v, gamma, vocab: int,
                  out_stride: Optional[int] = None):
    """Returns (n_acc, out_tok, accept_margin [sum gamma], draw_margin [batch])."""
    g = _c(gamma, np.int32)
    stride = int(out_stride if out_stride is not None else g.max() + 1)
    t, q = _c(tgt, np.float32), _c(drf, np.float32)
    d = _c(draft_tokens, np.int32)
    uu, vv = _c(u, np.float32), _c(v, np.float32)
    n_acc = np.zeros(g.shape[0], dtype=np.int32)
    out = np.full((g.shape[0], stride), -1, dtype=np.int32)
    am = np.full(max(1, int(g.sum())), np.nan, dtype=np.float64)
    dm = np.zeros(g.shape[0], dtype=np.float64)
    rc = lib().orc_accept_sample(_ptr(t), _ptr(q), _ptr(d), _ptr(uu), _ptr(vv), _ptr(g),
                                 g.shape[0], int(vocab), _ptr(n_acc), _ptr(out), stride,
                                 _ptr(am), _ptr(dm))
    _check(rc, "accept_sample")
    return n_acc, out, am[:int(g.sum())], dm


def cache_from_workload(w, kv_len=None) -> Cache:
    """Oracle cache over a workload object's arrays (duck-typed: dtype, k, v, paged, ...).

    ``kv_len`` defaults to the verify lengths (context plus the gamma+1 appended positions)."""
    kv_len = w.kv_len_verify if kv_len is None else kv_len
    if w.paged:
        return Cache(w.dtype, w.k, w.v, kv_len, w.h_kv, w.d, block_table=w.block_table,
                     page_size=16)
    return Cache(w.dtype, w.k, w.v, kv_len, w.h_kv, w.d)
