"""Thin Python binding of ``libsdattn.so`` (the C interface in ``include/sd_attn.h``).

Argument marshalling only: every step of the computation runs in the library's CUDA kernels.
Functions keep the C names and take torch CUDA tensors; descriptors are built from them.
Workspaces are allocated here with torch when the caller passes none (the C library itself
never allocates).  A status other than SD_OK raises :class:`SdError`.  There is no CPU
fallback: without the library, or without a GPU, calls raise.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

from . import build as _build

SD_OK, SD_ERR_INVALID_ARG, SD_ERR_UNSUPPORTED, SD_ERR_WORKSPACE, SD_ERR_CUDA = range(5)
SD_F32, SD_BF16 = 0, 1
SD_ATTN_VERIFY, SD_ATTN_TEXT_ANCHORED, SD_ATTN_SPARSE = 0, 1, 2
SD_ENGINE_CUDA_CORE, SD_ENGINE_TC, SD_ENGINE_TC_PERSISTENT = 0, 1, 2
SD_TOPK_LAST_QUERY, SD_TOPK_MEAN_TEXT_ATTENTION = 0, 1
SD_DEVERR_PAGE, SD_DEVERR_INDEX, SD_DEVERR_TOKEN, SD_DEVERR_NUMERIC, SD_DEVERR_SHAPE = 1, 2, 4, 8, 16
SD_DEVERR_TIMEOUT = 32
PAGE_SIZE = 16

_LIB = None
_LOCK = threading.Lock()


class SdError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib().sd_status_string(status).decode()}")


class sd_kv_desc(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("h_kv", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("stride_b", ctypes.c_int64), ("stride_h", ctypes.c_int64),
                ("stride_pos", ctypes.c_int64), ("block_table", ctypes.c_void_p),
                ("max_pages_per_seq", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("kv_len", ctypes.c_void_p)]


class sd_q_desc(ctypes.Structure):
    _fields_ = [("h_q", ctypes.c_int32), ("max_q_rows", ctypes.c_int32),
                ("max_kv_len", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
                ("q_start", ctypes.c_void_p)]


EXPORTS = ("sd_status_string", "sd_version", "sd_attention_workspace_size", "sd_verify_attention",
           "sd_text_anchored_attention", "sd_sparse_attention", "sd_topk_workspace_size",
           "sd_topk_select", "sd_hsr_project", "sd_accept_workspace_size", "sd_accept_greedy",
           "sd_accept_sample", "sd_verify_attention_noalloc", "sd_sparse_workspace_size",
           "sd_sparse_selection_size", "sd_sparse_stage", "sd_sparse_attention_staged",
           "sd_topk_scored_workspace_size", "sd_topk_select_scored", "sd_set_wait_timeout_ns",
           "sd_draft_layer_workspace_size", "sd_draft_layer", "sd_attention_plan")

# Size of the library's fixed scratch used by sd_verify_attention_noalloc.
SD_VERIFY_NOALLOC_SCRATCH_BYTES = 64 << 20


def lib():
    """The loaded library (built in-tree first when missing or older than its sources)."""
    global _LIB
    if _LIB is None:
        with _LOCK:
            if _LIB is None:
                path = _build.LIB
                if _build.is_stale():
                    path = _build.build()
                h = ctypes.CDLL(path)
                P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
                h.sd_status_string.restype = ctypes.c_char_p
                h.sd_status_string.argtypes = [ctypes.c_int]
                h.sd_version.restype = I32
                h.sd_draft_layer_workspace_size.argtypes = [P, I32, P, I32, I32, ctypes.POINTER(SZ)]
                h.sd_draft_layer.argtypes = [P, P, P, I32, P, I32, I32, P, P, SZ, P, P]
                h.sd_set_wait_timeout_ns.restype = ctypes.c_uint64
                h.sd_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
                h.sd_attention_workspace_size.argtypes = [ctypes.c_int, P, P, I32, ctypes.POINTER(SZ)]
                h.sd_attention_plan.argtypes = [ctypes.c_int, P, P, I32, I32, I32,
                                                ctypes.POINTER(I32), ctypes.POINTER(I32)]
                h.sd_verify_attention.argtypes = [P, P, P, I32, P, P, SZ, P, P]
                h.sd_text_anchored_attention.argtypes = [P, P, P, I32, P, P, P, I32, P, P, SZ, P, P]
                h.sd_sparse_attention.argtypes = [P, P, P, I32, P, I32, P, I32, P, P, SZ, P, P]
                h.sd_topk_workspace_size.argtypes = [P, I32, I32, I32, ctypes.POINTER(SZ)]
                h.sd_topk_select.argtypes = [P, P, P, I32, P, P, I32, I32, P, P, SZ, P, P]
                h.sd_hsr_project.argtypes = [P, P, I32, I32, P, P, P, P]
                h.sd_accept_workspace_size.argtypes = [I32, I32, I32, ctypes.POINTER(SZ)]
                h.sd_accept_greedy.argtypes = [P, P, P, I32, I32, I32, P, P, I32, P, SZ, P, P]
                h.sd_accept_sample.argtypes = [P, P, P, P, P, P, I32, I32, I32, P, P, I32, P, P, SZ,
                                               P, P]
                h.sd_verify_attention_noalloc.argtypes = [P, P, P, I32, P, P, P]
                h.sd_sparse_workspace_size.argtypes = [P, P, I32, I32, I32, ctypes.POINTER(SZ)]
                h.sd_sparse_selection_size.argtypes = [P, I32, I32, ctypes.POINTER(SZ)]
                h.sd_sparse_stage.argtypes = [P, I32, P, I32, P, P, SZ, P, P]
                h.sd_sparse_attention_staged.argtypes = [P, P, P, I32, P, I32, P, I32, P, P, SZ,
                                                         P, P]
                h.sd_topk_scored_workspace_size.argtypes = [ctypes.c_int, P, P, I32, I32, I32,
                                                            ctypes.POINTER(SZ)]
                h.sd_topk_select_scored.argtypes = [ctypes.c_int, P, P, P, I32, P, P, I32, I32, P,
                                                    P, P, SZ, P, P]
                for name in EXPORTS[2:]:
                    if name not in ("sd_set_wait_timeout_ns",):
                        getattr(h, name).restype = ctypes.c_int
                _LIB = h
    return _LIB


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("sdattn: tensors must live on the GPU")
    if not t.is_contiguous():
        raise ValueError("sdattn: tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _on(t: torch.Tensor):
    """Make the tensor's device current for the call (the library launches on the current
    device, and sd_verify_attention_noalloc picks its per-device scratch from it)."""
    if t.device.type == "cuda" and t.device.index is not None and \
            t.device.index != torch.cuda.current_device():
        return torch.cuda.device(t.device)
    return contextlib.nullcontext()


def _check(status: int, where: str):
    if status != SD_OK:
        raise SdError(status, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SD_BF16
    if t.dtype == torch.float32:
        return SD_F32
    raise ValueError(f"sdattn: unsupported dtype {t.dtype}")


class KVCache:
    """KV cache tensors plus the C descriptor.

    Contiguous: ``k``, ``v`` of shape [batch][h_kv][l_cap][head_dim].
    Paged: ``k``, ``v`` of shape [num_pages][h_kv][16][head_dim] with ``block_table``
    [batch][max_pages] int32.  ``kv_len``: int32 [batch] on the GPU.
    """

    def __init__(self, k: torch.Tensor, v: torch.Tensor, kv_len: torch.Tensor,
                 block_table: Optional[torch.Tensor] = None):
        if k.shape != v.shape or k.dtype != v.dtype or k.dim() != 4:
            raise ValueError("KVCache: k and v must be 4-D tensors of one shape and dtype")
        self.k, self.v, self.kv_len, self.block_table = k, v, kv_len, block_table
        d = sd_kv_desc()
        d.dtype = _dtype_code(k)
        d.h_kv = k.shape[1]
        d.head_dim = k.shape[3]
        d.k, d.v = _ptr(k), _ptr(v)
        if block_table is None:
            d.page_size = 0
            d.stride_b, d.stride_h, d.stride_pos = k.stride(0), k.stride(1), k.stride(2)
        else:
            if k.shape[2] != PAGE_SIZE:
                raise ValueError("KVCache: paged caches use pages of 16 positions")
            d.page_size = PAGE_SIZE
            d.block_table = _ptr(block_table)
            d.max_pages_per_seq = block_table.shape[1]
            d.num_pages = k.shape[0]
        d.kv_len = _ptr(kv_len)
        self.desc = d

    @property
    def batch(self) -> int:
        return self.kv_len.shape[0]

    @property
    def h_kv(self) -> int:
        return self.k.shape[1]

    @property
    def head_dim(self) -> int:
        return self.k.shape[3]


class Queries:
    """Query rows [rows][h_q][head_dim] with q_start [batch+1] (int32, GPU) and host hints."""

    def __init__(self, q: torch.Tensor, q_start: torch.Tensor, max_q_rows: int, max_kv_len: int,
                 softmax_scale: float = 0.0):
        self.q, self.q_start = q, q_start
        d = sd_q_desc()
        d.h_q = q.shape[1]
        d.max_q_rows = int(max_q_rows)
        d.max_kv_len = int(max_kv_len)
        d.softmax_scale = float(softmax_scale)
        d.q_start = _ptr(q_start)
        self.desc = d

    @property
    def rows(self) -> int:
        return self.q.shape[0]


def _workspace(nbytes, device, given: Optional[torch.Tensor]):
    """The caller's workspace (the library checks its size), or a new one of nbytes() bytes (the
    size query only runs when a workspace has to be allocated)."""
    if given is not None:
        return given
    return torch.empty(max(int(nbytes()), 16), dtype=torch.uint8, device=device)


def sd_set_wait_timeout_ns(ns: int) -> int:
    """Bound of the waits inside the tensor-core kernels (0 restores 1 s); returns the previous
    bound."""
    return int(lib().sd_set_wait_timeout_ns(int(ns)))


def sd_attention_workspace_size(kind: int, q: Queries, kv: KVCache) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().sd_attention_workspace_size(kind, ctypes.byref(q.desc), ctypes.byref(kv.desc),
                                             kv.batch, ctypes.byref(n)), "sd_attention_workspace_size")
    return n.value


def sd_attention_plan(kind: int, q: Queries, kv: KVCache, extent: int = 0,
                      max_tail: int = 0) -> Tuple[int, int]:
    """(engine, parts) of an attention call with these hints: SD_ENGINE_* and the split count
    (or the persistent plan's partial slots).  extent: max_window (text-anchored) or k (sparse)."""
    e, n = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib().sd_attention_plan(kind, ctypes.byref(q.desc), ctypes.byref(kv.desc), kv.batch,
                                   int(extent), int(max_tail), ctypes.byref(e), ctypes.byref(n)),
           "sd_attention_plan")
    return e.value, n.value


def _attn_out(q: Queries, out):
    return torch.empty_like(q.q) if out is None else out


def sd_verify_attention(q: Queries, kv: KVCache, out=None, workspace=None, dev_err=None,
                        stream=None) -> torch.Tensor:
    out = _attn_out(q, out)
    ws = _workspace(lambda: sd_attention_workspace_size(SD_ATTN_VERIFY, q, kv), q.q.device, workspace)
    with _on(q.q):
        _check(lib().sd_verify_attention(ctypes.byref(q.desc), _ptr(q.q), ctypes.byref(kv.desc),
                                         kv.batch, _ptr(out), _ptr(ws), ws.numel(), _ptr(dev_err),
                                         _stream(stream)), "sd_verify_attention")
    return out


def sd_verify_attention_noalloc(q: Queries, kv: KVCache, out: torch.Tensor, dev_err=None,
                                stream=None) -> torch.Tensor:
    """sd_verify_attention on the library's fixed scratch: the C call allocates nothing, so the
    caller passes ``out``.  Raises SdError (SD_ERR_WORKSPACE) when the call's workspace exceeds
    SD_VERIFY_NOALLOC_SCRATCH_BYTES."""
    with _on(q.q):
        _check(lib().sd_verify_attention_noalloc(ctypes.byref(q.desc), _ptr(q.q),
                                                 ctypes.byref(kv.desc), kv.batch, _ptr(out),
                                                 _ptr(dev_err), _stream(stream)),
               "sd_verify_attention_noalloc")
    return out


def sd_text_anchored_attention(q: Queries, kv: KVCache, vis_begin, vis_end, window,
                               max_window: int, out=None, workspace=None, dev_err=None,
                               stream=None) -> torch.Tensor:
    out = _attn_out(q, out)
    ws = _workspace(lambda: sd_attention_workspace_size(SD_ATTN_TEXT_ANCHORED, q, kv), q.q.device, workspace)
    with _on(q.q):
        _check(lib().sd_text_anchored_attention(
            ctypes.byref(q.desc), _ptr(q.q), ctypes.byref(kv.desc), kv.batch, _ptr(vis_begin),
            _ptr(vis_end), _ptr(window), int(max_window), _ptr(out), _ptr(ws), ws.numel(),
            _ptr(dev_err), _stream(stream)), "sd_text_anchored_attention")
    return out


def sd_sparse_attention(q: Queries, kv: KVCache, idx: torch.Tensor, tail_begin, max_tail: int,
                        out=None, workspace=None, dev_err=None, stream=None) -> torch.Tensor:
    out = _attn_out(q, out)
    ws = _workspace(lambda: sd_sparse_workspace_size(q, kv, int(idx.shape[-1]), max_tail), q.q.device,
                    workspace)
    with _on(q.q):
        _check(lib().sd_sparse_attention(
            ctypes.byref(q.desc), _ptr(q.q), ctypes.byref(kv.desc), kv.batch, _ptr(idx),
            int(idx.shape[-1]), _ptr(tail_begin), int(max_tail), _ptr(out), _ptr(ws), ws.numel(),
            _ptr(dev_err), _stream(stream)), "sd_sparse_attention")
    return out


def sd_sparse_workspace_size(q: Queries, kv: KVCache, k: int, max_tail: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().sd_sparse_workspace_size(ctypes.byref(q.desc), ctypes.byref(kv.desc), kv.batch,
                                          int(k), int(max_tail), ctypes.byref(n)),
           "sd_sparse_workspace_size")
    return n.value


def sd_sparse_selection_size(kv: KVCache, k: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().sd_sparse_selection_size(ctypes.byref(kv.desc), kv.batch, int(k),
                                          ctypes.byref(n)), "sd_sparse_selection_size")
    return n.value


def sd_sparse_stage(kv: KVCache, idx: torch.Tensor, tail_begin, selection=None, dev_err=None,
                    stream=None) -> torch.Tensor:
    """Stages the selected rows of idx [batch][h_kv][k]; returns the selection buffer."""
    k = int(idx.shape[-1])
    if selection is None:
        selection = torch.empty(max(sd_sparse_selection_size(kv, k), 16), dtype=torch.uint8,
                                device=kv.k.device)
    with _on(kv.k):
        _check(lib().sd_sparse_stage(ctypes.byref(kv.desc), kv.batch, _ptr(idx), k,
                                     _ptr(tail_begin), _ptr(selection), selection.numel(),
                                     _ptr(dev_err), _stream(stream)), "sd_sparse_stage")
    return selection


def sd_sparse_attention_staged(q: Queries, kv: KVCache, selection: torch.Tensor, k: int,
                               tail_begin, max_tail: int, out=None, workspace=None, dev_err=None,
                               stream=None) -> torch.Tensor:
    out = _attn_out(q, out)
    ws = _workspace(lambda: sd_sparse_workspace_size(q, kv, k, max_tail), q.q.device, workspace)
    with _on(q.q):
        _check(lib().sd_sparse_attention_staged(
            ctypes.byref(q.desc), _ptr(q.q), ctypes.byref(kv.desc), kv.batch, _ptr(selection),
            int(k), _ptr(tail_begin), int(max_tail), _ptr(out), _ptr(ws), ws.numel(), _ptr(dev_err),
            _stream(stream)), "sd_sparse_attention_staged")
    return out


def sd_topk_workspace_size(kv: KVCache, max_cand: int, k: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().sd_topk_workspace_size(ctypes.byref(kv.desc), kv.batch, int(max_cand), int(k),
                                        ctypes.byref(n)), "sd_topk_workspace_size")
    return n.value


def sd_topk_select(q: Queries, kv: KVCache, cand_begin, cand_end, max_cand: int, k: int,
                   idx_out=None, workspace=None, dev_err=None, stream=None) -> torch.Tensor:
    if idx_out is None:
        idx_out = torch.empty((kv.batch, kv.h_kv, int(k)), dtype=torch.int32, device=q.q.device)
    ws = _workspace(lambda: sd_topk_workspace_size(kv, max_cand, k), q.q.device, workspace)
    with _on(q.q):
        _check(lib().sd_topk_select(
            ctypes.byref(q.desc), _ptr(q.q), ctypes.byref(kv.desc), kv.batch, _ptr(cand_begin),
            _ptr(cand_end), int(max_cand), int(k), _ptr(idx_out), _ptr(ws), ws.numel(),
            _ptr(dev_err), _stream(stream)), "sd_topk_select")
    return idx_out


def sd_topk_scored_workspace_size(mode: int, q: Queries, kv: KVCache, max_cand: int,
                                  k: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().sd_topk_scored_workspace_size(int(mode), ctypes.byref(q.desc),
                                               ctypes.byref(kv.desc), kv.batch, int(max_cand),
                                               int(k), ctypes.byref(n)),
           "sd_topk_scored_workspace_size")
    return n.value


def sd_topk_select_scored(mode: int, q: Queries, kv: KVCache, cand_begin, cand_end,
                          max_cand: int, k: int, idx_out=None, scores_out=None, workspace=None,
                          dev_err=None, stream=None) -> torch.Tensor:
    """Top-K with a score mode: SD_TOPK_LAST_QUERY (as sd_topk_select) or
    SD_TOPK_MEAN_TEXT_ATTENTION (q holds the prefill text rows).  scores_out: optional float64
    [batch][h_kv][max_cand] tensor that receives every candidate's score."""
    if idx_out is None:
        idx_out = torch.empty((kv.batch, kv.h_kv, int(k)), dtype=torch.int32, device=q.q.device)
    ws = _workspace(lambda: sd_topk_scored_workspace_size(mode, q, kv, max_cand, k), q.q.device,
                    workspace)
    with _on(q.q):
        _check(lib().sd_topk_select_scored(
            int(mode), ctypes.byref(q.desc), _ptr(q.q), ctypes.byref(kv.desc), kv.batch,
            _ptr(cand_begin), _ptr(cand_end), int(max_cand), int(k), _ptr(idx_out),
            _ptr(scores_out), _ptr(ws), ws.numel(), _ptr(dev_err), _stream(stream)),
            "sd_topk_select_scored")
    return idx_out


class sd_draft_layer_desc(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("h_q", ctypes.c_int32), ("h_kv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("w_hsr", ctypes.c_void_p), ("ln1", ctypes.c_void_p), ("w_qkv", ctypes.c_void_p),
                ("b_qkv", ctypes.c_void_p), ("w_o", ctypes.c_void_p), ("ln2", ctypes.c_void_p),
                ("w_gate_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p)]


class DraftLayer:
    """The weights of one draft layer (bf16 tensors on the GPU) and their C descriptor."""

    NAMES = ("w_hsr", "ln1", "w_qkv", "b_qkv", "w_o", "ln2", "w_gate_up", "w_down")

    def __init__(self, d_model, h_q, h_kv, head_dim, d_ff, rms_eps, rope_theta, **weights):
        self.weights = weights
        d = sd_draft_layer_desc()
        d.d_model, d.h_q, d.h_kv, d.head_dim, d.d_ff = d_model, h_q, h_kv, head_dim, d_ff
        d.rms_eps, d.rope_theta = float(rms_eps), float(rope_theta)
        for name in self.NAMES:
            t = weights.get(name)
            setattr(d, name, _ptr(t))
        self.desc = d
        self.d_model = d_model


def sd_draft_layer_workspace_size(layer: DraftLayer, n_rows: int, cache: KVCache,
                                  max_kv_len: int, window: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().sd_draft_layer_workspace_size(ctypes.byref(layer.desc), int(n_rows),
                                               ctypes.byref(cache.desc), int(max_kv_len),
                                               int(window), ctypes.byref(n)),
           "sd_draft_layer_workspace_size")
    return n.value


def sd_draft_layer(layer: DraftLayer, emb: torch.Tensor, hid: torch.Tensor, cache: KVCache,
                   max_kv_len: int, window: int, out=None, workspace=None, dev_err=None,
                   stream=None) -> torch.Tensor:
    """One draft layer for the rows of emb / hid [n][d_model]; writes the rows' k and v into
    `cache` (whose kv_len already counts them)."""
    n = emb.shape[0]
    if out is None:
        out = torch.empty((n, layer.d_model), dtype=torch.bfloat16, device=emb.device)
    ws = _workspace(lambda: sd_draft_layer_workspace_size(layer, n, cache, max_kv_len, window),
                    emb.device, workspace)
    with _on(emb):
        _check(lib().sd_draft_layer(ctypes.byref(layer.desc), _ptr(emb), _ptr(hid), int(n),
                                    ctypes.byref(cache.desc), int(max_kv_len), int(window),
                                    _ptr(out), _ptr(ws), ws.numel(), _ptr(dev_err),
                                    _stream(stream)), "sd_draft_layer")
    return out


def sd_hsr_project(emb: torch.Tensor, hid: torch.Tensor, weight: torch.Tensor, bias=None,
                   out=None, stream=None) -> torch.Tensor:
    n, dm = emb.shape
    if out is None:
        out = torch.empty((n, dm), dtype=torch.bfloat16, device=emb.device)
    with _on(emb):
        _check(lib().sd_hsr_project(_ptr(emb), _ptr(hid), n, dm, _ptr(weight), _ptr(bias),
                                    _ptr(out), _stream(stream)), "sd_hsr_project")
    return out


def sd_accept_workspace_size(batch: int, max_gamma: int, vocab: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().sd_accept_workspace_size(int(batch), int(max_gamma), int(vocab), ctypes.byref(n)),
           "sd_accept_workspace_size")
    return n.value


def sd_accept_greedy(tgt_logits, draft_tok, gamma, max_gamma: int, n_acc=None, out_tok=None,
                     workspace=None, dev_err=None, stream=None):
    batch, vocab = gamma.shape[0], tgt_logits.shape[1]
    dev = tgt_logits.device
    n_acc = torch.empty(batch, dtype=torch.int32, device=dev) if n_acc is None else n_acc
    if out_tok is None:
        out_tok = torch.full((batch, max_gamma + 1), -1, dtype=torch.int32, device=dev)
    ws = _workspace(lambda: sd_accept_workspace_size(batch, max_gamma, vocab), dev, workspace)
    with _on(tgt_logits):
        _check(lib().sd_accept_greedy(_ptr(tgt_logits), _ptr(draft_tok), _ptr(gamma), batch,
                                      int(max_gamma), vocab, _ptr(n_acc), _ptr(out_tok),
                                      out_tok.shape[1], _ptr(ws), ws.numel(), _ptr(dev_err),
                                      _stream(stream)), "sd_accept_greedy")
    return n_acc, out_tok


def sd_accept_sample(tgt_logits, draft_logits, draft_tok, u, v, gamma, max_gamma: int,
                     n_acc=None, out_tok=None, near_boundary=None, workspace=None, dev_err=None,
                     stream=None):
    batch, vocab = gamma.shape[0], tgt_logits.shape[1]
    dev = tgt_logits.device
    n_acc = torch.empty(batch, dtype=torch.int32, device=dev) if n_acc is None else n_acc
    if out_tok is None:
        out_tok = torch.full((batch, max_gamma + 1), -1, dtype=torch.int32, device=dev)
    if near_boundary is None:
        near_boundary = torch.zeros(batch, dtype=torch.int32, device=dev)
    ws = _workspace(lambda: sd_accept_workspace_size(batch, max_gamma, vocab), dev, workspace)
    with _on(tgt_logits):
        _check(lib().sd_accept_sample(_ptr(tgt_logits), _ptr(draft_logits), _ptr(draft_tok),
                                      _ptr(u), _ptr(v), _ptr(gamma), batch, int(max_gamma), vocab,
                                      _ptr(n_acc), _ptr(out_tok), out_tok.shape[1],
                                      _ptr(near_boundary), _ptr(ws), ws.numel(), _ptr(dev_err),
                                      _stream(stream)), "sd_accept_sample")
    return n_acc, out_tok, near_boundary
