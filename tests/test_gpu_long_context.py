"""Contexts of an hour of video: 140,000 visual positions per sequence, within HBM.

Sparse-to-Dense's problem statement puts one hour of video above 140,000 visual tokens.  These
cases run every call of the path at that length (one 7B-like layer, or a paged batch of two
such sequences) and compare with the fp64 oracle at the usual tolerances: attention max-abs
2e-2 (bf16), top-K index sets bit-exact, the mean-text-attention scores within 1e-4 relative.
They exercise the position and offset arithmetic (tile starts, copy coordinates, split plans,
workspace sizes) far beyond the 25k-position workloads.
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_attention_verify_b200 import device as dev
from speculative_decoding_attention_verify_b200 import inputs as gen
from speculative_decoding_attention_verify_b200 import sdattn as sd

pytestmark = pytest.mark.gpu

L_VIS = 140_000
TOL = 2e-2


@pytest.fixture(scope="module")
def long_layer():
    w = gen.make_attn_workload(3, layers=1, l_vis=L_VIS)
    return w, dev.tensor(w.k, w.dtype), dev.tensor(w.v, w.dtype)


def _err(out, ref):
    got = dev.to_numpy_f64(out)
    assert np.isfinite(got).all()
    return float(np.abs(got - ref).max())


def test_verify_at_140k(long_layer):
    w, k, v = long_layer
    out = sd.sd_verify_attention(dev.verify_queries(w), dev.kv_cache(w, k=k, v=v))
    ref = oracle.verify_attention(w.h_q, w.q_verify, w.q_verify_start, oracle.cache_from_workload(w))
    assert _err(out, ref) <= TOL


def test_topk_and_staged_sparse_at_140k(long_layer):
    w, k, v = long_layer
    kv = dev.kv_cache(w, k=k, v=v)
    cb, ce = np.zeros(1, np.int32), w.l_vis.astype(np.int32)
    idx = sd.sd_topk_select(dev.verify_queries(w), kv, dev.int32(cb), dev.int32(ce), L_VIS,
                            w.topk).cpu().numpy()
    ref_idx, gap = oracle.topk_select(w.h_q, w.q_verify, w.q_verify_start,
                                      oracle.cache_from_workload(w), cb, ce, w.topk)
    assert np.array_equal(idx, ref_idx), gap
    tail = w.l_vis.astype(np.int32)
    for step in (0, 7):
        lens = w.kv_len_draft(step)
        kvd = dev.kv_cache(w, kv_len=lens, k=k, v=v)
        sel = sd.sd_sparse_stage(kvd, dev.int32(idx), dev.int32(tail))
        out = sd.sd_sparse_attention_staged(dev.draft_queries(w, step), kvd, sel, w.topk,
                                            dev.int32(tail), int((lens - tail).max()))
        ref = oracle.sparse_attention(w.h_q, w.q_draft[step], [0, 1],
                                      oracle.cache_from_workload(w, kv_len=lens), ref_idx, tail)
        assert _err(out, ref) <= TOL, step


def test_text_anchored_at_140k(long_layer):
    w, k, v = long_layer
    lens = w.kv_len_draft(3)
    vb, ve = np.zeros(1, np.int32), w.l_vis.astype(np.int32)
    out = sd.sd_text_anchored_attention(dev.draft_queries(w, 3), dev.kv_cache(w, kv_len=lens,
                                                                              k=k, v=v),
                                        dev.int32(vb), dev.int32(ve), dev.int32(w.window),
                                        int(w.window[0]))
    ref = oracle.text_anchored_attention(w.h_q, w.q_draft[3], [0, 1],
                                         oracle.cache_from_workload(w, kv_len=lens), vb, ve,
                                         w.window)
    assert _err(out, ref) <= TOL


def test_mean_text_attention_selection_at_140k():
    """64 prefill text rows score 140,000 visual keys."""
    w = gen.make_attn_workload(1, l_vis=L_VIS, l_txt=64)
    qt, qs = gen.make_text_queries(w)
    q = dev.queries(qt, qs, w.dtype, int(w.ctx_len.max()))
    kv = dev.kv_cache(w, kv_len=w.ctx_len)
    sc = torch.empty((1, w.h_kv, L_VIS), dtype=torch.float64, device="cuda")
    sd.sd_topk_select_scored(sd.SD_TOPK_MEAN_TEXT_ATTENTION, q, kv, dev.int32([0]),
                             dev.int32(w.l_vis), L_VIS, 1024, scores_out=sc)
    ref = oracle.topk_attention_scores(w.h_q, qt, qs, oracle.cache_from_workload(w, kv_len=w.ctx_len),
                                       [0], w.l_vis)
    got = sc.cpu().numpy()
    assert (np.abs(got - ref) / ref).max() <= 1e-4


def test_paged_verify_two_sequences_at_140k():
    w = gen.make_attn_workload(4, l_vis=L_VIS, l_txt=700, batch=2)
    out = sd.sd_verify_attention(dev.verify_queries(w), dev.kv_cache(w))
    ref = oracle.verify_attention(w.h_q, w.q_verify, w.q_verify_start, oracle.cache_from_workload(w))
    assert _err(out, ref) <= TOL
