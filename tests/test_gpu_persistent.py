"""GPU parity of the persistent tensor-core decomposition (one CTA per SM over an even share of
every (sequence, KV head) unit's tiles) against the fp64 oracle, through the C-ABI.

The planner takes it for long streams over many units; each case first asks the library's own
plan (sd_attention_plan) and checks that it is the persistent one, so that the case tests what
it is meant to.  The shapes make CTAs start and end inside units, split units between two or
three CTAs (partials merged by the merge kernel) and run several units back to back: paged
caches with ragged row counts, one-row decode, a text-anchored window that reaches below the
visual span (two position runs) and a sparse selection of 4,096 entries (the compacted run,
then the tail).  Tolerance: max-abs 2e-2 (bf16), as every attention test.
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_attention_verify_b200 import device as dev
from speculative_decoding_attention_verify_b200 import inputs as gen
from speculative_decoding_attention_verify_b200 import sdattn as sd

pytestmark = pytest.mark.gpu

TOL = 2e-2
SAMPLED = (0, 9, 27)


def _persistent(kind, q, kv, extent=0, max_tail=0):
    eng, parts = sd.sd_attention_plan(kind, q, kv, extent, max_tail)
    assert eng == sd.SD_ENGINE_TC_PERSISTENT, (eng, parts)
    return parts


def _layer_cache(w, layer, lens):
    return oracle.Cache(w.dtype, w.k[layer:layer + 1], w.v[layer:layer + 1],
                        lens[layer:layer + 1], w.h_kv, w.d)


def _check(got, ref, where):
    assert np.isfinite(got).all(), where
    err = float(np.abs(got - ref).max())
    assert err <= TOL, (where, err)


def test_persistent_verify_paged_ragged_rows():
    """28 paged sequences of 7,300 positions with 4, 6 or 8 rows each (NaN page tails): every
    sequence checked."""
    w = gen.make_attn_workload(4, batch=28, l_vis=7000, l_txt=300)
    q, kv = dev.verify_queries(w), dev.kv_cache(w)
    _persistent(sd.SD_ATTN_VERIFY, q, kv)
    out = sd.sd_verify_attention(q, kv)
    ref = oracle.verify_attention(w.h_q, w.q_verify, w.q_verify_start,
                                  oracle.cache_from_workload(w))
    _check(dev.to_numpy_f64(out), ref, "paged verify")


@pytest.fixture(scope="module")
def c2_long():
    """28 layers x (6,000 visual + 3,000 text) positions, 8 verify rows per layer."""
    w = gen.make_attn_workload(2, l_vis=6000, l_txt=3000)
    k, v = dev.tensor(w.k, w.dtype), dev.tensor(w.v, w.dtype)
    return w, k, v


def test_persistent_verify_and_decode_sampled_layers(c2_long):
    w, k, v = c2_long
    nq = int(w.n_q_verify[0])
    q, kv = dev.verify_queries(w), dev.kv_cache(w, k=k, v=v)
    _persistent(sd.SD_ATTN_VERIFY, q, kv)
    got = dev.to_numpy_f64(sd.sd_verify_attention(q, kv))
    lens = w.kv_len_draft(0)
    qd, kvd = dev.draft_queries(w, 0), dev.kv_cache(w, kv_len=lens, k=k, v=v)
    _persistent(sd.SD_ATTN_VERIFY, qd, kvd)
    dec = dev.to_numpy_f64(sd.sd_verify_attention(qd, kvd))
    for layer in SAMPLED:
        rows = slice(layer * nq, (layer + 1) * nq)
        ref = oracle.verify_attention(w.h_q, w.q_verify[rows], [0, nq],
                                      _layer_cache(w, layer, w.kv_len_verify))
        _check(got[rows], ref, ("verify", layer))
        ref = oracle.verify_attention(w.h_q, w.q_draft[0][layer:layer + 1], [0, 1],
                                      _layer_cache(w, layer, lens))
        _check(dec[layer:layer + 1], ref, ("decode", layer))


def test_persistent_text_anchored_window_below_the_span(c2_long):
    """Window 8,000 over 3,001 text positions: the window reaches 5,000 positions below the
    visual span, so every unit's stream is two runs."""
    w, k, v = c2_long
    L = w.n_seq
    lens = w.kv_len_draft(0)
    q, kv = dev.draft_queries(w, 0), dev.kv_cache(w, kv_len=lens, k=k, v=v)
    vb, ve = np.zeros(L, np.int32), w.l_vis.astype(np.int32)
    win = np.full(L, 8000, np.int32)
    _persistent(sd.SD_ATTN_TEXT_ANCHORED, q, kv, extent=8000)
    out = sd.sd_text_anchored_attention(q, kv, dev.int32(vb), dev.int32(ve), dev.int32(win), 8000)
    got = dev.to_numpy_f64(out)
    for layer in SAMPLED:
        sl = slice(layer, layer + 1)
        ref = oracle.text_anchored_attention(w.h_q, w.q_draft[0][sl], [0, 1],
                                             _layer_cache(w, layer, lens), vb[sl], ve[sl],
                                             win[sl])
        _check(got[sl], ref, ("text-anchored", layer))


def test_persistent_sparse_large_selection():
    """28 layers, 4,096 selected of 12,000 visual positions + the tail, direct and staged."""
    w = gen.make_attn_workload(3, l_vis=12000, l_txt=500)
    L, nq, K = w.n_seq, int(w.n_q_verify[0]), 4096
    k, v = dev.tensor(w.k, w.dtype), dev.tensor(w.v, w.dtype)
    kv_verify = dev.kv_cache(w, k=k, v=v)
    idx = sd.sd_topk_select(dev.verify_queries(w), kv_verify, dev.int32(np.zeros(L)),
                            dev.int32(w.l_vis), int(w.l_vis.max()), K)
    step = 2
    lens = w.kv_len_draft(step)
    tail = w.l_vis.astype(np.int32)
    max_tail = int((lens - tail).max())
    q, kv = dev.draft_queries(w, step), dev.kv_cache(w, kv_len=lens, k=k, v=v)
    _persistent(sd.SD_ATTN_SPARSE, q, kv, extent=K, max_tail=max_tail)
    direct = dev.to_numpy_f64(sd.sd_sparse_attention(q, kv, idx, dev.int32(tail), max_tail))
    sel = sd.sd_sparse_stage(kv, idx, dev.int32(tail))
    staged = dev.to_numpy_f64(sd.sd_sparse_attention_staged(q, kv, sel, K, dev.int32(tail),
                                                            max_tail))
    idx_h = idx.cpu().numpy()
    for layer in SAMPLED:
        ridx, gap = oracle.topk_select(w.h_q, w.q_verify[layer * nq:(layer + 1) * nq], [0, nq],
                                       _layer_cache(w, layer, w.kv_len_verify), [0],
                                       w.l_vis[layer:layer + 1], K)
        assert np.array_equal(idx_h[layer:layer + 1], ridx), (layer, gap)
        ref = oracle.sparse_attention(w.h_q, w.q_draft[step][layer:layer + 1], [0, 1],
                                      _layer_cache(w, layer, lens), ridx, tail[layer:layer + 1])
        _check(direct[layer:layer + 1], ref, ("sparse", layer))
        _check(staged[layer:layer + 1], ref, ("staged", layer))


def test_persistent_expired_waits_set_the_flag_and_the_device_recovers(c2_long):
    """With a 1 ns wait bound the persistent kernel's waits run out at once: SD_DEVERR_TIMEOUT,
    no CUDA error, and the next call with the default bound is correct.  (No wait here is
    endless: the bound is just shorter than the copies it waits for.)"""
    w, k, v = c2_long
    q, kv = dev.verify_queries(w), dev.kv_cache(w, k=k, v=v)
    _persistent(sd.SD_ATTN_VERIFY, q, kv)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    prev = sd.sd_set_wait_timeout_ns(1)
    try:
        sd.sd_verify_attention(q, kv, dev_err=flag)
        torch.cuda.synchronize()
    finally:
        sd.sd_set_wait_timeout_ns(prev)
    assert flag.item() & sd.SD_DEVERR_TIMEOUT
    flag.zero_()
    got = dev.to_numpy_f64(sd.sd_verify_attention(q, kv, dev_err=flag))
    assert flag.item() == 0
    nq = int(w.n_q_verify[0])
    ref = oracle.verify_attention(w.h_q, w.q_verify[:nq], [0, nq],
                                  _layer_cache(w, 0, w.kv_len_verify))
    _check(got[:nq], ref, "after timeout")
