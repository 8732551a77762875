"""GPU parity of Sparse-to-Dense's own selection score (mean text attention at prefill).

Scores: every candidate's device score against the fp64 oracle's, relative error <= 1e-4.  The
device forms the text rows' scores q . k in fp32 on the tensor core from bf16 inputs (absolute
error ~1e-5 on the scaled logits, so ~1e-5 relative on each weight), sums 128 weights per tile
in fp32 and the tiles in fp64: 1e-4 is ten times that bound.  Index sets: equal, except for
candidates whose oracle scores lie within that same relative tolerance of the selection boundary
(either choice is then correct up to rounding); such swaps are counted and must be few.
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_attention_verify_b200 import device as dev
from speculative_decoding_attention_verify_b200 import inputs as gen
from speculative_decoding_attention_verify_b200 import sdattn as sd

pytestmark = pytest.mark.gpu

REL = {gen.BF16: 1e-4, gen.F32: 1e-5}


def _run(w, k, cand=None):
    lens = w.ctx_len  # the prefill cache: visual span then the text rows
    qt, qs = gen.make_text_queries(w)
    cb = np.zeros(w.n_seq, np.int32) if cand is None else cand[0]
    ce = w.l_vis.astype(np.int32) if cand is None else cand[1]
    max_cand = int((ce - cb).max())
    q = dev.queries(qt, qs, w.dtype, int(lens.max()))
    kv = dev.kv_cache(w, kv_len=lens)
    scores = torch.full((w.n_seq, w.h_kv, max_cand), float("nan"), dtype=torch.float64,
                        device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx = sd.sd_topk_select_scored(sd.SD_TOPK_MEAN_TEXT_ATTENTION, q, kv, dev.int32(cb),
                                   dev.int32(ce), max_cand, k, scores_out=scores,
                                   dev_err=flag).cpu().numpy()
    torch.cuda.synchronize()
    assert flag.item() == 0
    cache = oracle.cache_from_workload(w, kv_len=lens)
    ref_sc = oracle.topk_attention_scores(w.h_q, qt, qs, cache, cb, ce)
    ref_idx, _ = oracle.topk_select_attention(w.h_q, qt, qs, cache, cb, ce, k)
    return idx, scores.cpu().numpy(), ref_idx, ref_sc, cb, ce


def _check(w, k, idx, sc, ref_idx, ref_sc, cb, ce):
    rel = REL[w.dtype]
    swaps = 0
    for b in range(w.n_seq):
        n = int(ce[b] - cb[b])
        for g in range(w.h_kv):
            want, got = ref_sc[b, g, :n], sc[b, g, :n]
            err = np.abs(got - want) / np.maximum(np.abs(want), 1e-300)
            assert err.max() <= rel, (b, g, float(err.max()))
            if np.array_equal(idx[b, g], ref_idx[b, g]):
                continue
            # boundary score of the oracle's selection, then every differing index must sit
            # within the tolerance of it
            kk = min(k, n)
            s_k = np.sort(want)[::-1][kk - 1]
            a = set(idx[b, g][idx[b, g] >= 0].tolist())
            o = set(ref_idx[b, g][ref_idx[b, g] >= 0].tolist())
            assert len(a) == len(o)
            for j in a ^ o:
                sj = want[j - cb[b]]
                assert abs(sj - s_k) <= 2 * rel * s_k, (b, g, j, sj, s_k)
            swaps += len(a - o)
    return swaps


CASES = [
    (1, dict(l_vis=2000, l_txt=128), 256, None),                      # one 7B-like layer
    (1, dict(l_vis=3000, l_txt=300), 1024, None),                     # ragged last row tile
    (3, dict(layers=2, l_vis=2500, l_txt=200), 512, None),            # two layers in one call
    (4, dict(l_vis=700, l_txt=150, batch=3), 300, None),              # paged, ragged lengths
    (0, dict(dtype="bf16", l_vis=1500, l_txt=70), 200, None),         # head_dim 64
    (0, {}, 32, None),                                                # fp32: CUDA cores
    (1, dict(l_vis=2000, l_txt=128), 2000, None),                     # K = every candidate
]


@pytest.mark.parametrize("cfg,kw,k,cand", CASES)
def test_text_attention_scores_and_selection_match_oracle(cfg, kw, k, cand):
    w = gen.make_attn_workload(cfg, **kw)
    idx, sc, ref_idx, ref_sc, cb, ce = _run(w, k, cand)
    swaps = _check(w, k, idx, sc, ref_idx, ref_sc, cb, ce)
    assert swaps <= max(2, w.n_seq * w.h_kv // 2), swaps


@pytest.mark.parametrize("paged", [False, True])
def test_text_attention_candidate_range_off_a_tile_boundary(paged):
    """Candidates [37, l_vis - 5): key tiles start at the range (its page boundary when
    paged), and the text rows' own positions are never candidates."""
    w = gen.make_attn_workload(4 if paged else 1, l_vis=1200, l_txt=100,
                               **({"batch": 2} if paged else {}))
    cb = np.full(w.n_seq, 37, np.int32)
    ce = (w.l_vis - 5).astype(np.int32)
    idx, sc, ref_idx, ref_sc, cb, ce = _run(w, 100, (cb, ce))
    _check(w, 100, idx, sc, ref_idx, ref_sc, cb, ce)


def test_text_attention_candidates_inside_the_text_span():
    """Candidates that text rows see only from their own position on (the causal mask inside
    the column sums)."""
    w = gen.make_attn_workload(1, l_vis=800, l_txt=260)
    cb = np.array([700], np.int32)
    ce = w.ctx_len.astype(np.int32)
    idx, sc, ref_idx, ref_sc, cb, ce = _run(w, 64, (cb, ce))
    _check(w, 64, idx, sc, ref_idx, ref_sc, cb, ce)


def test_text_attention_full_prefill_of_one_long_video_layer():
    """One layer of the long-video case: 25,000 visual keys scored by all 1,024 text rows."""
    w = gen.make_attn_workload(3, layers=1)
    idx, sc, ref_idx, ref_sc, cb, ce = _run(w, w.topk)
    swaps = _check(w, w.topk, idx, sc, ref_idx, ref_sc, cb, ce)
    assert swaps <= 4


def test_last_query_mode_equals_sd_topk_select():
    w = gen.make_attn_workload(1, l_vis=3000, l_txt=100)
    q, kv = dev.verify_queries(w), dev.kv_cache(w)
    cb, ce = dev.int32([0]), dev.int32(w.l_vis)
    a = sd.sd_topk_select(q, kv, cb, ce, int(w.l_vis[0]), 512)
    sc = torch.empty((1, w.h_kv, int(w.l_vis[0])), dtype=torch.float64, device="cuda")
    b = sd.sd_topk_select_scored(sd.SD_TOPK_LAST_QUERY, q, kv, cb, ce, int(w.l_vis[0]), 512,
                                 scores_out=sc)
    assert torch.equal(a, b)
    ref = oracle.topk_scores(w.h_q, w.q_verify, w.q_verify_start, oracle.cache_from_workload(w),
                             [0], w.l_vis)
    np.testing.assert_allclose(sc.cpu().numpy(), ref, rtol=1e-12, atol=1e-9)
