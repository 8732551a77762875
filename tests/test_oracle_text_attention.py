"""Pins for the oracle's mean-text-attention selection score (Sparse-to-Dense's own rule).

The score of candidate j for KV head g is the mean, over the prefill text rows and the group's
query heads, of the attention weight each row gives j (causal, each row with its own softmax
over every position it sees).  These pins tie it to a hand-derived golden case, to the
independently pinned verify oracle (one-hot values turn attention outputs into attention
weights), to a closed form and to two invariants.
"""
import json
import os

import numpy as np
import pytest

import oracle
from speculative_decoding_attention_verify_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_golden_text_attention_tiny():
    fx = json.load(open(os.path.join(GOLDEN, "topk_text_attention_tiny.json")))
    k = np.asarray(fx["k"], dtype=np.float32)[None, None]
    for grp in fx["groups"]:
        q = np.asarray(grp["q"], dtype=np.float32)
        cache = oracle.Cache("f32", k, np.zeros_like(k), [4], 1, 2)
        sc = oracle.topk_attention_scores(grp["h_q"], q, [0, 2], cache, [0], [4],
                                          scale=fx["scale"])
        np.testing.assert_allclose(sc[0, 0], grp["scores"], rtol=0, atol=1e-12)
        # a candidate range changes which scores are reported, not their values
        sub = oracle.topk_attention_scores(grp["h_q"], q, [0, 2], cache, [2], [4],
                                           scale=fx["scale"])
        np.testing.assert_allclose(sub[0, 0], grp["scores"][2:], rtol=0, atol=1e-12)
        for case in grp["cases"]:
            idx, _ = oracle.topk_select_attention(grp["h_q"], q, [0, 2], cache,
                                                  [case["cand"][0]], [case["cand"][1]],
                                                  case["k"], scale=fx["scale"])
            assert idx[0, 0].tolist() == case["expected"], (grp["h_q"], case)


def _problem(seed, n_seq=2, h_q=4, h_kv=2, d=16, ctx=(40, 33), n_q=(5, 3), dtype="f32"):
    """Random caches whose last n_q positions are the text rows of each sequence."""
    rng = np.random.default_rng(seed)
    cap = max(ctx)
    st = np.float32 if dtype == "f32" else np.uint16
    conv = (lambda x: x.astype(np.float32)) if dtype == "f32" else gen.bf16_bits_from_f32
    k = conv(rng.standard_normal((n_seq, h_kv, cap, d)).astype(np.float32))
    v = conv(rng.standard_normal((n_seq, h_kv, cap, d)).astype(np.float32))
    qs = np.concatenate([[0], np.cumsum(n_q)]).astype(np.int32)
    q = conv(rng.standard_normal((int(qs[-1]), h_q, d)).astype(np.float32) * 2.0)
    cache = oracle.Cache(dtype, k.astype(st), v.astype(st), np.asarray(ctx, np.int32), h_kv, d)
    return q, qs, cache, k, v


@pytest.mark.parametrize("seed", range(4))
def test_scores_over_every_position_sum_to_one(seed):
    """Each text row's weights sum to 1 over the positions it sees, so the mean over rows and
    heads of all positions' scores is 1."""
    q, qs, cache, _, _ = _problem(seed)
    ctx = cache.kv_len
    sc = oracle.topk_attention_scores(4, q, qs, cache, [0, 0], ctx)
    for b in range(2):
        for g in range(2):
            assert abs(np.nansum(sc[b, g, :ctx[b]]) - 1.0) < 1e-12


@pytest.mark.parametrize("seed,G", [(0, 1), (1, 3), (2, 2)])
def test_scores_equal_mean_attention_output_with_one_hot_values(seed, G):
    """With V row j = e_j (kv_len <= head_dim), the verify oracle's output for a text row is
    exactly that row's attention weight vector; its mean over the rows and the group's heads is
    the score."""
    d, h_kv, n = 32, 2, (29, 21)
    h_q = G * h_kv
    rng = np.random.default_rng(100 + seed)
    k = rng.standard_normal((2, h_kv, max(n), d)).astype(np.float32)
    v = np.zeros_like(k)
    for j in range(max(n)):
        v[:, :, j, j] = 1.0
    n_q = (6, 4)
    qs = np.concatenate([[0], np.cumsum(n_q)]).astype(np.int32)
    q = (rng.standard_normal((int(qs[-1]), h_q, d)) * 1.5).astype(np.float32)
    cache = oracle.Cache("f32", k, v, np.asarray(n, np.int32), h_kv, d)
    out = oracle.verify_attention(h_q, q, qs, cache)          # [rows][h_q][d]
    sc = oracle.topk_attention_scores(h_q, q, qs, cache, [0, 0], list(n))
    for b in range(2):
        rows = out[qs[b]:qs[b + 1]]
        for g in range(h_kv):
            want = rows[:, g * G:(g + 1) * G, :n[b]].mean(axis=(0, 1))
            np.testing.assert_allclose(sc[b, g, :n[b]], want, rtol=0, atol=1e-13)


def test_zero_keys_give_uniform_weights_closed_form():
    """All keys zero: row i spreads 1/(limit_i + 1) over positions 0..limit_i, so score_j is the
    mean over the rows that see j of 1/(limit_i + 1)."""
    d, kv_len, n_q = 8, 30, 7
    k = np.zeros((1, 1, kv_len, d), np.float32)
    q = np.random.default_rng(5).standard_normal((n_q, 3, d)).astype(np.float32)
    cache = oracle.Cache("f32", k, np.zeros_like(k), [kv_len], 1, d)
    sc = oracle.topk_attention_scores(3, q, [0, n_q], cache, [0], [kv_len])[0, 0]
    for j in range(kv_len):
        want = sum(1.0 / (kv_len - n_q + i + 1) for i in range(n_q) if j <= kv_len - n_q + i)
        assert abs(sc[j] - want / n_q) < 1e-15


@pytest.mark.parametrize("seed", range(5))
def test_one_text_row_one_head_ranks_like_the_query_key_score(seed):
    """One text row and one query head per KV head: the weight is increasing in q . k, so the
    selection equals the last-query dot-product selection (same ties, same order)."""
    q, qs, cache, _, _ = _problem(seed, h_q=2, h_kv=2, n_q=(1, 1), dtype="bf16")
    ce = np.asarray([28, 30], np.int32)
    a, _ = oracle.topk_select_attention(2, q, qs, cache, [3, 0], ce, 9)
    b, _ = oracle.topk_select(2, q, qs, cache, [3, 0], ce, 9)
    assert np.array_equal(a, b)


def test_candidates_beyond_a_rows_causal_limit_get_only_the_later_rows():
    """A candidate inside the text span is seen only by the rows at or after it."""
    q, qs, cache, _, _ = _problem(7, n_seq=1, ctx=(40,), n_q=(6,))
    full = oracle.topk_attention_scores(4, q, qs, cache, [0], [40])[0]
    part = oracle.topk_attention_scores(4, q, qs, cache, [36], [40])[0]
    np.testing.assert_array_equal(full[:, 36:40], part[:, :4])
    assert (full[:, 34:40] > 0).all()
