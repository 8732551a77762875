"""Pins for the oracle's top-K selection and hidden-state-reuse projection."""
import itertools
import json
import os

import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_attention_verify_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_golden_topk_tiny():
    fx = json.load(open(os.path.join(GOLDEN, "topk_tiny.json")))
    q = np.asarray(fx["q"], dtype=np.float32)
    k = np.asarray(fx["k"], dtype=np.float32)[None, None]
    cache = oracle.Cache("f32", k, np.zeros_like(k), [6], 1, 2)
    for case in fx["cases"]:
        idx, _ = oracle.topk_select(1, q, [0, 1], cache, [case["cand"][0]], [case["cand"][1]],
                                    case["k"])
        assert idx[0, 0].tolist() == case["expected"], case


def _integer_problem(seed, n, h_q=2, h_kv=1, d=4, lo=-3, hi=4):
    """Small integer-valued q and k, so every score and every subset sum is exact."""
    rng = np.random.default_rng(seed)
    k = rng.integers(lo, hi, size=(1, h_kv, n, d)).astype(np.float32)
    q = rng.integers(lo, hi, size=(1, h_q, d)).astype(np.float32)
    cache = oracle.Cache("f32", k, np.zeros_like(k), [n], h_kv, d)
    return q, k, cache


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("K", [1, 3, 5])
def test_topk_brute_force_over_all_subsets(seed, K):
    n = 11
    q, k, cache = _integer_problem(seed, n)
    idx, _ = oracle.topk_select(2, q, [0, 1], cache, [0], [n], K)
    s = (q[0].sum(axis=0) @ k[0, 0].T).astype(np.int64)  # exact integer scores
    best_sum = max(sum(s[list(c)]) for c in itertools.combinations(range(n), K))
    maximisers = [c for c in itertools.combinations(range(n), K) if sum(s[list(c)]) == best_sum]
    # The tie rule (equal scores go to the lower position) picks the lexicographically
    # smallest of the maximising subsets.
    assert tuple(idx[0, 0].tolist()) == min(maximisers)


def test_topk_duplicated_keys_tie_to_lower_positions():
    rng = np.random.default_rng(3)
    d, n = 8, 40
    k = rng.standard_normal((1, 1, n, d)).astype(np.float32)
    q = rng.standard_normal((1, 1, d)).astype(np.float32)
    salient = (4.0 * q[0, 0]).astype(np.float32)
    dup_pos = [5, 11, 17, 23, 29]
    k[0, 0, dup_pos] = salient
    cache = oracle.Cache("f32", k, np.zeros_like(k), [n], 1, d)
    idx, gap = oracle.topk_select(1, q, [0, 1], cache, [0], [n], 3)
    assert idx[0, 0].tolist() == [5, 11, 17]
    assert gap[0, 0] == 0.0  # the boundary falls between equal scores


def test_topk_scores_match_torch_fp64():
    w = gen.make_attn_workload(1, l_vis=300, l_txt=40, seed=5)
    cache = oracle.cache_from_workload(w)
    cb = np.zeros(1, np.int32)
    ce = w.l_vis.astype(np.int32)
    sc = oracle.topk_scores(w.h_q, w.q_verify, w.q_verify_start, cache, cb, ce)
    qf = torch.tensor(gen.as_f32(w.q_verify[-1], w.dtype), dtype=torch.float64)
    kf = torch.tensor(gen.as_f32(w.k[0], w.dtype), dtype=torch.float64)
    G = w.group
    for g in range(w.h_kv):
        ref = (qf[g * G:(g + 1) * G].sum(0) @ kf[g, :300].T).numpy()
        np.testing.assert_allclose(sc[0, g, :300], ref, rtol=1e-12, atol=1e-10)


def test_topk_selection_agrees_with_lexsort_of_scores():
    w = gen.make_attn_workload(1, l_vis=500, l_txt=40, seed=6)
    cache = oracle.cache_from_workload(w)
    cb, ce = np.array([20], np.int32), np.array([480], np.int32)
    sc = oracle.topk_scores(w.h_q, w.q_verify, w.q_verify_start, cache, cb, ce)
    idx, gap = oracle.topk_select(w.h_q, w.q_verify, w.q_verify_start, cache, cb, ce, 37)
    for g in range(w.h_kv):
        s = sc[0, g, :460]
        pos = np.arange(20, 480)
        order = np.lexsort((pos, -s))  # score descending, then position ascending
        assert idx[0, g].tolist() == sorted(pos[order[:37]].tolist())
        assert gap[0, g] >= 0.0


def test_topk_all_candidates_when_k_exceeds_count():
    q, k, cache = _integer_problem(7, 9)
    idx, gap = oracle.topk_select(2, q, [0, 1], cache, [2], [7], 8)
    assert idx[0, 0].tolist() == [2, 3, 4, 5, 6, -1, -1, -1]
    assert np.isinf(gap[0, 0])


def test_topk_salient_keys_are_selected_first():
    w = gen.make_attn_workload(1, l_vis=2000, l_txt=64, seed=8)
    cache = oracle.cache_from_workload(w)
    n_sal = len(w.salient[0][0])
    idx, _ = oracle.topk_select(w.h_q, w.q_verify, w.q_verify_start, cache, [0],
                                w.l_vis, n_sal)
    for g in range(w.h_kv):
        assert idx[0, g].tolist() == w.salient[0][g].tolist()


# ---------------------------------------------------------------- HSR ----------------------


def test_hsr_matches_torch_fp64_matmul():
    hw = gen.make_hsr_workload(n=3, d_model=64, seed=1, with_bias=True)
    y = oracle.hsr_project(hw.emb, hw.hid, hw.weight, hw.bias)
    x = np.concatenate([gen.f32_from_bf16_bits(hw.emb), gen.f32_from_bf16_bits(hw.hid)], axis=1)
    W = gen.f32_from_bf16_bits(hw.weight)
    b = gen.f32_from_bf16_bits(hw.bias)
    ref = torch.tensor(x, dtype=torch.float64) @ torch.tensor(W, dtype=torch.float64).T
    ref = ref + torch.tensor(b, dtype=torch.float64)
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_hsr_concatenation_order():
    """With h = 0 only the first D input columns act; with e = 0 only the last D."""
    hw = gen.make_hsr_workload(n=2, d_model=32, seed=2)
    W = gen.f32_from_bf16_bits(hw.weight).astype(np.float64)
    zero = np.zeros_like(hw.emb)
    e = gen.f32_from_bf16_bits(hw.emb).astype(np.float64)
    h = gen.f32_from_bf16_bits(hw.hid).astype(np.float64)
    np.testing.assert_allclose(oracle.hsr_project(hw.emb, zero, hw.weight), e @ W[:, :32].T,
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.hsr_project(zero, hw.hid, hw.weight), h @ W[:, 32:].T,
                               rtol=1e-12, atol=1e-12)


def test_hsr_full_size_matches_numpy():
    hw = gen.make_hsr_workload(n=1)
    y = oracle.hsr_project(hw.emb, hw.hid, hw.weight)
    x = np.concatenate([gen.f32_from_bf16_bits(hw.emb), gen.f32_from_bf16_bits(hw.hid)], axis=1)
    ref = x.astype(np.float64) @ gen.f32_from_bf16_bits(hw.weight).astype(np.float64).T
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-10)
    assert 0.5 < y.std() < 2.0  # W ~ N(0, 1/7168) keeps y ~ N(0, 1)
