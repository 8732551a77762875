"""Pins for the oracle's attention routines (verify, decode, text-anchored, sparse).

Each test checks the oracle against something other than itself: a hand-derived fixture, a
closed form, an invariant the method fixes, or a library routine on a special case (torch's
fp64 CPU scaled_dot_product_attention with an explicit boolean mask).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_attention_verify_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cache_contig(k, v, kv_len, dtype):
    """k, v: [B][h_kv][L][d] float32 values -> oracle cache in the given storage dtype."""
    ks, vs = gen.to_kv_dtype(k, dtype), gen.to_kv_dtype(v, dtype)
    return oracle.Cache(dtype, ks, vs, kv_len, k.shape[1], k.shape[3]), ks, vs


def _rand_problem(seed, B=2, h_q=6, h_kv=2, d=16, kv_lens=(37, 50), n_qs=(3, 5), dtype="f32"):
    rng = np.random.default_rng(seed)
    L = max(kv_lens)
    k = rng.standard_normal((B, h_kv, L, d)).astype(np.float32)
    v = rng.standard_normal((B, h_kv, L, d)).astype(np.float32)
    q_start = np.concatenate([[0], np.cumsum(n_qs)]).astype(np.int32)
    q = rng.standard_normal((int(q_start[-1]), h_q, d)).astype(np.float32)
    kv_len = np.asarray(kv_lens, dtype=np.int32)
    cache, ks, vs = _cache_contig(k, v, kv_len, dtype)
    qs = gen.to_kv_dtype(q, dtype)
    return dict(cache=cache, k=gen.as_f32(ks, dtype), v=gen.as_f32(vs, dtype), q=qs,
                qf=gen.as_f32(qs, dtype), q_start=q_start, kv_len=kv_len, h_q=h_q, h_kv=h_kv,
                d=d, dtype=dtype)


def _torch_masked_attention(qf, k, v, q_start, kv_len, h_q, allowed, scale=None):
    """Library reference: torch fp64 SDPA with an explicit boolean mask per (b, row).

    ``allowed(b, i, n_q, L, g)`` returns a boolean numpy vector over positions [0, L)."""
    B = len(kv_len)
    h_kv = k.shape[1]
    G = h_q // h_kv
    d = k.shape[-1]
    out = np.zeros((int(q_start[-1]), h_q, d))
    for b in range(B):
        L = int(kv_len[b])
        n_q = int(q_start[b + 1] - q_start[b])
        qb = torch.tensor(qf[q_start[b]:q_start[b + 1]], dtype=torch.float64).permute(1, 0, 2)
        kb = torch.tensor(k[b, :, :L], dtype=torch.float64).repeat_interleave(G, dim=0)
        vb = torch.tensor(v[b, :, :L], dtype=torch.float64).repeat_interleave(G, dim=0)
        mask = np.zeros((h_q, n_q, L), dtype=bool)
        for i in range(n_q):
            for h in range(h_q):
                mask[h, i] = allowed(b, i, n_q, L, h // G)
        o = torch.nn.functional.scaled_dot_product_attention(
            qb[None], kb[None], vb[None], attn_mask=torch.tensor(mask)[None],
            scale=scale)[0]
        out[q_start[b]:q_start[b + 1]] = o.permute(1, 0, 2).numpy()
    return out


def _causal(b, i, n_q, L, g):
    m = np.zeros(L, dtype=bool)
    m[:L - n_q + i + 1] = True
    return m


# ---------------------------------------------------------------- golden fixtures ---------


def test_golden_attention_tiny():
    fx = json.load(open(os.path.join(GOLDEN, "attention_tiny.json")))
    q = np.asarray(fx["q"], dtype=np.float32)
    k = np.asarray(fx["k"], dtype=np.float32)[None, None]
    v = np.asarray(fx["v"], dtype=np.float32)[None, None]
    cache = oracle.Cache("f32", k, v, [3], 1, fx["head_dim"])
    out = oracle.verify_attention(1, q, [0, 3], cache, scale=fx["softmax_scale"])
    np.testing.assert_allclose(out, np.asarray(fx["expected"]), rtol=0, atol=fx["tolerance"])


def test_golden_text_anchored_tiny():
    fx = json.load(open(os.path.join(GOLDEN, "text_anchored_tiny.json")))
    q = np.asarray(fx["q"], dtype=np.float32)
    k = np.asarray(fx["k"], dtype=np.float32)[None, None]
    v = np.asarray(fx["v"], dtype=np.float32)[None, None]
    cache = oracle.Cache("f32", k, v, [6], 1, 2)
    for case in fx["cases"]:
        out = oracle.text_anchored_attention(1, q, [0, 1], cache, [fx["vis_begin"]],
                                             [fx["vis_end"]], [case["window"]],
                                             scale=fx["softmax_scale"])
        np.testing.assert_allclose(out[0, 0], case["expected"], rtol=0, atol=fx["tolerance"])


# ---------------------------------------------------------------- verify -------------------


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_verify_matches_torch_sdpa(dtype):
    p = _rand_problem(1, dtype=dtype)
    got = oracle.verify_attention(p["h_q"], p["q"], p["q_start"], p["cache"])
    ref = _torch_masked_attention(p["qf"], p["k"], p["v"], p["q_start"], p["kv_len"], p["h_q"],
                                  _causal)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_verify_explicit_scale_matches_torch():
    p = _rand_problem(2)
    got = oracle.verify_attention(p["h_q"], p["q"], p["q_start"], p["cache"], scale=0.37)
    ref = _torch_masked_attention(p["qf"], p["k"], p["v"], p["q_start"], p["kv_len"], p["h_q"],
                                  _causal, scale=0.37)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_verify_gamma0_equals_single_token_decode():
    p = _rand_problem(3, n_qs=(1, 1))
    got = oracle.verify_attention(p["h_q"], p["q"], p["q_start"], p["cache"])
    dec = oracle.decode_attention(p["h_q"], p["q"], p["cache"])
    np.testing.assert_allclose(got, dec, rtol=1e-13, atol=1e-14)


def test_verify_single_position_returns_v0():
    rng = np.random.default_rng(4)
    k = rng.standard_normal((1, 1, 1, 8)).astype(np.float32)
    v = rng.standard_normal((1, 1, 1, 8)).astype(np.float32)
    cache = oracle.Cache("f32", k, v, [1], 1, 8)
    q = rng.standard_normal((1, 3, 8)).astype(np.float32)
    out = oracle.verify_attention(3, q, [0, 1], cache)
    for h in range(3):
        np.testing.assert_array_equal(out[0, h], v[0, 0, 0].astype(np.float64))


def test_verify_constant_values_give_the_constant():
    p = _rand_problem(5)
    c = np.linspace(-2, 2, p["d"]).astype(np.float32)
    v = np.broadcast_to(c, p["cache"].v.shape).copy()
    cache = oracle.Cache("f32", p["cache"].k, v, p["kv_len"], p["h_kv"], p["d"])
    out = oracle.verify_attention(p["h_q"], p["q"], p["q_start"], cache)
    np.testing.assert_allclose(out, np.broadcast_to(c.astype(np.float64), out.shape),
                               rtol=0, atol=1e-14)


def test_verify_zero_keys_give_running_mean():
    p = _rand_problem(6)
    k0 = np.zeros_like(p["cache"].k)
    cache = oracle.Cache("f32", k0, p["cache"].v, p["kv_len"], p["h_kv"], p["d"])
    out = oracle.verify_attention(p["h_q"], p["q"], p["q_start"], cache)
    G = p["h_q"] // p["h_kv"]
    for b in range(2):
        n_q = p["q_start"][b + 1] - p["q_start"][b]
        for i in range(n_q):
            lim = p["kv_len"][b] - n_q + i
            for h in range(p["h_q"]):
                want = p["v"][b, h // G, :lim + 1].astype(np.float64).mean(axis=0)
                np.testing.assert_allclose(out[p["q_start"][b] + i, h], want, rtol=1e-12,
                                           atol=1e-13)


def test_verify_causality_ignores_later_positions():
    p = _rand_problem(7)
    base = oracle.verify_attention(p["h_q"], p["q"], p["q_start"], p["cache"])
    k2, v2 = p["cache"].k.copy(), p["cache"].v.copy()
    b, n_q = 1, 5
    lim0 = p["kv_len"][b] - n_q  # row 0's last visible position
    k2[b, :, lim0 + 1:] = 1e3
    v2[b, :, lim0 + 1:] = -7.0
    cache = oracle.Cache("f32", k2, v2, p["kv_len"], p["h_kv"], p["d"])
    out = oracle.verify_attention(p["h_q"], p["q"], p["q_start"], cache)
    np.testing.assert_array_equal(out[p["q_start"][b]], base[p["q_start"][b]])
    assert not np.allclose(out[p["q_start"][b] + 1], base[p["q_start"][b] + 1])


def test_paged_layout_equals_contiguous():
    w = gen.make_attn_workload(4, l_vis=100, l_txt=20, batch=3, seed=11)
    assert w.paged
    cache_p = oracle.cache_from_workload(w)
    # The same logical rows laid out contiguously.
    L = int(w.kv_len_verify.max())
    kc = np.zeros((w.n_seq, w.h_kv, L, w.d), dtype=w.k.dtype)
    vc = np.zeros_like(kc)
    for s in range(w.n_seq):
        for j in range(int(w.kv_len_verify[s])):
            for g in range(w.h_kv):
                kc[s, g, j] = w.kv_row("k", s, g, j)
                vc[s, g, j] = w.kv_row("v", s, g, j)
    cache_c = oracle.Cache(w.dtype, kc, vc, w.kv_len_verify, w.h_kv, w.d)
    a = oracle.verify_attention(w.h_q, w.q_verify, w.q_verify_start, cache_p)
    b = oracle.verify_attention(w.h_q, w.q_verify, w.q_verify_start, cache_c)
    np.testing.assert_array_equal(a, b)
    assert np.isfinite(a).all()


def test_context_permutation_invariance():
    p = _rand_problem(8, B=1, kv_lens=(40,), n_qs=(4,))
    ctx = 40 - 4
    perm = np.random.default_rng(9).permutation(ctx)
    k2, v2 = p["cache"].k.copy(), p["cache"].v.copy()
    k2[:, :, :ctx] = k2[:, :, perm]
    v2[:, :, :ctx] = v2[:, :, perm]
    cache = oracle.Cache("f32", k2, v2, p["kv_len"], p["h_kv"], p["d"])
    a = oracle.verify_attention(p["h_q"], p["q"], p["q_start"], p["cache"])
    b = oracle.verify_attention(p["h_q"], p["q"], p["q_start"], cache)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_verify_c0_workload_matches_torch():
    w = gen.make_attn_workload(0)
    cache = oracle.cache_from_workload(w)
    got = oracle.verify_attention(w.h_q, w.q_verify, w.q_verify_start, cache)
    ref = _torch_masked_attention(w.q_verify, w.k, w.v, w.q_verify_start, w.kv_len_verify, w.h_q,
                                  _causal)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- text-anchored ------------


def test_text_anchored_wide_window_equals_dense_without_visual_span():
    p = _rand_problem(10, kv_lens=(45, 60), n_qs=(3, 4))
    vb, ve = np.array([5, 0], np.int32), np.array([25, 40], np.int32)
    window = np.array([1000, 1000], np.int32)
    got = oracle.text_anchored_attention(p["h_q"], p["q"], p["q_start"], p["cache"], vb, ve,
                                         window)
    # Physically delete the visual span and run plain verification on what remains.
    ks, vs, lens = [], [], []
    for b in range(2):
        keep = np.r_[0:vb[b], ve[b]:p["kv_len"][b]]
        ks.append(p["cache"].k[b][:, keep])
        vs.append(p["cache"].v[b][:, keep])
        lens.append(len(keep))
    L = max(lens)
    kk = np.zeros((2, p["h_kv"], L, p["d"]), np.float32)
    vv = np.zeros_like(kk)
    for b in range(2):
        kk[b, :, :lens[b]] = ks[b]
        vv[b, :, :lens[b]] = vs[b]
    cache = oracle.Cache("f32", kk, vv, lens, p["h_kv"], p["d"])
    ref = oracle.verify_attention(p["h_q"], p["q"], p["q_start"], cache)
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-14)


def test_text_anchored_window_one_returns_own_value():
    p = _rand_problem(12)
    z = np.zeros(2, np.int32)
    got = oracle.text_anchored_attention(p["h_q"], p["q"], p["q_start"], p["cache"],
                                         np.array([0, 0], np.int32), np.array([10, 10], np.int32),
                                         np.array([1, 1], np.int32))
    G = p["h_q"] // p["h_kv"]
    for b in range(2):
        n_q = p["q_start"][b + 1] - p["q_start"][b]
        for i in range(n_q):
            j = p["kv_len"][b] - n_q + i
            for h in range(p["h_q"]):
                np.testing.assert_array_equal(got[p["q_start"][b] + i, h],
                                              p["v"][b, h // G, j].astype(np.float64))
    assert z.sum() == 0


def test_text_anchored_empty_visual_span_is_sliding_window():
    p = _rand_problem(13)
    W = 9

    def band(b, i, n_q, L, g):
        lim = L - n_q + i
        m = np.zeros(L, dtype=bool)
        m[max(0, lim - W + 1):lim + 1] = True
        return m

    got = oracle.text_anchored_attention(p["h_q"], p["q"], p["q_start"], p["cache"],
                                         np.zeros(2, np.int32), np.zeros(2, np.int32),
                                         np.full(2, W, np.int32))
    ref = _torch_masked_attention(p["qf"], p["k"], p["v"], p["q_start"], p["kv_len"], p["h_q"],
                                  band)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("W", [3, 12, 20, 31])
def test_text_anchored_window_crossing_the_visual_span(W):
    p = _rand_problem(14, kv_lens=(48, 52), n_qs=(2, 4), dtype="bf16")
    vb, ve = np.array([10, 20], np.int32), np.array([30, 40], np.int32)

    def allowed(b, i, n_q, L, g):
        # Count non-visual positions from the row's own position downwards; keep the first W.
        lim = L - n_q + i
        nonvis = np.array([(j <= lim) and not (vb[b] <= j < ve[b]) for j in range(L)])
        from_right = np.cumsum(nonvis[::-1])[::-1]  # non-visual positions in [j, L)
        return nonvis & (from_right <= W)

    got = oracle.text_anchored_attention(p["h_q"], p["q"], p["q_start"], p["cache"], vb, ve,
                                         np.full(2, W, np.int32))
    ref = _torch_masked_attention(p["qf"], p["k"], p["v"], p["q_start"], p["kv_len"], p["h_q"],
                                  allowed)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- sparse -------------------


def test_sparse_with_all_candidates_equals_dense():
    p = _rand_problem(15, kv_lens=(30, 41), n_qs=(1, 1))
    ctx = p["kv_len"] - 1
    kmax = int(ctx.max())
    idx = np.full((2, p["h_kv"], kmax), -1, np.int32)
    for b in range(2):
        idx[b, :, :ctx[b]] = np.arange(ctx[b])
    got = oracle.sparse_attention(p["h_q"], p["q"], p["q_start"], p["cache"], idx, ctx)
    ref = oracle.verify_attention(p["h_q"], p["q"], p["q_start"], p["cache"])
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-14)


def test_sparse_with_no_selection_and_full_tail_equals_dense():
    p = _rand_problem(16)
    idx = np.full((2, p["h_kv"], 4), -1, np.int32)
    got = oracle.sparse_attention(p["h_q"], p["q"], p["q_start"], p["cache"], idx,
                                  np.zeros(2, np.int32))
    ref = oracle.verify_attention(p["h_q"], p["q"], p["q_start"], p["cache"])
    np.testing.assert_array_equal(got, ref)


def test_sparse_matches_torch_with_explicit_set_mask():
    p = _rand_problem(17, kv_lens=(60, 64), n_qs=(1, 3), dtype="bf16")
    rng = np.random.default_rng(18)
    tail = np.array([40, 44], np.int32)
    K = 7
    idx = np.full((2, p["h_kv"], K), -1, np.int32)
    for b in range(2):
        for g in range(p["h_kv"]):
            idx[b, g] = np.sort(rng.choice(tail[b], size=K, replace=False))

    def allowed(b, i, n_q, L, g):
        lim = L - n_q + i
        m = np.zeros(L, dtype=bool)
        m[idx[b, g]] = True
        m[tail[b]:] = True
        m[lim + 1:] = False
        return m

    got = oracle.sparse_attention(p["h_q"], p["q"], p["q_start"], p["cache"], idx, tail)
    ref = _torch_masked_attention(p["qf"], p["k"], p["v"], p["q_start"], p["kv_len"], p["h_q"],
                                  allowed)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_sparse_set_semantics_for_duplicates_and_tail_overlap():
    p = _rand_problem(19)
    tail = np.array([30, 40], np.int32)
    idx = np.array([[[3, 5, 9, -1, -1]] * 2, [[1, 2, 8, -1, -1]] * 2], np.int32)
    dup = np.array([[[3, 3, 5, 9, 31]] * 2, [[1, 2, 2, 8, 45]] * 2], np.int32)
    a = oracle.sparse_attention(p["h_q"], p["q"], p["q_start"], p["cache"], idx, tail)
    b = oracle.sparse_attention(p["h_q"], p["q"], p["q_start"], p["cache"], dup, tail)
    np.testing.assert_array_equal(a, b)
