"""Pins for the oracle's greedy and speculative-sampling acceptance."""
import json
import os

import numpy as np
import pytest

import oracle
from speculative_decoding_attention_verify_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _softmax64(z):
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(z - z.max())
    return e / e.sum()


# ---------------------------------------------------------------- greedy -------------------


def test_golden_accept_greedy_tiny():
    fx = json.load(open(os.path.join(GOLDEN, "accept_greedy_tiny.json")))
    tgt = np.array([[float(x) for x in row] for row in fx["target"]], dtype=np.float32)
    for case in fx["cases"]:
        n, out = oracle.accept_greedy(tgt, case["drafts"], [3], fx["vocab"])
        assert n[0] == case["n_acc"]
        assert out[0, :n[0] + 1].tolist() == case["tokens"]


def test_greedy_own_argmax_accepts_everything():
    aw = gen.make_accept_workload(2, vocab=5000, batch=3, gammas=[7, 2, 5])
    rows = np.split(aw.target_logits, np.cumsum(aw.gamma + 1)[:-1])
    drafts = np.concatenate([np.argmax(r[:-1], axis=1) for r in rows]).astype(np.int32)
    n, out = oracle.accept_greedy(aw.target_logits, drafts, aw.gamma, aw.vocab)
    assert n.tolist() == aw.gamma.tolist()
    for b, r in enumerate(rows):
        assert out[b, :n[b] + 1].tolist() == np.argmax(r, axis=1).tolist()


def test_greedy_first_mismatch_accepts_nothing():
    aw = gen.make_accept_workload(0, batch=2, gammas=[4, 4])
    rows = np.split(aw.target_logits, 2)
    drafts = np.concatenate([np.argmax(r[:-1], axis=1) for r in rows]).astype(np.int32)
    drafts[0] = (drafts[0] + 1) % aw.vocab
    drafts[4 + 2] = (drafts[4 + 2] + 1) % aw.vocab
    n, out = oracle.accept_greedy(aw.target_logits, drafts, aw.gamma, aw.vocab)
    assert n.tolist() == [0, 2]
    assert out[0, 0] == np.argmax(rows[0][0])
    assert out[1, 2] == np.argmax(rows[1][2])


def test_greedy_argmax_ties_nan_and_signed_zero():
    V = 6
    tgt = np.array([[1.0, 3.0, 3.0, 0.0, 3.0, -1.0],          # tie -> 1
                    [np.nan, -np.inf, -5.0, np.nan, -5.0, -6.0],  # NaN lowest, tie -> 2
                    [-0.0, 0.0, -1.0, -0.0, -2.0, -3.0],      # -0 == +0 -> 0
                    [np.nan] * 6], dtype=np.float32)           # all NaN -> 0
    n, out = oracle.accept_greedy(tgt, [1, 2, 0], [3], V)
    assert n[0] == 3 and out[0].tolist() == [1, 2, 0, 0]


# ---------------------------------------------------------------- sampling -----------------


def test_golden_accept_sample_tiny():
    fx = json.load(open(os.path.join(GOLDEN, "accept_sample_tiny.json")))
    tgt = np.asarray(fx["target"], dtype=np.float32)
    drf = np.asarray(fx["draft"], dtype=np.float32)
    for case in fx["cases"]:
        n, out, am, dm = oracle.accept_sample(tgt, drf, case["d"], case["u"], case["v"], [1],
                                              fx["vocab"])
        assert n[0] == case["n_acc"], case
        assert out[0, :n[0] + 1].tolist() == case["tokens"], case


def _enumerate(tgt, drf, gamma, M):
    """Every (drafted tokens, u grid, v grid) combination as one batch of sequences.

    Returns the oracle's outputs and each combination's probability weight.  u and v run over
    the M-point midpoint grid of (0, 1); one v value serves whichever row draws."""
    V = tgt.shape[1]
    grid = ((np.arange(M) + 0.5) / M).astype(np.float32)
    qs = [_softmax64(r) for r in drf]
    d_combos = np.array(np.meshgrid(*[np.arange(V)] * gamma, indexing="ij")).reshape(gamma, -1).T
    u_combos = np.array(np.meshgrid(*[np.arange(M)] * gamma, indexing="ij")).reshape(gamma, -1).T
    n_d, n_u = len(d_combos), len(u_combos)
    B = n_d * n_u * M
    di = np.repeat(d_combos, n_u * M, axis=0)
    ui = np.tile(np.repeat(u_combos, M, axis=0), (n_d, 1))
    vi = np.tile(np.arange(M), n_d * n_u)
    weight = np.ones(B)
    for t in range(gamma):
        weight *= qs[t][di[:, t]]
    weight /= float(M) ** (gamma + 1)
    T = np.tile(tgt, (B, 1))
    D = np.tile(drf, (B, 1))
    u = grid[ui].reshape(-1)
    v = np.repeat(grid[vi], gamma + 1)
    n, out, _, _ = oracle.accept_sample(T, D, di.reshape(-1).astype(np.int32), u, v,
                                        np.full(B, gamma, np.int32), V)
    return n, out, weight


@pytest.mark.parametrize("seed", [0, 1])
def test_sampling_brute_force_reproduces_target_distribution_gamma1(seed):
    rng = np.random.default_rng(seed)
    V, M = 4, 96
    tgt = (rng.standard_normal((2, V)) * 1.5).astype(np.float32)
    drf = (rng.standard_normal((1, V)) * 1.5).astype(np.float32)
    n, out, w = _enumerate(tgt, drf, 1, M)
    p0, p1 = _softmax64(tgt[0]), _softmax64(tgt[1])
    first = np.array([w[out[:, 0] == y].sum() for y in range(V)])
    np.testing.assert_allclose(first, p0, atol=2.0 / M)
    acc = n == 1
    second = np.array([w[acc & (out[:, 1] == y)].sum() for y in range(V)]) / w[acc].sum()
    np.testing.assert_allclose(second, p1, atol=2.0 / M)
    assert abs(w.sum() - 1.0) < 1e-12


def test_sampling_brute_force_reproduces_target_distribution_gamma2():
    rng = np.random.default_rng(7)
    V, M = 3, 28
    tgt = (rng.standard_normal((3, V)) * 1.5).astype(np.float32)
    drf = (rng.standard_normal((2, V)) * 1.5).astype(np.float32)
    n, out, w = _enumerate(tgt, drf, 2, M)
    p = [_softmax64(r) for r in tgt]
    first = np.array([w[out[:, 0] == y].sum() for y in range(V)])
    np.testing.assert_allclose(first, p[0], atol=2.0 / M)
    a1 = n >= 1
    second = np.array([w[a1 & (out[:, 1] == y)].sum() for y in range(V)]) / w[a1].sum()
    np.testing.assert_allclose(second, p[1], atol=3.0 / M)
    a2 = n == 2
    third = np.array([w[a2 & (out[:, 2] == y)].sum() for y in range(V)]) / w[a2].sum()
    np.testing.assert_allclose(third, p[2], atol=3.0 / M)


def test_sampling_identical_distributions_always_accept():
    aw = gen.make_accept_workload(0, batch=4, gammas=[4, 4, 4, 4])
    drf = aw.target_logits.reshape(4, 5, -1)[:, :4].reshape(16, -1).copy()
    u = np.full(16, 0.999999, np.float32)
    n, out, am, _ = oracle.accept_sample(aw.target_logits, drf, aw.draft_tokens_sampled, u,
                                         aw.v, aw.gamma, aw.vocab)
    assert n.tolist() == [4, 4, 4, 4]
    assert np.all(am <= 1e-6)


def test_sampling_disjoint_supports_reject_first_and_draw_from_target():
    V = 8
    tgt = np.full((3, V), -1e4, np.float32)
    tgt[:, :4] = np.array([1.0, 0.0, 2.0, 0.5], np.float32)
    drf = np.full((2, V), -1e4, np.float32)
    drf[:, 4:] = 0.0
    p0 = _softmax64(tgt[0])
    cdf = np.cumsum(p0)
    for vv in (0.05, 0.3, 0.62, 0.97):
        n, out, am, dm = oracle.accept_sample(tgt, drf, [5, 6], [0.5, 0.5], [vv, vv, vv], [2], V)
        assert n[0] == 0
        assert out[0, 0] == int(np.searchsorted(cdf, vv, side="right"))
        assert dm[0] > 0


def test_sampling_margins_are_consistent_with_decisions():
    aw = gen.make_accept_workload(0, batch=6)
    n, out, am, dm = oracle.accept_sample(aw.target_logits, aw.draft_logits,
                                          aw.draft_tokens_sampled, aw.u, aw.v, aw.gamma, aw.vocab)
    off = 0
    for b in range(aw.batch):
        g = int(aw.gamma[b])
        m = am[off:off + g]
        assert np.all(m[:n[b]] <= 0)
        if n[b] < g:
            assert m[n[b]] > 0 and np.all(np.isnan(m[n[b] + 1:]))
        off += g
    assert np.all((dm >= 0) & (dm <= 1))
