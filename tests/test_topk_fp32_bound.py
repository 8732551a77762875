"""The fp32 top-K scoring's error bound, checked numerically on the CPU.

The library's last-query top-K keeps the candidates of an fp64 scoring while computing the
scores in fp32: with y the fp32 score of a key row k, x its fp64 score, q the fp32 rounding of
the group-summed query qbar, Qu the fp32 round-up of the sum over the group of |q_h| plus
2^-126, and B the fp32 sum of Qu_i |k_i|, it relies on

    |y - x| <= 2^-15 B + 2^-140        (d <= 128)

This test emulates the fp32 accumulation with numpy float32 (a multiply, then an add: two
roundings per step, more error than the kernel's fused multiply-add) in several orders and
checks the inequality against an fp64 score, on rows that stress each term: ordinary values,
groups whose heads cancel (qbar much smaller than Q), subnormal keys and queries, and values
near the top of the fp32 range.  No GPU and no oracle code: it pins the bound itself.
"""
import numpy as np
import pytest

D, G = 128, 7
ERR_SCALE, ERR_FLOOR = 2.0 ** -15, 2.0 ** -140


def _bf16(x):
    """float32 values rounded to bf16 (round to nearest even), as float32."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32)


def _round_up_f32(v):
    f = np.float32(v)
    return np.nextafter(f, np.float32(np.inf)) if float(f) < v else f


def _fp32_dot(a, b, order):
    acc = np.float32(0.0)
    for i in order:
        acc = np.float32(acc + np.float32(a[i] * b[i]))
    return acc


def _check(qh, k, rng):
    """qh [G][D] and k [D] (bf16 values as float32)."""
    qbar = qh.astype(np.float64).sum(axis=0)
    Q = np.abs(qh.astype(np.float64)).sum(axis=0)
    q = qbar.astype(np.float32)
    Qu = np.array([np.float32(_round_up_f32(v)) + np.float32(2.0 ** -126) for v in Q],
                  np.float32)
    x = float(np.dot(qbar, k.astype(np.float64)))
    for order in (np.arange(D), np.arange(D)[::-1], rng.permutation(D)):
        y = _fp32_dot(q, k, order)
        B = _fp32_dot(Qu, np.abs(k), order)
        if not (np.isfinite(y) and np.isfinite(B)):
            continue  # (the kernel flags the unit and scores it in fp64)
        assert abs(float(y) - x) <= ERR_SCALE * float(B) + ERR_FLOOR, (float(y), x, float(B))


@pytest.mark.parametrize("case", ["normal", "cancelling", "subnormal", "wide", "huge"])
def test_fp32_score_bound_holds(case):
    rng = np.random.default_rng({"normal": 1, "cancelling": 2, "subnormal": 3, "wide": 4,
                                 "huge": 5}[case])
    for _ in range(40):
        qh = rng.standard_normal((G, D)).astype(np.float32)
        k = rng.standard_normal(D).astype(np.float32)
        if case == "cancelling":  # heads nearly cancel: qbar is a small fraction of Q
            qh[1:] = -qh[0] / (G - 1) * (1 + 1e-3 * rng.standard_normal((G - 1, D)))
        elif case == "subnormal":
            k *= np.float32(2.0 ** -133)
            qh *= np.float32(2.0 ** -10)
        elif case == "wide":  # elements spread over many binades
            k *= np.exp2(rng.integers(-40, 40, D)).astype(np.float32)
            qh *= np.exp2(rng.integers(-20, 20, (G, D))).astype(np.float32)
        elif case == "huge":
            k *= np.float32(2.0 ** 60)
            qh *= np.float32(2.0 ** 50)
        _check(_bf16(qh), _bf16(k), rng)


def test_the_bound_is_not_vacuous():
    """For ordinary rows the band 4E is about 0.3% of the spread of the scores: with 25,000
    candidates and the 1,024 best kept (the threshold near 1.75 standard deviations), about
    25,000 x 0.086 x 0.003 ~ 6 candidates fall in it, as the clock-stamped select kernel
    counts on the benchmark workload (a median of 7)."""
    rng = np.random.default_rng(7)
    qh = _bf16(rng.standard_normal((G, D)).astype(np.float32))
    ks = _bf16(rng.standard_normal((2000, D)).astype(np.float32))
    qbar = qh.astype(np.float64).sum(axis=0)
    Qu = np.abs(qh.astype(np.float64)).sum(axis=0)
    scores = ks.astype(np.float64) @ qbar
    E = ERR_SCALE * float((np.abs(ks.astype(np.float64)) @ Qu).max()) + ERR_FLOOR
    assert 4 * E < 5e-3 * scores.std()
