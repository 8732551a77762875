"""GPU parity of top-K selection (bit-exact index sets) and the HSR projection."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_attention_verify_b200 import device as dev
from speculative_decoding_attention_verify_b200 import inputs as gen
from speculative_decoding_attention_verify_b200 import sdattn as sd

pytestmark = pytest.mark.gpu

NEAR_TIE = 1e-9


def _run_topk(w, k, cand_begin=None, cand_end=None, lens=None):
    lens = w.kv_len_verify if lens is None else lens
    cb = np.zeros(w.n_seq, np.int32) if cand_begin is None else cand_begin
    ce = w.l_vis.astype(np.int32) if cand_end is None else cand_end
    kv = dev.kv_cache(w, kv_len=lens)
    q = dev.verify_queries(w)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = sd.sd_topk_select(q, kv, dev.int32(cb), dev.int32(ce), int((ce - cb).max()), k,
                            dev_err=flag).cpu().numpy()
    ref, gap = oracle.topk_select(w.h_q, w.q_verify, w.q_verify_start,
                                  oracle.cache_from_workload(w, kv_len=lens), cb, ce, k)
    assert flag.item() == 0
    return got, ref, gap


def _assert_same_sets(got, ref, gap):
    """Bit-exact, except where the oracle's boundary margin is a near-tie (counted)."""
    near = 0
    for b in range(got.shape[0]):
        for g in range(got.shape[1]):
            if not np.array_equal(got[b, g], ref[b, g]):
                assert gap[b, g] < NEAR_TIE, f"(b={b}, g={g}) differs with boundary gap {gap[b, g]}"
                near += 1
    return near


TOPK_CASES = [
    (0, {}, 32),
    (0, {}, 300),                                    # more than the 256 candidates
    (1, {}, 1024),
    (1, dict(l_vis=5000, l_txt=64), 7),
    (3, dict(layers=3, l_vis=6000, l_txt=100), 1024),
    (4, dict(l_vis=2500, l_txt=200, batch=6), 1024),
    (4, {}, 1024),
]


@pytest.mark.parametrize("cfg,kw,k", TOPK_CASES)
def test_topk_matches_oracle_exactly(cfg, kw, k):
    w = gen.make_attn_workload(cfg, **kw)
    got, ref, gap = _run_topk(w, k)
    near = _assert_same_sets(got, ref, gap)
    assert near == 0


def test_topk_ragged_batch_beyond_one_warp():
    """40 sequences, more than one warp's worth of the device's scan over the sequences' part
    counts, with candidate counts from 200 to 1,448: the scorer's parts follow each sequence's
    own count (one to three parts of 512), and the select reads exactly those parts."""
    w = gen.make_attn_workload(4, l_vis=1500, l_txt=100, batch=40)
    ce = (200 + 32 * np.arange(w.n_seq)).astype(np.int32)
    got, ref, gap = _run_topk(w, 128, cand_end=ce)
    assert _assert_same_sets(got, ref, gap) == 0


def test_topk_c3_full_launch_sampled_layers():
    w = gen.make_attn_workload(3)
    kv = dev.kv_cache(w)
    cb = np.zeros(w.n_seq, np.int32)
    ce = w.l_vis.astype(np.int32)
    got = sd.sd_topk_select(dev.verify_queries(w), kv, dev.int32(cb), dev.int32(ce), 25000,
                            1024).cpu().numpy()
    n_q = int(w.n_q_verify[0])
    for layer in (0, 11, 27):
        sub = oracle.Cache(w.dtype, w.k[layer:layer + 1], w.v[layer:layer + 1],
                           w.kv_len_verify[layer:layer + 1], w.h_kv, w.d)
        ref, gap = oracle.topk_select(w.h_q, w.q_verify[layer * n_q:(layer + 1) * n_q], [0, n_q],
                                      sub, [0], [25000], 1024)
        assert _assert_same_sets(got[layer:layer + 1], ref, gap) == 0
        # the salient keys (4x the query direction) are all selected
        for g in range(w.h_kv):
            assert set(w.salient[layer][g].tolist()) <= set(got[layer, g].tolist())


def test_topk_offset_candidate_range_and_ties():
    w = gen.make_attn_workload(1, l_vis=3000, l_txt=50)
    k_dup = w.k.copy()
    k_dup[0, :, 1000:1010] = k_dup[0, :, 999:1000]  # exact duplicate keys -> ties
    w.k = k_dup
    cb = np.array([500], np.int32)
    ce = np.array([2500], np.int32)
    got, ref, gap = _run_topk(w, 40, cand_begin=cb, cand_end=ce)
    assert _assert_same_sets(got, ref, gap) == 0


def test_topk_special_key_values():
    """Signed zeros, subnormals, the largest finite keys and non-finite keys score exactly.

    Head 0 holds only subnormal keys (every score is then a sum of subnormal products), head 1
    zeros and subnormals among normal keys, head 2 the largest finite bf16 values among normal
    keys, head 3 a few +inf, -inf and NaN elements.  A non-finite element makes the score the
    sum over the group's heads of +-inf products: +inf or -inf where every head's query agrees
    in sign there (dimension 9 of group 3 is set to 1.0 in every head), NaN otherwise.
    """
    w = gen.make_attn_workload(1, l_vis=3000, l_txt=50)
    rng = np.random.default_rng(11)
    k = w.k.copy()
    shape = k[0, 0, :3000].shape
    sign = rng.integers(0, 2, size=shape).astype(np.uint16) << 15
    sub = rng.integers(1, 128, size=shape).astype(np.uint16) | sign
    k[0, 0, :3000] = sub
    h1 = k[0, 1, :3000]
    r = rng.random(shape)
    h1[r < 0.2] = sub[r < 0.2]
    h1[(r >= 0.2) & (r < 0.3)] = sign[(r >= 0.2) & (r < 0.3)]  # +0 / -0
    h2 = k[0, 2, :3000]
    big = rng.random(shape) < 0.01
    h2[big] = np.uint16(0x7F7F) | sign[big]
    h3 = k[0, 3, :3000]
    PINF, NINF, QNAN = 0x7F80, 0xFF80, 0x7FC0
    for pos, dim, val in ((100, 9, PINF), (1500, 9, PINF), (101, 9, NINF), (700, 60, PINF),
                          (2000, 80, NINF), (2500, 4, QNAN), (2600, 9, PINF), (2600, 10, NINF)):
        h3[pos, dim] = val
    w.k = k
    q = w.q_verify.copy()
    last = int(w.q_verify_start[1]) - 1
    q[last, 21:28, 9] = 0x3F80  # 1.0: every head of group 3 agrees in sign at dimension 9
    w.q_verify = q
    got, ref, gap = _run_topk(w, 200)
    assert np.array_equal(got, ref)
    sel3 = set(got[0, 3].tolist())
    assert {100, 1500} <= sel3                       # +inf scores
    assert not {101, 700, 2000, 2500, 2600} & sel3   # -inf or NaN scores


def test_topk_huge_query_values():
    """Queries near the top of the bf16 range: |qbar| reaches 7 * 2^126 in one dimension."""
    w = gen.make_attn_workload(1, l_vis=3000, l_txt=50)
    q = w.q_verify.copy()
    last = int(w.q_verify_start[1]) - 1
    q[last, :7, 3] = 0x7E80  # 2^126 in seven heads of group 0: the group sum is 7 * 2^126
    q[last, 7:14, 5] = 0x7E00  # 2^125 in group 1
    w.q_verify = q
    got, ref, gap = _run_topk(w, 300)
    assert _assert_same_sets(got, ref, gap) == 0


def _boundary(w, k, cb, ce):
    """Oracle scores [b][g][t] and, per (b, g), the position of the k-th best candidate."""
    sc = oracle.topk_scores(w.h_q, w.q_verify, w.q_verify_start, oracle.cache_from_workload(w),
                            cb, ce)
    order = np.argsort(-sc, axis=-1, kind="stable")
    return sc, order[..., k - 1] + cb[:, None]


def test_topk_exact_ties_across_the_boundary():
    """Seven candidates share the k-th best score exactly (copies of its key row, placed below
    and above it): the lowest positions among them are kept, in every KV head."""
    w = gen.make_attn_workload(1, l_vis=3000, l_txt=50)
    k, cb, ce = 100, np.zeros(1, np.int32), np.array([3000], np.int32)
    _, jstar = _boundary(w, k, cb, ce)
    kk = w.k.copy()
    for g in range(w.h_kv):
        j = int(jstar[0, g])
        for dst in (5, 333, 1200, 1201, 2222, 2999):
            if dst != j:
                kk[0, g, dst] = kk[0, g, j]
    w.k = kk
    got, ref, gap = _run_topk(w, k, cand_begin=cb, cand_end=ce)
    assert np.array_equal(got, ref)


def test_topk_near_ties_finer_than_fp32_are_ranked_in_fp64():
    """Near-copies of the k-th best key row that differ in one dimension whose group query sum
    is 2^-20: their scores differ by ~1e-9 relative, far below the fp32 scores' resolution, so
    only the fp64 rescoring of the boundary band orders them (not by position)."""
    w = gen.make_attn_workload(1, l_vis=3000, l_txt=50)
    q = w.q_verify.copy()
    last = int(w.q_verify_start[1]) - 1
    e0 = 17
    G = w.h_q // w.h_kv
    for g in range(w.h_kv):
        q[last, g * G:(g + 1) * G, e0] = 0
        q[last, g * G, e0] = 0x3580  # 2^-20
    w.q_verify = q
    k, cb, ce = 150, np.zeros(1, np.int32), np.array([3000], np.int32)
    _, jstar = _boundary(w, k, cb, ce)
    kk = w.k.copy()
    for g in range(w.h_kv):
        j = int(jstar[0, g])
        base = int(kk[0, g, j, e0])
        if base & 0x7F80 in (0, 0x7F80):  # keep the edited element a normal number
            base = 0x3F80
            kk[0, g, j, e0] = base
        # (a positive bf16 value grows with its bit pattern; a negative one shrinks)
        for dst, step in ((7, 2), (400, -1), (1300, 3), (2100, -3), (2900, 1)):
            if dst != j:
                kk[0, g, dst] = kk[0, g, j]
                kk[0, g, dst, e0] = base + step
    w.k = kk
    got, ref, gap = _run_topk(w, k, cand_begin=cb, cand_end=ce)
    assert np.array_equal(got, ref)


def test_topk_band_wider_than_shared_memory_takes_the_fp64_path():
    """Every key row of one KV head identical: all 3,000 scores tie, the band around the
    threshold holds every candidate (more than the 1,024 ranked in shared memory), and the
    fp64 selection keeps the lowest positions; the other heads take the fp32 path."""
    w = gen.make_attn_workload(1, l_vis=3000, l_txt=50)
    kk = w.k.copy()
    kk[0, 2, :3000] = kk[0, 2, 1234]
    w.k = kk
    got, ref, gap = _run_topk(w, 200)
    assert np.array_equal(got, ref)
    assert np.array_equal(got[0, 2], np.arange(200))


# ---------------------------------------------------------------- HSR ----------------------


@pytest.mark.parametrize("n,bias,d_model", [(1, False, 3584), (3, True, 3584), (16, True, 3584),
                                            (2, False, 512), (4, True, 4096), (2, True, 4112),
                                            (1, False, 16), (5, False, 64)])
def test_hsr_matches_oracle(n, bias, d_model):
    hw = gen.make_hsr_workload(n=n, d_model=d_model, with_bias=bias)
    e = dev.tensor(hw.emb, gen.BF16)
    h = dev.tensor(hw.hid, gen.BF16)
    W = dev.tensor(hw.weight, gen.BF16)
    b = dev.tensor(hw.bias, gen.BF16) if bias else None
    y = sd.sd_hsr_project(e, h, W, b)
    ref = oracle.hsr_project(hw.emb, hw.hid, hw.weight, hw.bias)
    err = np.abs(dev.to_numpy_f64(y) - ref).max()
    assert err <= 2e-2, err


def test_hsr_is_deterministic():
    hw = gen.make_hsr_workload(n=3, d_model=3584, with_bias=True)
    e, h, W, b = (dev.tensor(a, gen.BF16) for a in (hw.emb, hw.hid, hw.weight, hw.bias))
    y1 = sd.sd_hsr_project(e, h, W, b)
    y2 = sd.sd_hsr_project(e, h, W, b)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
