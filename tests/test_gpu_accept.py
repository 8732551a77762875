"""GPU parity of greedy and speculative-sampling acceptance.

Greedy: accepted lengths and tokens bit-exact.  Sampling: bit-exact except where the oracle's
decision margin |u - p/q| < 1e-6, or its draw lies within 1e-6 * Z of a CDF edge (counted).
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_attention_verify_b200 import device as dev
from speculative_decoding_attention_verify_b200 import inputs as gen
from speculative_decoding_attention_verify_b200 import sdattn as sd

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _t(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda")


def _greedy(aw, drafts):
    n, out = sd.sd_accept_greedy(_t(aw.target_logits), _t(drafts.astype(np.int32)),
                                 _t(aw.gamma), aw.gamma_max)
    return n.cpu().numpy(), out.cpu().numpy()


def _assert_greedy(aw, drafts):
    n, out = _greedy(aw, drafts)
    rn, rout = oracle.accept_greedy(aw.target_logits, drafts, aw.gamma, aw.vocab)
    assert n.tolist() == rn.tolist()
    for b in range(aw.batch):
        assert out[b, :n[b] + 1].tolist() == rout[b, :rn[b] + 1].tolist()
    return n


GREEDY_CASES = [(0, {}), (2, {}), (4, {}), (0, dict(batch=37, vocab=5003))]


@pytest.mark.parametrize("cfg,kw", GREEDY_CASES)
def test_greedy_matches_oracle(cfg, kw):
    aw = gen.make_accept_workload(cfg, **kw)
    _assert_greedy(aw, aw.draft_tokens_greedy)
    _assert_greedy(aw, aw.draft_tokens_sampled)


@pytest.mark.parametrize("cfg", [0, 2, 4])
def test_greedy_own_argmax_accepts_all(cfg):
    aw = gen.make_accept_workload(cfg)
    rows = np.split(aw.target_logits, np.cumsum(aw.gamma + 1)[:-1])
    drafts = np.concatenate([np.argmax(r[:-1], axis=1) for r in rows]).astype(np.int32)
    n = _assert_greedy(aw, drafts)
    assert n.tolist() == aw.gamma.tolist()


def test_greedy_partial_prefix():
    aw = gen.make_accept_workload(4, batch=8, gammas=[7] * 8)
    rows = np.split(aw.target_logits, 8)
    drafts = np.concatenate([np.argmax(r[:-1], axis=1) for r in rows]).astype(np.int32)
    for b in range(8):  # break sequence b at draft position b (b=7 keeps all)
        if b < 7:
            drafts[7 * b + b] = (drafts[7 * b + b] + 1) % aw.vocab
    n = _assert_greedy(aw, drafts)
    assert n.tolist() == list(range(7)) + [7]


def test_greedy_ties_and_nan():
    V = 4099
    tgt = np.zeros((3, V), np.float32)
    tgt[0, [17, 4000, 2500]] = 5.0          # tie -> 17
    tgt[1, :] = -np.inf
    tgt[1, 3] = np.nan
    tgt[1, 9] = -1e30                        # -> 9
    tgt[2, :] = np.nan                       # all NaN -> 0
    aw = gen.AcceptWorkload(vocab=V, gamma=np.array([2], np.int32), target_logits=tgt,
                            draft_logits=np.zeros((2, V), np.float32),
                            draft_tokens_sampled=np.array([17, 9], np.int32),
                            draft_tokens_greedy=np.array([17, 9], np.int32),
                            u=np.zeros(2, np.float32), v=np.zeros(3, np.float32))
    n, out = _greedy(aw, np.array([17, 9], np.int32))
    assert n[0] == 2 and out[0].tolist() == [17, 9, 0]


def _sample(aw):
    n, out, near = sd.sd_accept_sample(_t(aw.target_logits), _t(aw.draft_logits),
                                       _t(aw.draft_tokens_sampled), _t(aw.u), _t(aw.v),
                                       _t(aw.gamma), aw.gamma_max)
    return n.cpu().numpy(), out.cpu().numpy(), near.cpu().numpy()


SAMPLE_CASES = [(0, {}), (0, dict(batch=64)), (2, {}), (4, {}), (4, dict(batch=24, vocab=32000)),
                (4, dict(batch=32))]  # 32 sequences over vocab 152,064: many residual draws


@pytest.mark.parametrize("cfg,kw", SAMPLE_CASES)
def test_sample_matches_oracle(cfg, kw):
    _check_sample(gen.make_accept_workload(cfg, **kw))


def test_sample_long_and_empty_drafts():
    """Draft lengths 24, 17 and 0 in one batch over vocab 152,064: the decision kernel's warps
    take several of the 2 gamma + 1 rows each, one CTA draws over ~300 vocabulary chunks of its
    own, and a sequence without drafts draws its bonus token from p."""
    aw = gen.make_accept_workload(4, batch=3, gammas=[24, 17, 0])
    _check_sample(aw)
    _assert_greedy(aw, aw.draft_tokens_greedy)


def test_sample_long_drafts_accept_all():
    """Draft rows equal to their target rows and u just below 1: all 24 and 17 drafts are kept
    and the bonus token is drawn from the last target row (as the oracle draws it)."""
    aw = gen.make_accept_workload(4, batch=3, gammas=[24, 17, 0])
    rows = np.split(aw.target_logits, np.cumsum(aw.gamma + 1)[:-1])
    aw.draft_logits = np.concatenate([r[:g] for r, g in zip(rows, aw.gamma)]).copy()
    aw.u = np.full(aw.u.shape, 0.999, np.float32)
    n, out, _ = _sample(aw)
    assert n.tolist() == [24, 17, 0]
    _check_sample(aw)


def _check_sample(aw):
    n, out, near = _sample(aw)
    rn, rout, am, dm = oracle.accept_sample(aw.target_logits, aw.draft_logits,
                                            aw.draft_tokens_sampled, aw.u, aw.v, aw.gamma,
                                            aw.vocab)
    exceptions = 0
    off = 0
    for b in range(aw.batch):
        g = int(aw.gamma[b])
        margins = am[off:off + g]
        same = n[b] == rn[b] and out[b, :n[b] + 1].tolist() == rout[b, :rn[b] + 1].tolist()
        if not same:
            seen = np.abs(margins[:min(n[b], rn[b]) + 1])
            near_decision = seen.size > 0 and np.nanmin(seen) < EPS
            near_draw = dm[b] < EPS
            assert near_decision or near_draw, f"sequence {b} differs away from any boundary"
            exceptions += 1
        off += g
    assert exceptions == 0, f"{exceptions} near-boundary exceptions"
    _assert_near_boundary_count(aw, near, am, dm)


def _assert_near_boundary_count(aw, near, am, dm):
    """The device's per-sequence near-boundary count equals the oracle's: decisions evaluated
    with |u - p/q| < 1e-6, plus a draw within 1e-6 * Z of a CDF edge.  A margin within a factor
    two of 1e-6 may be counted by one side only (the two sides round differently)."""
    off = 0
    for b in range(aw.batch):
        g = int(aw.gamma[b])
        m = np.abs(am[off:off + g])
        m = m[np.isfinite(m)]
        want = int((m < EPS).sum()) + int(dm[b] < EPS)
        loose = int(((m >= EPS / 2) & (m < 2 * EPS)).sum()) + int(EPS / 2 <= dm[b] < 2 * EPS)
        assert abs(int(near[b]) - want) <= loose, (b, int(near[b]), want)
        off += g


def test_sample_identical_distributions_accept_all():
    aw = gen.make_accept_workload(0, batch=6, gammas=[4] * 6)
    aw.draft_logits = aw.target_logits.reshape(6, 5, -1)[:, :4].reshape(24, -1).copy()
    aw.u = np.full(24, 0.999, np.float32)
    n, out, _ = _sample(aw)
    assert n.tolist() == [4] * 6


def test_sample_bad_token_sets_flag():
    aw = gen.make_accept_workload(0, batch=2, gammas=[3, 3])
    toks = aw.draft_tokens_sampled.copy()
    toks[0] = aw.vocab + 7  # position 0 is always evaluated
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    sd.sd_accept_sample(_t(aw.target_logits), _t(aw.draft_logits), _t(toks), _t(aw.u), _t(aw.v),
                        _t(aw.gamma), 3, dev_err=flag)
    torch.cuda.synchronize()
    assert flag.item() & sd.SD_DEVERR_TOKEN
