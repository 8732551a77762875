"""Checks of the seeded input generator (layout and determinism; it holds no method math)."""
import numpy as np

from speculative_decoding_attention_verify_b200 import inputs as gen


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.00390625, 1.01171875, 1.0078125 + 2**-9, -2.5, 3.0e38], np.float32)
    bits = gen.bf16_bits_from_f32(x)
    back = gen.f32_from_bf16_bits(bits)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1.0) wins; 1 + 3*2^-8 rounds up.
    assert back.tolist()[:3] == [1.0, 1.0, 1.015625]
    assert back[4] == -2.5
    assert np.all(np.abs(back - x) <= np.abs(x) * 2**-8)


def test_workload_is_deterministic_and_seed_dependent():
    a = gen.make_attn_workload(1, l_vis=64, l_txt=16)
    b = gen.make_attn_workload(1, l_vis=64, l_txt=16)
    c = gen.make_attn_workload(1, l_vis=64, l_txt=16, seed=99)
    assert np.array_equal(a.k, b.k) and np.array_equal(a.q_verify, b.q_verify)
    assert not np.array_equal(a.k, c.k)


def test_salient_keys_sit_in_the_visual_span():
    w = gen.make_attn_workload(1, l_vis=1000, l_txt=50)
    for g in range(w.h_kv):
        pos = w.salient[0][g]
        assert len(pos) == 10 and pos.max() < 1000
        rows = w.k[0, g, pos]
        assert (rows == rows[0]).all()


def test_paged_layout_round_trip_and_nan_tails():
    w = gen.make_attn_workload(4, l_vis=200, l_txt=30, seed=3)
    pages = (w.kv_len_verify + 15) // 16
    assert w.num_pages == pages.sum()
    used = np.concatenate([w.block_table[s, :pages[s]] for s in range(w.n_seq)])
    assert sorted(used.tolist()) == list(range(w.num_pages))
    for s in range(w.n_seq):
        L = int(w.kv_len_verify[s])
        last = w.block_table[s, (L - 1) // 16]
        if L % 16:
            assert (w.k[last, :, L % 16:] == 0x7FC0).all()
        assert np.isfinite(gen.f32_from_bf16_bits(w.kv_row("k", s, 0, L - 1))).all()


def test_accept_workload_shapes_and_uniform_range():
    aw = gen.make_accept_workload(4, vocab=1000)
    assert aw.target_logits.shape == (int((aw.gamma + 1).sum()), 1000)
    assert aw.draft_logits.shape == (int(aw.gamma.sum()), 1000)
    assert aw.u.min() >= 0 and aw.u.max() < 1 and aw.v.max() < 1
    assert set(aw.gamma.tolist()) <= {3, 5, 7}
