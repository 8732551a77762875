"""Pins for the oracle's draft-layer routines: RMSNorm, rotary embedding and the layer itself.

RMSNorm is checked against torch's fp64 implementation and a closed form; the rotary embedding
against its complex-number form (pairs (v_i, v_{i+d/2}) as complex numbers multiplied by
e^{j pos theta^(-2i/d)}), the identity at position 0, norm preservation and the dependence of
rotated dot products on the position difference only.  The layer is tied to the pinned HSR
and text-anchored attention routines and to closed forms of its special cases.
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_attention_verify_b200 import inputs as gen


def _small(n=2, **kw):
    args = dict(n=n, d_model=256, h_q=4, h_kv=2, head_dim=64, d_ff=512, l_txt=40)
    args.update(kw)
    return gen.make_draft_layer_workload(**args)


# ---------------------------------------------------------------- RMSNorm -----------------

def test_rmsnorm_matches_torch_fp64():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 97)) * 3.0
    g = gen.bf16_bits_from_f32((1.0 + 0.2 * rng.standard_normal(97)).astype(np.float32))
    gf = gen.f32_from_bf16_bits(g).astype(np.float64)
    want = torch.nn.functional.rms_norm(torch.from_numpy(x), (97,), torch.from_numpy(gf),
                                        eps=1e-6).numpy()
    np.testing.assert_allclose(oracle.rmsnorm(x, g, 1e-6), want, rtol=1e-13, atol=1e-14)


def test_rmsnorm_of_a_constant_vector():
    """x = c * 1: mean(x^2) = c^2, so y_i = c / sqrt(c^2 + eps) * gamma_i."""
    g = gen.bf16_bits_from_f32(np.linspace(0.5, 2.0, 16).astype(np.float32))
    for c in (-3.0, 0.25, 7.0):
        y = oracle.rmsnorm(np.full((1, 16), c), g, 1e-2)[0]
        want = c / np.sqrt(c * c + 1e-2) * gen.f32_from_bf16_bits(g)
        np.testing.assert_allclose(y, want, rtol=1e-14)


# ---------------------------------------------------------------- rotary embedding --------

def test_rope_equals_complex_rotation():
    rng = np.random.default_rng(2)
    d, theta = 64, 1e6
    v = rng.standard_normal((5, d))
    pos = np.array([0.0, 1.0, 17.0, 1000.0, 25_999.0])
    got = oracle.rope(v, pos, theta)
    half = d // 2
    z = v[:, :half] + 1j * v[:, half:]
    freq = theta ** (-np.arange(half) * 2.0 / d)
    zr = z * np.exp(1j * pos[:, None] * freq[None, :])
    np.testing.assert_allclose(got[:, :half], zr.real, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got[:, half:], zr.imag, rtol=1e-12, atol=1e-12)


def test_rope_identity_at_zero_and_norm_preserving():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((4, 128))
    np.testing.assert_array_equal(oracle.rope(v, np.zeros(4), 1e4), v)
    r = oracle.rope(v, np.array([3.0, 50.0, 700.0, 12345.0]), 1e4)
    np.testing.assert_allclose(np.linalg.norm(r, axis=1), np.linalg.norm(v, axis=1), rtol=1e-13)


def test_rope_dot_products_depend_on_the_position_difference():
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal((1, 64)), rng.standard_normal((1, 64))
    for m, n in ((10.0, 3.0), (500.0, 123.0), (7.0, 7.0)):
        a = float((oracle.rope(q, [m], 1e6) @ oracle.rope(k, [n], 1e6).T)[0, 0])
        b = float((oracle.rope(q, [m - n], 1e6) @ k.T)[0, 0])
        assert abs(a - b) < 1e-11


# ---------------------------------------------------------------- the layer ---------------

def _run(w, **over):
    for key, val in over.items():
        setattr(w, key, val)
    return oracle.draft_layer(w, w.emb, w.hid, w.k_cache, w.v_cache, w.kv_len, w.window)


def test_layer_input_is_the_hsr_projection_and_zero_projections_pass_it_through():
    w = _small()
    y, _, _, parts = _run(w, w_o=np.zeros_like(w.w_o), w_down=np.zeros_like(w.w_down))
    want = oracle.hsr_project(w.emb, w.hid, w.w_hsr)
    np.testing.assert_allclose(parts["x"], want, rtol=0, atol=1e-12)
    np.testing.assert_allclose(parts["x2"], want, rtol=0, atol=1e-12)
    np.testing.assert_allclose(y, want, rtol=0, atol=1e-12)


def test_layer_attention_is_the_text_anchored_attention_over_the_appended_cache():
    """o equals the pinned text-anchored routine run on the returned cache (the rows' k and v
    appended) with the rows' bf16 queries, no visual span and the window."""
    w = _small(n=3, window=17)
    y, k, v, parts = _run(w)
    cache = oracle.Cache("bf16", k, v, [w.kv_len], w.h_kv, w.head_dim)
    qb = gen.bf16_bits_from_f32(parts["q"].astype(np.float32)).reshape(w.n, w.h_q, w.head_dim)
    o = oracle.text_anchored_attention(w.h_q, qb, [0, w.n], cache, [0], [0], [w.window])
    np.testing.assert_allclose(parts["o"], o.reshape(w.n, -1), rtol=0, atol=1e-12)
    # positions before the rows are untouched
    np.testing.assert_array_equal(k[:, :, :w.l_txt], w.k_cache[:, :, :w.l_txt])
    np.testing.assert_array_equal(v[:, :, :w.l_txt], w.v_cache[:, :, :w.l_txt])


def test_layer_with_zero_norm_weights_has_closed_forms():
    """ln1 = 0 and no bias: q = k = v = 0, every score is 0, so each row's output is the mean of
    V over its window (the new rows' v are 0); ln2 = 0: the MLP sees 0 and adds silu(0) * 0 = 0,
    so y = x2 = x + W_o o."""
    w = _small(n=2, window=9)
    y, k, v, parts = _run(w, ln1=np.zeros_like(w.ln1), b_qkv=np.zeros_like(w.b_qkv),
                          ln2=np.zeros_like(w.ln2))
    assert (gen.f32_from_bf16_bits(k[:, :, w.l_txt:]) == 0).all()  # (signed zeros allowed)
    assert (gen.f32_from_bf16_bits(v[:, :, w.l_txt:]) == 0).all()
    vf = gen.f32_from_bf16_bits(v[0]).astype(np.float64)  # [h_kv][cap][d]
    G = w.h_q // w.h_kv
    for r in range(w.n):
        hi = w.kv_len - w.n + r
        mean = vf[:, hi - w.window + 1:hi + 1].mean(axis=1)  # [h_kv][d]
        want = np.repeat(mean, G, axis=0).reshape(-1)
        np.testing.assert_allclose(parts["o"][r], want, rtol=0, atol=1e-12)
    wo = gen.f32_from_bf16_bits(w.w_o).astype(np.float64)
    np.testing.assert_allclose(y, parts["x"] + parts["o"] @ wo.T, rtol=0, atol=1e-11)


def test_layer_queries_and_keys_are_rotated_at_their_positions():
    """Rotating the rows' queries back by their positions gives the unrotated projection,
    whatever the position: the last rows of a longer cache only differ by the angle."""
    a = _small(n=1, l_txt=40)
    b = _small(n=1, l_txt=40)
    b.k_cache = np.concatenate([b.k_cache[:, :, :40], b.k_cache[:, :, :40], b.k_cache[:, :, 40:]],
                               axis=2)
    b.v_cache = np.concatenate([b.v_cache[:, :, :40], b.v_cache[:, :, :40], b.v_cache[:, :, 40:]],
                               axis=2)
    b.l_txt = 80
    _, _, _, pa = _run(a)
    _, _, _, pb = _run(b)
    d = a.head_dim
    qa = oracle.rope(pa["q"].reshape(-1, d), np.full(a.h_q, -40.0), a.rope_theta)
    qb = oracle.rope(pb["q"].reshape(-1, d), np.full(b.h_q, -80.0), b.rope_theta)
    np.testing.assert_allclose(qa, qb, rtol=0, atol=1e-11)


def test_layer_with_zero_input_norm_projects_the_bias_rotated_at_the_row_positions():
    """ln1 = 0: the projection is the bias alone, so every row's q heads are the q bias rotated
    at the row's absolute position, the cache receives the k bias rotated the same way and the
    v bias, in bf16."""
    w = _small(n=3)
    _, k, v, parts = _run(w, ln1=np.zeros_like(w.ln1))
    d, hq, hk = w.head_dim, w.h_q, w.h_kv
    b = gen.f32_from_bf16_bits(w.b_qkv).astype(np.float64)
    for r in range(w.n):
        pos = float(w.kv_len - w.n + r)
        want_q = oracle.rope(b[:hq * d].reshape(hq, d), np.full(hq, pos), w.rope_theta)
        np.testing.assert_allclose(parts["q"][r].reshape(hq, d), want_q, rtol=0, atol=1e-12)
        want_k = oracle.rope(b[hq * d:(hq + hk) * d].reshape(hk, d), np.full(hk, pos),
                             w.rope_theta)
        j = w.kv_len - w.n + r
        np.testing.assert_array_equal(k[0, :, j], gen.bf16_bits_from_f32(want_k.astype(np.float32)))
        np.testing.assert_array_equal(v[0, :, j], w.b_qkv[(hq + hk) * d:].reshape(hk, d))


def test_layer_mlp_half_matches_torch_fp64():
    """y - x2 is the gated MLP of the normalised x2: torch's fp64 rms_norm, silu and matmul on
    the oracle's x2 give the same vector."""
    w = _small(n=2)
    y, _, _, parts = _run(w)
    f = lambda a: torch.from_numpy(gen.f32_from_bf16_bits(a).astype(np.float64))
    x2 = torch.from_numpy(parts["x2"])
    m = torch.nn.functional.rms_norm(x2, (w.d_model,), f(w.ln2), eps=w.rms_eps)
    gu = m @ f(w.w_gate_up).T
    g, u = gu[:, :w.d_ff], gu[:, w.d_ff:]
    want = x2 + (torch.nn.functional.silu(g) * u) @ f(w.w_down).T
    np.testing.assert_allclose(y, want.numpy(), rtol=0, atol=1e-11)
