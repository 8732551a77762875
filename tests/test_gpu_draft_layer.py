"""GPU parity of Sparrow's draft layer (through the C-ABI) against the fp64 oracle.

Output y: max-abs <= 2e-2.  y is rounded to bf16 (2^-9 relative: 0.008 at |y| = 4, about the
largest output of the 7B-like layer) after fp32 accumulation of every projection; the rows' q,
k and v pass through bf16 (the cache's type) and the MLP's input too, each perturbing the output
by a few 1e-3.

The rows' k and v written into the cache, element by element: the kernels feed every projection
a bf16 input vector (the normalised x here: relative error <= 2^-9 per entry), accumulate in
fp32 and round the result to bf16; the oracle keeps fp64 throughout and rounds only the stored
value.  So |k_gpu - k_oracle| <= E + 2^-8 (|k_gpu| + |k_oracle|), with E = 2^-8 sum_i |W_ji a_i|
(twice the input-rounding bound, the margin covering fp32 accumulation and the fp32 RMSNorm
scale) and, for keys, E of both members of the rotated pair added (RoPE mixes them with
|cos|, |sin| <= 1).  That worst case lets every rounding line up; the rounding errors are
independent, so over all the rows' elements the RMS difference must also stay below 2^-6 of the
oracle's RMS (about eight times the expected 2^-9).  The rest of the cache is untouched.
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_attention_verify_b200 import device as dev
from speculative_decoding_attention_verify_b200 import inputs as gen
from speculative_decoding_attention_verify_b200 import sdattn as sd

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _layer(w):
    t = lambda a: dev.tensor(a, gen.BF16)
    return sd.DraftLayer(w.d_model, w.h_q, w.h_kv, w.head_dim, w.d_ff, w.rms_eps, w.rope_theta,
                         **{name: t(getattr(w, name)) for name in sd.DraftLayer.NAMES})


def _run(w):
    layer = _layer(w)
    k, v = dev.tensor(w.k_cache, gen.BF16), dev.tensor(w.v_cache, gen.BF16)
    cache = sd.KVCache(k, v, dev.int32([w.kv_len]))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = sd.sd_draft_layer(layer, dev.tensor(w.emb, gen.BF16), dev.tensor(w.hid, gen.BF16), cache,
                          w.kv_len, w.window, dev_err=flag)
    torch.cuda.synchronize()
    assert flag.item() == 0
    ry, rk, rv, parts = oracle.draft_layer(w, w.emb, w.hid, w.k_cache, w.v_cache, w.kv_len,
                                           w.window)
    return y, k, v, ry, rk, rv, parts


def _kv_bounds(w, parts):
    """E for the rows' keys and values [h_kv][n][d] (see the module docstring)."""
    d, hq, hk, half = w.head_dim, w.h_q, w.h_kv, w.head_dim // 2
    a = np.abs(oracle.rmsnorm(parts["x"], w.ln1, w.rms_eps))          # [n][D]
    wq = np.abs(gen.f32_from_bf16_bits(w.w_qkv).astype(np.float64))  # [(hq + 2 hk) d][D]
    e = 2.0 ** -8 * (a @ wq.T)                                         # [n][(hq + 2 hk) d]
    ek = e[:, hq * d:(hq + hk) * d].reshape(w.n, hk, d)
    ek = ek + np.concatenate([ek[..., half:], ek[..., :half]], axis=-1)
    ev = e[:, (hq + hk) * d:].reshape(w.n, hk, d)
    return ek.transpose(1, 0, 2), ev.transpose(1, 0, 2)


def _check(w, y, k, v, ry, rk, rv, parts):
    err = float(np.abs(dev.to_numpy_f64(y) - ry).max())
    assert err <= TOL, err
    lo = w.kv_len - w.n
    gk = k.view(torch.int16).cpu().numpy().view(np.uint16)
    gv = v.view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(gk[:, :, :lo], w.k_cache[:, :, :lo])
    np.testing.assert_array_equal(gv[:, :, :lo], w.v_cache[:, :, :lo])
    ek, ev = _kv_bounds(w, parts)
    for got, want, bound in ((gk, rk, ek), (gv, rv, ev)):
        a = gen.f32_from_bf16_bits(got[0, :, lo:w.kv_len]).astype(np.float64)
        b = gen.f32_from_bf16_bits(want[0, :, lo:w.kv_len]).astype(np.float64)
        assert (np.abs(a - b) <= bound + 2.0 ** -8 * (np.abs(a) + np.abs(b))).all()
        assert np.sqrt(np.mean((a - b) ** 2)) <= 2.0 ** -6 * np.sqrt(np.mean(b ** 2))
    return err


@pytest.mark.parametrize("n,kw", [
    (1, dict(d_model=256, h_q=4, h_kv=2, head_dim=64, d_ff=512, l_txt=40, window=17)),
    (2, dict(d_model=256, h_q=4, h_kv=2, head_dim=64, d_ff=512, l_txt=40, window=17)),
    (4, dict(d_model=512, h_q=8, h_kv=2, head_dim=128, d_ff=1024, l_txt=300, window=300)),
    (3, dict(d_model=256, h_q=4, h_kv=1, head_dim=128, d_ff=512, l_txt=20_000, window=64)),
])
def test_draft_layer_matches_oracle_small(n, kw):
    w = gen.make_draft_layer_workload(n=n, **kw)
    _check(w, *_run(w))


@pytest.mark.parametrize("n", [1, 2])
def test_draft_layer_matches_oracle_7b_shapes(n):
    """D = 3584, 28 query / 4 KV heads of 128, d_ff = 18944, 1,024 earlier text positions."""
    w = gen.make_draft_layer_workload(n=n)
    _check(w, *_run(w))


def test_draft_layer_rejects_bad_arguments():
    w = gen.make_draft_layer_workload(n=1, d_model=256, h_q=4, h_kv=2, head_dim=64, d_ff=512,
                                      l_txt=40)
    layer = _layer(w)
    k, v = dev.tensor(w.k_cache, gen.BF16), dev.tensor(w.v_cache, gen.BF16)
    cache = sd.KVCache(k, v, dev.int32([w.kv_len]))
    e = dev.tensor(np.repeat(w.emb, 5, axis=0), gen.BF16)
    with pytest.raises(sd.SdError) as err:  # five rows: more than the layer takes
        sd.sd_draft_layer(layer, e, e, cache, w.kv_len, w.window)
    assert err.value.status == sd.SD_ERR_INVALID_ARG
