"""GPU parity of Sparrow's draft layer (through the C-ABI) against the fp64 oracle.

Output y: max-abs <= 2e-2.  y is rounded to bf16 (2^-9 relative: 0.008 at |y| = 4, about the
largest output of the 7B-like layer) after fp32 accumulation of every projection; the rows' q,
k and v pass through bf16 (the cache's type) and the MLP's input too, each perturbing the output
by a few 1e-3.  The rows' k and v written into the cache: within one bf16 step (2^-8 relative)
of the oracle's, which rounds its own fp64 values.  The rest of the cache is untouched.
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
    ry, rk, rv, _ = oracle.draft_layer(w, w.emb, w.hid, w.k_cache, w.v_cache, w.kv_len, w.window)
    return y, k, v, ry, rk, rv


def _check(w, y, k, v, ry, rk, rv):
    err = float(np.abs(dev.to_numpy_f64(y) - ry).max())
    assert err <= TOL, err
    lo = w.kv_len - w.n
    gk = k.view(torch.int16).cpu().numpy().view(np.uint16)
    gv = v.view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(gk[:, :, :lo], w.k_cache[:, :, :lo])
    np.testing.assert_array_equal(gv[:, :, :lo], w.v_cache[:, :, :lo])
    for got, want in ((gk, rk), (gv, rv)):
        a = gen.f32_from_bf16_bits(got[:, :, lo:w.kv_len]).astype(np.float64)
        b = gen.f32_from_bf16_bits(want[:, :, lo:w.kv_len]).astype(np.float64)
        assert (np.abs(a - b) <= 2.0 ** -8 * np.abs(b) + 1e-30).all()
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
