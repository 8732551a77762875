"""The allocation-free verify entry point against the workspace-taking one (through the C-ABI).

sd_verify_attention_noalloc serves callers that cannot allocate device memory when they call
(a serving engine whose KV page pool has taken the free HBM, or a host program that only holds
device pointers another runtime gave it).  It plans and launches exactly the kernels of
sd_verify_attention, with the split partials in the library's fixed scratch, so its output must
be bit-identical to sd_verify_attention's, on every call: the scratch keeps the previous call's
contents and nothing in it may leak into the next result.

This file is collected last, so that it also runs after every other GPU test in one process;
it passes alone in a fresh process as well.
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_attention_verify_b200 import device as dev
from speculative_decoding_attention_verify_b200 import inputs as gen
from speculative_decoding_attention_verify_b200 import sdattn as sd

pytestmark = pytest.mark.gpu

TOL = {gen.F32: 1e-4, gen.BF16: 2e-2}  # against the oracle, as every attention test

CASES = [
    (1, dict(l_vis=6000, l_txt=200, gamma=2)),     # 21 rows per KV head: tensor cores, split KV
    (1, dict(l_vis=3000, l_txt=100, gamma=0)),     # 7 rows per KV head: tensor cores, 4 row copies
    (1, dict(l_vis=2000, l_txt=150, gamma=19)),    # 140 rows per KV head: CUDA-core engine
    (0, dict(l_vis=20000, l_txt=64)),              # fp32: CUDA-core engine, many splits + merge
    (4, dict(l_vis=1500, l_txt=100, batch=5)),     # paged, ragged
    (3, {}),                                       # 28 layers x 9 rows over 26k positions
]


def _bits(t):
    return t.view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32)


@pytest.mark.parametrize("cfg,kw", CASES)
def test_noalloc_matches_workspace_entry_point_twice(cfg, kw):
    w = gen.make_attn_workload(cfg, **kw)
    kv, q = dev.kv_cache(w), dev.verify_queries(w)
    need = sd.sd_attention_workspace_size(sd.SD_ATTN_VERIFY, q, kv)
    assert 0 < need <= sd.SD_VERIFY_NOALLOC_SCRATCH_BYTES
    ref = sd.sd_verify_attention(q, kv)
    for call in range(2):
        out = torch.full_like(q.q, float("nan"))
        sd.sd_verify_attention_noalloc(q, kv, out)
        torch.cuda.synchronize()
        assert torch.equal(_bits(out), _bits(ref)), f"call {call}: differs from sd_verify_attention"


def test_noalloc_matches_oracle():
    """A direct check against the fp64 oracle, so that a fault shared by both entry points
    cannot hide."""
    for cfg, kw in ((1, dict(l_vis=6000, l_txt=200, gamma=2)), (0, dict(l_vis=20000, l_txt=64))):
        w = gen.make_attn_workload(cfg, **kw)
        kv, q = dev.kv_cache(w), dev.verify_queries(w)
        out = torch.empty_like(q.q)
        sd.sd_verify_attention_noalloc(q, kv, out)
        ref = oracle.verify_attention(w.h_q, w.q_verify, w.q_verify_start,
                                      oracle.cache_from_workload(w))
        err = float(np.abs(dev.to_numpy_f64(out) - ref).max())
        assert err <= TOL[w.dtype], (cfg, err)


def test_noalloc_rejects_a_plan_beyond_its_scratch():
    w = gen.make_attn_workload(3, l_vis=3000, l_txt=100)
    kv, q = dev.kv_cache(w), dev.verify_queries(w)
    # Same tensors; a much looser length hint (up to 2,000,000 positions) plans more splits
    # and a workspace of about 129 MiB.
    big = sd.Queries(q.q, q.q_start, max_q_rows=q.desc.max_q_rows, max_kv_len=2_000_000)
    assert sd.sd_attention_workspace_size(sd.SD_ATTN_VERIFY, big, kv) > \
        sd.SD_VERIFY_NOALLOC_SCRATCH_BYTES
    out = torch.zeros_like(q.q)
    with pytest.raises(sd.SdError) as e:
        sd.sd_verify_attention_noalloc(big, kv, out)
    assert e.value.status == sd.SD_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert not out.any()  # nothing was launched
