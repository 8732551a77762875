"""The allocation-free verify entry point against the workspace-taking one (through the C-ABI).

Kept in a file collected last so that it also runs after every other GPU test in one process;
it passes alone in a fresh process as well.  Tolerance as for the other bf16 attention tests.
"""
import pytest
import torch

from speculative_decoding_attention_verify_b200 import device as dev
from speculative_decoding_attention_verify_b200 import inputs as gen
from speculative_decoding_attention_verify_b200 import sdattn as sd

pytestmark = pytest.mark.gpu

TOL = 2e-2

CASES = [
    (1, dict(l_vis=6000, l_txt=200, gamma=2)),   # 21 rows per KV head: tensor cores, split KV
    (1, dict(l_vis=3000, l_txt=100, gamma=0)),   # 7 rows per KV head: CUDA-core engine
    (4, dict(l_vis=1500, l_txt=100, batch=5)),   # paged, ragged
    (3, {}),                                     # 28 layers x 9 rows over 26k positions
]


@pytest.mark.parametrize("cfg,kw", CASES)
def test_noalloc_matches_workspace_entry_point_twice(cfg, kw):
    w = gen.make_attn_workload(cfg, **kw)
    kv, q = dev.kv_cache(w), dev.verify_queries(w)
    need = sd.sd_attention_workspace_size(sd.SD_ATTN_VERIFY, q, kv)
    assert need <= sd.SD_VERIFY_NOALLOC_SCRATCH_BYTES
    ref = sd.sd_verify_attention(q, kv).float()
    for call in range(2):
        out = torch.full_like(q.q, float("nan"))
        sd.sd_verify_attention_noalloc(q, kv, out)
        torch.cuda.synchronize()
        got = out.float()
        assert torch.isfinite(got).all(), f"call {call}: non-finite output"
        err = (got - ref).abs().max().item()
        assert err <= TOL, f"call {call}: max-abs difference {err}"


def test_noalloc_rejects_a_plan_beyond_its_scratch():
    w = gen.make_attn_workload(3, l_vis=3000, l_txt=100)
    kv, q = dev.kv_cache(w), dev.verify_queries(w)
    # Same tensors; a looser row hint (18 rows per sequence) plans a workspace of about 66 MB.
    big = sd.Queries(q.q, q.q_start, max_q_rows=18, max_kv_len=int(w.kv_len_verify.max()))
    assert sd.sd_attention_workspace_size(sd.SD_ATTN_VERIFY, big, kv) > \
        sd.SD_VERIFY_NOALLOC_SCRATCH_BYTES
    out = torch.zeros_like(q.q)
    with pytest.raises(sd.SdError) as e:
        sd.sd_verify_attention_noalloc(big, kv, out)
    assert e.value.status == sd.SD_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert not out.any()  # nothing was launched
