"""Failure detection on the GPU without a fault: the tensor-core kernels' bounded waits.

With the wait bound set to 1 ns, the pipeline's waits run out at once: the kernel must record
SD_DEVERR_TIMEOUT in dev_err, drain its own copies and MMAs and exit, the launch must report no
CUDA error, and the device must stay usable: the next call with the default bound gives the
oracle's result and a clean flag.  Nothing here makes a wait that never ends, an invalid address
or a trap; the waits run out because their bound is shorter than the copies they wait for.
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_attention_verify_b200 import device as dev
from speculative_decoding_attention_verify_b200 import inputs as gen
from speculative_decoding_attention_verify_b200 import sdattn as sd

pytestmark = pytest.mark.gpu


@pytest.fixture
def short_wait_bound():
    prev = sd.sd_set_wait_timeout_ns(1)
    try:
        yield
    finally:
        sd.sd_set_wait_timeout_ns(prev)


def _verify_case():
    w = gen.make_attn_workload(1, l_vis=6000, l_txt=200, gamma=2)
    return w, dev.verify_queries(w), dev.kv_cache(w)


def test_expired_waits_set_the_timeout_flag_and_return(short_wait_bound):
    w, q, kv = _verify_case()
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(3):
        sd.sd_verify_attention(q, kv, dev_err=flag)
    torch.cuda.synchronize()  # raises if the kernel faulted
    assert flag.item() & sd.SD_DEVERR_TIMEOUT


def test_device_is_usable_after_expired_waits():
    w, q, kv = _verify_case()
    prev = sd.sd_set_wait_timeout_ns(1)
    try:
        flag = torch.zeros(1, dtype=torch.int32, device="cuda")
        sd.sd_verify_attention(q, kv, dev_err=flag)
        torch.cuda.synchronize()
    finally:
        sd.sd_set_wait_timeout_ns(prev)
    assert flag.item() & sd.SD_DEVERR_TIMEOUT
    flag.zero_()
    out = sd.sd_verify_attention(q, kv, dev_err=flag)
    torch.cuda.synchronize()
    assert flag.item() == 0
    ref = oracle.verify_attention(w.h_q, w.q_verify, w.q_verify_start, oracle.cache_from_workload(w))
    assert np.abs(dev.to_numpy_f64(out) - ref).max() <= 2e-2


def test_expired_waits_in_the_prefill_selection_kernels(short_wait_bound):
    w = gen.make_attn_workload(1, l_vis=1500, l_txt=130)
    qt, qs = gen.make_text_queries(w)
    q = dev.queries(qt, qs, w.dtype, int(w.ctx_len.max()))
    kv = dev.kv_cache(w, kv_len=w.ctx_len)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    sd.sd_topk_select_scored(sd.SD_TOPK_MEAN_TEXT_ATTENTION, q, kv, dev.int32([0]),
                             dev.int32(w.l_vis), int(w.l_vis[0]), 64, dev_err=flag)
    torch.cuda.synchronize()
    assert flag.item() & sd.SD_DEVERR_TIMEOUT
