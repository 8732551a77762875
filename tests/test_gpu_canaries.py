"""Writes stay inside their buffers: every output and workspace of every call sits between two
4 KB guard zones filled with a byte pattern, and the guards must be intact after the call (a
write past the end or before the start of an output, a workspace overrun, would change them).
"""
import numpy as np
import pytest
import torch

from speculative_decoding_attention_verify_b200 import device as dev
from speculative_decoding_attention_verify_b200 import inputs as gen
from speculative_decoding_attention_verify_b200 import sdattn as sd

pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5


class Guarded:
    """A tensor of `shape`/`dtype` carved out of a larger byte buffer with guard zones (the
    start of the tensor stays 256-byte aligned)."""

    def __init__(self, shape, dtype, fill=None):
        esz = torch.empty(0, dtype=dtype).element_size()
        n = int(np.prod(shape)) if len(shape) else 1
        self.nbytes = n * esz
        self.raw = torch.full((GUARD + self.nbytes + GUARD,), PATTERN, dtype=torch.uint8,
                              device="cuda")
        self.t = self.raw[GUARD:GUARD + self.nbytes].view(dtype).view(shape)
        if fill is not None:
            self.t.fill_(fill)

    def intact(self):
        torch.cuda.synchronize()
        return bool((self.raw[:GUARD] == PATTERN).all()) and \
            bool((self.raw[GUARD + self.nbytes:] == PATTERN).all())


def _ws(nbytes):
    return Guarded((max(int(nbytes), 16),), torch.uint8)


@pytest.mark.parametrize("cfg,kw", [(1, dict(l_vis=3000, l_txt=200)),
                                    (4, dict(l_vis=800, l_txt=100, batch=3)),
                                    (0, {})])
def test_attention_calls_stay_inside_their_buffers(cfg, kw):
    w = gen.make_attn_workload(cfg, **kw)
    kv, q = dev.kv_cache(w), dev.verify_queries(w)
    dt = torch.bfloat16 if w.dtype == gen.BF16 else torch.float32
    out, ws = Guarded(tuple(q.q.shape), dt), _ws(sd.sd_attention_workspace_size(sd.SD_ATTN_VERIFY, q, kv))
    sd.sd_verify_attention(q, kv, out=out.t, workspace=ws.t)
    assert out.intact() and ws.intact()
    lens = w.kv_len_draft(0)
    kvd, qd = dev.kv_cache(w, kv_len=lens), dev.draft_queries(w, 0)
    out = Guarded(tuple(qd.q.shape), dt)
    ws = _ws(sd.sd_attention_workspace_size(sd.SD_ATTN_TEXT_ANCHORED, qd, kvd))
    sd.sd_text_anchored_attention(qd, kvd, dev.int32(np.zeros(w.n_seq)), dev.int32(w.l_vis),
                                  dev.int32(w.window), int(w.window.max()), out=out.t,
                                  workspace=ws.t)
    assert out.intact() and ws.intact()
    k = min(w.topk, int(w.l_vis.min()))
    idx = Guarded((w.n_seq, w.h_kv, k), torch.int32)
    ws = _ws(sd.sd_topk_workspace_size(kv, int(w.l_vis.max()), k))
    sd.sd_topk_select(q, kv, dev.int32(np.zeros(w.n_seq)), dev.int32(w.l_vis), int(w.l_vis.max()),
                      k, idx_out=idx.t, workspace=ws.t)
    assert idx.intact() and ws.intact()
    tail = dev.int32(w.l_vis)
    max_tail = int((lens - w.l_vis).max())
    out = Guarded(tuple(qd.q.shape), dt)
    ws = _ws(sd.sd_sparse_workspace_size(qd, kvd, k, max_tail))
    sd.sd_sparse_attention(qd, kvd, idx.t, tail, max_tail, out=out.t, workspace=ws.t)
    assert out.intact() and ws.intact()
    if w.dtype == gen.BF16:
        sel = Guarded((max(sd.sd_sparse_selection_size(kvd, k), 16),), torch.uint8)
        # the selection must start 256-byte aligned: the guard keeps the offset a multiple of 4 KB
        sd.sd_sparse_stage(kvd, idx.t, tail, selection=sel.t)
        out = Guarded(tuple(qd.q.shape), dt)
        ws = _ws(sd.sd_sparse_workspace_size(qd, kvd, k, max_tail))
        sd.sd_sparse_attention_staged(qd, kvd, sel.t, k, tail, max_tail, out=out.t,
                                      workspace=ws.t)
        assert sel.intact() and out.intact() and ws.intact()
        qt, qs = gen.make_text_queries(w)
        qp = dev.queries(qt, qs, w.dtype, int(w.ctx_len.max()))
        kvp = dev.kv_cache(w, kv_len=w.ctx_len)
        idx = Guarded((w.n_seq, w.h_kv, k), torch.int32)
        sc = Guarded((w.n_seq, w.h_kv, int(w.l_vis.max())), torch.float64)
        ws = _ws(sd.sd_topk_scored_workspace_size(sd.SD_TOPK_MEAN_TEXT_ATTENTION, qp, kvp,
                                                  int(w.l_vis.max()), k))
        sd.sd_topk_select_scored(sd.SD_TOPK_MEAN_TEXT_ATTENTION, qp, kvp,
                                 dev.int32(np.zeros(w.n_seq)), dev.int32(w.l_vis),
                                 int(w.l_vis.max()), k, idx_out=idx.t, scores_out=sc.t,
                                 workspace=ws.t)
        assert idx.intact() and sc.intact() and ws.intact()


def test_hsr_and_acceptance_stay_inside_their_buffers():
    hw = gen.make_hsr_workload(n=3, d_model=1024, with_bias=True)
    y = Guarded((3, 1024), torch.bfloat16)
    sd.sd_hsr_project(dev.tensor(hw.emb, gen.BF16), dev.tensor(hw.hid, gen.BF16),
                      dev.tensor(hw.weight, gen.BF16), dev.tensor(hw.bias, gen.BF16), out=y.t)
    assert y.intact()
    aw = gen.make_accept_workload(4, batch=5, vocab=50000)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    B, gm = aw.batch, aw.gamma_max
    ws = _ws(sd.sd_accept_workspace_size(B, gm, aw.vocab))
    n, out = Guarded((B,), torch.int32), Guarded((B, gm + 1), torch.int32)
    sd.sd_accept_greedy(t(aw.target_logits), t(aw.draft_tokens_greedy), t(aw.gamma), gm,
                        n_acc=n.t, out_tok=out.t, workspace=ws.t)
    assert n.intact() and out.intact() and ws.intact()
    near = Guarded((B,), torch.int32)
    sd.sd_accept_sample(t(aw.target_logits), t(aw.draft_logits), t(aw.draft_tokens_sampled),
                        t(aw.u), t(aw.v), t(aw.gamma), gm, n_acc=n.t, out_tok=out.t,
                        near_boundary=near.t, workspace=ws.t)
    assert n.intact() and out.intact() and near.intact() and ws.intact()
