#!/usr/bin/env python
"""Benchmark: one speculative-decoding cycle through libsdattn, on synthetic seeded inputs.

Default workload (the long-video Sparse-to-Dense configuration, every call of the path): 28
independent layers (H_q=28, H_kv=4, d=128, bf16, 25,000 visual + 1,024 text positions),
gamma = 8, vocab 152,064.  One *step* is one cycle:
  top-K selection (K=1024 per KV head over the visual span) and staging of the kept rows
  8 draft steps x [sparse attention, HSR projection, text-anchored attention]   28 layers each
  dense verification of the 9 new rows                                         28 layers
  greedy acceptance and speculative-sampling acceptance                        batch 1
The metric is the algorithmic bytes the step must move (KV rows, queries, outputs, weights,
logits; implementation scratch not credited) over the step's device time: "spec-decode
attention KV-read GB/s".  The step reads 4 GB (1.49 GB of KV for verification alone), far
more than the 126 MB L2, so no flush is needed between steps; each of the 8 HSR projections
reads its own copy of the 51.4 MB weight.

Besides the headline the JSON line carries, per call kind, a roofline measured with L2
flushed before every call (`rooflines`), one-layer latencies, the cycle of each drafting
method against plain decoding (gamma single-row dense decode steps), the end-to-end figure
through the public API with host buffers, and the fp64 oracle timed on the host.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config C]

``--config 0..4`` prints the line of another workload instead (its own set of calls).  With
N > 1 (torchrun) every rank runs its own replica; the path has no exchange step, so there is
no data-path collective (time is the max over ranks).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "spec-decode attention KV-read GB/s (% of B200 HBM peak) at 25k vis tokens"
DEFAULT_CONFIG = 3
NOMINAL_HBM_GBS = 8000.0
FLUSH_BYTES = 1 << 30        # written before every separately timed call (L2 is 126 MB)
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "ncu_traffic.json")

# Calls of each workload's cycle.  sparse: "staged" (selection staged once per cycle, bf16),
# "direct" (gathered by every call) or None; draft_steps None means the workload's gamma.
SPECS = {
    0: dict(topk=True, sparse="direct", ta=True, hsr=False, accept=True, draft_steps=None),
    1: dict(topk=False, sparse=None, ta=True, hsr=True, accept=False, draft_steps=None),
    2: dict(topk=False, sparse=None, ta=True, hsr=True, accept=True, draft_steps=None),
    3: dict(topk=True, sparse="staged", ta=True, hsr=True, accept=True, draft_steps=None),
    4: dict(topk=True, sparse=None, ta=True, hsr=False, accept=True, draft_steps=1),
}

KERNELS = {  # call kind -> the library kernels one call launches
    "topk": "topk_score_fast_kernel + topk_select_fast_kernel",
    "stage": "sparse_compact_kernel",
    "sparse": "attn_tc_kernel (+ attn_merge_kernel when split)",
    "sparse_direct": "attn_* engine (+ attn_merge_kernel when split)",
    "hsr": "hsr_ring_kernel",
    "text_anchored": "attn_tc_kernel (+ attn_merge_kernel when split)",
    "verify": "attn_tc_persist_kernel + attn_merge_kernel (persistent plan)",
    "accept_greedy": "accept_argmax_kernel + accept_greedy_kernel",
    "accept_sample": "accept_stats/decide/wsum/draw kernels",
}


def env_rank():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def peak_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def strip_comments(src):
    """C/C++/CUDA source without its comments and with whitespace runs collapsed, so that a
    change to comments or layout alone leaves the hash of the code unchanged."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":  # string or character literal, escapes included
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash():
    """Hash of the library's code: every CUDA/C++ source and header of the package and the
    public header (comments and layout excluded), so that a change to any kernel or to the
    planner invalidates recorded counters."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "speculative_decoding_attention_verify_b200", "csrc")
    files = [os.path.join(csrc, n) for n in sorted(os.listdir(csrc))
             if n.endswith((".cu", ".cuh", ".h", ".cpp"))]
    files.append(os.path.join(ROOT, "include", "sd_attn.h"))
    for path in files:
        with open(path) as f:
            h.update(strip_comments(f.read()).encode())
    return h.hexdigest()[:12]


def recorded_traffic():
    """DRAM bytes (read + write) per launch of each call kind, from the committed ncu record,
    for the entries taken on the current code; {} when none matches."""
    try:
        with open(TRAFFIC_RECORD) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return {}
    want = kernel_source_hash()
    return {k: float(v["traffic_bytes_per_launch"]) for k, v in rec.get("calls", {}).items()
            if v.get("source_hash") == want}


# ---------------------------------------------------------------- algorithmic bytes --------

def call_bytes(w, kind, step=0, topk=None, hsr_d=None, aw=None):
    """Bytes one call must move (every operand it reads or writes once; scratch and staging
    not credited).  w: the attention workload; step: the draft step (0-based)."""
    d, hk, hq = w.d, w.h_kv, w.h_q
    s = 2 if w.dtype == "bf16" else 4
    row = hk * d * 2 * s  # K and V of one position, all KV heads
    L = w.n_seq
    qo = 2 * hq * d * s   # one query row in, one output row out
    nonvis = (w.l_txt + step + 1).astype(np.int64)  # text positions + the draft's own
    if kind == "verify":
        return int(w.kv_len_verify.astype(np.int64).sum()) * row + int(w.n_q_verify.sum()) * qo
    if kind == "text_anchored":
        return int(np.minimum(w.window, nonvis).sum()) * row + L * qo
    if kind in ("sparse", "sparse_direct"):
        kept = np.minimum(topk, w.l_vis).astype(np.int64)
        return int((kept + nonvis).sum()) * row + L * hk * topk * 4 + L * qo
    if kind == "topk":
        return int(w.l_vis.astype(np.int64).sum()) * hk * d * s + L * hq * d * s + L * hk * topk * 4
    if kind == "stage":  # staging copy of the kept rows (implementation traffic, not credited)
        kept = int(np.minimum(topk, w.l_vis).sum())
        return 2 * kept * row + L * hk * topk * 4
    if kind == "hsr":
        return hsr_d * 2 * hsr_d * 2 + 3 * hsr_d * 2
    g = aw.gamma.astype(np.int64)
    V = aw.vocab
    if kind == "accept_greedy":
        return int((g + 1).sum()) * V * 4 + int(g.sum()) * 4
    if kind == "accept_sample":
        return int((2 * g + 1).sum()) * V * 4 + 2 * V * 4 * aw.batch + int(g.sum()) * 8 + \
            int((g + 1).sum()) * 4
    raise ValueError(kind)


# ---------------------------------------------------------------- the GPU cycle ------------

class Cycle:
    """Device tensors and the ordered calls of one cycle of workload `cfg`.

    Per-step inputs that a caller would bring from the host (queries, embeddings, logits,
    drafted tokens, uniforms) exist twice on the device, so that the end-to-end run can copy
    the next step's inputs while the current step computes; `step(stream, buf)` uses set
    `buf`.  Everything else (caches, selection, workspaces, outputs) exists once."""

    def __init__(self, cfg, device):
        import torch
        from speculative_decoding_attention_verify_b200 import device as dev
        from speculative_decoding_attention_verify_b200 import inputs as gen
        from speculative_decoding_attention_verify_b200 import sdattn as sd
        self.torch, self.sd, self.dev, self.gen = torch, sd, dev, gen
        self.cfg, self.spec = cfg, SPECS[cfg]
        w = gen.make_attn_workload(cfg)
        self.w = w
        L = w.n_seq
        self.g = int(self.spec["draft_steps"] or w.gamma_max)
        i32 = lambda a: dev.int32(np.asarray(a), device)
        self.k = dev.tensor(w.k, w.dtype, device)
        self.v = dev.tensor(w.v, w.dtype, device)
        kvc = lambda lens: dev.kv_cache(w, kv_len=lens, device=device, k=self.k, v=self.v)
        self.kv_verify = kvc(w.kv_len_verify)
        self.kv_draft = [kvc(w.kv_len_draft(t)) for t in range(self.g)]
        # Sparrow's draft attends to its own keys and values (those of the draft layer), not to
        # the rows the Sparse-to-Dense draft reads in the same step: when both drafts run, the
        # text-anchored calls read a copy of the cache, so no byte that one call of a draft step
        # reads is credited again to a second call of that step (where L2 would serve it)
        self.kv_ta = self.kv_draft
        if self.spec["ta"] and self.spec["sparse"]:
            self.k_ta, self.v_ta = self.k.clone(), self.v.clone()
            self.kv_ta = [dev.kv_cache(w, kv_len=w.kv_len_draft(t), device=device, k=self.k_ta,
                                       v=self.v_ta) for t in range(self.g)]
        self.topk = w.topk
        # per-step inputs, two sets
        self.q_verify = [dev.verify_queries(w, device) for _ in range(2)]
        self.q_draft = [[dev.draft_queries(w, t, device) for t in range(self.g)] for _ in range(2)]
        self.cand_b, self.cand_e = i32(np.zeros(L)), i32(w.l_vis)
        self.max_cand = int(w.l_vis.max())
        self.tail = i32(w.l_vis)
        self.vis_b, self.vis_e, self.win = i32(np.zeros(L)), i32(w.l_vis), i32(w.window)
        self.max_win = int(w.window.max())
        self.max_tail = int(max(int((w.kv_len_draft(t) - w.l_vis).max()) for t in range(self.g)))
        self.idx = torch.empty((L, w.h_kv, w.topk), dtype=torch.int32, device=device)
        mk = lambda n: torch.empty(max(int(n), 16), dtype=torch.uint8, device=device)
        self.ws_verify = mk(sd.sd_attention_workspace_size(sd.SD_ATTN_VERIFY, self.q_verify[0],
                                                           self.kv_verify))
        self.ws_ta = mk(sd.sd_attention_workspace_size(sd.SD_ATTN_TEXT_ANCHORED,
                                                       self.q_draft[0][-1], self.kv_ta[-1]))
        self.o_verify = torch.empty_like(self.q_verify[0].q)
        self.o_draft = [torch.empty_like(q.q) for q in self.q_draft[0]]
        self.o_ta = [torch.empty_like(q.q) for q in self.q_draft[0]]
        if self.spec["topk"]:
            self.ws_topk = mk(sd.sd_topk_workspace_size(self.kv_verify, self.max_cand, w.topk))
        if self.spec["sparse"]:
            self.ws_sparse = mk(sd.sd_sparse_workspace_size(self.q_draft[0][-1],
                                                            self.kv_draft[-1], w.topk,
                                                            self.max_tail))
        if self.spec["sparse"] == "staged":
            self.sel = mk(sd.sd_sparse_selection_size(self.kv_draft[0], w.topk))
        self.hsr_d = None
        if self.spec["hsr"]:
            hw = gen.make_hsr_workload(n=1)
            self.hsr_d = hw.d_model
            base = dev.tensor(hw.weight, gen.BF16, device)
            # one weight copy per draft step: 8 x 51.4 MB, so no projection finds its weight
            # in L2
            self.W = [base] + [base.clone() for _ in range(self.g - 1)]
            self.emb = [[dev.tensor(hw.emb, gen.BF16, device) for _ in range(self.g)]
                        for _ in range(2)]
            self.hid = dev.tensor(hw.hid, gen.BF16, device)
            self.y = [torch.empty((1, hw.d_model), dtype=torch.bfloat16, device=device)
                      for _ in range(self.g)]
        self.aw = None
        if self.spec["accept"]:
            if cfg in (2, 3):  # one sequence whose 28 layers were attended above
                aw = gen.make_accept_workload(2, gammas=[self.g], batch=1)
            else:
                aw = gen.make_accept_workload(cfg, gammas=w.gamma)
            self.aw = aw
            t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
            self.acc_in = [dict(tgt=t(aw.target_logits), drf=t(aw.draft_logits),
                                tok_s=t(aw.draft_tokens_sampled),
                                tok_g=t(aw.draft_tokens_greedy), u=t(aw.u), v=t(aw.v))
                           for _ in range(2)]
            self.gam = t(aw.gamma)
            self.gmax = int(aw.gamma.max())
            B = aw.batch
            self.ws_acc = mk(sd.sd_accept_workspace_size(B, self.gmax, aw.vocab))
            # the greedy rule's own workspace: the two rules may run at the same time
            self.ws_acc_g = mk(sd.sd_accept_workspace_size(B, self.gmax, aw.vocab))
            # the step's results, views of one buffer (one device-to-host copy brings them back)
            nt = B * (self.gmax + 1)
            self.results = torch.empty(3 * B + 2 * nt, dtype=torch.int32, device=device)
            r = self.results
            self.n_acc_g = r[0:B]
            self.out_g = r[B:B + nt].view(B, self.gmax + 1)
            self.n_acc_s = r[B + nt:2 * B + nt]
            self.out_s = r[2 * B + nt:2 * B + 2 * nt].view(B, self.gmax + 1)
            self.near = r[2 * B + 2 * nt:3 * B + 2 * nt]
        self.calls = self._calls()
        self.side = torch.cuda.Stream(device)
        self.events = [torch.cuda.Event() for _ in range(4)]
        self.bytes = {}
        for kind, step, _ in self.calls:
            if kind == "stage":
                continue
            self.bytes[kind] = self.bytes.get(kind, 0) + self.call_bytes(kind, step)

    def call_bytes(self, kind, step=0):
        return call_bytes(self.w, kind, step, topk=self.topk, hsr_d=self.hsr_d, aw=self.aw)

    # ---- the calls, in cycle order: (kind, draft step, fn(stream, buf)) ----
    def _calls(self):
        sd, sp = self.sd, self.spec
        calls = []
        if sp["topk"]:
            calls.append(("topk", 0, lambda s, b: sd.sd_topk_select(
                self.q_verify[b], self.kv_verify, self.cand_b, self.cand_e, self.max_cand,
                self.topk, idx_out=self.idx, workspace=self.ws_topk, stream=s)))
        if sp["sparse"] == "staged":
            calls.append(("stage", 0, lambda s, b: sd.sd_sparse_stage(
                self.kv_draft[0], self.idx, self.tail, selection=self.sel, stream=s)))
        for t in range(self.g):
            if sp["sparse"] == "staged":
                calls.append(("sparse", t, lambda s, b, t=t: sd.sd_sparse_attention_staged(
                    self.q_draft[b][t], self.kv_draft[t], self.sel, self.topk, self.tail,
                    self.max_tail, out=self.o_draft[t], workspace=self.ws_sparse, stream=s)))
            elif sp["sparse"] == "direct":
                calls.append(("sparse_direct", t, lambda s, b, t=t: sd.sd_sparse_attention(
                    self.q_draft[b][t], self.kv_draft[t], self.idx, self.tail, self.max_tail,
                    out=self.o_draft[t], workspace=self.ws_sparse, stream=s)))
            if sp["hsr"]:
                calls.append(("hsr", t, lambda s, b, t=t: sd.sd_hsr_project(
                    self.emb[b][t], self.hid, self.W[t], out=self.y[t], stream=s)))
            if sp["ta"]:
                calls.append(("text_anchored", t, lambda s, b, t=t: sd.sd_text_anchored_attention(
                    self.q_draft[b][t], self.kv_ta[t], self.vis_b, self.vis_e, self.win,
                    self.max_win, out=self.o_ta[t], workspace=self.ws_ta, stream=s)))
        calls.append(("verify", 0, lambda s, b: sd.sd_verify_attention(
            self.q_verify[b], self.kv_verify, out=self.o_verify, workspace=self.ws_verify,
            stream=s)))
        if sp["accept"]:
            calls.append(("accept_greedy", 0, lambda s, b: sd.sd_accept_greedy(
                self.acc_in[b]["tgt"], self.acc_in[b]["tok_g"], self.gam, self.gmax,
                n_acc=self.n_acc_g, out_tok=self.out_g, workspace=self.ws_acc_g, stream=s)))
            calls.append(("accept_sample", 0, lambda s, b: sd.sd_accept_sample(
                self.acc_in[b]["tgt"], self.acc_in[b]["drf"], self.acc_in[b]["tok_s"],
                self.acc_in[b]["u"], self.acc_in[b]["v"], self.gam, self.gmax,
                n_acc=self.n_acc_s, out_tok=self.out_s, near_boundary=self.near,
                workspace=self.ws_acc, stream=s)))
        return calls

    def step(self, stream=None, buf=0, kinds=None):
        """Issues the cycle's calls on `stream` (None: the current stream), with input set
        `buf`.  With `kinds`, only those calls, in order on the one stream.

        The whole cycle is two chains that only verification joins: Sparse-to-Dense's (top-K,
        staging, the sparse draft steps) and Sparrow's (the HSR projection and text-anchored
        attention of every draft step); after verification the greedy and the sampling rule
        read the same logits, independently.  Sparrow's chain and the greedy rule run on a
        second stream, forked from and joined back to `stream` through events (a CUDA graph
        captured from the step holds the same edges), so one method's calls fill the SMs and
        the HBM time the other's leave idle (a call's start, its last tiles).  Every chain
        keeps its own order, and the results are those of the one-stream order."""
        if kinds is not None:
            for kind, _, fn in self.calls:
                if kind in kinds:
                    fn(stream, buf)
            return
        torch = self.torch
        main = stream if stream is not None else torch.cuda.current_stream()
        side, ev = self.side, self.events
        ev[0].record(main)
        side.wait_event(ev[0])
        for kind, _, fn in self.calls:
            if kind in ("hsr", "text_anchored"):
                fn(side, buf)
            elif kind == "verify":
                ev[1].record(side)
                main.wait_event(ev[1])
                fn(main, buf)
            elif kind == "accept_greedy":
                ev[2].record(main)
                side.wait_event(ev[2])
                fn(side, buf)
            else:
                fn(main, buf)
        ev[3].record(side)
        main.wait_event(ev[3])

    def decode_step_calls(self):
        """Plain decoding of the draft steps' tokens: each token is one dense single-row
        attention over the whole cache (verification attention with n_q = 1)."""
        sd = self.sd
        return [lambda s, t=t: sd.sd_verify_attention(
            self.q_draft[0][t], self.kv_draft[t], out=self.o_draft[t], workspace=self.ws_verify,
            stream=s) for t in range(self.g)]

    def one_layer(self, kind):
        """A call of `kind` over the first layer (sequence) alone: the one-launch-per-layer
        latency."""
        sd, dev, w = self.sd, self.dev, self.w
        if w.paged or w.n_seq == 1:
            return None
        k1, v1 = self.k[:1], self.v[:1]
        torch = self.torch
        dvc = self.k.device
        lens = w.kv_len_verify if kind == "verify" else w.kv_len_draft(0)
        kv = sd.KVCache(k1, v1, torch.tensor(lens[:1], dtype=torch.int32, device=dvc))
        if kind == "verify":
            nq = int(w.n_q_verify[0])
            q = sd.Queries(self.q_verify[0].q[:nq], torch.tensor([0, nq], dtype=torch.int32,
                                                                  device=dvc), nq, int(lens[0]))
            out = torch.empty_like(q.q)
            return lambda s: sd.sd_verify_attention(q, kv, out=out, workspace=self.ws_verify,
                                                    stream=s)
        q = sd.Queries(self.q_draft[0][0].q[:1], torch.tensor([0, 1], dtype=torch.int32,
                                                               device=dvc), 1, int(lens[0]))
        out = torch.empty_like(q.q)
        if kind == "text_anchored":
            return lambda s: sd.sd_text_anchored_attention(
                q, kv, self.vis_b[:1], self.vis_e[:1], self.win[:1], self.max_win, out=out,
                workspace=self.ws_ta, stream=s)
        if kind == "sparse" and self.spec["sparse"] == "staged":
            sel = self.torch.empty(max(sd.sd_sparse_selection_size(kv, self.topk), 16),
                                   dtype=torch.uint8, device=dvc)
            sd.sd_sparse_stage(kv, self.idx[:1].contiguous(), self.tail[:1], selection=sel)
            ws = self.torch.empty(max(sd.sd_sparse_workspace_size(q, kv, self.topk,
                                                                  self.max_tail), 16),
                                  dtype=torch.uint8, device=dvc)
            return lambda s: sd.sd_sparse_attention_staged(q, kv, sel, self.topk,
                                                           self.tail[:1], self.max_tail,
                                                           out=out, workspace=ws, stream=s)
        return None

    def count_graph_kernels(self, graph):
        """Kernel nodes of a captured CUDA graph (every kernel of the cycle is libsdattn's); from
        the call structure when the graph's nodes cannot be read."""
        try:
            from cuda.bindings import runtime as rt
            h = rt.cudaGraph_t(init_value=int(graph.raw_cuda_graph()))
            err, _, n = rt.cudaGraphGetNodes(h, 0)
            err2, nodes, n = rt.cudaGraphGetNodes(h, n)
            if err == rt.cudaError_t.cudaSuccess and err2 == rt.cudaError_t.cudaSuccess:
                kernel = rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
                return sum(1 for nd in nodes[:n] if rt.cudaGraphNodeGetType(nd)[1] == kernel)
        except Exception:  # noqa: BLE001 - counted from the call structure below instead
            pass
        per_call = {"topk": 2, "stage": 1, "sparse": 2, "sparse_direct": 3, "hsr": 1,
                    "text_anchored": 2, "verify": 2, "accept_greedy": 2, "accept_sample": 4}
        return sum(per_call[k] for k, _, _ in self.calls)  # upper bound (merges counted)


def capture(torch, fn):
    """Warm fn up eagerly, then capture one call of fn(stream) in a CUDA graph."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn(s)
        fn(s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph(keep_graph=True)  # the node list stays readable
    with torch.cuda.graph(graph, stream=s):
        fn(s)
    graph.instantiate()
    torch.cuda.synchronize()
    return graph


def time_graph(torch, graph, reps, warmup=3):
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


class Flusher:
    """Writes a buffer larger than L2 before a separately timed call, and times the call with
    CUDA events on the launching stream.  The write (~0.15 ms) also gives the host time to
    enqueue the call before the GPU reaches the first event."""

    def __init__(self, torch, device):
        self.torch = torch
        self.buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)

    def time_calls(self, fn, reps):
        torch = self.torch
        s = torch.cuda.current_stream()
        evs = []
        for _ in range(reps):
            self.buf.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            fn(s)
            e1.record(s)
            evs.append((e0, e1))
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs]


class Rotations:
    """Copies of a cycle's buffers for back-to-back timing of one call kind: consecutive calls
    read different memory, so that no call finds its operands in L2 (the rotation spans enough
    distinct buffers to exceed 4x the L2).  Rotation 0 is the cycle's own buffers;
    the others are clones on the device (the values do not change the work)."""

    def __init__(self, cyc, n_kv, n_small):
        torch, sd, dev, w = cyc.torch, cyc.sd, cyc.dev, cyc.w
        self.cyc = cyc
        dvc = cyc.k.device
        self.k = [cyc.k] + [cyc.k.clone() for _ in range(n_kv - 1)]
        self.v = [cyc.v] + [cyc.v.clone() for _ in range(n_kv - 1)]
        kvc = lambda lens, r: dev.kv_cache(w, kv_len=lens, device=dvc, k=self.k[r], v=self.v[r])
        self.kv_verify = [kvc(w.kv_len_verify, r) for r in range(n_kv)]
        self.kv_draft = [kvc(w.kv_len_draft(0), r) for r in range(n_kv)]
        self.sel = None
        if cyc.spec["sparse"] == "staged":
            self.sel = [cyc.sel] + [torch.empty_like(cyc.sel) for _ in range(n_kv - 1)]
            for r in range(1, n_kv):
                sd.sd_sparse_stage(self.kv_draft[r], cyc.idx, cyc.tail, selection=self.sel[r])
        self.W = None
        if cyc.spec["hsr"]:
            self.W = list(cyc.W) + [cyc.W[0].clone() for _ in range(max(0, n_small - len(cyc.W)))]
        self.acc = None
        if cyc.aw is not None:
            self.acc = [cyc.acc_in[0]] + [{k: v.clone() for k, v in cyc.acc_in[0].items()}
                                          for _ in range(n_small - 1)]
        torch.cuda.synchronize()

    def call(self, kind, r):
        """Draft step 0's call of `kind` on rotation r."""
        c, sd = self.cyc, self.cyc.sd
        if kind == "verify":
            return lambda s: sd.sd_verify_attention(c.q_verify[0], self.kv_verify[r],
                                                    out=c.o_verify, workspace=c.ws_verify,
                                                    stream=s)
        if kind == "topk":
            return lambda s: sd.sd_topk_select(c.q_verify[0], self.kv_verify[r], c.cand_b,
                                               c.cand_e, c.max_cand, c.topk, idx_out=c.idx,
                                               workspace=c.ws_topk, stream=s)
        if kind == "stage":
            return lambda s: sd.sd_sparse_stage(self.kv_draft[r], c.idx, c.tail,
                                                selection=self.sel[r], stream=s)
        if kind == "sparse":
            return lambda s: sd.sd_sparse_attention_staged(
                c.q_draft[0][0], self.kv_draft[r], self.sel[r], c.topk, c.tail, c.max_tail,
                out=c.o_draft[0], workspace=c.ws_sparse, stream=s)
        if kind == "sparse_direct":
            return lambda s: sd.sd_sparse_attention(c.q_draft[0][0], self.kv_draft[r], c.idx,
                                                    c.tail, c.max_tail, out=c.o_draft[0],
                                                    workspace=c.ws_sparse, stream=s)
        if kind == "text_anchored":
            return lambda s: sd.sd_text_anchored_attention(
                c.q_draft[0][0], self.kv_draft[r], c.vis_b, c.vis_e, c.win, c.max_win,
                out=c.o_ta[0], workspace=c.ws_ta, stream=s)
        if kind == "hsr":
            return lambda s: sd.sd_hsr_project(c.emb[0][0], c.hid, self.W[r], out=c.y[0],
                                               stream=s)
        a = self.acc[r]
        if kind == "accept_greedy":
            return lambda s: sd.sd_accept_greedy(a["tgt"], a["tok_g"], c.gam, c.gmax,
                                                 n_acc=c.n_acc_g, out_tok=c.out_g,
                                                 workspace=c.ws_acc, stream=s)
        return lambda s: sd.sd_accept_sample(a["tgt"], a["drf"], a["tok_s"], a["u"], a["v"],
                                             c.gam, c.gmax, n_acc=c.n_acc_s, out_tok=c.out_s,
                                             near_boundary=c.near, workspace=c.ws_acc,
                                             stream=s)


def rotations_needed(nbytes, l2_bytes, cap):
    """Distinct buffer sets so that consecutive calls span more than 4x the L2."""
    return int(min(cap, max(1, -(-4 * l2_bytes // max(int(nbytes), 1)))))


def roofline_entries(cyc, flusher, peak, traffic, reps, max_kv_rot=10, max_small_rot=16):
    """One entry per call kind.  launch_us: back-to-back calls replayed from a CUDA graph over
    rotated buffer sets (more than 4x the L2 between two uses of a set), per-call time =
    replay time / calls, median and p10/p90 over `reps` replays.  cold_launch_us: one call at
    a time with L2 flushed before it (a single call's latency from an idle device)."""
    torch = cyc.torch
    l2 = torch.cuda.get_device_properties(cyc.k.device).L2_cache_size
    kinds = []
    for kind, step, _ in cyc.calls:
        if kind not in kinds:
            kinds.append(kind)
    per_call = {k: statistics.mean(cyc.call_bytes(k, st) for kk, st, _ in cyc.calls if kk == k)
                for k in kinds}
    moved = dict(per_call)
    if "stage" in moved:
        moved["stage"] = cyc.call_bytes("stage")
    kv_kinds = ("verify", "topk", "stage", "sparse", "sparse_direct", "text_anchored")
    n_rot = {k: rotations_needed(moved[k], l2, max_kv_rot if k in kv_kinds else max_small_rot)
             for k in kinds}
    rot = Rotations(cyc, max([n_rot[k] for k in kinds if k in kv_kinds] or [1]),
                    max([n_rot[k] for k in kinds if k not in kv_kinds] or [1]))
    out = []
    for kind in kinds:
        n = n_rot[kind]
        fns = [rot.call(kind, r) for r in range(n)]
        calls = 2 * n
        g = capture(torch, lambda s, fns=fns: [f(s) for f in fns + fns])
        times = []
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) / calls)
        del g
        cold = statistics.median(flusher.time_calls(lambda s, f=fns[0]: f(s), 5))
        med = statistics.median(times)
        b = int(round(per_call[kind]))
        gbs = b / (med / 1e3) / 1e9
        out.append({
            "call": kind, "kernels": KERNELS[kind],
            "launches_per_step": sum(1 for k, _, _ in cyc.calls if k == kind),
            "bytes_per_launch": b, "credited": kind != "stage",
            "launch_us": round(med * 1e3, 2),
            "launch_us_p10_p90": [round(float(np.percentile(times, 10)) * 1e3, 2),
                                  round(float(np.percentile(times, 90)) * 1e3, 2)],
            "achieved_gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
            "frac_of_8TBps": round(gbs / NOMINAL_HBM_GBS, 4),
            "rotations": n, "rotated_bytes": int(n * moved[kind]),
            "cold_launch_us": round(cold * 1e3, 2),
            "traffic": traffic.get(kind)})
    del rot
    torch.cuda.empty_cache()
    return out


def plain_decoding(cyc, torch, reps):
    """Cycle of each drafting method against plain decoding, both replayed as CUDA graphs.

    Plain decoding spends one dense single-row attention over the whole cache per token.  A
    cycle yields n + 1 tokens (n accepted drafts plus the target's own next token); the
    attention-path speed-up at acceptance n is (n + 1) * t_token / t_cycle.  Only the
    attention and acceptance calls are timed: the models' other layers are outside this path."""
    sp = cyc.spec
    g = cyc.g
    res = {"decode_steps": g}
    dec = cyc.decode_step_calls()
    gd = capture(torch, lambda s: [f(s) for f in dec])
    t_dec = time_graph(torch, gd, reps) / g
    w = cyc.w
    row = w.h_kv * w.d * 2 * (2 if w.dtype == "bf16" else 4)
    tok_bytes = statistics.mean(int(w.kv_len_draft(t).astype(np.int64).sum()) * row
                                for t in range(g))
    res["plain_ms_per_token"] = round(t_dec, 4)
    res["plain_kv_bytes_per_token"] = int(tok_bytes)
    res["plain_gbs"] = round(tok_bytes / (t_dec / 1e3) / 1e9, 1)
    methods = {}
    if sp["sparse"]:
        methods["sparse_to_dense"] = ("topk", "stage", "sparse", "sparse_direct", "verify",
                                      "accept_greedy")
    if sp["ta"] and sp["hsr"]:
        methods["sparrow"] = ("hsr", "text_anchored", "verify", "accept_greedy")
    for name, kinds in methods.items():
        gc = capture(torch, lambda s, kinds=kinds: cyc.step(s, 0, kinds))
        t_cyc = time_graph(torch, gc, reps)
        byt = sum(cyc.call_bytes(k, st) for k, st, _ in cyc.calls if k in kinds and k != "stage")
        methods[name] = {
            "calls": [k for k in kinds if any(c[0] == k for c in cyc.calls)],
            "ms_per_cycle": round(t_cyc, 4), "bytes_per_cycle": int(byt),
            "kv_bytes_per_token_at_n": {str(n): int(byt / (n + 1)) for n in range(g + 1)},
            "speedup_at_n": {str(n): round((n + 1) * t_dec / t_cyc, 3) for n in range(g + 1)},
            "break_even_n": next((n for n in range(g + 1) if (n + 1) * t_dec >= t_cyc), None)}
        del gc
    if sp["ta"] and sp["hsr"] and cyc.w.dtype == "bf16" and cyc.w.d == 128:
        dl = DraftLayerSteps(cyc)
        kinds = ("verify", "accept_greedy")
        gc = capture(torch, lambda s: ([f(s) for f in dl.calls] + [cyc.step(s, 0, kinds)]))
        t_cyc = time_graph(torch, gc, reps)
        gl = capture(torch, lambda s: [f(s) for f in dl.calls])
        t_layer = time_graph(torch, gl, reps) / g
        byt = dl.bytes_per_call * g + sum(cyc.call_bytes(k, st) for k, st, _ in cyc.calls
                                          if k in kinds)
        methods["sparrow_draft_layer"] = {
            "calls": [f"{g} x sd_draft_layer (HSR, RMSNorm, QKV + RoPE, text-anchored "
                      "attention, O projection, RMSNorm, gated MLP)", *kinds],
            "ms_per_cycle": round(t_cyc, 4), "bytes_per_cycle": int(byt),
            "draft_layer_us": round(t_layer * 1e3, 2),
            "draft_layer_bytes": int(dl.bytes_per_call),
            "draft_layer_gbs": round(dl.bytes_per_call / (t_layer / 1e3) / 1e9, 1),
            "kv_bytes_per_token_at_n": {str(n): int(byt / (n + 1)) for n in range(g + 1)},
            "speedup_at_n": {str(n): round((n + 1) * t_dec / t_cyc, 3) for n in range(g + 1)},
            "break_even_n": next((n for n in range(g + 1) if (n + 1) * t_dec >= t_cyc), None)}
        del gc, gl, dl
    res["methods"] = methods
    return res


class DraftLayerSteps:
    """One Sparrow draft layer of the 7B-like shapes (random bf16 weights, 517 MB) run for each
    of the cycle's draft steps on its own text-only cache (1,024 earlier text positions, one row
    appended per step)."""

    def __init__(self, cyc):
        from speculative_decoding_attention_verify_b200 import sdattn as sd
        torch, dev, gen = cyc.torch, cyc.dev, cyc.gen
        g = cyc.g
        w = gen.make_draft_layer_workload(n=1, l_txt=int(cyc.w.l_txt[0]))
        dvc = cyc.k.device
        t = lambda a: dev.tensor(a, gen.BF16, dvc)
        self.layer = sd.DraftLayer(w.d_model, w.h_q, w.h_kv, w.head_dim, w.d_ff, w.rms_eps,
                                   w.rope_theta, **{n: t(getattr(w, n)) for n in sd.DraftLayer.NAMES})
        cap = w.l_txt + g
        k = torch.zeros((1, w.h_kv, cap, w.head_dim), dtype=torch.bfloat16, device=dvc)
        v = torch.zeros_like(k)
        k[:, :, :w.l_txt] = t(w.k_cache[:, :, :w.l_txt])
        v[:, :, :w.l_txt] = t(w.v_cache[:, :, :w.l_txt])
        self.caches = [sd.KVCache(k, v, dev.int32([w.l_txt + i + 1], dvc)) for i in range(g)]
        self.emb = [t(w.emb) for _ in range(g)]
        self.hid = t(w.hid)
        self.y = [torch.empty((1, w.d_model), dtype=torch.bfloat16, device=dvc) for _ in range(g)]
        nb = sd.sd_draft_layer_workspace_size(self.layer, 1, self.caches[-1], cap, w.window)
        self.ws = torch.empty(nb, dtype=torch.uint8, device=dvc)
        self.calls = [lambda s, i=i: sd.sd_draft_layer(self.layer, self.emb[i], self.hid,
                                                       self.caches[i], cap, w.window,
                                                       out=self.y[i], workspace=self.ws, stream=s)
                      for i in range(g)]
        D, F, HD = w.d_model, w.d_ff, w.h_q * w.head_dim
        nqkv = (w.h_q + 2 * w.h_kv) * w.head_dim
        weights = 2 * (D * 2 * D + nqkv * D + D * HD + 2 * F * D + D * F + 2 * D + nqkv)
        window = min(w.window, w.l_txt + 1) * w.h_kv * w.head_dim * 2 * 2
        self.bytes_per_call = weights + window + 3 * D * 2 + 2 * w.h_kv * w.head_dim * 2


def long_context(torch, sd, flusher, peak, l_vis=140_000, layers=28, topk=1024, reps=3):
    """The path at an hour of video: 28 layers x 140,000 visual + 1,024 text positions (8.1 GB
    of KV, drawn on the device), each call timed with L2 flushed before it."""
    from speculative_decoding_attention_verify_b200 import inputs as gen
    L, g = layers, 8
    t = gen.make_device_workload(layers, l_vis, 1024, g)
    dvc = t["k"].device
    i32 = lambda a: torch.tensor(a, dtype=torch.int32, device=dvc)
    ctx = l_vis + 1024
    kv = lambda n: sd.KVCache(t["k"], t["v"], i32([n] * L))
    kv_verify, kv_draft = kv(ctx + g + 1), kv(ctx + 1)
    qv = sd.Queries(t["q_verify"], i32(list(range(0, L * (g + 1) + 1, g + 1))), g + 1, ctx + g + 1)
    qd = sd.Queries(t["q_draft"], i32(list(range(L + 1))), 1, ctx + 1)
    row = 4 * 128 * 2 * 2
    cb, ce, tail = i32([0] * L), i32([l_vis] * L), i32([l_vis] * L)
    idx = sd.sd_topk_select(qv, kv_verify, cb, ce, l_vis, topk)
    sel = sd.sd_sparse_stage(kv_draft, idx, tail)
    vb, ve, win = i32([0] * L), i32([l_vis] * L), i32([1024] * L)
    outs = {}
    calls = {
        "verify": (lambda s: sd.sd_verify_attention(qv, kv_verify, stream=s),
                   L * (ctx + g + 1) * row + 2 * L * (g + 1) * 28 * 128 * 2),
        "decode": (lambda s: sd.sd_verify_attention(qd, kv_draft, stream=s),
                   L * (ctx + 1) * row + 2 * L * 28 * 128 * 2),
        "topk": (lambda s: sd.sd_topk_select(qv, kv_verify, cb, ce, l_vis, topk, idx_out=idx,
                                             stream=s),
                 L * l_vis * 4 * 128 * 2 + L * 28 * 128 * 2 + L * 4 * topk * 4),
        "sparse": (lambda s: sd.sd_sparse_attention_staged(qd, kv_draft, sel, topk, tail, 1025,
                                                           stream=s),
                   L * (topk + 1025) * row + L * 4 * topk * 4 + 2 * L * 28 * 128 * 2),
        "text_anchored": (lambda s: sd.sd_text_anchored_attention(qd, kv_draft, vb, ve, win,
                                                                  1024, stream=s),
                          L * 1024 * row + 2 * L * 28 * 128 * 2),
    }
    for name, (fn, byt) in calls.items():
        fn(None)
        ms = statistics.median(flusher.time_calls(fn, reps))
        gbs = byt / (ms / 1e3) / 1e9
        outs[name] = {"launch_us": round(ms * 1e3, 1), "bytes": int(byt),
                      "achieved_gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}
    del t, sel, idx
    torch.cuda.empty_cache()
    return {"workload": f"{L} layers x ({l_vis} visual + 1024 text) positions, H_q=28, H_kv=4, "
                        "d=128, bf16, gamma 8, top-K 1024, window 1024 (device-drawn N(0,1))",
            "kv_bytes": int(L * (ctx + g + 1) * row), "calls": outs}


def peak_bf16():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def prefill_selection(cyc, torch, reps=3):
    """Sparse-to-Dense's own selection (mean text attention at prefill) over the workload's
    layers: the text rows of every layer score every visual key; timed with CUDA events.
    FLOPs: both passes' Q.K products (pass 1 over every position a row sees, pass 2 over the
    candidates), 2 * d per product."""
    sd, dev, gen, w = cyc.sd, cyc.dev, cyc.gen, cyc.w
    if w.dtype != "bf16":
        return None
    qt, qs = gen.make_text_queries(w)
    device = cyc.k.device
    q = dev.queries(qt, qs, w.dtype, int(w.ctx_len.max()), device)
    kv = dev.kv_cache(w, kv_len=w.ctx_len, device=device, k=cyc.k, v=cyc.v)
    cb = dev.int32(np.zeros(w.n_seq), device)
    ce = dev.int32(w.l_vis, device)
    max_cand = int(w.l_vis.max())
    idx = torch.empty((w.n_seq, w.h_kv, w.topk), dtype=torch.int32, device=device)
    ws = torch.empty(sd.sd_topk_scored_workspace_size(sd.SD_TOPK_MEAN_TEXT_ATTENTION, q, kv,
                                                      max_cand, w.topk),
                     dtype=torch.uint8, device=device)
    call = lambda: sd.sd_topk_select_scored(sd.SD_TOPK_MEAN_TEXT_ATTENTION, q, kv, cb, ce,
                                            max_cand, w.topk, idx_out=idx, workspace=ws)
    call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        call()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    flop = 0
    for s in range(w.n_seq):
        n_q, ctx = int(w.l_txt[s]), int(w.ctx_len[s])
        seen = sum(ctx - n_q + i + 1 for i in range(n_q))  # pass 1
        flop += w.h_q * 2 * w.d * (seen + n_q * int(w.l_vis[s]))  # + pass 2
    peak, kind = peak_bf16()
    tf = flop / (ms / 1e3) / 1e12
    return {"call": "sd_topk_select_scored (SD_TOPK_MEAN_TEXT_ATTENTION)",
            "kernels": "text_lse_tc_kernel + text_colsum_tc_kernel + topk_select_smem_kernel",
            "layers": w.n_seq, "text_rows": int(w.l_txt.max()), "visual_keys": max_cand,
            "ms": round(ms, 3), "flop": int(flop), "achieved_tflops": round(tf, 1),
            "bound": "tensor (and the exponentials)", "peak_tflops": peak,
            "peak_source": f"{kind} bf16_tflops", "frac": round(tf / peak, 4),
            "exp2_per_launch": int(flop // (2 * w.d))}


class HostIO:
    """Per-step inputs in pinned host memory and the end-to-end loop: the next step's inputs
    (the new K/V rows among them, into a device staging buffer) are copied on a second stream
    while the current step computes (two device input sets); the new K/V rows go from staging
    into the cache at the start of each step (a device copy: a host copy issued there would
    queue on the copy engine behind the next step's upload); the accepted counts and tokens
    come back at its end."""

    def __init__(self, cyc):
        torch = cyc.torch
        sets = []
        for b in range(2):
            d = [cyc.q_verify[b].q] + [q.q for q in cyc.q_draft[b]]
            if cyc.spec["hsr"]:
                d += list(cyc.emb[b])
            if cyc.aw is not None:
                d += [cyc.acc_in[b][k] for k in ("tgt", "drf", "tok_s", "tok_g", "u", "v")]
            sets.append(d)
        self.dev_sets = sets
        # one pinned host copy serves both device sets (the inputs are the same every step)
        self.host = [t.cpu().pin_memory() for t in sets[0]]
        w = cyc.w
        self.kv_rows = None
        if not w.paged:
            n_new = int(w.n_q_verify[0])
            ctx = int(w.ctx_len[0])
            assert (w.ctx_len == ctx).all() and (w.n_q_verify == n_new).all()
            self.kv_rows = (ctx, n_new,
                            cyc.k[:, :, ctx:ctx + n_new].contiguous().cpu().pin_memory(),
                            cyc.v[:, :, ctx:ctx + n_new].contiguous().cpu().pin_memory())
            # device staging of the new rows, one per input set, filled by the upload
            for b in range(2):
                sets[b] += [torch.empty_like(t, device=cyc.k.device) for t in self.kv_rows[2:]]
            self.host += list(self.kv_rows[2:])
        if cyc.aw is not None:
            self.outs = [cyc.results]  # accepted counts and tokens of both rules, near-ties
        else:
            self.outs = [cyc.o_verify]
        self.res = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in self.outs]
        self.h2d_bytes = sum(t.numel() * t.element_size() for t in self.host)
        self.d2h_bytes = sum(t.numel() * t.element_size() for t in self.res)

    def upload(self, b):
        """Copies on the current stream."""
        for h, d in zip(self.host, self.dev_sets[b]):
            d.copy_(h, non_blocking=True)

    def kv_rows_in(self, cyc, b):
        """The new K/V rows of every (layer, KV head), uploaded into staging set b, into the
        cache (a strided device copy on the current stream)."""
        if self.kv_rows is None:
            return
        ctx, n = self.kv_rows[:2]
        sk, sv = self.dev_sets[b][-2:]
        cyc.k[:, :, ctx:ctx + n].copy_(sk, non_blocking=True)
        cyc.v[:, :, ctx:ctx + n].copy_(sv, non_blocking=True)

    def download(self):
        for dst, src in zip(self.res, self.outs):
            dst.copy_(src, non_blocking=True)

    def run(self, cyc, steps, graphs=None):
        """Returns the device time of `steps` end-to-end steps (ms).  graphs: one CUDA graph of
        the step's public-API calls per input set, replayed instead of calling them eagerly."""
        torch = cyc.torch
        comp = torch.cuda.current_stream()
        copy = torch.cuda.Stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        done = [torch.cuda.Event() for _ in range(steps)]
        up = [torch.cuda.Event() for _ in range(steps)]
        e0.record(comp)
        copy.wait_event(e0)
        with torch.cuda.stream(copy):
            self.upload(0)
            up[0].record(copy)
        for k in range(steps):
            b = k % 2
            if k + 1 < steps:  # next step's inputs, once the step that last used them is done
                with torch.cuda.stream(copy):
                    if k >= 1:
                        copy.wait_event(done[k - 1])
                    self.upload((k + 1) % 2)
                    up[k + 1].record(copy)
            comp.wait_event(up[k])
            self.kv_rows_in(cyc, b)
            if graphs is None:
                cyc.step(comp, b)
            else:
                graphs[b].replay()
            self.download()
            done[k].record(comp)
        e1.record(comp)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)


def reduce_max(x: float, world: int, device=None) -> float:
    """Maximum of a per-rank scalar over all ranks (identity on one rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(bytes_per_step: int, steps: int, max_ms: float, world: int) -> float:
    """GB/s of the whole job: every rank processed its own replica in at most max_ms."""
    return world * bytes_per_step * steps / (max_ms / 1e3) / 1e9


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        busy = [s for s in sm if mx and s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def workload_config(cyc):
    w = cyc.w
    sp = cyc.spec
    calls = ["topk" if sp["topk"] else None, "stage" if sp["sparse"] == "staged" else None,
             f"{cyc.g} x draft step [" + ", ".join(x for x in (
                 "sparse" if sp["sparse"] else None, "hsr" if sp["hsr"] else None,
                 "text_anchored" if sp["ta"] else None) if x) + "]",
             "verify", "accept_greedy + accept_sample" if sp["accept"] else None]
    lv = (int(w.l_vis.min()), int(w.l_vis.max()))
    lt = (int(w.l_txt.min()), int(w.l_txt.max()))
    desc = (f"{w.name}: {w.n_seq} {'layers' if w.n_seq > 1 and not w.paged else 'sequences'}"
            f", H_q={w.h_q}, H_kv={w.h_kv}, d={w.d}, {w.dtype}, L_vis="
            f"{lv[0] if lv[0] == lv[1] else lv}, L_txt={lt[0] if lt[0] == lt[1] else lt}, "
            f"gamma={int(w.gamma_max)}" + (", paged (16)" if w.paged else "") +
            (f", top-K {w.topk}" if sp["topk"] else "") +
            (f", window {int(w.window.max())}" if sp["ta"] else "") +
            (f", vocab {cyc.aw.vocab}" if cyc.aw is not None else ""))
    return dict(workload=desc, config_index=cyc.cfg, calls=[c for c in calls if c],
                layers_or_sequences=w.n_seq, l_vis=lv, l_txt=lt, gamma=int(w.gamma_max),
                h_q=w.h_q, h_kv=w.h_kv, head_dim=w.d, kv_dtype=w.dtype,
                topk=w.topk if sp["topk"] else None,
                hsr_weight_copies=len(cyc.W) if sp["hsr"] else 0,
                vocab=cyc.aw.vocab if cyc.aw is not None else None,
                parallelism="replicas (no data-path collective)",
                streams=("2: Sparrow's chain (HSR, text-anchored) and the greedy rule on a "
                         "second stream beside Sparse-to-Dense's chain, joined at verification"))


def run_ours(args):
    import torch
    import torch.distributed as dist
    rank, world, local = env_rank()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=300))
    device = torch.device("cuda", torch.cuda.current_device())
    cyc = Cycle(args.config, device)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    max_over_ranks = lambda x: reduce_max(x, world, device)

    # ---- device-resident timing of the whole step, replayed from a CUDA graph ----
    graph = capture(torch, lambda s: cyc.step(s, 0))
    for _ in range(args.warmup):
        graph.replay()
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        ev0.record()
        for _ in range(args.steps):
            graph.replay()
        ev1.record()
        barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1))
    ms_per_step = ms / args.steps
    bytes_step = sum(cyc.bytes.values())
    value = whole_job_value(bytes_step, args.steps, ms, world)
    n_kernels = cyc.count_graph_kernels(graph)

    # ---- per call kind, L2 flushed before every call ----
    peak, peak_kind = peak_hbm()
    traffic = recorded_traffic()
    flusher = Flusher(torch, device)
    rooflines = roofline_entries(cyc, flusher, peak, traffic, reps=args.call_reps)
    for r in rooflines:
        r["cold_launch_us"] = round(max_over_ranks(r["cold_launch_us"]), 2)
    for r in rooflines:
        r["launch_us"] = round(max_over_ranks(r["launch_us"]), 2)
    dom = max((r for r in rooflines if r["credited"]),
              key=lambda r: r["launch_us"] * r["launches_per_step"])
    roofline = {"bound": "hbm", "kernel": f"{dom['call']}: {dom['kernels']}",
                "achieved": dom["achieved_gbs"], "peak": peak, "unit": "GB/s",
                "frac": dom["frac"], "peak_source": f"{peak_kind} hbm_gbs",
                "frac_of_8TBps": dom["frac_of_8TBps"], "bytes_per_launch": dom["bytes_per_launch"],
                "launch_ms": round(dom["launch_us"] / 1e3, 4), "traffic": dom["traffic"],
                "timing": ("CUDA events on the launching stream around back-to-back launches "
                           "replayed from a CUDA graph, buffers rotated over more than 4x the "
                           "L2")}
    layer_latency = []
    for kind in ("verify", "sparse", "text_anchored"):
        fn = cyc.one_layer(kind)
        if fn is None:
            continue
        ms1 = statistics.median(flusher.time_calls(fn, args.call_reps))
        b1 = cyc.call_bytes(kind, 0) // cyc.w.n_seq  # the layers are alike
        layer_latency.append({"call": kind, "layers": 1, "launch_us": round(ms1 * 1e3, 2),
                              "bytes": b1, "achieved_gbs": round(b1 / (ms1 / 1e3) / 1e9, 1),
                              "frac": round(b1 / (ms1 / 1e3) / 1e9 / peak, 4)})
    longctx = long_context(torch, cyc.sd, flusher, peak) \
        if args.long_context and args.config == DEFAULT_CONFIG else None
    del flusher
    torch.cuda.empty_cache()

    # ---- each drafting method's cycle against plain decoding (CUDA graphs) ----
    plain = plain_decoding(cyc, torch, reps=max(5, args.steps // 2)) if not args.no_plain \
        else None

    # ---- Sparse-to-Dense's prefill selection (once per video, outside the decode cycle) ----
    prefill = prefill_selection(cyc, torch) if cyc.spec["topk"] and not args.no_prefill \
        else None
    torch.cuda.empty_cache()

    # ---- end to end through the public API, host buffers, copies inside the timed region ----
    # The step's calls captured once per input set into a CUDA graph (what a decoder loop
    # does), replayed every step between the host copies; and the same calls made eagerly.
    host = HostIO(cyc)
    step_graphs = [capture(torch, lambda s, b=b: cyc.step(s, b)) for b in range(2)]
    host.run(cyc, 2, step_graphs)
    barrier()
    e2e_ms = max_over_ranks(host.run(cyc, args.steps, step_graphs))
    e2e_value = whole_job_value(bytes_step, args.steps, e2e_ms, world)
    host.run(cyc, 2)
    barrier()
    eager_ms = max_over_ranks(host.run(cyc, args.steps))
    eager_value = whole_job_value(bytes_step, args.steps, eager_ms, world)
    del step_graphs

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_report(cyc, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if cyc.w.dtype == "bf16" else "f32",
            "data": "synthetic (seeded; stands in for the pages' long-video benchmarks)",
            "config": dict(workload_config(cyc), graph=True, bytes_per_step=bytes_step,
                           bytes_per_call_kind=cyc.bytes,
                           l2=("the step reads more than the 126 MB L2 (no flush between "
                               "steps); per-call rooflines rotate buffers over more than 4x "
                               "the L2; cold per-call latencies flush L2 before every call; "
                               "the text-anchored calls read their own copy of the cache, so "
                               "no call of a draft step is credited bytes that another call "
                               "of that step has just read")
                           if cyc.kv_ta is not cyc.kv_draft else
                           ("the step reads more than the 126 MB L2 (no flush between "
                            "steps); per-call rooflines rotate buffers over more than 4x "
                            "the L2; cold per-call latencies flush L2 before every call")),
            "roofline": roofline,
            "rooflines": rooflines,
            "layer_latency": layer_latency,
            "plain_decoding": plain,
            "prefill_selection": prefill,
            "long_context": longctx,
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                    "h2d_bytes_per_step": host.h2d_bytes, "d2h_bytes_per_step": host.d2h_bytes,
                    "ms_per_step": round(e2e_ms / args.steps, 4),
                    "path": ("the step's C-ABI calls (through the Python binding) captured in "
                             "a CUDA graph per input set and replayed each step; the step's "
                             "inputs (the new K/V rows among them, into device staging) copied "
                             "from pinned host memory on a second stream during the previous "
                             "step; the new K/V rows moved into the cache and the results "
                             "copied back inside the step")},
            "e2e_eager": {"value": round(eager_value, 2), "unit": "GB/s",
                          "ms_per_step": round(eager_ms / args.steps, 4),
                          "path": "the same step, its calls made eagerly each step"},
            "gpu_launches": (n_kernels if n_kernels is not None else -1) * args.steps,
            "clocks": clocks.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------- oracle on the host -------

def cpu_cycle(w, spec, g, layers, hsr_d, aw, topk):
    """Run the fp64 oracle over one cycle of the workload restricted to its first `layers`
    sequences (the acceptance and HSR calls in full); returns (seconds, algorithmic bytes)."""
    import oracle
    from speculative_decoding_attention_verify_b200 import inputs as gen
    sub = lambda lens: oracle.Cache(w.dtype, w.k[:layers], w.v[:layers], lens[:layers], w.h_kv,
                                    w.d) if not w.paged else oracle.cache_from_workload(w, lens)
    if w.paged:
        layers = w.n_seq
    nq = w.n_q_verify
    qs = np.concatenate([[0], np.cumsum(nq[:layers])]).astype(np.int32)
    hw = gen.make_hsr_workload(n=1) if spec["hsr"] else None
    frac = layers / w.n_seq
    byt = 0
    t0 = time.perf_counter()
    idx = None
    if spec["topk"]:
        idx, _ = oracle.topk_select(w.h_q, w.q_verify[:qs[-1]], qs, sub(w.kv_len_verify),
                                    np.zeros(layers, np.int32), w.l_vis[:layers], topk)
        byt += call_bytes(w, "topk", topk=topk) * frac
    for t in range(g):
        lens = w.kv_len_draft(t)
        if spec["sparse"]:
            oracle.sparse_attention(w.h_q, w.q_draft[t][:layers], np.arange(layers + 1),
                                    sub(lens), idx, w.l_vis[:layers])
            byt += call_bytes(w, "sparse", t, topk=topk) * frac
        if spec["hsr"]:
            oracle.hsr_project(hw.emb, hw.hid, hw.weight)
            byt += call_bytes(w, "hsr", hsr_d=hsr_d)
        if spec["ta"]:
            oracle.text_anchored_attention(w.h_q, w.q_draft[t][:layers], np.arange(layers + 1),
                                           sub(lens), np.zeros(layers, np.int32),
                                           w.l_vis[:layers], w.window[:layers])
            byt += call_bytes(w, "text_anchored", t) * frac
    oracle.verify_attention(w.h_q, w.q_verify[:qs[-1]], qs, sub(w.kv_len_verify))
    byt += call_bytes(w, "verify") * frac
    if spec["accept"]:
        oracle.accept_greedy(aw.target_logits, aw.draft_tokens_greedy, aw.gamma, aw.vocab)
        oracle.accept_sample(aw.target_logits, aw.draft_logits, aw.draft_tokens_sampled, aw.u,
                             aw.v, aw.gamma, aw.vocab)
        byt += call_bytes(w, "accept_greedy", aw=aw) + call_bytes(w, "accept_sample", aw=aw)
    return time.perf_counter() - t0, byt


def cpu_baseline_at(w, spec, g, hsr_d, aw, topk, threads, seconds):
    """The oracle on `threads` host threads (0: all), on as many layers of one cycle as fit in
    about `seconds`."""
    import oracle
    used = oracle.set_threads(threads if threads > 0 else os.cpu_count() or 1)
    t1, _ = cpu_cycle(w, spec, g, 1, hsr_d, aw, topk)
    layers = int(max(1, min(w.n_seq, seconds / max(t1, 1e-3))))
    t, byt = cpu_cycle(w, spec, g, layers, hsr_d, aw, topk)
    return {"value": round(byt / t / 1e9, 4), "unit": "GB/s", "cores": used, "kind": "oracle",
            "seconds": round(t, 3),
            "sample": f"one whole cycle on {layers} of {w.n_seq} "
                      f"{'layers' if w.n_seq > 1 and not w.paged else 'sequences'} "
                      f"({t:.1f} s on {used} threads)"}


def cpu_baseline_report(cyc, seconds):
    import oracle
    cores = len(os.sched_getaffinity(0))
    args = (cyc.w, cyc.spec, cyc.g, cyc.hsr_d, cyc.aw, cyc.topk)
    multi = cpu_baseline_at(*args, threads=cores, seconds=seconds)
    single = cpu_baseline_at(*args, threads=1, seconds=seconds / 2)
    oracle.set_threads(cores)
    multi["single_thread"] = {k: single[k] for k in ("value", "unit", "cores", "seconds", "sample")}
    multi["cpu_model"] = cpu_model()
    return multi


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def run_reference(args):
    """The reference arm: the fp64 oracle (the pages hold no code to install), timed on the
    host's cores on bounded samples of the same workload."""
    rank, world, _ = env_rank()
    if rank != 0:
        return
    from speculative_decoding_attention_verify_b200 import inputs as gen
    import oracle
    cfg = args.config
    spec = SPECS[cfg]
    w = gen.make_attn_workload(cfg)
    g = int(spec["draft_steps"] or w.gamma_max)
    aw = None
    if spec["accept"]:
        aw = gen.make_accept_workload(2, gammas=[g], batch=1) if cfg in (2, 3) else \
            gen.make_accept_workload(cfg, gammas=w.gamma)
    hsr_d = gen.HSR_D_MODEL if spec["hsr"] else None
    cores = len(os.sched_getaffinity(0))
    used = oracle.set_threads(cores)
    vals = []
    t0 = time.perf_counter()
    cpu = None
    for _ in range(args.steps):
        t, byt = cpu_cycle(w, spec, g, 1, hsr_d, aw, w.topk)
        vals.append(byt / t / 1e9)
    elapsed = time.perf_counter() - t0
    value = statistics.mean(vals)
    cpu = {"value": round(value, 4), "unit": "GB/s", "cores": used, "kind": "oracle",
           "sample": f"one whole cycle on 1 of {w.n_seq} layers/sequences per step "
                     f"({elapsed / max(args.steps, 1):.1f} s per step on {used} threads)"}
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * elapsed / max(args.steps, 1), 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": {"workload": w.name, "config_index": cfg},
            "cpu_baseline": cpu,
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


CASES = ("verify", "sparse", "sparse_staged", "stage", "text_anchored", "topk", "hsr",
         "accept_greedy", "accept_sample", "decode", "prefill_select", "draft_layer")


def run_case(args):
    """One call kind of the default workload on a reduced layer count (``--layers``), or of
    workload ``--config`` as it is, repeated ``--steps`` times after ``--warmup``; prints its
    device time.  Used for ncu captures of one kernel on a small case."""
    import torch
    from speculative_decoding_attention_verify_b200 import device as dev
    from speculative_decoding_attention_verify_b200 import inputs as gen
    from speculative_decoding_attention_verify_b200 import sdattn as sd
    # the default workload on --layers layers, or another configuration as it is (--config)
    w = gen.make_attn_workload(DEFAULT_CONFIG, layers=args.layers) \
        if args.config == DEFAULT_CONFIG else gen.make_attn_workload(args.config)
    L, g = w.n_seq, int(w.gamma[0])
    k = dev.tensor(w.k, w.dtype)
    v = dev.tensor(w.v, w.dtype)
    kv_verify = dev.kv_cache(w, k=k, v=v)
    lens = w.kv_len_draft(0)
    kv_draft = dev.kv_cache(w, kv_len=lens, k=k, v=v)
    qv, qd = dev.verify_queries(w), dev.draft_queries(w, 0)
    i32 = dev.int32
    tail = i32(w.l_vis)
    max_tail = int((lens - w.l_vis).max())
    if args.case == "verify":
        call = lambda: sd.sd_verify_attention(qv, kv_verify)
    elif args.case == "decode":
        call = lambda: sd.sd_verify_attention(qd, kv_draft)
    elif args.case == "topk":
        call = lambda: sd.sd_topk_select(qv, kv_verify, i32(np.zeros(L)), i32(w.l_vis),
                                         int(w.l_vis.max()), w.topk)
    elif args.case == "prefill_select":
        qt, qs = gen.make_text_queries(w)
        qp = dev.queries(qt, qs, w.dtype, int(w.ctx_len.max()))
        kvp = dev.kv_cache(w, kv_len=w.ctx_len, k=k, v=v)
        call = lambda: sd.sd_topk_select_scored(sd.SD_TOPK_MEAN_TEXT_ATTENTION, qp, kvp,
                                                i32(np.zeros(L)), i32(w.l_vis),
                                                int(w.l_vis.max()), w.topk)
    elif args.case in ("sparse", "sparse_staged", "stage"):
        idx = sd.sd_topk_select(qv, kv_verify, i32(np.zeros(L)), i32(w.l_vis),
                                int(w.l_vis.max()), w.topk)
        sel = sd.sd_sparse_stage(kv_draft, idx, tail)
        if args.case == "sparse":
            call = lambda: sd.sd_sparse_attention(qd, kv_draft, idx, tail, max_tail)
        elif args.case == "stage":
            call = lambda: sd.sd_sparse_stage(kv_draft, idx, tail, selection=sel)
        else:
            call = lambda: sd.sd_sparse_attention_staged(qd, kv_draft, sel, w.topk, tail,
                                                         max_tail)
    elif args.case == "text_anchored":
        vb, ve, win = i32(np.zeros(L)), i32(w.l_vis), i32(w.window)
        call = lambda: sd.sd_text_anchored_attention(qd, kv_draft, vb, ve, win, int(w.window.max()))
    elif args.case == "hsr":
        hw = gen.make_hsr_workload(n=1)
        e, h, W = (dev.tensor(a, gen.BF16) for a in (hw.emb, hw.hid, hw.weight))
        call = lambda: sd.sd_hsr_project(e, h, W)
    elif args.case == "draft_layer":  # Sparrow's full draft layer, 7B shapes, one row
        dw = gen.make_draft_layer_workload(n=1)
        t = lambda a: dev.tensor(a, gen.BF16)
        layer = sd.DraftLayer(dw.d_model, dw.h_q, dw.h_kv, dw.head_dim, dw.d_ff, dw.rms_eps,
                              dw.rope_theta, **{n: t(getattr(dw, n)) for n in sd.DraftLayer.NAMES})
        cache = sd.KVCache(t(dw.k_cache), t(dw.v_cache), dev.int32([dw.kv_len]))
        e, h = t(dw.emb), t(dw.hid)
        call = lambda: sd.sd_draft_layer(layer, e, h, cache, dw.kv_len, dw.window)
    else:
        aw = gen.make_accept_workload(2, gammas=[g], batch=1)
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
        tg, dr, ts, u, vv, gm = (t(a) for a in (aw.target_logits, aw.draft_logits,
                                                aw.draft_tokens_sampled, aw.u, aw.v, aw.gamma))
        if args.case == "accept_greedy":
            call = lambda: sd.sd_accept_greedy(tg, ts, gm, g)
        else:
            call = lambda: sd.sd_accept_sample(tg, dr, ts, u, vv, gm, g)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        call()
    e1.record()
    torch.cuda.synchronize()
    print(json.dumps({"case": args.case, "config": args.config, "layers": w.n_seq,
                      "ms_per_call": round(e0.elapsed_time(e1) / args.steps, 4)}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, choices=sorted(SPECS), default=DEFAULT_CONFIG,
                    help="workload (default: the 28-layer 25k-visual-token Sparse-to-Dense case)")
    ap.add_argument("--call-reps", type=int, default=10,
                    help="separately timed repetitions of every call for the per-call rooflines")
    ap.add_argument("--no-plain", action="store_true", help="skip the plain-decoding comparison")
    ap.add_argument("--no-long-context", dest="long_context", action="store_false",
                    help="skip the 140,000-position measurement")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the prefill (mean text attention) selection")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--case", choices=CASES, default=None,
                    help="time one call kind on a reduced workload (for ncu captures)")
    ap.add_argument("--layers", type=int, default=4)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.case is not None:
        run_case(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
