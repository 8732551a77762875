#!/usr/bin/env python
"""Benchmark: one speculative-decoding cycle at 25k visual tokens through libsdattn.

One *step* runs every call of the hot path once per its role in a cycle, over 28 independent
layers (H_q=28, H_kv=4, d=128, bf16, 25,000 visual + 1,024 text positions, gamma = 8, vocab
152,064), on synthetic seeded inputs:
  top-K selection (K=1024 per KV head over the visual span)              1 launch group
  8 draft steps x [sparse attention, HSR projection, text-anchored]       28 layers each
  dense verification of the 9 new rows                                   28 layers
  greedy acceptance and speculative-sampling acceptance                  batch 1
The metric is algorithmic bytes moved by the step (KV, queries, outputs, weights, logits;
implementation scratch not credited) divided by the step's device time: "spec-decode
attention KV-read GB/s".  Inputs (1.49 GB of KV) exceed the L2 cache, so no flush is needed.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun) every rank runs its own replica of the workload; the path has no
exchange step, so there is no data-path collective (time is the max over ranks).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = dict(workload="spec-decode cycle, 28 layers, L_vis=25000, L_txt=1024, gamma=8, "
                         "H_q=28, H_kv=4, d=128, bf16, top-K 1024, window 1024, vocab 152064",
                layers=28, l_vis=25000, l_txt=1024, gamma=8, h_q=28, h_kv=4, head_dim=128,
                topk=1024, window=1024, vocab=152064, hsr_d_model=3584,
                l2="inputs larger than L2 (1.49 GB of KV per step)",
                parallelism="replicas (no data-path collective)")
METRIC = "spec-decode attention KV-read GB/s (% of B200 HBM peak) at 25k vis tokens"
CFG_INDEX = 3  # the Sparse-to-Dense configuration carries every call of the path


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
    """Hash of the attention kernels' code (comments and layout excluded)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "speculative_decoding_attention_verify_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.startswith("attn_") or name in ("sd_common.cuh", "sd_internal.h", "tc_ptx.cuh"):
            with open(os.path.join(csrc, name)) as f:
                h.update(strip_comments(f.read()).encode())
    return h.hexdigest()[:12]


def recorded_traffic():
    """DRAM bytes per verify launch from the committed ncu summary, if the kernel is unchanged."""
    path = os.path.join(ROOT, "profiles", "verify_attention_c3_ncu.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    want = kernel_source_hash()
    for line in text.splitlines():
        if line.startswith("traffic_bytes_per_full_launch:"):
            parts = line.split()
            if len(parts) >= 4 and parts[3] == want:
                return float(parts[1])
    return None


# ---------------------------------------------------------------- algorithmic bytes --------

def cycle_bytes(w, lens_draft, topk):
    """Bytes the method must move in one step, per call kind (algorithmic bytes: every operand
    the step reads or writes once; scratch is not credited)."""
    d, hk, hq, s = w.d, w.h_kv, w.h_q, 2
    row = hk * d * 2 * s  # K and V of one position, all KV heads
    L = w.n_seq
    n_q = int(w.n_q_verify[0])
    out = {}
    out["verify"] = int(w.kv_len_verify.sum()) * row + 2 * L * n_q * hq * d * s
    ctx_txt = int(w.l_txt[0])
    ta = 0
    sp = 0
    for t in range(len(lens_draft)):
        nonvis = ctx_txt + t + 1
        ta += L * min(int(w.window[0]), nonvis) * row + 2 * L * hq * d * s
        tail = nonvis
        sp += L * (topk + tail) * row + L * hk * topk * 4 + 2 * L * hq * d * s
    out["text_anchored"] = ta
    out["sparse"] = sp
    out["topk"] = L * int(w.l_vis[0]) * hk * d * s + L * hq * d * s + L * hk * topk * 4
    D = WORKLOAD["hsr_d_model"]
    out["hsr"] = len(lens_draft) * (D * 2 * D * 2 + (2 * D + D) * 2)
    V, g = WORKLOAD["vocab"], WORKLOAD["gamma"]
    out["accept_greedy"] = (g + 1) * V * 4 + g * 4
    out["accept_sample"] = (2 * g + 1) * V * 4 + 2 * V * 4 + g * 4 + (2 * g + 1) * 4
    return out


# ---------------------------------------------------------------- the GPU step -------------

class Cycle:
    def __init__(self, device):
        import torch
        from speculative_decoding_attention_verify_b200 import device as dev
        from speculative_decoding_attention_verify_b200 import inputs as gen
        from speculative_decoding_attention_verify_b200 import sdattn as sd
        self.torch, self.sd, self.dev, self.gen = torch, sd, dev, gen
        w = gen.make_attn_workload(CFG_INDEX)
        self.w = w
        g = int(w.gamma[0])
        self.gamma = g
        L = w.n_seq
        self.k = dev.tensor(w.k, w.dtype, device)
        self.v = dev.tensor(w.v, w.dtype, device)
        self.kv_verify = dev.kv_cache(w, device=device, k=self.k, v=self.v)
        self.lens_draft = [w.kv_len_draft(t) for t in range(g)]
        self.kv_draft = [dev.kv_cache(w, kv_len=l, device=device, k=self.k, v=self.v)
                         for l in self.lens_draft]
        self.q_verify = dev.verify_queries(w, device)
        self.q_draft = [dev.draft_queries(w, t, device) for t in range(g)]
        self.cand_b = dev.int32(np.zeros(L, np.int32), device)
        self.cand_e = dev.int32(w.l_vis, device)
        self.tail = dev.int32(w.l_vis, device)
        self.vis_b = dev.int32(np.zeros(L, np.int32), device)
        self.vis_e = dev.int32(w.l_vis, device)
        self.win = dev.int32(w.window, device)
        self.topk = w.topk
        self.idx = torch.empty((L, w.h_kv, w.topk), dtype=torch.int32, device=device)
        self.max_tail = int(max(int((l - w.l_vis).max()) for l in self.lens_draft))
        hw = gen.make_hsr_workload(n=1)
        self.hsr_np = hw
        self.emb = [dev.tensor(hw.emb, gen.BF16, device) for _ in range(g)]
        self.hid = dev.tensor(hw.hid, gen.BF16, device)
        self.W = dev.tensor(hw.weight, gen.BF16, device)
        self.y = torch.empty((1, hw.d_model), dtype=torch.bfloat16, device=device)
        aw = gen.make_accept_workload(2, gammas=[g], batch=1)
        self.aw = aw
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        self.tgt, self.drf = t(aw.target_logits), t(aw.draft_logits)
        self.tok_s, self.tok_g = t(aw.draft_tokens_sampled), t(aw.draft_tokens_greedy)
        self.u, self.vv, self.gam = t(aw.u), t(aw.v), t(aw.gamma)
        # outputs and workspaces allocated once
        self.o_verify = torch.empty_like(self.q_verify.q)
        self.o_draft = [torch.empty_like(q.q) for q in self.q_draft]
        self.o_ta = [torch.empty_like(q.q) for q in self.q_draft]
        mk = lambda n: torch.empty(max(int(n), 16), dtype=torch.uint8, device=device)
        self.ws_verify = mk(sd.sd_attention_workspace_size(sd.SD_ATTN_VERIFY, self.q_verify,
                                                           self.kv_verify))
        self.ws_sparse = mk(sd.sd_sparse_workspace_size(self.q_draft[-1], self.kv_draft[-1],
                                                        w.topk, self.max_tail))
        self.ws_ta = mk(sd.sd_attention_workspace_size(sd.SD_ATTN_TEXT_ANCHORED, self.q_draft[-1],
                                                       self.kv_draft[-1]))
        self.ws_topk = mk(sd.sd_topk_workspace_size(self.kv_verify, int(w.l_vis.max()), w.topk))
        # the top-K rows are staged once per cycle and read by every draft step
        self.sel = mk(sd.sd_sparse_selection_size(self.kv_draft[0], w.topk))
        self.ws_acc = mk(sd.sd_accept_workspace_size(1, g, aw.vocab))
        self.n_acc_g = torch.empty(1, dtype=torch.int32, device=device)
        self.out_g = torch.empty((1, g + 1), dtype=torch.int32, device=device)
        self.n_acc_s = torch.empty(1, dtype=torch.int32, device=device)
        self.out_s = torch.empty((1, g + 1), dtype=torch.int32, device=device)
        self.near = torch.empty(1, dtype=torch.int32, device=device)
        self.bytes = cycle_bytes(w, self.lens_draft, w.topk)
        self.verify_events = []

    def launches_per_step(self, graph=None):
        """Kernels one step launches: counted from the captured CUDA graph (kernel nodes; every
        kernel of the step is libsdattn's), else an upper bound from the call structure."""
        if graph is not None:
            try:
                from cuda.bindings import runtime as rt
                h = rt.cudaGraph_t(init_value=int(graph.raw_cuda_graph()))
                err, _, n = rt.cudaGraphGetNodes(h, 0)
                err2, nodes, n = rt.cudaGraphGetNodes(h, n)
                if err == rt.cudaError_t.cudaSuccess and err2 == rt.cudaError_t.cudaSuccess:
                    kernel = rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
                    return sum(1 for nd in nodes[:n] if rt.cudaGraphNodeGetType(nd)[1] == kernel)
            except Exception:  # noqa: BLE001 - fall back to the structural count
                pass
        g = self.gamma
        # top-K (score, select), staging; per draft step sparse (attention, merge), HSR,
        # text-anchored (attention, merge); verify (attention, merge); greedy (2); sampling (4)
        return 2 + 1 + g * 2 + g + g * 2 + 2 + 2 + 4

    def step(self, stream=None, time_verify=False):
        sd = self.sd
        sd.sd_topk_select(self.q_verify, self.kv_verify, self.cand_b, self.cand_e,
                          int(self.w.l_vis.max()), self.topk, idx_out=self.idx,
                          workspace=self.ws_topk, stream=stream)
        sd.sd_sparse_stage(self.kv_draft[0], self.idx, self.tail, selection=self.sel,
                           stream=stream)
        for t in range(self.gamma):
            sd.sd_sparse_attention_staged(self.q_draft[t], self.kv_draft[t], self.sel, self.topk,
                                          self.tail, self.max_tail, out=self.o_draft[t],
                                          workspace=self.ws_sparse, stream=stream)
            sd.sd_hsr_project(self.emb[t], self.hid, self.W, out=self.y, stream=stream)
            sd.sd_text_anchored_attention(self.q_draft[t], self.kv_draft[t], self.vis_b,
                                          self.vis_e, self.win, int(self.w.window.max()),
                                          out=self.o_ta[t], workspace=self.ws_ta, stream=stream)
        if time_verify:
            e0 = self.torch.cuda.Event(enable_timing=True)
            e1 = self.torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        sd.sd_verify_attention(self.q_verify, self.kv_verify, out=self.o_verify,
                               workspace=self.ws_verify, stream=stream)
        if time_verify:
            e1.record(stream)
            self.verify_events.append((e0, e1))
        sd.sd_accept_greedy(self.tgt, self.tok_g, self.gam, self.gamma, n_acc=self.n_acc_g,
                            out_tok=self.out_g, workspace=self.ws_acc, stream=stream)
        sd.sd_accept_sample(self.tgt, self.drf, self.tok_s, self.u, self.vv, self.gam, self.gamma,
                            n_acc=self.n_acc_s, out_tok=self.out_s, near_boundary=self.near,
                            workspace=self.ws_acc, stream=stream)


class HostInputs:
    """Per-step inputs in pinned host memory for the end-to-end measurement."""

    def __init__(self, cyc):
        torch = cyc.torch
        w = cyc.w
        pin = lambda t: t.cpu().pin_memory()
        self.q_verify = pin(cyc.q_verify.q)
        self.q_draft = [pin(q.q) for q in cyc.q_draft]
        n_new = int(w.n_q_verify[0])
        ctx = int(w.ctx_len[0])
        self.ctx, self.n_new = ctx, n_new
        self.k_new = pin(cyc.k[:, :, ctx:ctx + n_new].contiguous())
        self.v_new = pin(cyc.v[:, :, ctx:ctx + n_new].contiguous())
        self.emb = [pin(e) for e in cyc.emb]
        self.tgt, self.drf = pin(cyc.tgt), pin(cyc.drf)
        self.tok_s, self.tok_g = pin(cyc.tok_s), pin(cyc.tok_g)
        self.u, self.v = pin(cyc.u), pin(cyc.vv)
        self.res = [torch.empty(t.shape, dtype=t.dtype).pin_memory()
                    for t in (cyc.n_acc_g, cyc.out_g, cyc.n_acc_s, cyc.out_s)]
        tensors = [self.q_verify, *self.q_draft, self.k_new, self.v_new, *self.emb, self.tgt,
                   self.drf, self.tok_s, self.tok_g, self.u, self.v]
        self.h2d_bytes = sum(t.numel() * t.element_size() for t in tensors)
        self.d2h_bytes = sum(t.numel() * t.element_size() for t in self.res)

    def upload(self, cyc):
        nb = True
        cyc.q_verify.q.copy_(self.q_verify, non_blocking=nb)
        for dq, hq in zip(cyc.q_draft, self.q_draft):
            dq.q.copy_(hq, non_blocking=nb)
        cyc.k[:, :, self.ctx:self.ctx + self.n_new].copy_(self.k_new, non_blocking=nb)
        cyc.v[:, :, self.ctx:self.ctx + self.n_new].copy_(self.v_new, non_blocking=nb)
        for de, he in zip(cyc.emb, self.emb):
            de.copy_(he, non_blocking=nb)
        for dst, src in ((cyc.tgt, self.tgt), (cyc.drf, self.drf), (cyc.tok_s, self.tok_s),
                         (cyc.tok_g, self.tok_g), (cyc.u, self.u), (cyc.vv, self.v)):
            dst.copy_(src, non_blocking=nb)

    def download(self, cyc):
        for dst, src in zip(self.res, (cyc.n_acc_g, cyc.out_g, cyc.n_acc_s, cyc.out_s)):
            dst.copy_(src, non_blocking=True)


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


def run_ours(args):
    import torch
    import torch.distributed as dist
    rank, world, local = env_rank()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=300))
    device = torch.device("cuda", torch.cuda.current_device())
    cyc = Cycle(device)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    max_over_ranks = lambda x: reduce_max(x, world, device)

    # ---- device-resident timing (optionally replayed from a CUDA graph) ----
    graph = None
    if args.graph:
        for _ in range(2):
            cyc.step()
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            cyc.step(stream=s)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            cyc.step(stream=s)
        torch.cuda.synchronize()
    run = (lambda: graph.replay()) if graph is not None else (lambda: cyc.step())
    for _ in range(args.warmup):
        run()
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        ev0.record()
        for _ in range(args.steps):
            run()
        ev1.record()
        barrier()
    ms = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms)
    ms_per_step = ms / args.steps
    bytes_step = sum(cyc.bytes.values())
    value = whole_job_value(bytes_step, args.steps, ms, world)

    # ---- dominant kernel: verify, timed live with events on the launching stream ----
    cyc.verify_events = []
    for _ in range(args.steps):
        cyc.step(time_verify=True)
    barrier()
    vt = [a.elapsed_time(b) for a, b in cyc.verify_events]
    verify_ms = statistics.mean(vt)
    verify_ms = max_over_ranks(verify_ms)
    peak, peak_kind = peak_hbm()
    achieved = cyc.bytes["verify"] / (verify_ms / 1e3) / 1e9
    traffic = recorded_traffic()

    # ---- end to end through the public API, host buffers, copies inside the timed region ----
    host = HostInputs(cyc)
    for _ in range(2):
        host.upload(cyc)
        cyc.step()
        host.download(cyc)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        host.upload(cyc)
        cyc.step()
        host.download(cyc)
    e1.record()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    e2e_value = whole_job_value(bytes_step, args.steps, e2e_ms, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        probe = cpu_baseline(cyc.w, layers=1)
        layers = int(max(1, min(cyc.w.n_seq, args.cpu_seconds / max(probe["seconds"], 1e-3))))
        cpu = cpu_baseline(cyc.w, layers=layers)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; stands in for the pages' long-video benchmarks)",
            "config": dict(WORKLOAD, graph=bool(graph is not None),
                           bytes_per_step=bytes_step,
                           bytes_per_call_kind=cyc.bytes),
            "roofline": {"bound": "hbm", "kernel": "sd_verify_attention (28 layers, one call)",
                         "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} hbm_gbs",
                         "frac_of_8TBps": round(achieved / 8000.0, 4),
                         "bytes_per_launch": cyc.bytes["verify"],
                         "launch_ms": round(verify_ms, 4), "traffic": traffic},
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                    "h2d_bytes_per_step": host.h2d_bytes, "d2h_bytes_per_step": host.d2h_bytes,
                    "ms_per_step": round(e2e_ms / args.steps, 4)},
            "gpu_launches": cyc.launches_per_step(graph) * args.steps,
            "clocks": clocks.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        del graph
        dist.destroy_process_group()


# ---------------------------------------------------------------- oracle on the host -------

def cpu_baseline(w, layers=1):
    """Time the fp64 oracle on a bounded sample of the same workload: one whole cycle (top-K,
    every draft step's sparse attention, HSR projection and text-anchored attention, verify,
    greedy and sampling acceptance) restricted to the first `layers` layers of the attention
    calls; report GB/s of algorithmic bytes."""
    import oracle
    threads = oracle.set_threads(0)
    g = int(w.gamma[0])
    n_q = int(w.n_q_verify[0])
    sub = lambda lens: oracle.Cache(w.dtype, w.k[:layers], w.v[:layers], lens[:layers], w.h_kv, w.d)
    full = cycle_bytes(w, [w.kv_len_draft(t) for t in range(g)], w.topk)
    L = w.n_seq
    from speculative_decoding_attention_verify_b200 import inputs as gen
    hw = gen.make_hsr_workload(n=1)
    aw = gen.make_accept_workload(2, gammas=[g], batch=1)
    t0 = time.perf_counter()
    idx, _ = oracle.topk_select(w.h_q, w.q_verify[:layers * n_q], w.q_verify_start[:layers + 1],
                                sub(w.kv_len_verify), np.zeros(layers, np.int32),
                                w.l_vis[:layers], w.topk)
    for t in range(g):
        lens = w.kv_len_draft(t)
        oracle.sparse_attention(w.h_q, w.q_draft[t][:layers], np.arange(layers + 1), sub(lens),
                                idx, w.l_vis[:layers])
        oracle.hsr_project(hw.emb, hw.hid, hw.weight)
        oracle.text_anchored_attention(w.h_q, w.q_draft[t][:layers], np.arange(layers + 1),
                                       sub(lens), np.zeros(layers, np.int32), w.l_vis[:layers],
                                       w.window[:layers])
    oracle.verify_attention(w.h_q, w.q_verify[:layers * n_q], w.q_verify_start[:layers + 1],
                            sub(w.kv_len_verify))
    oracle.accept_greedy(aw.target_logits, aw.draft_tokens_greedy, aw.gamma, aw.vocab)
    oracle.accept_sample(aw.target_logits, aw.draft_logits, aw.draft_tokens_sampled, aw.u, aw.v,
                         aw.gamma, aw.vocab)
    t_total = time.perf_counter() - t0
    per_layer = full["topk"] + full["verify"] + full["sparse"] + full["text_anchored"]
    bytes_total = per_layer * layers // L + full["hsr"] + full["accept_greedy"] + \
        full["accept_sample"]
    return {"value": round(bytes_total / t_total / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": "oracle", "seconds": round(t_total, 3),
            "sample": f"one whole cycle on {layers} of {L} layers: top-K, {g} x (sparse draft "
                      f"step, HSR projection, text-anchored draft step), verify, greedy + "
                      f"sampling acceptance ({t_total:.1f} s on {threads} threads)"}


def run_reference(args):
    rank, world, _ = env_rank()
    if rank != 0:
        return
    from speculative_decoding_attention_verify_b200 import inputs as gen
    w = gen.make_attn_workload(CFG_INDEX)
    for _ in range(args.warmup):
        pass  # the oracle has no warm-up state; warm-up steps are skipped deliberately
    vals = []
    t0 = time.perf_counter()
    cpu = None
    for _ in range(args.steps):
        cpu = cpu_baseline(w, layers=1)
        vals.append(cpu["value"])
    elapsed = time.perf_counter() - t0
    value = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * elapsed / max(args.steps, 1), 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": WORKLOAD,
            "cpu_baseline": dict(cpu, value=round(value, 4)),
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


CASES = ("verify", "sparse", "text_anchored", "topk", "hsr", "accept_greedy", "accept_sample")


def run_case(args):
    """One call kind of the cycle on a reduced workload (``--layers``), repeated ``--steps``
    times after ``--warmup``; prints its device time.  Used for ncu captures of one kernel."""
    import torch
    from speculative_decoding_attention_verify_b200 import device as dev
    from speculative_decoding_attention_verify_b200 import inputs as gen
    from speculative_decoding_attention_verify_b200 import sdattn as sd
    w = gen.make_attn_workload(CFG_INDEX, layers=args.layers)
    L, g = w.n_seq, int(w.gamma[0])
    k = dev.tensor(w.k, w.dtype)
    v = dev.tensor(w.v, w.dtype)
    kv_verify = dev.kv_cache(w, k=k, v=v)
    lens = w.kv_len_draft(0)
    kv_draft = dev.kv_cache(w, kv_len=lens, k=k, v=v)
    qv, qd = dev.verify_queries(w), dev.draft_queries(w, 0)
    i32 = dev.int32
    if args.case == "verify":
        call = lambda: sd.sd_verify_attention(qv, kv_verify)
    elif args.case == "topk":
        call = lambda: sd.sd_topk_select(qv, kv_verify, i32(np.zeros(L)), i32(w.l_vis),
                                         int(w.l_vis.max()), w.topk)
    elif args.case == "sparse":
        idx = sd.sd_topk_select(qv, kv_verify, i32(np.zeros(L)), i32(w.l_vis),
                                int(w.l_vis.max()), w.topk)
        tail = i32(w.l_vis)
        call = lambda: sd.sd_sparse_attention(qd, kv_draft, idx, tail, int((lens - w.l_vis).max()))
    elif args.case == "text_anchored":
        vb, ve, win = i32(np.zeros(L)), i32(w.l_vis), i32(w.window)
        call = lambda: sd.sd_text_anchored_attention(qd, kv_draft, vb, ve, win, int(w.window.max()))
    elif args.case == "hsr":
        hw = gen.make_hsr_workload(n=1)
        e, h, W = (dev.tensor(a, gen.BF16) for a in (hw.emb, hw.hid, hw.weight))
        call = lambda: sd.sd_hsr_project(e, h, W)
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
    print(json.dumps({"case": args.case, "layers": args.layers,
                      "ms_per_call": round(e0.elapsed_time(e1) / args.steps, 4)}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-graph", dest="graph", action="store_false")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
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
