"""Seeded synthetic inputs for the speculative-decoding attention path.

This module only draws random numbers and lays them out in memory.  It computes none of the
method's arithmetic: no attention, no softmax statistics, no key scoring or selection and no
acceptance rule.  The same bytes feed the CUDA path (tests, benchmark) and the fp64 CPU oracle
(tests only), so both sides always see identical inputs.

Shapes and value distributions follow the five synthetic workloads that stand in for the
long-video benchmarks the pages evaluate on (Sparrow: LLaVA-OneVision-7B / Qwen2.5-VL-7B with up
to 25k visual tokens; Sparse-to-Dense: Qwen2-VL-7B with top-K KV and about 9 drafted tokens; the
pages publish no dataset items, and none are reproduced here):

* ``C0`` tiny fp32 case (1 head group, d=64, 256 visual + 64 text positions, gamma 4).
* ``C1`` one 7B-like layer (28 query / 4 KV heads, d=128, 8192 + 512, gamma 5), 1% salient keys.
* ``C2`` 28 independent layers at 25,000 visual + 1,024 text positions, gamma 7.
* ``C3`` as C2 with gamma 8 and 2% salient keys (Sparse-to-Dense: top-K 1024 per KV head).
* ``C4`` ragged paged batch of 8 sequences (visual 4096..32768, text 256..2048, gamma 3/5/7).

Salient keys: a chosen fraction of visual positions per (sequence, KV head) hold 4x the mean of
the group's last verify query row (rounded to the KV dtype); the Sparse-to-Dense page reports
that a few top-K entries carry the attention mass, and SpecTemp that >90% of visual tokens get
weight below 1e-3, which this reproduces (scaled logit ~6.5 against N(0,1) noise).

All draws use ``numpy.random.Generator(PCG64(seed))``; normals are drawn in float32 and rounded
to bfloat16 by round-to-nearest-even where the KV dtype is bf16.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

F32 = "f32"
BF16 = "bf16"
PAGE_SIZE = 16
HSR_D_MODEL = 3584

# Seed base: 20260 + config index; per-layer tensors add 1000 * layer.
SEED_BASE = 20260

CONFIGS = {
    0: dict(name="C0-tiny-fp32", layers=1, batch=1, h_q=4, h_kv=1, d=64, dtype=F32,
            l_vis=(256, 256), l_txt=(64, 64), gammas=(4,), window=None, topk=32,
            vocab=1000, logits="independent", logit_sigma=2.0, salient=0.0, paged=False,
            hsr=False),
    1: dict(name="C1-7B-layer", layers=1, batch=1, h_q=28, h_kv=4, d=128, dtype=BF16,
            l_vis=(8192, 8192), l_txt=(512, 512), gammas=(5,), window=512, topk=1024,
            vocab=None, logits=None, logit_sigma=None, salient=0.01, paged=False, hsr=True),
    2: dict(name="C2-long-video-28L", layers=28, batch=1, h_q=28, h_kv=4, d=128, dtype=BF16,
            l_vis=(25000, 25000), l_txt=(1024, 1024), gammas=(7,), window=1024, topk=1024,
            vocab=152064, logits="target+noise", logit_sigma=3.0, salient=0.01, paged=False,
            hsr=True),
    3: dict(name="C3-sparse-to-dense-28L", layers=28, batch=1, h_q=28, h_kv=4, d=128,
            dtype=BF16, l_vis=(25000, 25000), l_txt=(1024, 1024), gammas=(8,), window=1024,
            topk=1024, vocab=152064, logits="target+noise", logit_sigma=3.0, salient=0.02,
            paged=False, hsr=True),
    4: dict(name="C4-ragged-paged-B8", layers=1, batch=8, h_q=28, h_kv=4, d=128, dtype=BF16,
            l_vis=(4096, 32768), l_txt=(256, 2048), gammas=(3, 5, 7), window=None, topk=1024,
            vocab=152064, logits="target+noise", logit_sigma=3.0, salient=0.01, paged=True,
            hsr=False),
}


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bits to float32 (for building inputs and for display)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_kv_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Store float32 values in the KV storage type: float32 as is, bf16 as uint16 bits."""
    if dtype == F32:
        return np.ascontiguousarray(x, dtype=np.float32)
    return bf16_bits_from_f32(x)


def as_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    return f32_from_bf16_bits(x) if dtype == BF16 else np.asarray(x, dtype=np.float32)


def uniform01_f32(rng: np.random.Generator, n: int) -> np.ndarray:
    """Uniforms in [0, 1) on the 2^-24 grid, exactly representable in float32."""
    raw = rng.integers(0, 1 << 24, size=n, dtype=np.int64)
    return (raw.astype(np.float64) * (1.0 / (1 << 24))).astype(np.float32)


@dataclasses.dataclass
class AttnWorkload:
    """KV caches and query rows for a batch of independent sequences.

    A multi-layer workload (C2, C3) is a batch of ``layers * batch`` sequences, one cache each.
    Contiguous caches are ``[n_seq][h_kv][l_cap][d]``; paged caches are a page pool
    ``[num_pages][h_kv][PAGE_SIZE][d]`` plus ``block_table[n_seq][max_pages]`` (-1 padded).
    Position layout of every sequence: ``l_vis`` visual positions, then ``l_txt`` text positions,
    then the new positions appended for drafting / verification.
    """

    cfg_index: int
    name: str
    dtype: str
    n_seq: int
    h_q: int
    h_kv: int
    d: int
    l_vis: np.ndarray          # [n_seq] int32
    l_txt: np.ndarray          # [n_seq] int32
    gamma: np.ndarray          # [n_seq] int32 (draft length of the sequence's cycle)
    l_cap: int                 # contiguous layout: positions allocated per sequence
    k: np.ndarray              # storage dtype (float32 or uint16 bf16 bits)
    v: np.ndarray
    paged: bool
    block_table: Optional[np.ndarray]  # [n_seq][max_pages] int32, or None
    num_pages: int
    q_verify: np.ndarray       # [sum(gamma+1)][h_q][d] storage dtype
    q_verify_start: np.ndarray  # [n_seq + 1] int32
    q_draft: np.ndarray        # [gamma_max][n_seq][h_q][d]: draft-step queries (one row each)
    salient: list              # salient[s][g] -> sorted int array of salient positions
    window: np.ndarray         # [n_seq] int32: text-anchored window (W)
    topk: int

    @property
    def ctx_len(self) -> np.ndarray:
        return (self.l_vis + self.l_txt).astype(np.int32)

    @property
    def n_q_verify(self) -> np.ndarray:
        return (self.gamma + 1).astype(np.int32)

    @property
    def kv_len_verify(self) -> np.ndarray:
        """Verify step: the gamma+1 new positions are already appended to the cache."""
        return (self.ctx_len + self.gamma + 1).astype(np.int32)

    def kv_len_draft(self, step: int) -> np.ndarray:
        """Draft step ``step`` (0-based) appends one position: kv_len = ctx + step + 1."""
        return (self.ctx_len + step + 1).astype(np.int32)

    @property
    def group(self) -> int:
        return self.h_q // self.h_kv

    @property
    def gamma_max(self) -> int:
        return int(self.gamma.max())

    def kv_row(self, which: str, s: int, g: int, j: int) -> np.ndarray:
        """Row ``j`` of sequence ``s``, KV head ``g`` of K or V (storage dtype), for tests."""
        arr = self.k if which == "k" else self.v
        if not self.paged:
            return arr[s, g, j]
        page = self.block_table[s, j // PAGE_SIZE]
        return arr[page, g, j % PAGE_SIZE]


def _ragged_lengths(rng, cfg, n_seq):
    lo_v, hi_v = cfg["l_vis"]
    lo_t, hi_t = cfg["l_txt"]
    l_vis = rng.integers(lo_v, hi_v + 1, size=n_seq).astype(np.int32)
    l_txt = rng.integers(lo_t, hi_t + 1, size=n_seq).astype(np.int32)
    gammas = np.asarray(cfg["gammas"], dtype=np.int32)
    gamma = gammas[rng.integers(0, len(gammas), size=n_seq)].astype(np.int32)
    return l_vis, l_txt, gamma


def make_attn_workload(cfg_index: int, layers: Optional[int] = None, l_vis: Optional[int] = None,
                       l_txt: Optional[int] = None, gamma: Optional[int] = None,
                       batch: Optional[int] = None, seed: Optional[int] = None,
                       l_cap_pad: int = 0, nan_tail: bool = True,
                       salient: Optional[float] = None, paged: Optional[bool] = None,
                       dtype: Optional[str] = None) -> AttnWorkload:
    """Build the attention inputs of configuration ``cfg_index``.

    Keyword overrides shrink a configuration for fast tests (fewer layers, shorter spans).
    ``l_cap_pad`` adds unused positions after each contiguous sequence; with ``nan_tail`` the
    unused positions (contiguous padding and the tail of each last page) hold NaN, so any read
    of them shows up as a NaN in the output.
    """
    cfg = dict(CONFIGS[cfg_index])
    if l_vis is not None:
        cfg["l_vis"] = (l_vis, l_vis)
    if l_txt is not None:
        cfg["l_txt"] = (l_txt, l_txt)
    if gamma is not None:
        cfg["gammas"] = (gamma,)
    if salient is not None:
        cfg["salient"] = salient
    if paged is not None:
        cfg["paged"] = paged
    if dtype is not None:
        cfg["dtype"] = dtype
    n_layers = cfg["layers"] if layers is None else layers
    n_batch = cfg["batch"] if batch is None else batch
    n_seq = n_layers * n_batch
    seed0 = SEED_BASE + cfg_index if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed0))
    l_vis_a, l_txt_a, gamma_a = _ragged_lengths(rng, cfg, n_seq)
    h_q, h_kv, d, dt = cfg["h_q"], cfg["h_kv"], cfg["d"], cfg["dtype"]
    G = h_q // h_kv
    kv_cap = (l_vis_a + l_txt_a + gamma_a + 1).astype(np.int64)
    l_cap = int(kv_cap.max()) + int(l_cap_pad)
    nan_bits = np.uint16(0x7FC0) if dt == BF16 else np.float32(np.nan)
    store_dt = np.uint16 if dt == BF16 else np.float32

    n_q = gamma_a + 1
    q_start = np.zeros(n_seq + 1, dtype=np.int32)
    q_start[1:] = np.cumsum(n_q)
    q_verify = np.empty((int(q_start[-1]), h_q, d), dtype=store_dt)
    g_max = int(gamma_a.max())
    q_draft = np.empty((g_max, n_seq, h_q, d), dtype=store_dt)

    paged_layout = bool(cfg["paged"])
    if paged_layout:
        pages = (kv_cap + PAGE_SIZE - 1) // PAGE_SIZE
        num_pages = int(pages.sum())
        max_pages = int(pages.max())
        perm = rng.permutation(num_pages).astype(np.int32)
        block_table = np.full((n_seq, max_pages), -1, dtype=np.int32)
        off = 0
        for s in range(n_seq):
            block_table[s, :pages[s]] = perm[off:off + pages[s]]
            off += int(pages[s])
        k = np.empty((num_pages, h_kv, PAGE_SIZE, d), dtype=store_dt)
        v = np.empty((num_pages, h_kv, PAGE_SIZE, d), dtype=store_dt)
    else:
        num_pages = 0
        block_table = None
        k = np.empty((n_seq, h_kv, l_cap, d), dtype=store_dt)
        v = np.empty((n_seq, h_kv, l_cap, d), dtype=store_dt)

    salient_pos = []
    for s in range(n_seq):
        srng = np.random.Generator(np.random.PCG64(seed0 + 1000 * (s + 1)))
        cap = int(kv_cap[s])
        qv = srng.standard_normal((int(n_q[s]), h_q, d), dtype=np.float32)
        qv_store = to_kv_dtype(qv, dt)
        q_verify[q_start[s]:q_start[s + 1]] = qv_store
        qd = srng.standard_normal((g_max, h_q, d), dtype=np.float32)
        q_draft[:, s] = to_kv_dtype(qd, dt)
        ks = srng.standard_normal((h_kv, cap, d), dtype=np.float32)
        vs = srng.standard_normal((h_kv, cap, d), dtype=np.float32)
        ks_store = to_kv_dtype(ks, dt)
        # Salient keys: 4x the mean of the group's last verify query row, in the KV dtype.
        last = as_f32(qv_store[-1], dt).astype(np.float64)  # [h_q][d]
        n_sal = int(round(cfg["salient"] * int(l_vis_a[s])))
        per_g = []
        for g in range(h_kv):
            if n_sal > 0:
                pos = np.sort(srng.choice(int(l_vis_a[s]), size=n_sal, replace=False))
                qbar = last[g * G:(g + 1) * G].mean(axis=0)
                row = to_kv_dtype((4.0 * qbar).astype(np.float32)[None, :], dt)[0]
                ks_store[g, pos] = row
            else:
                pos = np.zeros(0, dtype=np.int64)
            per_g.append(pos.astype(np.int64))
        salient_pos.append(per_g)
        vs_store = to_kv_dtype(vs, dt)
        if paged_layout:
            pg = int((cap + PAGE_SIZE - 1) // PAGE_SIZE)
            padded = pg * PAGE_SIZE
            kpad = np.empty((h_kv, padded, d), dtype=store_dt)
            vpad = np.empty((h_kv, padded, d), dtype=store_dt)
            kpad[:, :cap] = ks_store
            vpad[:, :cap] = vs_store
            fill = nan_bits if nan_tail else store_dt(0)
            kpad[:, cap:] = fill
            vpad[:, cap:] = fill
            kp = kpad.reshape(h_kv, pg, PAGE_SIZE, d).transpose(1, 0, 2, 3)
            vp = vpad.reshape(h_kv, pg, PAGE_SIZE, d).transpose(1, 0, 2, 3)
            k[block_table[s, :pg]] = kp
            v[block_table[s, :pg]] = vp
        else:
            k[s, :, :cap] = ks_store
            v[s, :, :cap] = vs_store
            if l_cap > cap:
                fill = nan_bits if nan_tail else store_dt(0)
                k[s, :, cap:] = fill
                v[s, :, cap:] = fill

    if cfg["window"] is None:
        window = l_txt_a.copy()
    else:
        window = np.full(n_seq, cfg["window"], dtype=np.int32)
    return AttnWorkload(
        cfg_index=cfg_index, name=cfg["name"], dtype=dt, n_seq=n_seq, h_q=h_q, h_kv=h_kv, d=d,
        l_vis=l_vis_a, l_txt=l_txt_a, gamma=gamma_a, l_cap=l_cap, k=k, v=v, paged=paged_layout,
        block_table=block_table, num_pages=num_pages, q_verify=q_verify,
        q_verify_start=q_start, q_draft=q_draft, salient=salient_pos,
        window=window.astype(np.int32), topk=int(cfg["topk"]))


def make_text_queries(w: AttnWorkload, seed: Optional[int] = None):
    """Prefill query rows of every sequence's text tokens, for selecting the kept KV entries at
    prefill: ``(q_text [sum(l_txt)][h_q][d] in the KV storage type, q_start [n_seq + 1])``.

    The text tokens are the positions [l_vis, l_vis + l_txt) of each cache, i.e. the last
    ``l_txt`` positions of a cache holding the ``ctx_len`` prefill positions.  Rows are N(0, 1)
    drawn per sequence (seed ``SEED_BASE + cfg + 2000 * (sequence + 1)``)."""
    q_start = np.zeros(w.n_seq + 1, dtype=np.int32)
    q_start[1:] = np.cumsum(w.l_txt)
    st = np.uint16 if w.dtype == BF16 else np.float32
    q = np.empty((int(q_start[-1]), w.h_q, w.d), dtype=st)
    base = SEED_BASE + w.cfg_index if seed is None else seed
    for s in range(w.n_seq):
        rng = np.random.Generator(np.random.PCG64(base + 2000 * (s + 1)))
        rows = rng.standard_normal((int(w.l_txt[s]), w.h_q, w.d), dtype=np.float32)
        q[q_start[s]:q_start[s + 1]] = to_kv_dtype(rows, w.dtype)
    return q, q_start


def make_device_workload(layers: int, l_vis: int, l_txt: int, gamma: int, h_q: int = 28,
                         h_kv: int = 4, d: int = 128, seed: int = SEED_BASE + 5, device="cuda"):
    """bf16 caches and queries drawn directly on the device with a seeded torch generator, for
    benchmark workloads too large to draw on the host (e.g. 28 layers x 140,000 positions):
    K, V [layers][h_kv][l_vis + l_txt + gamma + 1][d] and verify / draft query rows, all
    N(0, 1).  No salient keys: timing only, no oracle comparison."""
    import torch
    gen_ = torch.Generator(device=device)
    gen_.manual_seed(int(seed))
    cap = l_vis + l_txt + gamma + 1
    draw = lambda *shape: torch.randn(*shape, generator=gen_, device=device,
                                      dtype=torch.float32).to(torch.bfloat16)
    k = draw(layers, h_kv, cap, d)
    v = draw(layers, h_kv, cap, d)
    q_verify = draw(layers * (gamma + 1), h_q, d)
    q_draft = draw(layers, h_q, d)
    return dict(k=k, v=v, q_verify=q_verify, q_draft=q_draft, layers=layers, l_vis=l_vis,
                l_txt=l_txt, gamma=gamma, h_q=h_q, h_kv=h_kv, d=d, cap=cap)


@dataclasses.dataclass
class DraftLayerWorkload:
    """Weights and inputs of one draft layer (all bf16 bits): the HSR FC, two RMSNorm weights,
    the QKV projection with bias, the output projection, the gate/up and down projections;
    the rows' embeddings and reused hidden states; the draft's own text-only KV cache
    [1][h_kv][cap][d] whose last n positions are the rows' (their k, v are written there)."""

    n: int
    d_model: int
    h_q: int
    h_kv: int
    head_dim: int
    d_ff: int
    rms_eps: float
    rope_theta: float
    l_txt: int
    window: int
    w_hsr: np.ndarray
    ln1: np.ndarray
    w_qkv: np.ndarray
    b_qkv: np.ndarray
    w_o: np.ndarray
    ln2: np.ndarray
    w_gate_up: np.ndarray
    w_down: np.ndarray
    emb: np.ndarray
    hid: np.ndarray
    k_cache: np.ndarray
    v_cache: np.ndarray

    @property
    def kv_len(self) -> int:
        return self.l_txt + self.n


def make_draft_layer_workload(n: int = 1, d_model: int = HSR_D_MODEL, h_q: int = 28,
                              h_kv: int = 4, head_dim: int = 128, d_ff: int = 18944,
                              l_txt: int = 1024, window: Optional[int] = None,
                              seed: Optional[int] = None) -> DraftLayerWorkload:
    """Random weights of the 7B-like shapes by default (N(0, 1/fan_in) matrices, RMSNorm weights
    1 + N(0, 0.1^2), QKV bias N(0, 0.1^2)), N(0, 1) embeddings, hidden states and cache rows;
    the cache holds l_txt earlier text positions and room for the n new rows."""
    rng = np.random.Generator(np.random.PCG64(SEED_BASE + 9 + 800_000 if seed is None else seed))
    D, F, d = d_model, d_ff, head_dim
    nqkv = (h_q + 2 * h_kv) * d
    mat = lambda m, k: bf16_bits_from_f32(rng.standard_normal((m, k), dtype=np.float32) *
                                          np.float32(1.0 / np.sqrt(k)))
    vec = lambda m, mu, sd: bf16_bits_from_f32(
        (mu + sd * rng.standard_normal(m)).astype(np.float32))
    w_hsr = mat(D, 2 * D)
    ln1 = vec(D, 1.0, 0.1)
    w_qkv = mat(nqkv, D)
    b_qkv = vec(nqkv, 0.0, 0.1)
    w_o = mat(D, h_q * d)
    ln2 = vec(D, 1.0, 0.1)
    w_gate_up = mat(2 * F, D)
    w_down = mat(D, F)
    emb = bf16_bits_from_f32(rng.standard_normal((n, D), dtype=np.float32))
    hid = bf16_bits_from_f32(rng.standard_normal((n, D), dtype=np.float32))
    cap = l_txt + n
    k_cache = bf16_bits_from_f32(rng.standard_normal((1, h_kv, cap, d), dtype=np.float32))
    v_cache = bf16_bits_from_f32(rng.standard_normal((1, h_kv, cap, d), dtype=np.float32))
    return DraftLayerWorkload(n=n, d_model=D, h_q=h_q, h_kv=h_kv, head_dim=d, d_ff=F,
                              rms_eps=1e-6, rope_theta=1e6, l_txt=l_txt,
                              window=l_txt if window is None else window, w_hsr=w_hsr, ln1=ln1,
                              w_qkv=w_qkv, b_qkv=b_qkv, w_o=w_o, ln2=ln2, w_gate_up=w_gate_up,
                              w_down=w_down, emb=emb, hid=hid, k_cache=k_cache,
                              v_cache=v_cache)


@dataclasses.dataclass
class AcceptWorkload:
    """Logits, drafted tokens and uniforms for a batch of acceptance problems.

    Rows are packed per sequence: target rows ``[sum(gamma+1)][vocab]``, draft rows
    ``[sum(gamma)][vocab]``, drafted tokens and ``u`` ``[sum(gamma)]``, ``v`` ``[sum(gamma+1)]``.
    ``draft_tokens_sampled`` are drawn from the draft distribution with the Gumbel-max trick
    (argmax of logits plus Gumbel noise is an exact draw from the softmax); ``draft_tokens_greedy``
    are the draft rows' argmax.  Both are inputs: how the draft chose them is not part of the
    acceptance method.
    """

    vocab: int
    gamma: np.ndarray
    target_logits: np.ndarray
    draft_logits: np.ndarray
    draft_tokens_sampled: np.ndarray
    draft_tokens_greedy: np.ndarray
    u: np.ndarray
    v: np.ndarray

    @property
    def batch(self) -> int:
        return int(self.gamma.shape[0])

    @property
    def gamma_max(self) -> int:
        return int(self.gamma.max())


def make_accept_workload(cfg_index: int, vocab: Optional[int] = None,
                         gammas: Optional[np.ndarray] = None, batch: Optional[int] = None,
                         seed: Optional[int] = None, logits: Optional[str] = None,
                         sigma: Optional[float] = None) -> AcceptWorkload:
    cfg = CONFIGS[cfg_index]
    V = int(vocab if vocab is not None else cfg["vocab"])
    B = int(batch if batch is not None else cfg["batch"])
    seed0 = (SEED_BASE + cfg_index + 500_000) if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed0))
    if gammas is None:
        gs = np.asarray(cfg["gammas"], dtype=np.int32)
        gamma = gs[rng.integers(0, len(gs), size=B)].astype(np.int32)
    else:
        gamma = np.asarray(gammas, dtype=np.int32)
        B = gamma.shape[0]
    mode = logits if logits is not None else cfg["logits"]
    sig = float(sigma if sigma is not None else cfg["logit_sigma"])
    n_t = int((gamma + 1).sum())
    n_d = int(gamma.sum())
    tgt = np.empty((n_t, V), dtype=np.float32)
    drf = np.empty((n_d, V), dtype=np.float32)
    ot = od = 0
    for b in range(B):
        g = int(gamma[b])
        t_rows = rng.standard_normal((g + 1, V), dtype=np.float32) * np.float32(sig)
        tgt[ot:ot + g + 1] = t_rows
        if mode == "independent":
            drf[od:od + g] = rng.standard_normal((g, V), dtype=np.float32) * np.float32(sig)
        else:  # draft = target + N(0, 1) noise, aligned row for row (draft row i ~ target row i)
            drf[od:od + g] = t_rows[:g] + rng.standard_normal((g, V), dtype=np.float32)
        ot += g + 1
        od += g
    gum = -np.log(-np.log(rng.random((n_d, V))))
    sampled = np.argmax(drf.astype(np.float64) + gum, axis=1).astype(np.int32)
    greedy = np.argmax(drf, axis=1).astype(np.int32)
    u = uniform01_f32(rng, n_d)
    v = uniform01_f32(rng, n_t)
    return AcceptWorkload(vocab=V, gamma=gamma, target_logits=tgt, draft_logits=drf,
                          draft_tokens_sampled=sampled, draft_tokens_greedy=greedy, u=u, v=v)


@dataclasses.dataclass
class HsrWorkload:
    """Inputs of the hidden-state-reuse projection: e, h [n][D] and W [D][2D], all bf16 bits."""

    n: int
    d_model: int
    emb: np.ndarray
    hid: np.ndarray
    weight: np.ndarray
    bias: Optional[np.ndarray]


def make_hsr_workload(n: int = 1, d_model: int = HSR_D_MODEL, seed: Optional[int] = None,
                      with_bias: bool = False) -> HsrWorkload:
    rng = np.random.Generator(np.random.PCG64(SEED_BASE + 1 + 700_000 if seed is None else seed))
    emb = bf16_bits_from_f32(rng.standard_normal((n, d_model), dtype=np.float32))
    hid = bf16_bits_from_f32(rng.standard_normal((n, d_model), dtype=np.float32))
    w = rng.standard_normal((d_model, 2 * d_model), dtype=np.float32)
    w *= np.float32(1.0 / np.sqrt(2 * d_model))
    weight = bf16_bits_from_f32(w)
    bias = None
    if with_bias:
        bias = bf16_bits_from_f32(rng.standard_normal(d_model, dtype=np.float32))
    return HsrWorkload(n=n, d_model=d_model, emb=emb, hid=hid, weight=weight, bias=bias)
