"""GPU parity of the three attention calls against the fp64 oracle (through the C-ABI).

Tolerances (max-abs over every output element): 2e-2 for bf16 KV, 1e-4 for fp32 KV.
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_attention_verify_b200 import device as dev
from speculative_decoding_attention_verify_b200 import inputs as gen
from speculative_decoding_attention_verify_b200 import sdattn as sd

pytestmark = pytest.mark.gpu

TOL = {gen.F32: 1e-4, gen.BF16: 2e-2}


def _assert_close(out, ref, dtype, where=""):
    got = dev.to_numpy_f64(out)
    assert got.shape == ref.shape, where
    assert np.isfinite(got).all(), f"{where}: non-finite output"
    err = float(np.abs(got - ref).max())
    assert err <= TOL[dtype], f"{where}: max-abs error {err} > {TOL[dtype]}"
    return err


# ---------------------------------------------------------------- verify -------------------

VERIFY_CASES = [
    (0, {}),                                                   # C0 tiny fp32
    (0, dict(l_vis=1000, l_txt=333, gamma=6)),                 # fp32, several tiles, ragged tail
    (1, {}),                                                   # C1 7B-like layer
    (1, dict(l_vis=777, l_txt=45, gamma=1)),                   # bf16, ragged, R = 14 rows
    (1, dict(l_vis=3000, l_txt=100, gamma=0)),                 # gamma = 0: one row per head
    (1, dict(l_vis=5000, l_txt=300, gamma=4, l_cap_pad=37)),   # NaN-filled unused capacity
    (2, dict(layers=3, l_vis=4000, l_txt=200)),                # multi-layer batch
    (3, dict(layers=2, l_vis=2500, l_txt=300)),                # gamma 8: R = 63 rows
    (4, dict(l_vis=1500, l_txt=100, batch=5)),                 # paged, ragged gammas, NaN page tails
    (4, {}),                                                   # C4 full: 8 sequences up to 34.8k
    (0, dict(dtype="bf16")),                                   # d=64, G=4: R = 20 (tensor cores)
    (0, dict(dtype="bf16", l_vis=3000, l_txt=77, gamma=7)),    # d=64: R = 32 rows, ragged tail
    (4, dict(l_vis=1500, l_txt=100, batch=5, gamma=2)),        # paged ragged, R = 21
    (2, dict(layers=48, l_vis=600, l_txt=50, gamma=1)),        # 192 (sequence, KV head) units
    (1, dict(l_vis=40, l_txt=9, gamma=3)),                     # a single tile
    (1, dict(l_vis=3000, l_txt=100, gamma=11)),                # R = 84 rows: one row copy
    (1, dict(l_vis=3000, l_txt=100, gamma=8)),                 # R = 63: two row copies
    (0, dict(dtype="bf16", l_vis=1500, l_txt=90, gamma=10)),   # d=64: R = 44, two row copies
    (0, dict(dtype="bf16", l_vis=1500, l_txt=90, gamma=20)),   # d=64: R = 84, one row copy
]


@pytest.mark.parametrize("cfg,kw", VERIFY_CASES)
def test_verify_matches_oracle(cfg, kw):
    w = gen.make_attn_workload(cfg, **kw)
    out = sd.sd_verify_attention(dev.verify_queries(w), dev.kv_cache(w))
    ref = oracle.verify_attention(w.h_q, w.q_verify, w.q_verify_start, oracle.cache_from_workload(w))
    _assert_close(out, ref, w.dtype, f"verify cfg{cfg} {kw}")


def test_verify_c2_full_launch_sampled_layers():
    """All 28 layers of the long-video case in one launch; three layers checked in full."""
    w = gen.make_attn_workload(2)
    out = sd.sd_verify_attention(dev.verify_queries(w), dev.kv_cache(w))
    got = dev.to_numpy_f64(out)
    n_q = int(w.n_q_verify[0])
    for layer in (0, 13, 27):
        sub = oracle.Cache(w.dtype, w.k[layer:layer + 1], w.v[layer:layer + 1],
                           w.kv_len_verify[layer:layer + 1], w.h_kv, w.d)
        rows = slice(layer * n_q, (layer + 1) * n_q)
        ref = oracle.verify_attention(w.h_q, w.q_verify[rows], [0, n_q], sub)
        err = np.abs(got[rows] - ref).max()
        assert err <= TOL[w.dtype], (layer, err)


def test_verify_gamma0_equals_single_token_decode():
    w = gen.make_attn_workload(1, l_vis=2000, l_txt=64, gamma=0, layers=1)
    out = sd.sd_verify_attention(dev.verify_queries(w), dev.kv_cache(w))
    ref = oracle.decode_attention(w.h_q, w.q_verify, oracle.cache_from_workload(w))
    _assert_close(out, ref, w.dtype, "gamma0")


def test_verify_engines_and_schedules_agree():
    """The same call under looser (still valid) host hints: a larger max_q_rows plans 56 rows
    per KV head instead of 21; a larger max_kv_len plans another split of the positions.  All
    must match the oracle."""
    w = gen.make_attn_workload(1, l_vis=6000, l_txt=200, gamma=2)
    kv = dev.kv_cache(w)
    ref = oracle.verify_attention(w.h_q, w.q_verify, w.q_verify_start, oracle.cache_from_workload(w))
    n = int(w.kv_len_verify.max())
    base = dev.verify_queries(w)
    variants = {
        "default": base,
        "rows8": sd.Queries(base.q, base.q_start, max_q_rows=8, max_kv_len=n),
        "len4x": sd.Queries(base.q, base.q_start, max_q_rows=base.desc.max_q_rows,
                            max_kv_len=4 * n),
    }
    outs = {}
    for name, q in variants.items():
        outs[name] = sd.sd_verify_attention(q, kv)
        _assert_close(outs[name], ref, w.dtype, name)
    for name in ("rows8", "len4x"):
        diff = (outs[name].float() - outs["default"].float()).abs().max().item()
        assert diff <= 2e-2, name


def test_verify_is_deterministic():
    w = gen.make_attn_workload(4, l_vis=3000, l_txt=150, batch=4)
    kv, q = dev.kv_cache(w), dev.verify_queries(w)
    a = sd.sd_verify_attention(q, kv)
    b = sd.sd_verify_attention(q, kv)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("gamma", [None, 2])   # R = 56 and R = 21 rows per KV head
def test_verify_bad_page_sets_flag_without_fault(gamma):
    w = gen.make_attn_workload(4, l_vis=500, l_txt=40, batch=2, gamma=gamma)
    bt = w.block_table.copy()
    bt[1, 3] = w.num_pages + 5  # out of the pool
    kv = dev.kv_cache(w)
    kv = sd.KVCache(kv.k, kv.v, kv.kv_len, block_table=dev.int32(bt))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    sd.sd_verify_attention(dev.verify_queries(w), kv, dev_err=flag)
    torch.cuda.synchronize()
    assert flag.item() & sd.SD_DEVERR_PAGE


# ---------------------------------------------------------------- text-anchored ------------


def _text_anchored_case(w, step=0, vis=None, window=None):
    lens = w.kv_len_draft(step)
    kv = dev.kv_cache(w, kv_len=lens)
    q = dev.draft_queries(w, step)
    vb = np.zeros(w.n_seq, np.int32) if vis is None else np.full(w.n_seq, vis[0], np.int32)
    ve = w.l_vis.astype(np.int32) if vis is None else np.full(w.n_seq, vis[1], np.int32)
    win = w.window if window is None else np.full(w.n_seq, window, np.int32)
    out = sd.sd_text_anchored_attention(q, kv, dev.int32(vb), dev.int32(ve), dev.int32(win),
                                        int(win.max()))
    ref = oracle.text_anchored_attention(w.h_q, w.q_draft[step], np.arange(w.n_seq + 1),
                                         oracle.cache_from_workload(w, kv_len=lens), vb, ve, win)
    return out, ref


TA_CASES = [
    (0, {}, {}),
    (1, {}, {}),
    (1, dict(l_vis=3000, l_txt=700), dict(step=3)),
    (1, dict(l_vis=3000, l_txt=300), dict(vis=(1000, 2500), window=900)),   # window crosses span
    (1, dict(l_vis=3000, l_txt=300), dict(vis=(0, 0), window=777)),        # no visual span
    (1, dict(l_vis=3000, l_txt=300), dict(window=1)),
    (2, dict(layers=4, l_vis=3000), {}),
    (4, dict(l_vis=2000, l_txt=300, batch=6), {}),
    (4, {}, {}),
    (0, dict(dtype="bf16", l_vis=2000, l_txt=500), dict(window=300)),     # d=64 tensor cores
    (2, dict(layers=40, l_vis=2000, l_txt=900), dict(vis=(100, 1500), window=1000)),
]


@pytest.mark.parametrize("cfg,kw,case", TA_CASES)
def test_text_anchored_matches_oracle(cfg, kw, case):
    w = gen.make_attn_workload(cfg, **kw)
    out, ref = _text_anchored_case(w, **case)
    _assert_close(out, ref, w.dtype, f"text-anchored cfg{cfg} {kw} {case}")


@pytest.mark.parametrize("window", [900, 960, 1000, 1023])
def test_text_anchored_window_shorter_than_cache_fits_reported_workspace(window):
    """The workspace query knows only max_kv_len; a call whose window makes the streams shorter
    plans from the window, and its split count (the split model is not monotone in the stream
    length) must not outgrow the workspace the query reported.  No visual span, 7 rows per KV
    head, about 1,025 positions: the draft layer's own attention."""
    w = gen.make_attn_workload(1, l_vis=64, l_txt=960)
    out, ref = _text_anchored_case(w, vis=(0, 0), window=window)
    _assert_close(out, ref, w.dtype, f"text-anchored window {window}")


def test_text_anchored_multi_row_verify_shape():
    """Text-anchored attention over gamma+1 rows at once (rows slide the window up)."""
    w = gen.make_attn_workload(1, l_vis=2000, l_txt=400, gamma=5)
    kv, q = dev.kv_cache(w), dev.verify_queries(w)
    vb = np.zeros(1, np.int32)
    ve = w.l_vis.astype(np.int32)
    win = np.array([300], np.int32)
    out = sd.sd_text_anchored_attention(q, kv, dev.int32(vb), dev.int32(ve), dev.int32(win), 300)
    ref = oracle.text_anchored_attention(w.h_q, w.q_verify, w.q_verify_start,
                                         oracle.cache_from_workload(w), vb, ve, win)
    _assert_close(out, ref, w.dtype, "text-anchored multi-row")


# ---------------------------------------------------------------- sparse -------------------


def _oracle_topk(w, lens, k):
    cache = oracle.cache_from_workload(w, kv_len=lens)
    idx, _ = oracle.topk_select(w.h_q, w.q_verify, w.q_verify_start, cache,
                                np.zeros(w.n_seq, np.int32), w.l_vis, k)
    return idx


SPARSE_CASES = [
    (0, {}, 0),
    (1, dict(l_vis=4000, l_txt=300), 0),
    (3, dict(layers=3, l_vis=5000, l_txt=600), 2),
    (4, dict(l_vis=3000, l_txt=200, batch=5), 0),
    (4, {}, 1),
    (0, dict(dtype="bf16", l_vis=2000, l_txt=100), 3),                     # d=64
    (2, dict(layers=40, l_vis=3000, l_txt=300), 5),                        # 160 units
]


@pytest.mark.parametrize("cfg,kw,step", SPARSE_CASES)
def test_sparse_matches_oracle(cfg, kw, step):
    w = gen.make_attn_workload(cfg, **kw)
    lens = w.kv_len_draft(step)
    idx = _oracle_topk(w, w.kv_len_verify, w.topk)
    kv = dev.kv_cache(w, kv_len=lens)
    q = dev.draft_queries(w, step)
    tail = w.l_vis.astype(np.int32)
    max_tail = int((lens - tail).max())
    out = sd.sd_sparse_attention(q, kv, dev.int32(idx), dev.int32(tail), max_tail)
    ref = oracle.sparse_attention(w.h_q, w.q_draft[step], np.arange(w.n_seq + 1),
                                  oracle.cache_from_workload(w, kv_len=lens), idx, tail)
    _assert_close(out, ref, w.dtype, f"sparse cfg{cfg} {kw}")


def test_sparse_with_every_candidate_equals_dense():
    w = gen.make_attn_workload(1, l_vis=1500, l_txt=100)
    lens = w.kv_len_draft(0)
    ctx = int(lens[0]) - 1
    idx = np.arange(ctx, dtype=np.int32).reshape(1, 1, -1).repeat(w.h_kv, axis=1)
    kv = dev.kv_cache(w, kv_len=lens)
    q = dev.draft_queries(w, 0)
    sparse = sd.sd_sparse_attention(q, kv, dev.int32(idx), dev.int32([ctx]), 1)
    dense = sd.sd_verify_attention(q, kv)
    ref = oracle.verify_attention(w.h_q, w.q_draft[0], [0, 1],
                                  oracle.cache_from_workload(w, kv_len=lens))
    _assert_close(sparse, ref, w.dtype, "sparse-all")
    _assert_close(dense, ref, w.dtype, "dense")


@pytest.mark.parametrize("cfg,kw", [(1, dict(l_vis=4000, l_txt=300)),
                                    (3, dict(layers=3, l_vis=5000, l_txt=600)),
                                    (4, dict(l_vis=3000, l_txt=200, batch=5))])
def test_sparse_staged_selection_reused_across_draft_steps(cfg, kw):
    """One staged selection serves every draft step (the tail grows, the selection does not);
    each step matches the oracle and the unstaged call."""
    w = gen.make_attn_workload(cfg, **kw)
    idx = _oracle_topk(w, w.kv_len_verify, w.topk)
    tail = w.l_vis.astype(np.int32)
    kv0 = dev.kv_cache(w, kv_len=w.kv_len_draft(0))
    sel = sd.sd_sparse_stage(kv0, dev.int32(idx), dev.int32(tail))
    for step in range(int(w.gamma.min())):  # steps every sequence drafts
        lens = w.kv_len_draft(step)
        kv = dev.kv_cache(w, kv_len=lens)
        q = dev.draft_queries(w, step)
        max_tail = int((lens - tail).max())
        out = sd.sd_sparse_attention_staged(q, kv, sel, w.topk, dev.int32(tail), max_tail)
        ref = oracle.sparse_attention(w.h_q, w.q_draft[step], np.arange(w.n_seq + 1),
                                      oracle.cache_from_workload(w, kv_len=lens), idx, tail)
        _assert_close(out, ref, w.dtype, f"staged cfg{cfg} step {step}")
        direct = sd.sd_sparse_attention(q, kv, dev.int32(idx), dev.int32(tail), max_tail)
        assert (out.float() - direct.float()).abs().max().item() <= TOL[w.dtype]


@pytest.mark.parametrize("tail_back", [1, 3, 40])
def test_sparse_multi_row_tail_above_row_limits(tail_back):
    """Several rows per sequence with the tail starting above the lowest rows' causal limit:
    some selected positions are then invisible to some rows (the positions are checked one by
    one)."""
    w = gen.make_attn_workload(1, l_vis=3000, l_txt=200, gamma=4)
    kv, q = dev.kv_cache(w), dev.verify_queries(w)
    kv_len = int(w.kv_len_verify[0])
    tail = np.array([kv_len - tail_back], np.int32)
    cache = oracle.cache_from_workload(w)
    idx, _ = oracle.topk_select(w.h_q, w.q_verify, w.q_verify_start, cache,
                                np.zeros(1, np.int32), tail, 256)
    out = sd.sd_sparse_attention(q, kv, dev.int32(idx), dev.int32(tail), tail_back)
    ref = oracle.sparse_attention(w.h_q, w.q_verify, w.q_verify_start, cache, idx, tail)
    _assert_close(out, ref, w.dtype, f"sparse multi-row tail_back={tail_back}")


def test_sparse_unsorted_indices_set_flag():
    w = gen.make_attn_workload(0)
    lens = w.kv_len_draft(0)
    idx = np.array([[[5, 3, 9, 9, 100]]], np.int32)
    kv = dev.kv_cache(w, kv_len=lens)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    sd.sd_sparse_attention(dev.draft_queries(w, 0), kv, dev.int32(idx),
                           dev.int32(w.l_vis), 100, dev_err=flag)
    torch.cuda.synchronize()
    assert flag.item() & sd.SD_DEVERR_INDEX


@pytest.mark.parametrize("l_vis,l_txt,batch", [(300, 40, 7), (1500, 100, 5), (700, 33, 9)])
def test_verify_short_chunks_repeated(l_vis, l_txt, batch):
    """Short sequences split into CTAs of one to three tiles, run repeatedly: every run must
    match the oracle and be bitwise identical (catches pipeline races in the epilogue)."""
    w = gen.make_attn_workload(4, l_vis=l_vis, l_txt=l_txt, batch=batch)
    kv, q = dev.kv_cache(w), dev.verify_queries(w)
    ref = oracle.verify_attention(w.h_q, w.q_verify, w.q_verify_start, oracle.cache_from_workload(w))
    first = None
    for _ in range(12):
        out = sd.sd_verify_attention(q, kv)
        _assert_close(out, ref, w.dtype, "short chunks")
        bits = out.view(torch.int16).clone()
        if first is None:
            first = bits
        else:
            assert torch.equal(first, bits)


# ---------------------------------------------------------------- CUDA-core engine ---------
# The tensor-core kernel serves bf16 calls with at most 128 planned rows per KV head whose Q
# and O are 16-byte aligned and whose cache the copy engine can describe; every other call runs
# on the CUDA-core engine.  These cases reach that engine on purpose.


def _unaligned_like(t):
    """A contiguous copy of t whose data starts 2 bytes past a 16-byte boundary."""
    flat = torch.empty(t.numel() + 8, dtype=t.dtype, device=t.device)
    view = flat[1:1 + t.numel()].view(t.shape)
    view.copy_(t)
    assert view.data_ptr() % 16 != 0
    return view


@pytest.mark.parametrize("cfg,kw", [
    (1, dict(l_vis=2000, l_txt=150, gamma=19)),               # 140 rows per KV head
    (0, dict(dtype="bf16", l_vis=1500, l_txt=90, gamma=33)),  # d=64, 136 rows
])
def test_verify_cuda_core_engine_more_than_128_rows(cfg, kw):
    w = gen.make_attn_workload(cfg, **kw)
    assert w.group * int(w.n_q_verify.max()) > 128
    out = sd.sd_verify_attention(dev.verify_queries(w), dev.kv_cache(w))
    ref = oracle.verify_attention(w.h_q, w.q_verify, w.q_verify_start, oracle.cache_from_workload(w))
    _assert_close(out, ref, w.dtype, f"verify >128 rows cfg{cfg}")


@pytest.mark.parametrize("kind", ["verify", "text_anchored", "sparse"])
def test_cuda_core_engine_unaligned_q_and_out_bf16(kind):
    """Q and O that start off a 16-byte boundary cannot feed the tensor-core kernel."""
    w = gen.make_attn_workload(1, l_vis=3000, l_txt=200, gamma=3)
    q0 = dev.verify_queries(w)
    q = sd.Queries(_unaligned_like(q0.q), q0.q_start, q0.desc.max_q_rows, q0.desc.max_kv_len)
    out = _unaligned_like(torch.zeros_like(q0.q))
    kv = dev.kv_cache(w)
    cache = oracle.cache_from_workload(w)
    if kind == "verify":
        sd.sd_verify_attention(q, kv, out=out)
        ref = oracle.verify_attention(w.h_q, w.q_verify, w.q_verify_start, cache)
    elif kind == "text_anchored":
        vb, ve, win = np.zeros(1, np.int32), w.l_vis.astype(np.int32), np.array([150], np.int32)
        sd.sd_text_anchored_attention(q, kv, dev.int32(vb), dev.int32(ve), dev.int32(win), 150,
                                      out=out)
        ref = oracle.text_anchored_attention(w.h_q, w.q_verify, w.q_verify_start, cache, vb, ve,
                                             win)
    else:
        idx, _ = oracle.topk_select(w.h_q, w.q_verify, w.q_verify_start, cache,
                                    np.zeros(1, np.int32), w.l_vis, 300)
        tail = w.l_vis.astype(np.int32)
        sd.sd_sparse_attention(q, kv, dev.int32(idx), dev.int32(tail),
                               int(w.kv_len_verify[0] - tail[0]), out=out)
        ref = oracle.sparse_attention(w.h_q, w.q_verify, w.q_verify_start, cache, idx, tail)
    _assert_close(out, ref, w.dtype, f"unaligned {kind}")


@pytest.mark.parametrize("kw", [dict(gamma=5), dict(gamma=0, l_vis=3000, l_txt=100),
                                dict(gamma=2, l_vis=700, l_txt=33, layers=3)])
def test_verify_fp32_head_dim_128(kw):
    """fp32 caches with the 7B-like head shapes (d=128, G=7): CUDA cores, 1e-4."""
    w = gen.make_attn_workload(1, dtype="f32", **kw)
    out = sd.sd_verify_attention(dev.verify_queries(w), dev.kv_cache(w))
    ref = oracle.verify_attention(w.h_q, w.q_verify, w.q_verify_start, oracle.cache_from_workload(w))
    _assert_close(out, ref, w.dtype, f"fp32 d=128 {kw}")


def test_draft_calls_fp32_head_dim_128():
    w = gen.make_attn_workload(1, dtype="f32", l_vis=2500, l_txt=300)
    out, ref = _text_anchored_case(w, step=2, window=200)
    _assert_close(out, ref, w.dtype, "fp32 text-anchored d=128")
    lens = w.kv_len_draft(1)
    idx = _oracle_topk(w, w.kv_len_verify, 256)
    tail = w.l_vis.astype(np.int32)
    out = sd.sd_sparse_attention(dev.draft_queries(w, 1), dev.kv_cache(w, kv_len=lens),
                                 dev.int32(idx), dev.int32(tail), int((lens - tail).max()))
    ref = oracle.sparse_attention(w.h_q, w.q_draft[1], np.arange(w.n_seq + 1),
                                  oracle.cache_from_workload(w, kv_len=lens), idx, tail)
    _assert_close(out, ref, w.dtype, "fp32 sparse d=128")


# ---------------------------------------------------------------- full-size draft calls ----


@pytest.fixture(scope="module")
def c3_full():
    """The 28-layer Sparse-to-Dense workload (25,000 visual + 1,024 text positions) on the GPU,
    with the device's own top-K selection, as the benchmark cycle runs it."""
    w = gen.make_attn_workload(3)
    k, v = dev.tensor(w.k, w.dtype), dev.tensor(w.v, w.dtype)
    kv_verify = dev.kv_cache(w, k=k, v=v)
    L = w.n_seq
    idx = sd.sd_topk_select(dev.verify_queries(w), kv_verify, dev.int32(np.zeros(L)),
                            dev.int32(w.l_vis), int(w.l_vis.max()), w.topk).cpu().numpy()
    return w, k, v, idx


SAMPLED_LAYERS = (0, 13, 27)


def _layer_cache(w, layer, lens):
    return oracle.Cache(w.dtype, w.k[layer:layer + 1], w.v[layer:layer + 1],
                        lens[layer:layer + 1], w.h_kv, w.d)


@pytest.mark.parametrize("step", [0, 7])
def test_staged_sparse_full_launch_sampled_layers(c3_full, step):
    """The benchmark's exact staged sparse call: 28 layers x (1,024 selected + tail) in one
    launch, three layers checked in full against the oracle (with the oracle's own top-K)."""
    w, k, v, idx = c3_full
    nq = int(w.n_q_verify[0])
    tail = w.l_vis.astype(np.int32)
    kv0 = dev.kv_cache(w, kv_len=w.kv_len_draft(0), k=k, v=v)
    sel = sd.sd_sparse_stage(kv0, dev.int32(idx), dev.int32(tail))
    lens = w.kv_len_draft(step)
    max_tail = int(max(int((w.kv_len_draft(t) - w.l_vis).max()) for t in range(int(w.gamma[0]))))
    out = sd.sd_sparse_attention_staged(dev.draft_queries(w, step),
                                        dev.kv_cache(w, kv_len=lens, k=k, v=v), sel, w.topk,
                                        dev.int32(tail), max_tail)
    got = dev.to_numpy_f64(out)
    assert np.isfinite(got).all()
    for layer in SAMPLED_LAYERS:
        ridx, gap = oracle.topk_select(w.h_q, w.q_verify[layer * nq:(layer + 1) * nq], [0, nq],
                                       _layer_cache(w, layer, w.kv_len_verify), [0],
                                       w.l_vis[layer:layer + 1], w.topk)
        assert np.array_equal(idx[layer:layer + 1], ridx), (layer, gap)
        ref = oracle.sparse_attention(w.h_q, w.q_draft[step][layer:layer + 1], [0, 1],
                                      _layer_cache(w, layer, lens), ridx, tail[layer:layer + 1])
        err = np.abs(got[layer:layer + 1] - ref).max()
        assert err <= TOL[w.dtype], (layer, step, err)


@pytest.mark.parametrize("step", [0, 7])
def test_text_anchored_full_launch_sampled_layers(c3_full, step):
    """The benchmark's exact text-anchored call: 28 layers, window 1,024 above a 25,000-position
    visual span, one launch; three layers checked in full."""
    w, k, v, _ = c3_full
    L = w.n_seq
    lens = w.kv_len_draft(step)
    vb, ve = np.zeros(L, np.int32), w.l_vis.astype(np.int32)
    out = sd.sd_text_anchored_attention(dev.draft_queries(w, step),
                                        dev.kv_cache(w, kv_len=lens, k=k, v=v), dev.int32(vb),
                                        dev.int32(ve), dev.int32(w.window), int(w.window.max()))
    got = dev.to_numpy_f64(out)
    assert np.isfinite(got).all()
    for layer in SAMPLED_LAYERS:
        sl = slice(layer, layer + 1)
        ref = oracle.text_anchored_attention(w.h_q, w.q_draft[step][sl], [0, 1],
                                             _layer_cache(w, layer, lens), vb[sl], ve[sl],
                                             w.window[sl])
        err = np.abs(got[sl] - ref).max()
        assert err <= TOL[w.dtype], (layer, step, err)
