"""C-ABI checks that need no GPU: the library builds, loads and exports every symbol the
public header declares, and host-side validation rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

from speculative_decoding_attention_verify_b200 import sdattn as sd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sd_attn.h")
FAKE = ctypes.c_void_p(0x7f0000001000)  # 16-byte aligned, never dereferenced by the host


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^SD_API\s+[\w\s\*]+?\b(sd_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("sd_verify_attention", "sd_text_anchored_attention", "sd_sparse_attention",
              "sd_topk_select", "sd_hsr_project", "sd_accept_greedy", "sd_accept_sample"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = sd.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(sd.EXPORTS) == set(declared_functions())


def test_status_strings_and_version():
    lib = sd.lib()
    assert lib.sd_status_string(0) == b"SD_OK"
    assert b"workspace" in lib.sd_status_string(3)
    assert lib.sd_version() >= 100


def _descs(h_q=28, h_kv=4, d=128, dtype=sd.SD_BF16, max_q=8, max_kv=4096):
    kv = sd.sd_kv_desc()
    kv.dtype, kv.h_kv, kv.head_dim, kv.page_size = dtype, h_kv, d, 0
    kv.k = kv.v = kv.kv_len = FAKE
    kv.stride_b, kv.stride_h, kv.stride_pos = h_kv * max_kv * d, max_kv * d, d
    q = sd.sd_q_desc()
    q.h_q, q.max_q_rows, q.max_kv_len, q.softmax_scale, q.q_start = h_q, max_q, max_kv, 0.0, FAKE
    return q, kv


def _verify(q, kv, batch=2, ws_bytes=0, ws=None):
    return sd.lib().sd_verify_attention(ctypes.byref(q), FAKE, ctypes.byref(kv), batch, FAKE, ws,
                                        ws_bytes, None, None)


def test_sparse_workspace_query_includes_the_staged_selection():
    q, kv = _descs(max_q=1, max_kv=30000)
    n = ctypes.c_size_t(0)
    assert sd.lib().sd_attention_workspace_size(sd.SD_ATTN_SPARSE, ctypes.byref(q),
                                                ctypes.byref(kv), 28,
                                                ctypes.byref(n)) == sd.SD_ERR_INVALID_ARG
    assert sd.lib().sd_sparse_workspace_size(ctypes.byref(q), ctypes.byref(kv), 28, 1024, 1100,
                                             ctypes.byref(n)) == sd.SD_OK
    staged = 28 * 4 * 1024 * 128 * 2 * 2  # compact K and V, bf16
    assert n.value >= staged
    m = ctypes.c_size_t(0)
    assert sd.lib().sd_sparse_workspace_size(ctypes.byref(q), ctypes.byref(kv), 28, 512, 1100,
                                             ctypes.byref(m)) == sd.SD_OK
    assert m.value < n.value
    # too small a workspace is rejected before any launch
    assert sd.lib().sd_sparse_attention(ctypes.byref(q), FAKE, ctypes.byref(kv), 28, FAKE, 1024,
                                        FAKE, 1100, FAKE, FAKE, n.value - 1, None,
                                        None) == sd.SD_ERR_WORKSPACE


def test_workspace_query_and_undersized_workspace_is_rejected():
    q, kv = _descs()
    n = ctypes.c_size_t(0)
    assert sd.lib().sd_attention_workspace_size(sd.SD_ATTN_VERIFY, ctypes.byref(q),
                                                ctypes.byref(kv), 2, ctypes.byref(n)) == 0
    if n.value > 0:
        assert _verify(q, kv, ws_bytes=n.value - 1, ws=FAKE) == sd.SD_ERR_WORKSPACE
        assert _verify(q, kv, ws_bytes=n.value, ws=None) == sd.SD_ERR_WORKSPACE


@pytest.mark.parametrize("mutate,expected", [
    (lambda q, kv: setattr(q, "h_q", 27), sd.SD_ERR_INVALID_ARG),          # not a multiple of h_kv
    (lambda q, kv: (setattr(kv, "head_dim", 96), setattr(kv, "stride_pos", 96)), sd.SD_ERR_UNSUPPORTED),
    (lambda q, kv: setattr(kv, "dtype", 7), sd.SD_ERR_INVALID_ARG),
    (lambda q, kv: setattr(kv, "k", None), sd.SD_ERR_INVALID_ARG),
    (lambda q, kv: setattr(kv, "k", ctypes.c_void_p(0x7f0000001002)), sd.SD_ERR_INVALID_ARG),
    (lambda q, kv: setattr(kv, "stride_pos", 256), sd.SD_ERR_INVALID_ARG),
    (lambda q, kv: setattr(q, "max_q_rows", 0), sd.SD_ERR_INVALID_ARG),
    (lambda q, kv: setattr(q, "softmax_scale", float("nan")), sd.SD_ERR_INVALID_ARG),
    (lambda q, kv: setattr(kv, "page_size", 8), sd.SD_ERR_INVALID_ARG),
])
def test_invalid_descriptors_are_rejected_before_launch(mutate, expected):
    q, kv = _descs()
    mutate(q, kv)
    assert _verify(q, kv) == expected


def test_other_entry_points_validate_on_the_host():
    lib = sd.lib()
    q, kv = _descs()
    P = FAKE
    # sparse: negative k
    assert lib.sd_sparse_attention(ctypes.byref(q), P, ctypes.byref(kv), 1, P, -1, P, 10, P, None,
                                   0, None, None) == sd.SD_ERR_INVALID_ARG
    # text-anchored: window hint must be >= 1
    assert lib.sd_text_anchored_attention(ctypes.byref(q), P, ctypes.byref(kv), 1, P, P, P, 0, P,
                                          None, 0, None, None) == sd.SD_ERR_INVALID_ARG
    # top-K: k < 1, and an undersized workspace
    assert lib.sd_topk_select(ctypes.byref(q), P, ctypes.byref(kv), 1, P, P, 100, 0, P, None, 0,
                              None, None) == sd.SD_ERR_INVALID_ARG
    assert lib.sd_topk_select(ctypes.byref(q), P, ctypes.byref(kv), 1, P, P, 100, 10, P, P, 8,
                              None, None) == sd.SD_ERR_WORKSPACE
    # HSR: too many rows, misaligned pointer, d_model not a multiple of 8
    assert lib.sd_hsr_project(P, P, 17, 3584, P, None, P, None) == sd.SD_ERR_INVALID_ARG
    assert lib.sd_hsr_project(ctypes.c_void_p(0x7f0000001002), P, 1, 3584, P, None, P,
                              None) == sd.SD_ERR_INVALID_ARG
    assert lib.sd_hsr_project(P, P, 1, 3580, P, None, P, None) == sd.SD_ERR_INVALID_ARG
    assert lib.sd_hsr_project(P, P, 1, 3592, P, None, P, None) == sd.SD_ERR_INVALID_ARG
    # acceptance: out_stride too small, missing workspace
    assert lib.sd_accept_greedy(P, P, P, 2, 7, 1000, P, P, 7, P, 1 << 20, None,
                                None) == sd.SD_ERR_INVALID_ARG
    assert lib.sd_accept_greedy(P, P, P, 2, 7, 1000, P, P, 8, None, 0, None,
                                None) == sd.SD_ERR_WORKSPACE
    assert lib.sd_accept_sample(P, P, P, P, None, P, 2, 7, 1000, P, P, 8, None, P, 1 << 20, None,
                                None) == sd.SD_ERR_INVALID_ARG


def test_workspace_sizes_scale_with_the_problem():
    lib = sd.lib()
    n1, n2 = ctypes.c_size_t(0), ctypes.c_size_t(0)
    assert lib.sd_accept_workspace_size(1, 7, 152064, ctypes.byref(n1)) == 0
    assert lib.sd_accept_workspace_size(8, 7, 152064, ctypes.byref(n2)) == 0
    assert n1.value > 0 and n2.value > 0
    _, kv = _descs()
    assert lib.sd_topk_workspace_size(ctypes.byref(kv), 28, 25000, 1024, ctypes.byref(n1)) == 0
    # 64-bit key slots per candidate, then the fp32 scoring's per-split partials (8 bytes for
    # each of up to ceil(25000 / 128) / 4 = 49 splits)
    assert n1.value == 28 * 4 * 25000 * 8 + 28 * 4 * 49 * 8


def test_topk_scored_validation():
    q, kv = _descs(max_q=64, max_kv=4096)
    lib = sd.lib()
    n = ctypes.c_size_t(0)
    assert lib.sd_topk_scored_workspace_size(7, ctypes.byref(q), ctypes.byref(kv), 2, 4000, 64,
                                             ctypes.byref(n)) == sd.SD_ERR_INVALID_ARG
    assert lib.sd_topk_scored_workspace_size(sd.SD_TOPK_MEAN_TEXT_ATTENTION, ctypes.byref(q),
                                             ctypes.byref(kv), 2, 4000, 64,
                                             ctypes.byref(n)) == sd.SD_OK
    keys = 2 * 4 * 4000 * 8
    assert n.value >= keys + 2 * 64 * 28 * 4
    call = lambda mode, ws, nbytes: lib.sd_topk_select_scored(
        mode, ctypes.byref(q), FAKE, ctypes.byref(kv), 2, FAKE, FAKE, 4000, 64, FAKE, None, ws,
        nbytes, None, None)
    assert call(5, FAKE, n.value) == sd.SD_ERR_INVALID_ARG
    assert call(sd.SD_TOPK_MEAN_TEXT_ATTENTION, FAKE, n.value - 1) == sd.SD_ERR_WORKSPACE
    assert call(sd.SD_TOPK_MEAN_TEXT_ATTENTION, ctypes.c_void_p(0x7f0000001010),
                n.value) == sd.SD_ERR_WORKSPACE  # not 256-byte aligned
    assert call(sd.SD_TOPK_MEAN_TEXT_ATTENTION, None, n.value) == sd.SD_ERR_WORKSPACE


def test_wait_timeout_setting_round_trips():
    lib = sd.lib()
    prev = sd.sd_set_wait_timeout_ns(5000)
    assert prev == 10**9  # the default bound of 1 s
    assert sd.sd_set_wait_timeout_ns(0) == 5000   # 0 restores the default ...
    assert sd.sd_set_wait_timeout_ns(0) == 10**9  # ... which is what is now set
    assert lib.sd_version() >= 200


def _plan(kind, q, kv, batch, extent=0, max_tail=0):
    e, n = ctypes.c_int32(-1), ctypes.c_int32(-1)
    st = sd.lib().sd_attention_plan(kind, ctypes.byref(q), ctypes.byref(kv), batch, extent,
                                    max_tail, ctypes.byref(e), ctypes.byref(n))
    return st, e.value, n.value


def test_attention_plan_picks_the_decomposition():
    """Host-only planning (148 SMs assumed without a device): long streams over many units get
    the persistent tensor-core decomposition, the short draft calls the per-unit one, fp32 and
    more than 128 rows per KV head the CUDA-core engine; the workspace covers the plan."""
    # 28 layers x 9 rows x 7 heads per KV head over 26,033 positions: persistent
    q, kv = _descs(max_q=9, max_kv=26033)
    st, eng, parts = _plan(sd.SD_ATTN_VERIFY, q, kv, 28)
    assert st == sd.SD_OK and eng == sd.SD_ENGINE_TC_PERSISTENT and 2 <= parts <= 8
    n = ctypes.c_size_t(0)
    assert sd.lib().sd_attention_workspace_size(sd.SD_ATTN_VERIFY, ctypes.byref(q),
                                                ctypes.byref(kv), 28, ctypes.byref(n)) == 0
    assert n.value >= parts * 28 * 9 * 28 * (128 + 2) * 4
    # one layer: the per-unit kernel with splits
    st, eng, parts = _plan(sd.SD_ATTN_VERIFY, q, kv, 1)
    assert st == sd.SD_OK and eng == sd.SD_ENGINE_TC and parts > 1
    # the draft calls of the benchmark cycle: per-unit, one split
    q1, kv1 = _descs(max_q=1, max_kv=26025)
    assert _plan(sd.SD_ATTN_TEXT_ANCHORED, q1, kv1, 28, extent=1024)[1:] == (sd.SD_ENGINE_TC, 1)
    assert _plan(sd.SD_ATTN_SPARSE, q1, kv1, 28, extent=1024, max_tail=1025)[1:] == \
        (sd.SD_ENGINE_TC, 1)
    # a large selection or a wide window make the draft streams long: persistent
    assert _plan(sd.SD_ATTN_SPARSE, q1, kv1, 28, extent=8192, max_tail=1025)[1] == \
        sd.SD_ENGINE_TC_PERSISTENT
    assert _plan(sd.SD_ATTN_TEXT_ANCHORED, q1, kv1, 28, extent=8000)[1] == \
        sd.SD_ENGINE_TC_PERSISTENT
    # fp32 caches and more than 128 rows per KV head: CUDA cores
    qf, kvf = _descs(dtype=sd.SD_F32, max_q=9, max_kv=26033)
    assert _plan(sd.SD_ATTN_VERIFY, qf, kvf, 28)[1] == sd.SD_ENGINE_CUDA_CORE
    qr, kvr = _descs(max_q=20, max_kv=26033)
    assert _plan(sd.SD_ATTN_VERIFY, qr, kvr, 28)[1] == sd.SD_ENGINE_CUDA_CORE
    # host validation
    assert _plan(7, q, kv, 28)[0] == sd.SD_ERR_INVALID_ARG
    assert _plan(sd.SD_ATTN_TEXT_ANCHORED, q1, kv1, 28, extent=0)[0] == sd.SD_ERR_INVALID_ARG
    assert _plan(sd.SD_ATTN_VERIFY, q, kv, 0)[0] == sd.SD_ERR_INVALID_ARG
    qd, kvd = _descs(d=96)
    assert _plan(sd.SD_ATTN_VERIFY, qd, kvd, 2)[0] == sd.SD_ERR_UNSUPPORTED
