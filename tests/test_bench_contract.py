"""The benchmark's host-side contract on CPU: the algorithmic byte count of a cycle and the
JSON line of the reference arm (the fp64 oracle timed on the host cores)."""
import json
import os
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_call_bytes_count_each_operand_once():
    import bench
    from speculative_decoding_attention_verify_b200 import inputs as gen
    w = gen.make_attn_workload(1)  # one layer: 8,192 visual + 512 text positions, gamma 5
    g = int(w.gamma[0])
    kv_row = w.h_kv * w.d * 2 * 2  # K and V of one position over all KV heads, bf16
    n_q = int(w.n_q_verify[0])
    q_and_o = 2 * n_q * w.h_q * w.d * 2
    assert bench.call_bytes(w, "verify") == int(w.kv_len_verify[0]) * kv_row + q_and_o
    # top-K reads K of every visual candidate once, the last query row, writes K indices
    assert bench.call_bytes(w, "topk", topk=w.topk) == int(w.l_vis[0]) * w.h_kv * w.d * 2 + \
        w.h_q * w.d * 2 + w.h_kv * w.topk * 4
    # each draft step: the window (or all non-visual positions) for text-anchored attention,
    # the selection plus the dense tail for sparse attention, one query row and one output row
    for t in range(g):
        ta = min(int(w.window[0]), int(w.l_txt[0]) + t + 1) * kv_row + 2 * w.h_q * w.d * 2
        sp = (w.topk + int(w.l_txt[0]) + t + 1) * kv_row + w.h_kv * w.topk * 4 + \
            2 * w.h_q * w.d * 2
        assert bench.call_bytes(w, "text_anchored", t) == ta
        assert bench.call_bytes(w, "sparse", t, topk=w.topk) == sp
    # HSR: the [D][2D] weight once, [e ; h] in and y out
    D = 3584
    assert bench.call_bytes(w, "hsr", hsr_d=D) == D * 2 * D * 2 + 3 * D * 2
    aw = gen.make_accept_workload(2, gammas=[7], batch=1)
    V = aw.vocab
    assert bench.call_bytes(w, "accept_greedy", aw=aw) == 8 * V * 4 + 7 * 4
    assert bench.call_bytes(w, "accept_sample", aw=aw) == 15 * V * 4 + 2 * V * 4 + 7 * 8 + 8 * 4


def test_traffic_record_is_used_only_for_the_current_code(tmp_path, monkeypatch):
    import bench
    rec = {"calls": {"verify": {"traffic_bytes_per_launch": 123.0,
                                "source_hash": bench.kernel_source_hash()},
                     "topk": {"traffic_bytes_per_launch": 456.0, "source_hash": "stale"}}}
    path = tmp_path / "ncu_traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", str(path))
    assert bench.recorded_traffic() == {"verify": 123.0}
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", str(tmp_path / "missing.json"))
    assert bench.recorded_traffic() == {}


def test_committed_traffic_record_is_well_formed():
    import bench
    with open(bench.TRAFFIC_RECORD) as f:
        rec = json.load(f)
    for kind, entry in rec["calls"].items():
        assert kind in bench.KERNELS
        for key in ("kernel", "traffic_bytes_per_launch", "source_hash", "workload", "command"):
            assert key in entry, (kind, key)


def test_reference_arm_prints_the_contract_line():
    env = dict(os.environ, PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["value"] > 0 and np.isfinite(line["value"])
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"].startswith("C3")


def test_code_hash_ignores_comments_but_not_code():
    import bench
    a = 'int f(int x) { // scale\n    return 2 * x; /* twice */ }\nconst char *s = "a // b";\n'
    b = 'int f(int x) {\n  return 2 * x;\n}\n// a new comment line\nconst char *s = "a // b";'
    c = 'int f(int x) { return 3 * x; }\nconst char *s = "a // b";'
    d = 'int f(int x) { return 2 * x; }\nconst char *s = "a /* b";'
    assert bench.strip_comments(a) == bench.strip_comments(b)
    assert bench.strip_comments(a) != bench.strip_comments(c)
    assert bench.strip_comments(a) != bench.strip_comments(d)  # string contents count
