"""The algorithmic counts behind the bench's roofline figures, against hand-derived
closed forms (no GPU).

Decode step (per query head, at t = L - 1 with C_e = floor(t / 64) eligible chunks):
the summary table row of every eligible chunk (d bf16 values and a float32 b'), the K
kept chunks and the W window tokens of K and V (read once per key-value head), and
the small per-query vectors. Prefill (per head, queries i = 0..N-1, e_i = floor(i / 64)
eligible chunks): scores 2d per (query, eligible chunk), chunk attention 4dS per
(query, kept chunk), window 4d per (query, window token), summaries 4dS per chunk.
Backward: 10d per (query, attended token), 4d per (query, kept chunk), 8dS per chunk.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from hils_synth import WORKLOADS  # noqa: E402


def test_decode_bytes_512k():
    by = bench.decode_bytes(WORKLOADS[4])  # B1 H32 d128, L = 524288, K16, W512, bf16
    heads, eligible = 32, 524287 // 64  # 8191 chunks strictly before the query's own
    table = heads * eligible * (128 * 2 + 4)
    kv = heads * (16 * 64 + 512) * 128 * 2 * 2
    small = heads * (2 * 128 * 2 + 16 * 8 + 4)
    assert table == 68_149_120 and kv == 25_165_824
    assert by == {"select": table + small, "attend": kv + small, "step": table + kv + small}
    assert by["select"] == 68_169_728 and by["step"] == 93_335_552


def test_decode_bytes_grouped_reads_kv_once_per_key_value_head():
    mh, gq = bench.decode_bytes(WORKLOADS[4]), bench.decode_bytes(WORKLOADS[8])  # 32 vs 8 KV heads
    small = 32 * (2 * 128 * 2 + 16 * 8 + 4)
    assert gq["select"] == mh["select"]
    assert gq["attend"] - small == (mh["attend"] - small) // 4


def test_prefill_flops_8k():
    w = WORKLOADS[2]  # B1 H32 d128 N8192, K16, W512
    d, S, H = 128, 64, 32
    # sum over queries of min(K, e_i): 64 queries per e = 0..127
    kept = 64 * (sum(range(16)) + (128 - 16) * 16)
    assert kept == 122_368
    # sum over queries of min(W, i + 1)
    win_tok = sum(range(1, 513)) + (8192 - 512) * 512
    assert win_tok == 4_063_488
    eligible = 64 * sum(range(128))
    attend = H * (4 * d * S * kept + 4 * d * win_tok)
    step = attend + H * (2 * d * eligible + 4 * d * S * 128)
    assert bench.prefill_flops(w, "attend") == pytest.approx(attend, rel=0, abs=0)
    assert bench.prefill_flops(w) == pytest.approx(step, rel=0, abs=0)
    assert round(attend / 1e9, 1) == 194.9 and round(step / 1e9, 1) == 199.3


def test_backward_flops_8k():
    w = WORKLOADS[2]
    d, S, H = 128, 64, 32
    kept = 64 * (sum(range(16)) + (128 - 16) * 16)
    tok = S * kept + sum(range(1, 513)) + (8192 - 512) * 512
    want = H * (10 * d * tok + 4 * d * kept + 8 * d * S * 128)
    assert bench.backward_flops(w) == want
    assert round(want / 1e9, 1) == 489.5


def test_decode_input_copies_cover_three_l2_sizes():
    """Decode steps cycle over R input copies; R is the least count >= 2 whose bytes per
    cycle reach three L2 sizes, so a copy is evicted before it is read again."""
    l2 = 126 * 2**20
    for cfg in (3, 4, 5, 8, 9):
        w = WORKLOADS[cfg]
        step = bench.decode_bytes(w)["step"]
        R = bench.decode_sets(w, l2)
        assert R >= 2 and R * step >= 3 * l2
        assert R == 2 or (R - 1) * step < 3 * l2
    assert bench.decode_sets(WORKLOADS[4], l2) == 5  # 93.3 MB per step


def test_traffic_record_goes_null_when_the_kernel_changes(monkeypatch):
    """A traffic capture counts only for the source it was taken on."""
    dig = bench.source_digest("summarize")
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, "summarize", (17000.0, dig))
    assert bench.measured_traffic("summarize", scale=10) == 170000.0
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, "summarize", (17000.0, "0" * 16))
    assert bench.measured_traffic("summarize", scale=10) is None


def test_reference_arm_runs_the_oracle_alone(tmp_path):
    """The reference arm on a small decode workload: one JSON line with the config of
    the library's arm, and the CUDA library never imported."""
    import json
    import subprocess

    code = (
        "import sys, json, types; sys.path.insert(0, %r); import bench; from hils_synth import WORKLOADS;"
        "w = WORKLOADS[4].replace(H=4, N=64 * 300, needles=1);"
        "bench.run_reference(types.SimpleNamespace(gpus=1, steps=2, warmup=1), w);"
        "assert 'hierarchical_chunk_sparse_b200' not in sys.modules;"
        "print(json.dumps(bench.decode_config(w, 1)))" % ROOT)
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0, out.stderr
    lines = [json.loads(x) for x in out.stdout.strip().splitlines()]
    ref, cfg = lines[0], lines[1]
    assert ref["impl"] == "reference" and ref["config"] == cfg
    assert ref["value"] > 0 and ref["steps"] == 2 and ref["warmup"] == 1
    assert ref["e2e"]["h2d_bytes_per_step"] == 0 and ref["cpu_baseline"]["kind"] == "oracle"
