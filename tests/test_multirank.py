"""Host logic of the multi-rank bench on CPU: two gloo ranks, no GPU.

The forward path has no exchange step, so N GPUs run N independent replicas; what
the ranks share is the timing protocol: a barrier on both sides of the timed region,
the maximum of the per-rank step times, the job value as all ranks' units over that
maximum, and rank 0 alone printing (the reference arm runs on rank 0 only).
"""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench.dist_ctx()
        assert (w, r, lr) == (world, rank, rank)
        bench.barrier(world)
        # rank r timed (r + 1) ms per step: the job time is the slowest rank's
        ms = bench.max_over_ranks(float(rank + 1), world, torch.device("cpu"))
        value = bench.job_throughput(units_per_rank=3, world=world, ms_per_step=ms)
        # the reference arm: every rank but 0 leaves without work or output
        buf = io.StringIO()
        if rank != 0:
            with redirect_stdout(buf):
                bench.run_reference(None, None)
        bench.barrier(world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms": ms, "value": value, "ref_out": buf.getvalue()}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_the_timing_protocol(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(world)]
    for r in res:
        assert r["ms"] == pytest.approx(2.0)  # max over ranks of 1 ms and 2 ms
        assert r["value"] == pytest.approx(world * 3 / 2e-3)  # 6 tokens per 2 ms
    assert res[1]["ref_out"] == ""


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert not dist.is_initialized()
    assert bench.max_over_ranks(4.5, 1, torch.device("cpu")) == 4.5
    bench.barrier(1)
    assert bench.job_throughput(units_per_rank=1, world=1, ms_per_step=0.5) == pytest.approx(2000.0)


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` at N=1 runs on the host cores only: one JSON line with
    the arm's metric, unit and workload, the oracle's throughput as `value`, a
    `cpu_baseline` describing the run and an `e2e` with no host-device bytes, and at
    least three warm-up steps whatever is asked."""
    import subprocess

    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["n_gpus"] == 1 and j["steps"] == 1 and j["warmup"] >= 3
    assert j["unit"] == "tokens/s" and j["higher_is_better"] is True and j["value"] > 0
    assert j["ms_per_step"] > 0 and j["dtype"] == "f64" and j["data"] == "synthetic"
    assert j["config"]["workload"] == "decode_bf16_512k" and j["config"]["kv_len"] == 524288
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == j["value"] and cb["cores"] >= 1 and cb["sample"]
    assert j["e2e"] == {"value": j["value"], "unit": j["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
