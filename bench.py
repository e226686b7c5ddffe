#!/usr/bin/env python
"""Benchmark of the HiLS-Attention forward hot path on B200.

Headline (one JSON line on rank 0):
  decode tokens/s at a 512K-token KV cache (B=1, H=32, d=128, chunk 64, top-K 16,
  window 512; synthetic Gaussian K/V with one needle key per head). One step = one
  new token through the whole decode path in one call, hils_decode: the select (Eq. 7
  scores over 8191 chunk summaries + exact top-K) then the attend (Eq. 10 over 16
  chunks + the window). Summaries are built once beforehand (hils_summarize), as a
  server keeps them with its KV cache.
Beside it, in the same line:
  "roofline": the dominant decode kernel against the measured HBM copy bandwidth;
  "e2e": the same decode metric through the Python binding with pinned host
  buffers: the step's query (Q, Q_cal, positions) copied in and (O, lse) copied out
  inside the timed region; KV cache and summaries stay resident in HBM;
  "cold_single_step": the same step with L2 flushed before it, timed alone;
  "prefill", "prefill_local", "prefill_gqa": algorithmic TFLOP/s of summarise + select +
  prefill attend on the 8K prefill workloads (B=1, H=32, d=128, K=16, W=512);
  "decode_b8_128k", "decode_1m" (with the full summary rebuild at 1M, timed alone),
  "decode_gqa", "decode_retrieval": the other decode workloads, each with its own
  roofline;
  "prefill_backward": the backward of the 8K prefill for its selection;
  "cpu_baseline": the float64 oracle on this host's cores, on a sample of heads (also
  inside the B8 128K and 1M decode entries, on smaller samples).

Timing: decode steps run back to back over R independent copies of the workload's
inputs (R copies of KV cache, summaries, queries and outputs, cycled in order) whose
bytes per cycle are at least three times the L2 size, so every step reads its data
cold, as each layer of a model reads its own cache. W warm-up steps, then exactly K
timed steps between two CUDA events on the launching stream; barrier + synchronize
around the region; the max over ranks is reported. Prefill and backward passes (and
the cold single step) are timed one at a time with L2 flushed before each. Multi-GPU
(torchrun): every rank runs its own replica of the workload (weak scaling; the path
has no exchange step) and value = all ranks' tokens / max time. Per-step timings also
report their median and 90th percentile (p50_ms, p90_ms); fractions are given against
the measured peaks (HBM copy, bf16 burst) and against 8 TB/s or the sustained bf16 peak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hils|reference]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hils_synth import WORKLOADS, make_decode, make_prefill  # noqa: E402

METRIC = "HiLS decode tokens/s @512K ctx (%HBM roofline); prefill TFLOP/s @8K (%TC peak)"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- clocks (NVML, read-only)

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    """Polls the SM clock and clock-event reasons of this process's GPU every ~1 ms."""

    def __init__(self, device: torch.device):
        self.samples = []
        self.ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.nv = pynvml
            self.ok = True
        except Exception as e:  # no NVML: report that clocks were not sampled
            self.err = repr(e)

    def _reasons(self):
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return fn(self.h)

    def _loop(self):
        while not self._stop.is_set():
            try:
                self.samples.append((self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM),
                                     self._reasons()))
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._loop, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= int(r)
        reasons = sorted(n for b, n in _REASONS.items() if bits & b and n != "gpu_idle")
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz)}


# ----------------------------------------------------------------- timing helpers

class Flusher:
    """Writes a buffer of twice the L2 size, then reads another of twice the L2 size, so
    that no step starts with warm L2, nor with the flush's dirty lines still to be written
    back (which would charge the step with 126 MB of write-backs it did not cause)."""

    DESCRIPTION = "flushed before every step: 2x L2 written, then 2x L2 read"

    def __init__(self, dev):
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.buf = torch.empty(2 * l2 // 4, dtype=torch.float32, device=dev)
        self.rbuf = torch.ones(2 * l2 // 4, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.buf.fill_(1.0)
        torch.sum(self.rbuf, dim=0, out=self.sink)


def time_steps(fn, steps, flush, stream):
    """Per-step device milliseconds of `fn` on `stream`, L2 flushed before each step."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    with torch.cuda.stream(stream):
        for s, e in ev:
            flush()
            s.record(stream)
            fn()
            e.record(stream)
    stream.synchronize()
    return [s.elapsed_time(e) for s, e in ev]


def spread(ms_list):
    """Median and 90th percentile of per-step milliseconds."""
    v = sorted(ms_list)
    return {"p50_ms": statistics.median(v), "p90_ms": v[min(len(v) - 1, int(round(0.9 * (len(v) - 1))))]}


def graphed(fn, stream):
    """Captures fn (already warmed up) into a CUDA graph on `stream`; returns replay()."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    stream.synchronize()
    return g.replay


def dist_ctx():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, dev) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job rate: every rank processes its own replica's units in each step, and
    the step takes as long as the slowest rank (ms_per_step is already that maximum)."""
    return world * units_per_rank / (ms_per_step / 1e3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ----------------------------------------------------------------- decode workload

def decode_bytes(w) -> dict:
    """Algorithmic HBM bytes of one decode step (per the whole batch). The summary table
    is per query head; the kept chunks and the window of K and V are read once per
    key-value head (a group of query heads shares them)."""
    t = w.N - 1
    c_elig = min(t // w.S, w.C)
    es = 2
    n, nk = w.B * w.H, w.B * w.Hkv
    table = n * c_elig * (w.d * es + 4)
    kv = nk * (w.K * w.S + w.W) * w.d * es * 2
    small = n * (2 * w.d * es + w.K * 8 + 4)  # q~, q, o, kept lists, lse
    return {"select": table + small, "attend": kv + small, "step": table + kv + small}


# Decode steps are timed back to back over R independent copies of the workload's inputs
# (R copies of the KV cache, summary table, queries and outputs, cycled in order), with R
# chosen so that the R steps together touch at least three times the L2 size: every step
# reads its data cold, as each layer of a model reads its own KV cache and summaries.
DECODE_L2 = ("inputs larger than L2: steps cycle over R independent input copies whose bytes per "
             "cycle are >= 3x L2; timed back to back")


def decode_sets(w, l2_bytes: int) -> int:
    step = decode_bytes(w)["step"]
    return max(2, -(-3 * l2_bytes // step))


class DecodeSet:
    """One copy of a decode workload's inputs, summaries, outputs and workspaces."""

    def __init__(self, hils, p, w, inp, Ksum, Bsum, dev):
        self.hils, self.p, self.w = hils, p, w
        self.inp, self.Ksum, self.Bsum = inp, Ksum, Bsum
        C = w.C
        self.qpos = (inp["cache_len"] - 1).reshape(w.B, 1).contiguous()
        self.idx = torch.empty(w.B, w.Hkv, 1, w.K, dtype=torch.int32, device=dev)
        self.score = torch.empty(w.B, w.H, 1, w.K, dtype=torch.float32, device=dev)
        self.nsel = torch.empty(w.B, w.Hkv, 1, dtype=torch.int32, device=dev)
        self.ws_sel = hils.alloc_workspace(p, hils.HILS_CALL_SELECT, 1, C, device=dev)
        self.ws_dec = hils.alloc_workspace(p, hils.HILS_CALL_ATTEND_DECODE, 1, 0, device=dev)
        self.ws_step = hils.alloc_workspace(p, hils.HILS_CALL_DECODE, 1, C, device=dev)
        self.O = torch.empty_like(inp["Q"])
        self.lse = torch.empty(w.B, w.H, dtype=torch.float32, device=dev)

    def select(self):
        i = self.inp
        self.hils.hils_select(self.p, i["Qcal"], self.Ksum, self.Bsum, self.idx, self.score, self.nsel,
                              qpos=self.qpos, workspace=self.ws_sel)

    def attend(self):
        i = self.inp
        self.hils.hils_attend_decode(self.p, i["Q"], i["K"], i["V"], i["cache_len"], self.idx, self.score,
                                     self.nsel, self.O, self.lse, workspace=self.ws_dec)

    def step(self):
        i = self.inp
        self.hils.hils_decode(self.p, i["Qcal"], self.Ksum, self.Bsum, i["Q"], i["K"], i["V"], i["cache_len"],
                              self.idx, self.score, self.nsel, self.O, self.lse, workspace=self.ws_step)

    def e2e_setup(self):
        """The step's inputs (query, calibrated query, cache lengths) and results (O, lse)
        move through one pinned host buffer each way: the device tensors the library
        reads and writes become views of one staging buffer per direction, so a step
        costs one host-to-device and one device-to-host copy."""
        i = self.inp
        ins = [("Q", i["Q"]), ("Qcal", i["Qcal"]), ("cache_len", i["cache_len"])]
        outs = [("O", self.O), ("lse", self.lse)]
        self.d_in, views_in = _staging(ins, self.O.device)
        self.d_out, views_out = _staging(outs, self.O.device)
        for k, v in views_in.items():
            v.copy_(i[k])
            i[k] = v
        self.O, self.lse = views_out["O"], views_out["lse"]
        self.h_in = self.d_in.cpu().pin_memory()
        self.h_out = torch.empty(self.d_out.shape, dtype=torch.uint8).pin_memory()
        return self.h_in.numel(), self.h_out.numel()

    def e2e_step(self):
        self.d_in.copy_(self.h_in, non_blocking=True)
        self.step()
        self.h_out.copy_(self.d_out, non_blocking=True)


def _staging(named, dev):
    """One device byte buffer holding every tensor of `named` (16-byte aligned offsets),
    and a view of the buffer for each tensor with its shape and dtype."""
    off, spans = 0, []
    for name, t in named:
        off = (off + 15) // 16 * 16
        n = t.numel() * t.element_size()
        spans.append((name, t, off, n))
        off += n
    buf = torch.zeros(off, dtype=torch.uint8, device=dev)
    views = {name: buf[o:o + n].view(t.dtype).view(t.shape) for name, t, o, n in spans}
    return buf, views


class DecodeBench:
    """R copies of a decode workload (R >= 2, see decode_sets); summaries built once by
    hils_summarize (untimed), as a server keeps them with its KV cache."""

    def __init__(self, w, dev, sets: int | None = None):
        import hierarchical_chunk_sparse_b200 as hils

        self.hils, self.w, self.dev = hils, w, dev
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.R = sets if sets is not None else decode_sets(w, l2)
        self.p = hils.Params(B=w.B, H=w.H, d=w.d, K=w.K, W=w.W, dtype=w.dtype, H_kv=w.Hk)
        inp = make_decode(w, device=dev)
        Ksum = torch.empty(w.B, w.H, w.C, w.d, dtype=w.dtype, device=dev)
        Bsum = torch.empty(w.B, w.H, w.C, dtype=torch.float32, device=dev)
        hils.hils_summarize(self.p, inp["K"], inp["LQ"], Ksum, Bsum)
        self.needles = inp["needles"]
        self.sets = []
        for r in range(self.R):
            if r == 0:
                ir, kr, br = inp, Ksum, Bsum
            else:
                ir = {k: (v.clone() if isinstance(v, torch.Tensor) and v.is_cuda else v) for k, v in inp.items()}
                kr, br = Ksum.clone(), Bsum.clone()
            ir.pop("LQ", None)  # landmark queries are only needed for the summaries
            self.sets.append(DecodeSet(hils, self.p, w, ir, kr, br, dev))
        del inp
        torch.cuda.synchronize()
        # one step = hils_decode: the screen and pick kernels of the select, then the attend
        self.launches_per_step = 3

    def graphs(self, name, stream):
        """CUDA graphs of `name` (step, select, attend or e2e_step): one over all R sets in
        order, and one per set."""
        fns = [getattr(s, name) for s in self.sets]
        with torch.cuda.stream(stream):
            for f in fns:  # warm (and, for e2e_step, not captured cold)
                f()
        stream.synchronize()

        def run_all():
            for f in fns:
                f()

        return graphed(run_all, stream), [graphed(f, stream) for f in fns]


def time_rotating(graphs, steps: int, stream) -> float:
    """Device milliseconds per step of `steps` steps run back to back: whole cycles over
    the R sets, then the first steps % R sets."""
    g_all, g_one = graphs
    R = len(g_one)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        s.record(stream)
        for _ in range(steps // R):
            g_all()
        for r in range(steps % R):
            g_one[r]()
        e.record(stream)
    stream.synchronize()
    return s.elapsed_time(e) / steps


# ----------------------------------------------------------------- prefill workload

def prefill_flops(w, part: str = "step") -> float:
    """Algorithmic flops of one prefill (per batch): the whole step (summarise + score +
    chunk attention + window) or only the attend's share (chunk attention + window)."""
    d, S, K, W, N, C = w.d, w.S, w.K, w.W, w.N, w.C
    score = chunk = win = 0
    for i in range(N):
        e = min(i // S, C)
        score += 2 * d * e
        chunk += 4 * d * S * min(K, e)
        win += 4 * d * min(W, i + 1)
    summ = 4 * d * S * C
    total = chunk + win if part == "attend" else score + chunk + win + summ
    return float(w.B * w.H * total)


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) that Nsight Compute
# measured, each with its command in profiles/, keyed by the kernel it describes and the
# digest of that kernel's source files at capture time. A kernel whose sources changed
# after its capture reports null until it is captured again.
CSRC = os.path.join(ROOT, "hierarchical_chunk_sparse_b200", "csrc")
KERNEL_SOURCES = {
    "decode_select": ["select.cu", "screen_stage.cuh", "select_pick.cuh", "select_common.cuh", "tc_common.cuh",
                      "hils_internal.cuh"],
    "decode_attend": ["attend.cu", "attend_common.cuh", "hils_internal.cuh"],
    "attend_prefill": ["attend_prefill_tc.cu", "tc_common.cuh", "fast_math.cuh", "hils_internal.cuh"],
    "summarize": ["summarize.cu", "tc_common.cuh", "hils_internal.cuh"],
}
# kernel -> (DRAM bytes per unit, source digest at capture). Units: decode_select and
# decode_attend per algorithmic byte of the launch (the captured traffic / algorithmic
# bytes), summarize per chunk, attend_prefill per launch of the 8K prefill workload.
MEASURED_TRAFFIC = {
    'decode_select': (1.0160202487532295, 'bee0ccd8a98086ff'),
    'decode_attend': (1.0020989078564204, 'cb90a6455b1fa122'),
    'summarize': (16926.2578125, '853b63865c7de306'),
    'attend_prefill': (661702656, '04b39bda6acf4099'),
}


def source_digest(kernel: str) -> str:
    import hashlib

    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, scale: float = 1.0):
    """DRAM bytes of one timed launch of `kernel`: the captured bytes per unit times the
    launch's units (`scale`), or None if the kernel's sources changed since its capture."""
    rec = MEASURED_TRAFFIC.get(kernel)
    if rec is None or rec[1] != source_digest(kernel):
        return None
    return rec[0] * scale


class PrefillBench:
    def __init__(self, w, dev):
        import hierarchical_chunk_sparse_b200 as hils

        self.hils, self.w = hils, w
        self.inp = make_prefill(w, device=dev)
        self.p = hils.Params(B=w.B, H=w.H, d=w.d, K=w.K, W=w.W, dtype=w.dtype, H_kv=w.Hk)
        C = w.C
        self.Ksum = torch.empty(w.B, w.H, C, w.d, dtype=w.dtype, device=dev)
        self.Bsum = torch.empty(w.B, w.H, C, dtype=torch.float32, device=dev)
        self.idx = torch.empty(w.B, w.Hkv, w.N, w.K, dtype=torch.int32, device=dev)
        self.score = torch.empty(w.B, w.H, w.N, w.K, dtype=torch.float32, device=dev)
        self.nsel = torch.empty(w.B, w.Hkv, w.N, dtype=torch.int32, device=dev)
        self.ws = hils.alloc_workspace(self.p, hils.HILS_CALL_SELECT, w.N, C, device=dev)
        self.ws_att = hils.alloc_workspace(self.p, hils.HILS_CALL_ATTEND_PREFILL, w.N, C, device=dev)
        self.O = torch.empty_like(self.inp["Q"])
        self.lse = torch.empty(w.B, w.H, w.N, dtype=torch.float32, device=dev)
        torch.cuda.synchronize()

    def summarize(self):
        i = self.inp
        self.hils.hils_summarize(self.p, i["K"], i["LQ"], self.Ksum, self.Bsum)

    def select(self):
        i = self.inp
        self.hils.hils_select(self.p, i["Qcal"], self.Ksum, self.Bsum, self.idx, self.score, self.nsel,
                              workspace=self.ws)

    def check_status(self):
        """The status words of select and attend: nonzero if a bounded wait expired."""
        for name, ws in (("select", self.ws), ("attend", self.ws_att)):
            if ws is not None and int(ws[:4].view(torch.int32)[0].item()) != 0:
                raise RuntimeError(f"prefill {name}: a bounded wait expired (status word set)")

    def attend(self):
        i = self.inp
        self.hils.hils_attend_prefill(self.p, i["Q"], i["K"], i["V"], self.idx, self.score, self.nsel,
                                      self.O, self.lse, workspace=self.ws_att)

    def step(self):
        self.summarize()
        self.select()
        self.attend()


# ----------------------------------------------------------------- CPU oracle baseline

def oracle_decode_sample(w, dev, heads: int):
    """Host copies of the first `heads` heads of a decode workload, with their Eq. 8
    summaries from the oracle. The inputs are drawn by hils_synth (on the GPU when one is
    present, through torch alone: the same values as the first heads of the full
    workload), so nothing here touches the CUDA library."""
    import oracle

    ws = w.replace(H=heads)
    inp = make_decode(ws, device=dev if dev is not None else "cpu")
    host = {k: v.cpu() for k, v in inp.items() if isinstance(v, torch.Tensor)}
    del inp
    if dev is not None:
        torch.cuda.empty_cache()
    ks, bs = oracle.summarize(host["K"], host["LQ"], ws.S, ws.scale)
    host["Ksum"], host["Bsum"] = torch.from_numpy(ks).to(ws.dtype), torch.from_numpy(bs).float()
    host["qpos"] = (host["cache_len"] - 1).reshape(ws.B, 1)
    return ws, host


def oracle_decode_step(ws, host):
    import oracle

    idx, score, nsel = oracle.select(host["Qcal"], host["Ksum"], host["Bsum"], ws.S, ws.K, ws.scale,
                                     qpos=host["qpos"])
    oracle.attend(host["Q"], host["K"], host["V"], idx, score, nsel, ws.S, ws.W, ws.scale, qpos=host["qpos"])


def oracle_single_thread():
    """One-thread oracle times (seconds): the tiny float32 prefill (summarise, select,
    attend over all 512 queries) and one head of the 8K prefill."""
    import oracle

    out = {}
    n0 = oracle.get_threads()
    oracle.set_threads(1)
    try:
        for name, w in (("tiny_fp32_prefill_s", WORKLOADS[1]), ("prefill_8k_one_head_s", WORKLOADS[2].replace(H=1))):
            inp = make_prefill(w)
            t0 = time.perf_counter()
            ks, bs = oracle.summarize(inp["K"], inp["LQ"], w.S, w.scale)
            ksum, bsum = torch.from_numpy(ks).to(w.dtype), torch.from_numpy(bs).float()
            idx, score, nsel = oracle.select(inp["Qcal"], ksum, bsum, w.S, w.K, w.scale)
            oracle.attend(inp["Q"], inp["K"], inp["V"], idx, score, nsel, w.S, w.W, w.scale)
            out[name] = time.perf_counter() - t0
    finally:
        oracle.set_threads(n0)
    return out


def cpu_baseline(w, dev, heads=4, min_s=5.0, max_s=20.0, single_thread=True):
    import oracle

    oracle.build()
    ws, host = oracle_decode_sample(w, dev, heads)
    oracle_decode_step(ws, host)  # warm
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle_decode_step(ws, host)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_s or (el >= max_s):
            break
    per_step = el / reps * (w.H / heads)  # seconds for all heads of one token
    out = {"value": w.B / per_step, "unit": "tokens/s", "cores": oracle.get_threads(), "kind": "oracle",
           "sample": f"{heads} of {w.H} heads of one decode step (select over {w.C - 1} chunks + attend), "
                     f"{reps} repetitions in {el:.1f} s, time scaled by {w.H}/{heads}; summaries by the "
                     f"oracle (untimed)"}
    if single_thread:
        out["single_thread"] = oracle_single_thread()
    return out


def decode_config(w, world: int) -> dict:
    """The `config` of a decode line, the same for both arms."""
    return {"workload": w.name, "B": w.B, "H": w.H, "H_kv": w.Hkv, "d": w.d, "kv_len": w.N, "chunk": w.S,
            "top_k": w.K, "window": w.W, "parallelism": f"replicas{world}", "l2": DECODE_L2}


# ----------------------------------------------------------------- main

def run_reference(args, w):
    """The oracle as the reference arm: same metric, workload and config, on host cores;
    the CUDA library is never loaded."""
    world, rank, local = dist_ctx()
    if world > 1 and rank != 0:
        return
    import oracle

    oracle.build()
    dev = torch.device("cuda", local) if torch.cuda.is_available() else None
    heads = 2
    ws, host = oracle_decode_sample(w, dev, heads)
    for _ in range(args.warmup):
        oracle_decode_step(ws, host)
    t = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_decode_step(ws, host)
        t.append((time.perf_counter() - t0) * (w.H / heads))
    ms = 1e3 * statistics.mean(t)
    value = world * w.B / (ms / 1e3)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": decode_config(w, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.get_threads(),
                             "kind": "oracle",
                             "sample": f"{heads} of {w.H} heads per step, time scaled by {w.H}/{heads}; "
                                       f"summaries by the oracle (untimed)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile_case(args):
    """Small cases for Nsight Compute captures (a few GB on the device at most).

    decode-select: the 512K decode geometry (H=32, 8191 eligible chunks, K=16) on a
                   random summary table (68 MB) without a KV cache;
    decode-select-gqa: the same with 8 key-value heads (groups of 4 query heads);
    decode-attend: the decode attend with H=32, K=16, W=512 on a 128K-token cache (2.1 GB);
    decode-step:   the whole hils_decode step on that cache (select over 2047 chunks, attend);
    summarize:     hils_summarize over a 1M-token cache of 4 heads (16384 chunks each, 1.1 GB of keys);
    prefill:       the full 8K prefill workload (summarise, select, attend);
    prefill-select: the select of the 8K prefill, multi-head then grouped-query (32 query
                   heads, 8 key-value heads), `warmup + steps` launches each;
    prefill-backward: the attend backward of the 8K prefill for the forward's selection, then
                   its score backward (hils_select_backward), `warmup + steps` launches each.
    Runs `warmup + steps` plain launches of the case and exits."""
    import hierarchical_chunk_sparse_b200 as hils

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    hils.load_library()
    case = args.profile
    if case in ("decode-select", "decode-select-gqa"):
        w = WORKLOADS[4] if case == "decode-select" else WORKLOADS[8]
        g = torch.Generator(device=dev).manual_seed(1)
        Q = torch.randn(w.B, w.H, 1, w.d, generator=g, device=dev).to(w.dtype)
        Ksum = (torch.randn(w.B, w.H, w.C, w.d, generator=g, device=dev) * 0.3).to(w.dtype)
        Bsum = torch.rand(w.B, w.H, w.C, generator=g, device=dev) * 0.5 + 3.7
        p = hils.Params(B=w.B, H=w.H, d=w.d, K=w.K, W=w.W, dtype=w.dtype, H_kv=w.Hk)
        qpos = torch.full((w.B, 1), w.N - 1, dtype=torch.int32, device=dev)
        idx = torch.empty(w.B, w.Hkv, 1, w.K, dtype=torch.int32, device=dev)
        score = torch.empty(w.B, w.H, 1, w.K, device=dev)
        nsel = torch.empty(w.B, w.Hkv, 1, dtype=torch.int32, device=dev)
        ws = hils.alloc_workspace(p, hils.HILS_CALL_SELECT, 1, w.C, device=dev)
        fn = lambda: hils.hils_select(p, Q, Ksum, Bsum, idx, score, nsel, qpos=qpos, workspace=ws)  # noqa
    elif case in ("decode-attend", "decode-step"):
        db = DecodeBench(WORKLOADS[4].replace(N=131072, needles=0), dev, sets=1)
        db.sets[0].select()
        fn = db.sets[0].attend if case == "decode-attend" else db.sets[0].step
    elif case == "summarize":
        w = WORKLOADS[5].replace(H=4, needles=0)
        p = hils.Params(B=w.B, H=w.H, d=w.d, K=w.K, W=w.W, dtype=w.dtype)
        g = torch.Generator(device=dev).manual_seed(11)
        K = torch.randn(w.B, w.H, w.N, w.d, generator=g, device=dev).to(w.dtype)
        LQ = torch.randn(w.B, w.H, w.C, w.d, generator=g, device=dev).to(w.dtype)
        Ksum = torch.empty(w.B, w.H, w.C, w.d, dtype=w.dtype, device=dev)
        Bsum = torch.empty(w.B, w.H, w.C, dtype=torch.float32, device=dev)
        fn = lambda: hils.hils_summarize(p, K, LQ, Ksum, Bsum)  # noqa
    elif case == "prefill":
        fn = PrefillBench(WORKLOADS[2], dev).step
    elif case == "prefill-backward":
        pb = PrefillBench(WORKLOADS[2], dev)
        pb.step()
        w = WORKLOADS[2]
        f32 = dict(dtype=torch.float32, device=dev)
        g = torch.Generator(device=dev).manual_seed(3)
        dO = torch.randn(w.B, w.H, w.N, w.d, generator=g, **f32)
        dQ, dscore = torch.empty(w.B, w.H, w.N, w.d, **f32), torch.empty(w.B, w.H, w.N, w.K, **f32)
        dK, dV = torch.zeros(w.B, w.Hkv, w.N, w.d, **f32), torch.zeros(w.B, w.Hkv, w.N, w.d, **f32)
        ws = hils.alloc_workspace(pb.p, hils.HILS_CALL_ATTEND_BACKWARD, w.N, 0, device=dev)
        i = pb.inp
        dQcal = torch.empty(w.B, w.H, w.N, w.d, **f32)
        dKsum, dBsum = torch.zeros(w.B, w.H, w.C, w.d, **f32), torch.zeros(w.B, w.H, w.C, **f32)
        for _ in range(args.warmup + args.steps):
            hils.hils_attend_prefill_backward(pb.p, i["Q"], i["K"], i["V"], pb.idx, pb.score, pb.nsel, pb.O, pb.lse,
                                              dO, dQ, dK, dV, dscore, workspace=ws)
        fn = lambda: hils.hils_select_backward(pb.p, i["Qcal"], pb.Ksum, pb.idx, pb.nsel, dscore, dQcal,  # noqa
                                               dKsum, dBsum)
    elif case == "prefill-select":
        benches = [PrefillBench(WORKLOADS[n], dev) for n in (2, 7)]
        for pb in benches:
            pb.summarize()
        torch.cuda.synchronize()
        for pb in benches:
            for _ in range(args.warmup + args.steps):
                pb.select()
        torch.cuda.synchronize()
        print(json.dumps({"profile_case": case, "launches": 2 * (args.warmup + args.steps)}))
        return
    else:
        raise SystemExit(f"unknown profile case {case}")
    for _ in range(args.warmup + args.steps):
        fn()
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": case, "launches": args.warmup + args.steps}))


def mean_item_union(idx: torch.Tensor, nsel: torch.Tensor, C: int, q: int = 256) -> float:
    """Mean number of distinct chunks kept by the q consecutive queries of one work item of
    the tensor-core prefill attend (256 queries of one head, or 256 / P queries of P
    packed heads of a group, which share one kept list)."""
    B, H, N, K = idx.shape
    nb = N // q
    if nb == 0:
        return 0.0
    i = idx[:, :, : nb * q].reshape(B, H, nb, q * K).long()
    keep = (torch.arange(K, device=idx.device).view(1, 1, 1, K) < nsel[:, :, : nb * q, None]).reshape(B, H, nb, q * K)
    bits = torch.zeros(B, H, nb, C + 1, dtype=torch.int32, device=idx.device)
    bits.scatter_(3, torch.where(keep & (i >= 0), i, torch.full_like(i, C)), 1)
    return float(bits[..., :C].sum(-1).float().mean())


def packed_heads(G: int) -> int:
    """Query heads the tensor-core prefill attend packs into one tile: the largest power of
    two <= 8 that divides the group size."""
    p = 1
    while p < 8 and G % (2 * p) == 0:
        p *= 2
    return p


def measure_prefill(wp, dev, stream, flush, args, world, peaks, peak_src, traffic):
    """One prefill workload: step and per-kernel times (L2 flushed), TFLOP/s, roofline of
    the attend kernel, mean chunk union per 256-query item."""
    pb = PrefillBench(wp, dev)
    with torch.cuda.stream(stream):
        for _ in range(3):
            pb.step()
    stream.synchronize()
    n = max(3, min(args.steps, 20))
    with ClockSampler(dev) as pclk:
        pts = time_steps(graphed(pb.step, stream), n, flush, stream)
    pt = max_over_ranks(statistics.mean(pts), world, dev)
    ks = {k: statistics.mean(time_steps(graphed(getattr(pb, k), stream), n, flush, stream))
          for k in ("summarize", "select", "attend")}
    torch.cuda.synchronize()
    pb.check_status()
    fl = prefill_flops(wp)
    tf = fl / (pt * 1e-3) / 1e12
    fl_att = prefill_flops(wp, "attend")
    tf_att = fl_att / (ks["attend"] * 1e-3) / 1e12
    out = {"value": tf * world, "unit": "TFLOP/s", "ms_per_step": pt, **spread(pts), "workload": wp.name,
           "algorithmic_gflop_per_step": fl / 1e9, "steps": n,
           "kernel_ms": ks, "clocks": pclk.summary(),
           "step_frac_of_peak": tf / peaks["bf16_tflops"],
           "step_frac_of_sustained_peak": tf / peaks["bf16_tflops_sustained"],
           "mean_item_union_chunks": mean_item_union(pb.idx, pb.nsel, wp.C, 256 // packed_heads(wp.G)),
           "roofline": {"bound": "tensor", "kernel": "attend", "achieved": tf_att,
                        "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                        "frac": tf_att / peaks["bf16_tflops"], "traffic": traffic,
                        "frac_sustained": tf_att / peaks["bf16_tflops_sustained"],
                        "algorithmic_gflop": fl_att / 1e9,
                        "peak_source": f"{peak_src} bf16 dense (burst)"}}
    del pb
    torch.cuda.empty_cache()
    return out


def backward_flops(w) -> float:
    """Algorithmic flops of the backward pass for the kept chunks and window of every
    query (recomputed logits, dO.v, and the dq, dk, dv products: 10 d per query-token),
    the score backward (4 d per kept chunk) and the summaries' backward (8 d per chunk
    token): per batch."""
    d, S, K, W, N, C = w.d, w.S, w.K, w.W, w.N, w.C
    tok = sel = 0
    for i in range(N):
        e = min(i // S, C)
        tok += S * min(K, e) + min(W, i + 1)
        sel += min(K, e)
    return float(w.B * w.H * (10 * d * tok + 4 * d * sel + 8 * d * S * C))


def measure_prefill_backward(w, dev, stream, flush, args, world, peaks):
    """The three backward calls of the 8K prefill for the forward's selection (L2
    flushed before each timed pass; the accumulated gradients are zeroed inside it)."""
    import hierarchical_chunk_sparse_b200 as hils

    pb = PrefillBench(w, dev)
    pb.step()
    torch.cuda.synchronize()
    B, H, N, d, Hk, K, C = w.B, w.H, w.N, w.d, w.Hkv, w.K, w.C
    f32 = dict(dtype=torch.float32, device=dev)
    g = torch.Generator(device=dev).manual_seed(3)
    dO = torch.randn(B, H, N, d, generator=g, **f32)
    dQ, dK, dV = torch.empty(B, H, N, d, **f32), torch.zeros(B, Hk, N, d, **f32), torch.zeros(B, Hk, N, d, **f32)
    dscore, dQcal = torch.empty(B, H, N, K, **f32), torch.empty(B, H, N, d, **f32)
    dKsum, dBsum, dLQ = torch.zeros(B, H, C, d, **f32), torch.zeros(B, H, C, **f32), torch.empty(B, H, C, d, **f32)
    i = pb.inp
    ws = hils.alloc_workspace(pb.p, hils.HILS_CALL_ATTEND_BACKWARD, N, 0, device=dev)

    def bwd():
        for t in (dK, dV, dKsum, dBsum):
            t.zero_()
        hils.hils_attend_prefill_backward(pb.p, i["Q"], i["K"], i["V"], pb.idx, pb.score, pb.nsel, pb.O, pb.lse, dO,
                                          dQ, dK, dV, dscore, workspace=ws)
        hils.hils_select_backward(pb.p, i["Qcal"], pb.Ksum, pb.idx, pb.nsel, dscore, dQcal, dKsum, dBsum)
        hils.hils_summarize_backward(pb.p, i["K"], i["LQ"], dKsum, dBsum, dK, dLQ)

    with torch.cuda.stream(stream):
        for _ in range(3):
            bwd()
    stream.synchronize()
    n = 3
    bts = time_steps(bwd, n, flush, stream)
    ms = max_over_ranks(statistics.mean(bts), world, dev)

    # each call timed alone (L2 flushed), with the zeroing of what it accumulates into
    def attend_bwd():
        dK.zero_()
        dV.zero_()
        hils.hils_attend_prefill_backward(pb.p, i["Q"], i["K"], i["V"], pb.idx, pb.score, pb.nsel, pb.O, pb.lse, dO,
                                          dQ, dK, dV, dscore, workspace=ws)

    def select_bwd():
        dKsum.zero_()
        dBsum.zero_()
        hils.hils_select_backward(pb.p, i["Qcal"], pb.Ksum, pb.idx, pb.nsel, dscore, dQcal, dKsum, dBsum)

    def summarize_bwd():
        hils.hils_summarize_backward(pb.p, i["K"], i["LQ"], dKsum, dBsum, dK, dLQ)

    split = {name: statistics.mean(time_steps(f, n, flush, stream))
             for name, f in (("attend_backward", attend_bwd), ("select_backward", select_bwd),
                             ("summarize_backward", summarize_bwd))}
    fl = backward_flops(w)
    tf = fl / (ms * 1e-3) / 1e12
    out = {"ms_per_step": ms, **spread(bts), "unit": "TFLOP/s", "value": tf * world, "workload": w.name,
           "algorithmic_gflop_per_step": fl / 1e9, "steps": n, "ms_per_call": split,
           "frac_of_peak": tf / peaks["bf16_tflops"], "frac_of_sustained_peak": tf / peaks["bf16_tflops_sustained"],
           "note": "key-major attend backward on tcgen05 (bf16, d = 128: 128 queries per step of a 64-key block, dK and dV accumulated in TMEM per work item, Q and dO rows by TMA row gathers), float32 atomics for dQ (vector) and dK, dV; dKsum and dBsum summed per CTA in shared memory first; ms_per_call times each call alone"}
    del pb
    torch.cuda.empty_cache()
    return out


def measure_decode(w, dev, stream, flush, args, world, peaks, peak_src, steps: int, headline: bool = False,
                   rebuild: bool = False):
    """One decode workload: the hils_decode step back to back over rotating input copies
    (value, clocks), its select and attend kernels timed alone the same way, the same
    step with per-step L2 flushes and events (cold single step), the HBM roofline of the
    dominant kernel, and needle retention for workloads with planted needles.
    headline: also the end-to-end figure with host buffers. rebuild: also a full
    hils_summarize pass over every chunk of the cache, timed alone."""
    db = DecodeBench(w, dev)
    g_step = db.graphs("step", stream)
    g_sel = db.graphs("select", stream)
    g_att = db.graphs("attend", stream)
    for _ in range(max(1, args.warmup // db.R)):
        time_rotating(g_step, db.R, stream)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        ms = time_rotating(g_step, steps, stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(ms, world, dev)
    t_sel = time_rotating(g_sel, steps, stream)
    t_att = time_rotating(g_att, steps, stream)
    n_cold = max(3, min(steps, 50))
    cold = time_steps(g_step[1][0], n_cold, flush, stream)
    ms_cold = statistics.mean(cold)
    by = decode_bytes(w)
    hbm = peaks["hbm_gbs"]
    sel_gbs = by["select"] / (t_sel * 1e-3) / 1e9
    att_gbs = by["attend"] / (t_att * 1e-3) / 1e9
    step_gbs = by["step"] / (ms * 1e-3) / 1e9
    dominant = "select" if t_sel >= t_att else "attend"
    dom_gbs, dom_bytes = {"select": (sel_gbs, by["select"]), "attend": (att_gbs, by["attend"])}[dominant]
    traffic = measured_traffic("decode_" + dominant, scale=dom_bytes)
    out = {"value": job_throughput(w.B, world, ms), "unit": "tokens/s", "ms_per_step": ms, "workload": w.name,
           "config": decode_config(w, world), "steps": steps, "input_copies": db.R, "clocks": clk.summary(),
           "kernel_us": {"select": 1e3 * t_sel, "attend": 1e3 * t_att, "select_gbs": sel_gbs,
                         "attend_gbs": att_gbs},
           "algorithmic_bytes": by,
           "roofline": {"bound": "hbm", "kernel": dominant, "achieved": dom_gbs, "peak": hbm, "unit": "GB/s",
                        "frac": dom_gbs / hbm, "traffic": traffic, "algorithmic_bytes": dom_bytes,
                        "frac_8tbs": dom_gbs / 8000.0, "peak_source": f"{peak_src} HBM copy"},
           "step_roofline": {"bytes": by["step"], "achieved_gbs": step_gbs, "frac_measured": step_gbs / hbm,
                             "frac_8tbs": step_gbs / 8000.0},
           "cold_single_step": {"ms": ms_cold, **spread(cold), "tokens_per_s": job_throughput(w.B, world, ms_cold),
                                "protocol": Flusher.DESCRIPTION + "; CUDA events around each step"},
           "gpu_launches": steps * db.launches_per_step}
    if w.needles:
        s0 = db.sets[0]
        ih, nh = s0.idx.cpu().numpy(), s0.nsel.cpu().numpy()
        kept = total = 0
        for b in range(w.B):
            for h in range(w.Hkv):
                ks = set(ih[b, h, 0, : nh[b, h, 0]].tolist())
                for pos in db.needles[b, h].tolist():
                    total += 1
                    kept += (pos // w.S) in ks
        out["needle_chunks_kept"] = {"kept": kept, "of": total}
    if headline:
        sizes = [s.e2e_setup() for s in db.sets]
        h2d, d2h = sizes[0]
        try:
            g_e2e = db.graphs("e2e_step", stream)
            mode = "CUDA graph of the binding calls: H2D copies, hils_decode, D2H copies"
        except Exception as e:  # noqa: BLE001  (capture of the copies refused: time the calls themselves)
            def run_all():
                for s in db.sets:
                    s.e2e_step()
            g_e2e = (run_all, [s.e2e_step for s in db.sets])
            mode = f"binding calls launched eagerly (graph capture failed: {type(e).__name__})"
        time_rotating(g_e2e, db.R, stream)
        ms_e2e = max_over_ranks(time_rotating(g_e2e, steps, stream), world, dev)
        out["e2e"] = {"value": job_throughput(w.B, world, ms_e2e), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h, "mode": mode}
    del db, g_step, g_sel, g_att
    torch.cuda.empty_cache()
    if rebuild:
        out["summary_rebuild"] = measure_rebuild(w, dev, stream, flush, peaks, peak_src)
    return out


def measure_rebuild(w, dev, stream, flush, peaks, peak_src, reps: int = 5):
    """hils_summarize over every chunk of every head of the cache (Eq. 8), timed alone with
    L2 flushed before each pass: algorithmic bytes = the keys, the landmark queries and
    the written summaries."""
    import hierarchical_chunk_sparse_b200 as hils

    p = hils.Params(B=w.B, H=w.H, d=w.d, K=w.K, W=w.W, dtype=w.dtype, H_kv=w.Hk)
    g = torch.Generator(device=dev).manual_seed(11)
    K = torch.randn(w.B, w.Hkv, w.N, w.d, generator=g, device=dev).to(w.dtype)
    LQ = torch.randn(w.B, w.H, w.C, w.d, generator=g, device=dev).to(w.dtype)
    Ksum = torch.empty(w.B, w.H, w.C, w.d, dtype=w.dtype, device=dev)
    Bsum = torch.empty(w.B, w.H, w.C, dtype=torch.float32, device=dev)

    def fn():
        hils.hils_summarize(p, K, LQ, Ksum, Bsum)

    with torch.cuda.stream(stream):
        for _ in range(2):
            fn()
    stream.synchronize()
    ms = statistics.mean(time_steps(fn, reps, flush, stream))
    es = 2 if w.dtype == torch.bfloat16 else 4
    nbytes = w.B * w.H * w.C * (w.S * w.d * es + w.d * es + w.d * es + 4)
    gbs = nbytes / (ms * 1e-3) / 1e9
    del K, LQ, Ksum, Bsum
    torch.cuda.empty_cache()
    return {"ms": ms, "chunks": w.B * w.H * w.C, "algorithmic_bytes": nbytes,
            "roofline": {"bound": "hbm", "kernel": "summarize", "achieved": gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "frac_8tbs": gbs / 8000.0,
                         "traffic": measured_traffic("summarize", scale=w.B * w.H * w.C),
                         "peak_source": f"{peak_src} HBM copy"},
            "protocol": Flusher.DESCRIPTION + f"; {reps} passes, CUDA events around each"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--profile", default=None,
                    choices=["decode-select", "decode-select-gqa", "decode-attend", "decode-step", "prefill",
                             "prefill-select", "prefill-backward", "summarize"],
                    help="run a small case for an ncu capture and exit")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="hils", choices=["hils", "reference"])
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill and backward measurements")
    ap.add_argument("--no-extra-decode", action="store_true",
                    help="skip the decode workloads other than the 512K headline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.profile:
        run_profile_case(args)
        return
    w = WORKLOADS[4]
    if args.impl == "reference":
        run_reference(args, w)
        return

    world, rank, local = dist_ctx()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    import hierarchical_chunk_sparse_b200 as hils

    hils.load_library()
    peaks, peak_src = load_peaks()
    stream = torch.cuda.Stream(dev)
    flush = Flusher(dev)

    # ---------------- headline: decode @512K, one step = hils_decode (select then attend)
    head = measure_decode(w, dev, stream, flush, args, world, peaks, peak_src, args.steps, headline=True)

    # ---------------- prefill @8K (iid queries; query locality; grouped-query heads)
    prefill = prefill_local = prefill_gqa = prefill_bwd = None
    if not args.no_prefill:
        prefill = measure_prefill(WORKLOADS[2], dev, stream, flush, args, world, peaks, peak_src,
                                  measured_traffic("attend_prefill"))
        prefill_local = measure_prefill(WORKLOADS[6], dev, stream, flush, args, world, peaks, peak_src, None)
        prefill_gqa = measure_prefill(WORKLOADS[7], dev, stream, flush, args, world, peaks, peak_src, None)
    # ---------------- the other decode workloads: batch of 8 at 128K, 1M (with the summary
    # rebuild), grouped-query 512K, retrieval 512K
    extra = {}
    if not args.no_extra_decode:
        n_extra = max(3, min(args.steps, 50))
        for key, cfg, rb in (("decode_b8_128k", 3, False), ("decode_1m", 5, True), ("decode_gqa", 8, False),
                             ("decode_retrieval", 9, False)):
            extra[key] = measure_decode(WORKLOADS[cfg], dev, stream, flush, args, world, peaks, peak_src, n_extra,
                                        rebuild=rb)
    # ---------------- backward of the 8K prefill (fixed selection)
    if not args.no_prefill:
        prefill_bwd = measure_prefill_backward(WORKLOADS[2], dev, stream, flush, args, world, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, dev)
        # the oracle beside the other decode configurations too (a smaller sample each)
        for key, cfg in (("decode_b8_128k", 3), ("decode_1m", 5)):
            if key in extra:
                extra[key]["cpu_baseline"] = cpu_baseline(WORKLOADS[cfg], dev, heads=2, min_s=3.0, max_s=8.0,
                                                          single_thread=False)

    if rank == 0:
        line = {
            "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": head["config"],
            "roofline": head["roofline"],
            "step_roofline": head["step_roofline"],
            "kernel_us": head["kernel_us"],
            "cold_single_step": head["cold_single_step"],
            "input_copies": head["input_copies"],
            "needle_chunks_kept": head.get("needle_chunks_kept"),
            "e2e": head["e2e"],
            "gpu_launches": head["gpu_launches"],
            "clocks": head["clocks"],
            "prefill": prefill,
            "prefill_local": prefill_local,
            "prefill_gqa": prefill_gqa,
            **extra,
            "prefill_backward": prefill_bwd,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
