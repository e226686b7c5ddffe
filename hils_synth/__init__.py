"""Seeded synthetic inputs for the HiLS-Attention forward pass.

This module only draws random tensors with the shapes, value distributions and
planted structure of the workloads below. It holds none of the method's
arithmetic, and it is the one module that both the CUDA path's callers (tests,
bench, smoke check) and the oracle's callers share.

Workloads (one attention layer; chunk size S = 64 everywhere):
  1 tiny fp32 prefill:   B1 H1 d64 N512, K2 W64; Q, Q_cal, LQ, K, V iid N(0,1).
  2 prefill bf16 8K:     B1 H32 d128 N8192, K16 W512; Q, Q_cal, K, V iid N(0,1)/sqrt(d),
                         LQ iid N(0,1).
  3 decode bf16 batch:   B8 H32 d128, KV cache 131072, K16 W512; K, V, Q iid N(0,1),
                         Q_cal a separate buffer with Q's values, LQ iid N(0,1).
  4 decode bf16 512K:    B1 H32 d128, KV cache 524288, K16 W512; as 3, plus one needle
                         key per head whose logit against the query is 8.
  5 decode bf16 1M:      B1 H32 d128, KV cache 1048576, K32 W1024; as 4 with four
                         needles per head in distinct chunks.
  6 prefill bf16 8K with query locality: as 2, except that Q_cal changes slowly along
                         the sequence: Q_cal[t] = (u[t // 256] + 0.25 e[t]) / sqrt(d), with
                         u one N(0,1) vector per 256-token block and e iid N(0,1), so that
                         adjacent queries keep overlapping chunk sets (the regime in which
                         the query-packing kernel shares chunks between queries).
  7 prefill bf16 8K, grouped-query: as 2 with 8 key-value heads for the 32 query heads
                         (groups of 4): K and V are [B, 8, N, d].
  8 decode bf16 512K, grouped-query: as 4 with 8 key-value heads (groups of 4); the
                         needle of each key-value head is planted against the query of
                         the group's first head.
  9 decode bf16 512K, retrieval: as 4 with four needles per head, and the landmark query
                         of each needle's chunk set to point at the needle key, with a
                         landmark logit of 8: the summary of that chunk then concentrates
                         on the needle, as a trained landmark would for a salient token.
Every workload with Hk = 0 has as many key-value heads as query heads.
bf16 tensors are drawn in float32 and rounded to nearest-even.

Seeds: base 20260709; the tensor with id k of workload n uses base + 100 n + k,
with ids Q 1, Q_cal 2, LQ 3, K 4, V 5, needles 6.
"""
from __future__ import annotations

import dataclasses
import math

import torch

BASE_SEED = 20260709
TENSOR_IDS = {"Q": 1, "Qcal": 2, "LQ": 3, "K": 4, "V": 5, "needles": 6}


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and value recipe of one workload."""

    cfg: int
    name: str
    mode: str  # "prefill" or "decode"
    B: int
    H: int
    d: int
    S: int
    K: int
    W: int
    N: int  # prefill sequence length, or decode KV cache length
    dtype: torch.dtype
    qkv_scaled: bool = False  # Q, Q_cal, K, V divided by sqrt(d)
    needles: int = 0  # planted needle keys per (b, h)
    needle_logit: float = 8.0
    qcal_block: int = 0  # > 0: Q_cal = block base vector + qcal_noise * iid noise
    qcal_noise: float = 0.0
    needle_landmark: bool = False  # the needle chunk's landmark query points at the needle
    Hk: int = 0  # key-value heads (0: one per query head)

    @property
    def Hkv(self) -> int:
        return self.Hk if self.Hk > 0 else self.H

    @property
    def G(self) -> int:
        return self.H // self.Hkv

    @property
    def C(self) -> int:
        return self.N // self.S

    @property
    def scale(self) -> float:
        """Softmax scale 1/sqrt(d) as the float32 value the library uses."""
        return float(torch.tensor(1.0 / math.sqrt(self.d), dtype=torch.float32))

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    1: Workload(1, "tiny_fp32_prefill", "prefill", 1, 1, 64, 64, 2, 64, 512, torch.float32),
    2: Workload(2, "prefill_bf16_8k", "prefill", 1, 32, 128, 64, 16, 512, 8192, torch.bfloat16,
                qkv_scaled=True),
    3: Workload(3, "decode_bf16_b8_128k", "decode", 8, 32, 128, 64, 16, 512, 131072,
                torch.bfloat16),
    4: Workload(4, "decode_bf16_512k", "decode", 1, 32, 128, 64, 16, 512, 524288,
                torch.bfloat16, needles=1),
    5: Workload(5, "decode_bf16_1m", "decode", 1, 32, 128, 64, 32, 1024, 1048576,
                torch.bfloat16, needles=4),
    6: Workload(6, "prefill_bf16_8k_local", "prefill", 1, 32, 128, 64, 16, 512, 8192,
                torch.bfloat16, qkv_scaled=True, qcal_block=256, qcal_noise=0.25),
    7: Workload(7, "prefill_bf16_8k_gqa", "prefill", 1, 32, 128, 64, 16, 512, 8192, torch.bfloat16,
                qkv_scaled=True, Hk=8),
    8: Workload(8, "decode_bf16_512k_gqa", "decode", 1, 32, 128, 64, 16, 512, 524288,
                torch.bfloat16, needles=1, Hk=8),
    9: Workload(9, "decode_bf16_512k_retrieval", "decode", 1, 32, 128, 64, 16, 512, 524288,
                torch.bfloat16, needles=4, needle_landmark=True),
}


def _gen(w: Workload, tensor: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(BASE_SEED + 100 * w.cfg + TENSOR_IDS[tensor])
    return g


def _randn(shape, g, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def make_prefill(w: Workload, device="cpu") -> dict:
    """Q, Q_cal [B,H,N,d], K, V [B,Hk,N,d] and LQ [B,H,C,d] for a prefill workload."""
    B, H, N, d, C, Hk = w.B, w.H, w.N, w.d, w.C, w.Hkv
    s = 1.0 / math.sqrt(d) if w.qkv_scaled else 1.0
    out = {}
    for name, shape, scaled in (("Q", (B, H, N, d), True), ("Qcal", (B, H, N, d), True),
                                ("LQ", (B, H, C, d), False), ("K", (B, Hk, N, d), True),
                                ("V", (B, Hk, N, d), True)):
        g = _gen(w, name, device)
        if name == "Qcal" and w.qcal_block > 0:
            nb = (N + w.qcal_block - 1) // w.qcal_block
            base = _randn((B, H, nb, d), g, device)
            x = base.repeat_interleave(w.qcal_block, dim=2)[:, :, :N] + w.qcal_noise * _randn(shape, g, device)
        else:
            x = _randn(shape, g, device)
        if scaled and s != 1.0:
            x = x * s
        out[name] = x.to(w.dtype)
    return out


def needle_positions(w: Workload, device="cpu") -> torch.Tensor:
    """[B, Hk, needles] token positions of the planted needle keys (decode workloads).

    Positions lie in [0, t - W] with t = N - 1, so no needle is in the window; the
    needles of one (b, h) sit in distinct chunks."""
    if w.needles == 0:
        return torch.zeros(w.B, w.Hkv, 0, dtype=torch.int64)
    g = _gen(w, "needles", "cpu")
    t = w.N - 1
    last_chunk = (t - w.W + 1) // w.S  # chunks [0, last_chunk) lie wholly before the window
    pos = torch.empty(w.B, w.Hkv, w.needles, dtype=torch.int64)
    for b in range(w.B):
        for h in range(w.Hkv):
            chunks = torch.randperm(last_chunk, generator=g)[: w.needles]
            offs = torch.randint(0, w.S, (w.needles,), generator=g)
            pos[b, h] = chunks * w.S + offs
    return pos


def make_decode(w: Workload, device="cpu") -> dict:
    """Decode inputs: Q, Q_cal [B,H,1,d], LQ [B,H,C,d], Kc, Vc [B,Hk,N,d] KV cache,
    cache_len [B] int32 (= N; the query sits at t = N - 1) and needle positions.

    K and V are drawn one (b, h) slice at a time so that the float32 staging
    buffer stays at one head's size."""
    B, H, N, d, C, Hk = w.B, w.H, w.N, w.d, w.C, w.Hkv
    q32 = _randn((B, H, 1, d), _gen(w, "Q", device), device)
    lq = torch.empty((B, H, C, d), dtype=w.dtype, device=device)
    kc = torch.empty((B, Hk, N, d), dtype=w.dtype, device=device)
    vc = torch.empty((B, Hk, N, d), dtype=w.dtype, device=device)
    pos = needle_positions(w)
    g_lq, g_k, g_v = _gen(w, "LQ", device), _gen(w, "K", device), _gen(w, "V", device)
    for b in range(B):
        for h in range(H):
            lq[b, h] = _randn((C, d), g_lq, device).to(w.dtype)
    for b in range(B):
        for h in range(Hk):
            k = _randn((N, d), g_k, device)
            q = q32[b, h * w.G, 0]
            for p in pos[b, h].tolist():
                # k_p <- k_p + (L/scale - q.k_p) q / |q|^2, so that scale * q.k_p = L
                k[p] += (w.needle_logit / w.scale - torch.dot(q, k[p])) * q / torch.dot(q, q)
                if w.needle_landmark:
                    # landmark query L/scale * k_p / |k_p|^2: scale * q'_c . k_p = L
                    lm = (w.needle_logit / w.scale) * k[p] / torch.dot(k[p], k[p])
                    for hq in range(h * w.G, (h + 1) * w.G):
                        lq[b, hq, p // w.S] = lm.to(w.dtype)
            kc[b, h] = k.to(w.dtype)
            vc[b, h] = _randn((N, d), g_v, device).to(w.dtype)
            del k
    q = q32.to(w.dtype)
    return {
        "Q": q,
        "Qcal": q.clone(),
        "LQ": lq,
        "K": kc,
        "V": vc,
        "cache_len": torch.full((B,), N, dtype=torch.int32, device=device),
        "needles": pos,
    }
