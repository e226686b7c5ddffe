"""float64 CPU oracle for the HiLS-Attention forward pass (ctypes wrapper).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this module. The CUDA library never loads
it, and it never loads the CUDA library.

Each function wraps the C routine of the same name in ``hils_oracle.c``; see that
file for the passages of "Hierarchical Sparse Attention Done Right" each one
follows. Inputs are CPU torch tensors (float32, bfloat16 or float64), read in place
through their strides; outputs are float64 / int32 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hils_oracle.c")
_HDR = os.path.join(_HERE, "hils_oracle.h")
LIB_PATH = os.path.join(_HERE, "libhils_oracle.so")

CFLAGS = ["-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

OR_F32, OR_BF16, OR_F64 = 0, 1, 2
_DTYPES = {torch.float32: OR_F32, torch.bfloat16: OR_BF16, torch.float64: OR_F64}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc if the shared library is missing or stale."""
    stale = not os.path.exists(LIB_PATH) or any(
        os.path.getmtime(p) > os.path.getmtime(LIB_PATH) for p in (_SRC, _HDR)
    )
    if force or stale:
        tmp = LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


class _Tensor(ctypes.Structure):
    _fields_ = [
        ("ptr", ctypes.c_void_p),
        ("dtype", ctypes.c_int),
        ("sb", ctypes.c_longlong),
        ("sh", ctypes.c_longlong),
        ("st", ctypes.c_longlong),
    ]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        T = _Tensor
        i, d_, p = ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        lib.or_set_threads.argtypes = [i]
        lib.or_get_threads.restype = i
        lib.or_summarize.argtypes = [i, i, i, i, i, d_, T, i, T, p, p]
        lib.or_score_all.argtypes = [i, i, i, i, i, d_, T, i, p, T, T, i, p]
        lib.or_select.argtypes = [i, i, i, i, i, i, i, d_, T, i, p, T, T, i, p, p, p]
        lib.or_attend.argtypes = [i, i, i, i, i, i, i, d_, T, i, p, T, T, p, T, p, p, p]
        lib.or_brute_weights.argtypes = [i, i, i, i, i, d_, T, i, i, i, i, T, p, T,
                                         ctypes.c_longlong, i, p]
        lib.or_chunk_logmass.argtypes = [i, i, i, i, i, d_, T, i, T, p, p, p]
        for name in ("or_summarize", "or_score_all", "or_select", "or_attend",
                     "or_brute_weights", "or_chunk_logmass"):
            getattr(lib, name).restype = i
        _lib = lib
    return _lib


def _desc(t: torch.Tensor) -> _Tensor:
    """Describe a CPU tensor [B,H,T,D] (innermost stride 1) or [B,H,T]."""
    if t.device.type != "cpu":
        raise ValueError("oracle inputs must live on the CPU")
    if t.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {t.dtype}")
    if t.dim() == 4:
        if t.stride(3) != 1 and t.shape[3] > 1:
            raise ValueError("innermost dimension must be contiguous")
        sb, sh, st = t.stride(0), t.stride(1), t.stride(2)
    elif t.dim() == 3:
        sb, sh, st = t.stride()
    else:
        raise ValueError("expected a 3-D or 4-D tensor")
    return _Tensor(t.data_ptr(), _DTYPES[t.dtype], sb, sh, st)


def _i32(a) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        a = a.cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, name: str) -> None:
    if rc != 0:
        raise ValueError(f"{name}: invalid arguments")


def set_threads(n: int) -> None:
    _load().or_set_threads(int(n))


def get_threads() -> int:
    return int(_load().or_get_threads())


def _group(h_query: int, h_kv: int) -> int:
    if h_kv <= 0 or h_query % h_kv != 0:
        raise ValueError(f"{h_query} query heads do not form groups over {h_kv} key-value heads")
    return h_query // h_kv


def summarize(K: torch.Tensor, LQ: torch.Tensor, S: int, scale: float):
    """Eq. 8 summaries of every query head (LQ [B,H,C,d]) over the keys of its key-value
    head (K [B,H/G,N,d]). Returns (Ksum [B,H,C,d], Bsum [B,H,C]) in float64."""
    K, LQ = _as_tensor(K), _as_tensor(LQ)
    B, Hk, N, d = K.shape
    H = LQ.shape[1]
    G = _group(H, Hk)
    C = N // S
    ksum = np.zeros((B, H, C, d), np.float64)
    bsum = np.zeros((B, H, C), np.float64)
    _check(_load().or_summarize(B, H, G, d, S, float(scale), _desc(K), N, _desc(LQ),
                                _ptr(ksum), _ptr(bsum)), "summarize")
    return ksum, bsum


def _as_tensor(a) -> torch.Tensor:
    return a if isinstance(a, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(a))


def score_all(Qcal, Ksum, Bsum, S: int, scale: float, qpos=None, exclude_window: int = 0):
    """Eq. 7 scores of every chunk for every query; -inf where not eligible
    (exclude_window = W > 0: chunks wholly inside the query's window are not eligible)."""
    Qcal, Ksum, Bsum = _as_tensor(Qcal), _as_tensor(Ksum), _as_tensor(Bsum)
    B, H, Lq, d = Qcal.shape
    C = Ksum.shape[2]
    out = np.zeros((B, H, Lq, C), np.float64)
    qp = None if qpos is None else _i32(qpos)
    _check(_load().or_score_all(B, H, d, S, int(exclude_window), float(scale), _desc(Qcal), Lq,
                                None if qp is None else _ptr(qp), _desc(Ksum), _desc(Bsum), C,
                                _ptr(out)), "score_all")
    return out


def select(Qcal, Ksum, Bsum, S: int, K: int, scale: float, qpos=None, group: int = 1, exclude_window: int = 0):
    """Top-K selection, shared by each group of `group` consecutive query heads; with
    exclude_window = W > 0, chunks wholly inside the query's window are not eligible.
    Returns (idx int32 [B,H/G,Lq,K], score float64 [B,H,Lq,K], nsel int32 [B,H/G,Lq])."""
    Qcal, Ksum, Bsum = _as_tensor(Qcal), _as_tensor(Ksum), _as_tensor(Bsum)
    B, H, Lq, d = Qcal.shape
    G = _group(H, H // group if group > 0 and H % group == 0 else 0)
    C = Ksum.shape[2]
    idx = np.zeros((B, H // G, Lq, K), np.int32)
    score = np.zeros((B, H, Lq, K), np.float64)
    nsel = np.zeros((B, H // G, Lq), np.int32)
    qp = None if qpos is None else _i32(qpos)
    _check(_load().or_select(B, H, G, d, S, K, int(exclude_window), float(scale), _desc(Qcal), Lq,
                             None if qp is None else _ptr(qp), _desc(Ksum), _desc(Bsum), C,
                             _ptr(idx), _ptr(score), _ptr(nsel)), "select")
    return idx, score, nsel


def attend(Q, Kc, Vc, idx, score, nsel, S: int, W: int, scale: float, qpos=None):
    """Eq. 10 output for query heads Q [B,H,Lq,d] over key-value heads Kc, Vc [B,H/G,L,d]
    with the groups' kept chunks idx [B,H/G,Lq,K], nsel [B,H/G,Lq] and each head's scores
    [B,H,Lq,K]. Returns (O [B,H,Lq,d] float64, lse [B,H,Lq] float64)."""
    Q, Kc, Vc = _as_tensor(Q), _as_tensor(Kc), _as_tensor(Vc)
    B, H, Lq, d = Q.shape
    G = _group(H, Kc.shape[1])
    idx = _i32(idx)
    K = idx.shape[-1]
    idx = idx.reshape(B, H // G, Lq, K)
    score = _as_tensor(score).reshape(B, H, Lq, K).contiguous()
    nsel = _i32(nsel).reshape(B, H // G, Lq)
    O = np.zeros((B, H, Lq, d), np.float64)
    lse = np.zeros((B, H, Lq), np.float64)
    qp = None if qpos is None else _i32(qpos)
    _check(_load().or_attend(B, H, G, d, S, K, W, float(scale), _desc(Q), Lq,
                             None if qp is None else _ptr(qp), _desc(Kc), _desc(Vc),
                             _ptr(idx), _desc(score), _ptr(nsel), _ptr(O), _ptr(lse)), "attend")
    return O, lse


def brute_weights(Q, Kc, idx_row, score_row, nsel_row: int, b: int, h: int, i: int, t: int,
                  S: int, W: int, scale: float):
    """Token-level Eq. 10 weights w[j], j in [0, t], for one query."""
    Q, Kc = _as_tensor(Q), _as_tensor(Kc)
    H, d = Q.shape[1], Q.shape[3]
    idx_row = _i32(idx_row).reshape(-1)
    K = idx_row.shape[0]
    srow = _as_tensor(score_row).reshape(1, 1, 1, K).to(torch.float64).contiguous()
    w = np.zeros(t + 1, np.float64)
    _check(_load().or_brute_weights(H, d, S, K, W, float(scale), _desc(Q), b, h, i, t,
                                    _desc(Kc), _ptr(idx_row), _desc(srow), 0, int(nsel_row),
                                    _ptr(w)), "brute_weights")
    return w


def chunk_logmass(Q, Kc, idx, nsel, S: int, scale: float):
    """Exact log Z_{i,c} of each selected chunk (Introduction, chunk mass)."""
    Q, Kc = _as_tensor(Q), _as_tensor(Kc)
    B, H, Lq, d = Q.shape
    idx = _i32(idx)
    K = idx.shape[-1]
    idx = idx.reshape(B, H, Lq, K)
    nsel = _i32(nsel).reshape(B, H, Lq)
    out = np.zeros((B, H, Lq, K), np.float64)
    _check(_load().or_chunk_logmass(B, H, d, S, K, float(scale), _desc(Q), Lq, _desc(Kc),
                                    _ptr(idx), _ptr(nsel), _ptr(out)), "chunk_logmass")
    return out
