"""Python binding of libhils, the HiLS-Attention forward pass for B200 (sm_100a).

Argument marshalling only: every function here turns torch CUDA tensors into the
pointers and element strides of the C ABI (``include/hils.h``) and calls the entry
point of the same name; all work runs in the library's CUDA kernels. There is no
CPU fallback: if the compiled library is missing, loading fails with an error.

    import hierarchical_chunk_sparse_b200 as hils
    p = hils.Params(B=1, H=32, d=128, K=16, W=512, dtype=torch.bfloat16)
    hils.hils_summarize(p, K, LQ, Ksum, Bsum)
    hils.hils_select(p, Qcal, Ksum, Bsum, idx, score, nsel, workspace=ws)
    hils.hils_attend_prefill(p, Q, K, V, idx, score, nsel, O, lse)
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhils.so")

HILS_F32, HILS_BF16 = 0, 1
HILS_CALL_SELECT, HILS_CALL_ATTEND_PREFILL, HILS_CALL_ATTEND_DECODE, HILS_CALL_DECODE = 0, 1, 2, 3
HILS_CALL_ATTEND_BACKWARD = 4
# hils_params.flags: chunks wholly inside a query's window are not selected
HILS_FLAG_EXCLUDE_WINDOW_CHUNKS = 1
# hils_params.flags, diagnostic: the tensor-core kernels' waits on work in progress expire at once
HILS_FLAG_DIAG_EXPIRE_WAITS = 0x80000000
STATUS = {0: "HILS_OK", 1: "HILS_ERR_INVALID_ARG", 2: "HILS_ERR_UNSUPPORTED",
          3: "HILS_ERR_ALIGNMENT", 4: "HILS_ERR_WORKSPACE", 5: "HILS_ERR_CUDA"}
_DTYPES = {torch.float32: HILS_F32, torch.bfloat16: HILS_BF16}

# Every function the C header declares (checked by the tests against the header).
EXPORTS = ("hils_summarize", "hils_select", "hils_attend_prefill", "hils_attend_decode", "hils_decode",
           "hils_attend_decode_noalloc", "hils_workspace_bytes", "hils_workspace_init",
           "hils_status_string", "hils_last_cuda_error", "hils_summarize_append", "hils_attend_prefill_backward",
           "hils_select_backward", "hils_summarize_backward", "hils_selftest_fast_math")


class HilsError(RuntimeError):
    def __init__(self, call: str, status: int, detail: str = ""):
        self.status = status
        msg = f"{call}: {STATUS.get(status, status)}"
        super().__init__(msg + (f" ({detail})" if detail else ""))


class _CTensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("sb", ctypes.c_int64), ("sh", ctypes.c_int64),
                ("st", ctypes.c_int64)]


class _Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int), ("S", ctypes.c_int),
                ("K", ctypes.c_int), ("W", ctypes.c_int), ("dtype", ctypes.c_int),
                ("scale", ctypes.c_float), ("flags", ctypes.c_uint32), ("H_kv", ctypes.c_int)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libhils.so; raises if it has not been built (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(f"libhils.so not built at {path}; run "
                              "python -m hierarchical_chunk_sparse_b200.build")
        lib = ctypes.CDLL(path)
        T, P, vp, i, sz = _CTensor, ctypes.POINTER(_Params), ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        lib.hils_summarize.argtypes = [P, T, i, T, T, vp, vp]
        lib.hils_summarize_append.argtypes = [P, T, vp, T, T, vp, i, vp]
        lib.hils_attend_prefill_backward.argtypes = [P, T, T, T, i, vp, vp, vp, T, vp, vp, vp, vp, vp, vp, vp, sz,
                                                     vp]
        lib.hils_select_backward.argtypes = [P, T, i, T, i, vp, vp, vp, vp, vp, vp, vp]
        lib.hils_summarize_backward.argtypes = [P, T, i, T, vp, vp, vp, vp, vp]
        lib.hils_select.argtypes = [P, T, i, vp, T, vp, i, vp, vp, vp, vp, sz, vp]
        lib.hils_attend_prefill.argtypes = [P, T, T, T, i, vp, vp, vp, T, vp, vp, sz, vp]
        lib.hils_attend_decode.argtypes = [P, T, T, T, vp, vp, vp, vp, T, vp, vp, sz, vp]
        lib.hils_attend_decode_noalloc.argtypes = [P, T, T, T, vp, vp, vp, vp, T, vp, vp]
        lib.hils_decode.argtypes = [P, T, T, vp, i, T, T, T, vp, vp, vp, vp, T, vp, vp, sz, vp]
        lib.hils_workspace_bytes.argtypes = [P, i, i, i]
        lib.hils_workspace_bytes.restype = sz
        lib.hils_workspace_init.argtypes = [vp, sz, vp]
        lib.hils_status_string.argtypes = [i]
        lib.hils_status_string.restype = ctypes.c_char_p
        lib.hils_last_cuda_error.restype = ctypes.c_char_p
        lib.hils_selftest_fast_math.argtypes = [vp, vp, i, vp, vp, vp]
        for name in ("hils_summarize", "hils_summarize_append", "hils_attend_prefill_backward",
                     "hils_select_backward", "hils_summarize_backward", "hils_select", "hils_attend_prefill",
                     "hils_attend_decode", "hils_decode", "hils_attend_decode_noalloc", "hils_workspace_init",
                     "hils_selftest_fast_math"):
            getattr(lib, name).restype = i
        _lib = lib
    return _lib


class Params:
    """hils_params: B, H query heads, d, chunk size S (64), top-K, window W, dtype, scale
    (0 = 1/sqrt(d)), H_kv key-value heads (0 or H: multi-head; a divisor of H: groups of
    H / H_kv query heads share a key-value head and one chunk selection)."""

    def __init__(self, B: int, H: int, d: int, K: int, W: int, dtype: torch.dtype = torch.bfloat16,
                 S: int = 64, scale: float = 0.0, flags: int = 0, H_kv: int = 0):
        self.B, self.H, self.d, self.K, self.W, self.S = B, H, d, K, W, S
        self.dtype, self.scale, self.flags, self.H_kv = dtype, scale, flags, H_kv

    @property
    def Hk(self) -> int:
        """Key-value heads (= the number of selection groups)."""
        return self.H_kv if self.H_kv > 0 else self.H

    def c(self) -> _Params:
        dt = _DTYPES.get(self.dtype, -1) if isinstance(self.dtype, torch.dtype) else int(self.dtype)
        return _Params(self.B, self.H, self.d, self.S, self.K, self.W, dt, self.scale, self.flags, self.H_kv)


def _view(t) -> _CTensor:
    """[B, H, T, d] torch tensor (innermost stride 1) -> pointer + element strides."""
    if t is None:
        return _CTensor(None, 0, 0, 0)
    if t.dim() != 4:
        raise ValueError("expected a [B, H, T, d] tensor")
    if t.shape[3] > 1 and t.stride(3) != 1:
        raise ValueError("the head dimension must be contiguous")
    return _CTensor(t.data_ptr(), t.stride(0), t.stride(1), t.stride(2))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _expect(call: str, name: str, t, shape, dtype=None) -> None:
    """Shape (and dtype) check of one argument against the parameters; raises before the
    C call, so that a mismatched tensor can never be read or written out of bounds."""
    if t is None:
        return
    got = tuple(t.shape)
    if got != tuple(shape):
        raise ValueError(f"{call}: {name} has shape {got}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{call}: {name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_cuda:
        raise ValueError(f"{call}: {name} must be a CUDA tensor")


def _check(call: str, rc: int) -> None:
    if rc != 0:
        lib = load_library()
        detail = lib.hils_last_cuda_error().decode() if rc == 5 else lib.hils_status_string(rc).decode()
        raise HilsError(call, rc, detail)


def hils_workspace_bytes(p: Params, call: int, Lq: int, C: int) -> int:
    return int(load_library().hils_workspace_bytes(ctypes.byref(p.c()), call, Lq, C))


def hils_workspace_init(workspace, ws_bytes: int | None = None, stream=None) -> None:
    n = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    _check("hils_workspace_init", load_library().hils_workspace_init(_ptr(workspace), n, _stream(stream)))


def _ws(workspace):
    if workspace is None:
        return None, 0
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


def hils_summarize(p: Params, K, LQ, Ksum, Bsum, N: int | None = None, stream=None) -> None:
    """Eq. 8 summaries of every complete chunk of every query head: K [B,Hk,N,d],
    Ksum [B,H,C,d], Bsum [B,H,C] float32."""
    n = K.shape[2] if N is None else N
    B, H, d, C = p.B, p.H, p.d, n // p.S
    if K.shape[0] != B or K.shape[1] != p.Hk or K.shape[3] != d or K.shape[2] < C * p.S:
        raise ValueError(f"hils_summarize: K has shape {tuple(K.shape)} for B={B} H={H} d={d} N={n}")
    if K.dtype != p.dtype:
        raise ValueError("hils_summarize: K dtype differs from params")
    _expect("hils_summarize", "LQ", LQ, (B, H, C, d), p.dtype)
    _expect("hils_summarize", "Ksum", Ksum, (B, H, C, d), p.dtype)
    _expect("hils_summarize", "Bsum", Bsum, (B, H, C), torch.float32)
    _check("hils_summarize", load_library().hils_summarize(
        ctypes.byref(p.c()), _view(K), n, _view(LQ), _view(Ksum), _ptr(Bsum), _stream(stream)))


def hils_summarize_append(p: Params, K, cache_len, LQ, Ksum, Bsum, stream=None) -> None:
    """Decode-time summary of the chunk each sequence's newest token completed: for b
    with cache_len[b] a positive multiple of 64, chunk cache_len[b] / 64 - 1 of every
    head into Ksum [B,H,C,d] and Bsum [B,H,C]; everything else is left as it was.
    K [B,Hk,T,d] is the KV cache's keys, LQ [B,H,C,d] the landmark queries."""
    B, H, d = p.B, p.H, p.d
    C = Ksum.shape[2]
    if K.shape[0] != B or K.shape[1] != p.Hk or K.shape[3] != d or K.dtype != p.dtype or not K.is_cuda:
        raise ValueError(f"hils_summarize_append: K has shape {tuple(K.shape)} / {K.dtype}")
    if K.shape[2] < C * p.S:
        raise ValueError("hils_summarize_append: the cache holds fewer than C chunks")
    _expect("hils_summarize_append", "cache_len", cache_len, (B,), torch.int32)
    _expect("hils_summarize_append", "LQ", LQ, (B, H, C, d), p.dtype)
    _expect("hils_summarize_append", "Ksum", Ksum, (B, H, C, d), p.dtype)
    _expect("hils_summarize_append", "Bsum", Bsum, (B, H, C), torch.float32)
    _check("hils_summarize_append", load_library().hils_summarize_append(
        ctypes.byref(p.c()), _view(K), _ptr(cache_len), _view(LQ), _view(Ksum), _ptr(Bsum), C, _stream(stream)))


def hils_select(p: Params, Qcal, Ksum, Bsum, idx, score, nsel, qpos=None, workspace=None,
                Lq: int | None = None, C: int | None = None, stream=None) -> None:
    """Eq. 7 scores and exact top-K: idx [B,Hk,Lq,K] and nsel [B,Hk,Lq] per selection
    group, score [B,H,Lq,K] per query head."""
    lq = Qcal.shape[2] if Lq is None else Lq
    c = Ksum.shape[2] if C is None else C
    B, H, d, K, Hk = p.B, p.H, p.d, p.K, p.Hk
    _expect("hils_select", "Qcal", Qcal, (B, H, lq, d), p.dtype)
    _expect("hils_select", "Ksum", Ksum, (B, H, c, d), p.dtype)
    _expect("hils_select", "Bsum", Bsum, (B, H, c), torch.float32)
    _expect("hils_select", "idx", idx, (B, Hk, lq, K), torch.int32)
    _expect("hils_select", "score", score, (B, H, lq, K), torch.float32)
    _expect("hils_select", "nsel", nsel, (B, Hk, lq), torch.int32)
    if qpos is not None:
        _expect("hils_select", "qpos", qpos, (B, lq), torch.int32)
    wp, wn = _ws(workspace)
    _check("hils_select", load_library().hils_select(
        ctypes.byref(p.c()), _view(Qcal), lq, _ptr(qpos), _view(Ksum), _ptr(Bsum), c,
        _ptr(idx), _ptr(score), _ptr(nsel), wp, wn, _stream(stream)))


def hils_attend_prefill(p: Params, Q, K, V, idx, score, nsel, O, lse=None, workspace=None,
                        N: int | None = None, stream=None) -> None:
    """Eq. 10 for every position: Q, O [B,H,N,d], K, V [B,Hk,N,d], lse [B,H,N] float32
    (optional)."""
    n = Q.shape[2] if N is None else N
    B, H, d, k, Hk = p.B, p.H, p.d, p.K, p.Hk
    for name, t, h in (("Q", Q, H), ("K", K, Hk), ("V", V, Hk), ("O", O, H)):
        _expect("hils_attend_prefill", name, t, (B, h, n, d), p.dtype)
    if k > 0:
        _expect("hils_attend_prefill", "idx", idx, (B, Hk, n, k), torch.int32)
        _expect("hils_attend_prefill", "score", score, (B, H, n, k), torch.float32)
        _expect("hils_attend_prefill", "nsel", nsel, (B, Hk, n), torch.int32)
    _expect("hils_attend_prefill", "lse", lse, (B, H, n), torch.float32)
    wp, wn = _ws(workspace)
    _check("hils_attend_prefill", load_library().hils_attend_prefill(
        ctypes.byref(p.c()), _view(Q), _view(K), _view(V), n, _ptr(idx), _ptr(score), _ptr(nsel),
        _view(O), _ptr(lse), wp, wn, _stream(stream)))


def hils_attend_decode(p: Params, Q, Kc, Vc, cache_len, idx, score, nsel, O, lse=None,
                       workspace=None, stream=None) -> None:
    """Eq. 10 for one new token per sequence: O [B,H,1,d], lse [B,H] float32 (optional).

    The cache tensors may be longer than any cache_len; the kernels read positions
    below cache_len[b] only, which must not exceed the cache tensors' length."""
    B, H, d, k = p.B, p.H, p.d, p.K
    _expect("hils_attend_decode", "Q", Q, (B, H, 1, d), p.dtype)
    _expect("hils_attend_decode", "O", O, (B, H, 1, d), p.dtype)
    for name, t in (("Kc", Kc), ("Vc", Vc)):
        if t.shape[0] != B or t.shape[1] != p.Hk or t.shape[3] != d or t.dtype != p.dtype or not t.is_cuda:
            raise ValueError(f"hils_attend_decode: {name} has shape {tuple(t.shape)} / {t.dtype}")
    _expect("hils_attend_decode", "cache_len", cache_len, (B,), torch.int32)
    if k > 0:
        _expect("hils_attend_decode", "idx", idx, (B, p.Hk, 1, k), torch.int32)
        _expect("hils_attend_decode", "score", score, (B, H, 1, k), torch.float32)
        _expect("hils_attend_decode", "nsel", nsel, (B, p.Hk, 1), torch.int32)
    _expect("hils_attend_decode", "lse", lse, (B, H), torch.float32)
    wp, wn = _ws(workspace)
    _check("hils_attend_decode", load_library().hils_attend_decode(
        ctypes.byref(p.c()), _view(Q), _view(Kc), _view(Vc), _ptr(cache_len), _ptr(idx), _ptr(score),
        _ptr(nsel), _view(O), _ptr(lse), wp, wn, _stream(stream)))


def hils_decode(p: Params, Qcal, Ksum, Bsum, Q, Kc, Vc, cache_len, idx, score, nsel, O, lse=None,
                workspace=None, stream=None) -> None:
    """One decode step: hils_select with qpos = cache_len - 1, then hils_attend_decode,
    as one chain. Outputs as the two calls: idx [B,Hk,1,K], score [B,H,1,K], nsel [B,Hk,1], O, lse."""
    B, H, d, k = p.B, p.H, p.d, p.K
    c = Ksum.shape[2]
    _expect("hils_decode", "Qcal", Qcal, (B, H, 1, d), p.dtype)
    _expect("hils_decode", "Ksum", Ksum, (B, H, c, d), p.dtype)
    _expect("hils_decode", "Bsum", Bsum, (B, H, c), torch.float32)
    _expect("hils_decode", "Q", Q, (B, H, 1, d), p.dtype)
    _expect("hils_decode", "O", O, (B, H, 1, d), p.dtype)
    for name, t in (("Kc", Kc), ("Vc", Vc)):
        if t.shape[0] != B or t.shape[1] != p.Hk or t.shape[3] != d or t.dtype != p.dtype or not t.is_cuda:
            raise ValueError(f"hils_decode: {name} has shape {tuple(t.shape)} / {t.dtype}")
    _expect("hils_decode", "cache_len", cache_len, (B,), torch.int32)
    _expect("hils_decode", "idx", idx, (B, p.Hk, 1, k), torch.int32)
    _expect("hils_decode", "score", score, (B, H, 1, k), torch.float32)
    _expect("hils_decode", "nsel", nsel, (B, p.Hk, 1), torch.int32)
    _expect("hils_decode", "lse", lse, (B, H), torch.float32)
    wp, wn = _ws(workspace)
    _check("hils_decode", load_library().hils_decode(
        ctypes.byref(p.c()), _view(Qcal), _view(Ksum), _ptr(Bsum), c, _view(Q), _view(Kc), _view(Vc),
        _ptr(cache_len), _ptr(idx), _ptr(score), _ptr(nsel), _view(O), _ptr(lse), wp, wn, _stream(stream)))


def hils_attend_decode_noalloc(p: Params, Q, Kc, Vc, cache_len, idx, score, nsel, O, lse=None,
                               stream=None) -> None:
    """hils_attend_decode with the library's built-in scratch instead of a workspace.

    For callers that cannot allocate device memory; the scratch is one fixed 4 MiB
    array per GPU, shared by every call (calls that overlap on the GPU race on it)."""
    B, H, d, k = p.B, p.H, p.d, p.K
    _expect("hils_attend_decode_noalloc", "Q", Q, (B, H, 1, d), p.dtype)
    _expect("hils_attend_decode_noalloc", "O", O, (B, H, 1, d), p.dtype)
    for name, t in (("Kc", Kc), ("Vc", Vc)):
        if t.shape[0] != B or t.shape[1] != p.Hk or t.shape[3] != d or t.dtype != p.dtype or not t.is_cuda:
            raise ValueError(f"hils_attend_decode_noalloc: {name} has shape {tuple(t.shape)} / {t.dtype}")
    _expect("hils_attend_decode_noalloc", "cache_len", cache_len, (B,), torch.int32)
    if k > 0:
        _expect("hils_attend_decode_noalloc", "idx", idx, (B, p.Hk, 1, k), torch.int32)
        _expect("hils_attend_decode_noalloc", "score", score, (B, H, 1, k), torch.float32)
        _expect("hils_attend_decode_noalloc", "nsel", nsel, (B, p.Hk, 1), torch.int32)
    _expect("hils_attend_decode_noalloc", "lse", lse, (B, H), torch.float32)
    _check("hils_attend_decode_noalloc", load_library().hils_attend_decode_noalloc(
        ctypes.byref(p.c()), _view(Q), _view(Kc), _view(Vc), _ptr(cache_len), _ptr(idx), _ptr(score),
        _ptr(nsel), _view(O), _ptr(lse), _stream(stream)))


def _dense32(call: str, name: str, t, shape) -> None:
    _expect(call, name, t, shape, torch.float32)
    if not t.is_contiguous():
        raise ValueError(f"{call}: {name} must be dense (contiguous)")


def hils_attend_prefill_backward(p: Params, Q, K, V, idx, score, nsel, O, lse, dO, dQ, dK, dV, dscore,
                                 workspace=None, stream=None) -> None:
    """Eq. 10 backward for the kept chunks of hils_select: dQ [B,H,N,d] (written),
    dK, dV [B,Hk,N,d] (accumulated: zero them first), dscore [B,H,N,K] (written); all
    float32 and dense. O, lse are the forward's outputs, dO [B,H,N,d] float32."""
    n = Q.shape[2]
    B, H, d, k, Hk = p.B, p.H, p.d, p.K, p.Hk
    for name, t, h in (("Q", Q, H), ("K", K, Hk), ("V", V, Hk), ("O", O, H)):
        _expect("hils_attend_prefill_backward", name, t, (B, h, n, d), p.dtype)
    if k > 0:
        _expect("hils_attend_prefill_backward", "idx", idx, (B, Hk, n, k), torch.int32)
        _expect("hils_attend_prefill_backward", "score", score, (B, H, n, k), torch.float32)
        _expect("hils_attend_prefill_backward", "nsel", nsel, (B, Hk, n), torch.int32)
        _dense32("hils_attend_prefill_backward", "dscore", dscore, (B, H, n, k))
    _expect("hils_attend_prefill_backward", "lse", lse, (B, H, n), torch.float32)
    for name, t, h in (("dO", dO, H), ("dQ", dQ, H), ("dK", dK, Hk), ("dV", dV, Hk)):
        _dense32("hils_attend_prefill_backward", name, t, (B, h, n, d))
    if workspace is None:
        workspace = alloc_workspace(p, HILS_CALL_ATTEND_BACKWARD, n, 0, device=Q.device)
    wp, wn = _ws(workspace)
    _check("hils_attend_prefill_backward", load_library().hils_attend_prefill_backward(
        ctypes.byref(p.c()), _view(Q), _view(K), _view(V), n, _ptr(idx), _ptr(score), _ptr(nsel), _view(O),
        _ptr(lse), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dscore), wp, wn, _stream(stream)))


def hils_select_backward(p: Params, Qcal, Ksum, idx, nsel, dscore, dQcal, dKsum, dBsum, stream=None) -> None:
    """Eq. 7 backward: dQcal [B,H,Lq,d] (written), dKsum [B,H,C,d] and dBsum [B,H,C]
    (accumulated), float32 and dense, from dscore [B,H,Lq,K]."""
    lq, c = Qcal.shape[2], Ksum.shape[2]
    B, H, d, k, Hk = p.B, p.H, p.d, p.K, p.Hk
    _expect("hils_select_backward", "Qcal", Qcal, (B, H, lq, d), p.dtype)
    _expect("hils_select_backward", "Ksum", Ksum, (B, H, c, d), p.dtype)
    _expect("hils_select_backward", "idx", idx, (B, Hk, lq, k), torch.int32)
    _expect("hils_select_backward", "nsel", nsel, (B, Hk, lq), torch.int32)
    _dense32("hils_select_backward", "dscore", dscore, (B, H, lq, k))
    _dense32("hils_select_backward", "dQcal", dQcal, (B, H, lq, d))
    _dense32("hils_select_backward", "dKsum", dKsum, (B, H, c, d))
    _dense32("hils_select_backward", "dBsum", dBsum, (B, H, c))
    _check("hils_select_backward", load_library().hils_select_backward(
        ctypes.byref(p.c()), _view(Qcal), lq, _view(Ksum), c, _ptr(idx), _ptr(nsel), _ptr(dscore), _ptr(dQcal),
        _ptr(dKsum), _ptr(dBsum), _stream(stream)))


def hils_summarize_backward(p: Params, K, LQ, dKsum, dBsum, dK, dLQ, N: int | None = None, stream=None) -> None:
    """Eq. 8 backward over the complete chunks: dLQ [B,H,C,d] (written), dK [B,Hk,N,d]
    (accumulated), float32 and dense, from dKsum [B,H,C,d] and dBsum [B,H,C]."""
    n = K.shape[2] if N is None else N
    B, H, d, Hk = p.B, p.H, p.d, p.Hk
    C = n // p.S
    if K.shape[0] != B or K.shape[1] != Hk or K.shape[3] != d or K.shape[2] < n or K.dtype != p.dtype:
        raise ValueError(f"hils_summarize_backward: K has shape {tuple(K.shape)}")
    _expect("hils_summarize_backward", "LQ", LQ, (B, H, C, d), p.dtype)
    _dense32("hils_summarize_backward", "dKsum", dKsum, (B, H, C, d))
    _dense32("hils_summarize_backward", "dBsum", dBsum, (B, H, C))
    _dense32("hils_summarize_backward", "dK", dK, (B, Hk, n, d))
    _dense32("hils_summarize_backward", "dLQ", dLQ, (B, H, C, d))
    _check("hils_summarize_backward", load_library().hils_summarize_backward(
        ctypes.byref(p.c()), _view(K), n, _view(LQ), _ptr(dKsum), _ptr(dBsum), _ptr(dK), _ptr(dLQ),
        _stream(stream)))


def alloc_workspace(p: Params, call: int, Lq: int, C: int, device="cuda") -> torch.Tensor | None:
    """Allocates (torch) and zeroes a workspace of the size the call needs, or None."""
    n = hils_workspace_bytes(p, call, Lq, C)
    if n == 0:
        return None
    ws = torch.empty((n + 15) // 16 * 16, dtype=torch.uint8, device=device)
    hils_workspace_init(ws)
    return ws


def hils_selftest_fast_math(x, z, exp2_out, recip_out, stream=None) -> None:
    """The library's FMA-pipe 2^x and 1/z helpers on every element of x and z (float32
    CUDA tensors of one size), written to exp2_out and recip_out."""
    n = x.numel()
    for name, t in (("x", x), ("z", z), ("exp2_out", exp2_out), ("recip_out", recip_out)):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or t.numel() != n:
            raise ValueError(f"hils_selftest_fast_math: {name} must be a dense float32 CUDA tensor of {n} elements")
    _check("hils_selftest_fast_math", load_library().hils_selftest_fast_math(
        _ptr(x), _ptr(z), n, _ptr(exp2_out), _ptr(recip_out), _stream(stream)))
