"""C-ABI checks that need no GPU: the library builds and loads, it exports every
function include/hils.h declares, and invalid arguments are rejected by the host
checks before any launch (so these calls never touch a device)."""
import ctypes
import os
import re

import pytest
import torch

import hierarchical_chunk_sparse_b200 as hils
from hierarchical_chunk_sparse_b200 import build as hbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hils.h")


@pytest.fixture(scope="module")
def lib():
    hbuild.build()
    return hils.load_library()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hils_[a-z_]+)\s*\(", text)))


def test_header_declarations_are_exported(lib):
    names = _declared()
    assert "hils_summarize" in names and "hils_attend_decode" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in hils.h but not exported"
    assert set(hils.EXPORTS) <= set(names)


def test_library_exports_no_undeclared_entry_points(lib):
    out = os.popen(f"nm -D --defined-only {hils.LIB_PATH}").read()
    exported = set(re.findall(r"\b(hils_[a-z_]+)$", out, flags=re.M))
    assert exported == set(_declared())


def _p(**kw):
    base = dict(B=1, H=2, d=128, K=16, W=512, dtype=hils.torch.bfloat16)
    base.update(kw)
    return hils.Params(**base)


T = hils._CTensor
ALIGNED = 0x10000  # never dereferenced: every call below fails its host checks first


def _summ(lib, p, K=None, N=256, LQ=None, Ksum=None, Bsum=ALIGNED):
    K = K or T(ALIGNED, 32768, 32768, 128)
    LQ = LQ or T(ALIGNED, 512, 512, 128)
    Ksum = Ksum or T(ALIGNED, 512, 512, 128)
    return lib.hils_summarize(ctypes.byref(p.c()), K, N, LQ, Ksum, Bsum, None)


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), 2), (dict(S=32), 2), (dict(K=33), 2), (dict(flags=2), 2), (dict(flags=3), 2),
    (dict(B=-1), 1), (dict(W=-1), 1), (dict(K=-2), 1), (dict(scale=float("nan")), 1),
])
def test_invalid_params_rejected(lib, kw, code):
    p = _p(**{k: v for k, v in kw.items() if k not in ("S", "flags")})
    if "S" in kw:
        p.S = kw["S"]
    if "flags" in kw:
        p.flags = kw["flags"]
    assert _summ(lib, p, Bsum=None if code == 1 else ALIGNED) == code


def test_bad_dtype_rejected(lib):
    p = _p()
    c = p.c()
    c.dtype = 7
    assert lib.hils_summarize(ctypes.byref(c), T(ALIGNED, 0, 0, 128), 64, T(ALIGNED, 0, 0, 128),
                              T(ALIGNED, 0, 0, 128), ALIGNED, None) == 2


def test_null_params_and_pointers(lib):
    assert lib.hils_summarize(None, T(ALIGNED, 0, 0, 128), 64, T(ALIGNED, 0, 0, 128),
                              T(ALIGNED, 0, 0, 128), ALIGNED, None) == 1
    assert _summ(lib, _p(), K=T(None, 0, 0, 128)) == 1
    assert _summ(lib, _p(), Bsum=None) == 1
    assert _summ(lib, _p(), N=-5) == 1


@pytest.mark.parametrize("view", [T(ALIGNED + 2, 32768, 32768, 128), T(ALIGNED, 32768, 32768, 132),
                                  T(ALIGNED, 32769, 32768, 128)])
def test_misalignment_rejected(lib, view):
    assert _summ(lib, _p(), K=view) == 3


def test_select_workspace_too_small(lib):
    p = _p(B=1, H=2)
    c = p.c()
    need = lib.hils_workspace_bytes(ctypes.byref(c), hils.HILS_CALL_SELECT, 1, 8000)
    # a 256-byte status header, then a screen value and radius per (query, chunk) and
    # one (max, max) pair per 64 chunks
    assert need == 256 + 2 * (8000 + 125) * 8
    rc = lib.hils_select(ctypes.byref(c), T(ALIGNED, 256, 128, 128), 1, ALIGNED, T(ALIGNED, 0, 0, 128),
                         ALIGNED, 8000, ALIGNED, ALIGNED, ALIGNED, ALIGNED, need - 16, None)
    assert rc == 4
    rc = lib.hils_select(ctypes.byref(c), T(ALIGNED, 256, 128, 128), 1, ALIGNED, T(ALIGNED, 0, 0, 128),
                         ALIGNED, 8000, ALIGNED, ALIGNED, ALIGNED, None, need, None)
    assert rc == 4


def test_decode_workspace_too_small(lib):
    p = _p(B=1, H=2)
    c = p.c()
    need = lib.hils_workspace_bytes(ctypes.byref(c), hils.HILS_CALL_ATTEND_DECODE, 1, 0)
    units = 16 + 512 // 64
    assert need >= 2 * units * 128 * 4
    v = T(ALIGNED, 256, 128, 128)
    rc = lib.hils_attend_decode(ctypes.byref(c), v, v, v, ALIGNED, ALIGNED, ALIGNED, ALIGNED, v,
                                ALIGNED, ALIGNED, need - 1, None)
    assert rc == 4


def test_decode_chain_workspace_and_validation(lib):
    p = _p(B=1, H=2)
    c = p.c()
    sel = lib.hils_workspace_bytes(ctypes.byref(c), hils.HILS_CALL_SELECT, 1, 8000)
    att = lib.hils_workspace_bytes(ctypes.byref(c), hils.HILS_CALL_ATTEND_DECODE, 1, 0)
    need = lib.hils_workspace_bytes(ctypes.byref(c), hils.HILS_CALL_DECODE, 1, 8000)
    assert need == (sel + 255) // 256 * 256 + att  # select part, aligned, then the attend part
    v = T(ALIGNED, 256, 128, 128)
    args = [ctypes.byref(c), v, T(ALIGNED, 0, 0, 128), ALIGNED, 8000, v, v, v, ALIGNED, ALIGNED, ALIGNED, ALIGNED,
            v, None]
    assert lib.hils_decode(*args, ALIGNED, need - 1, None) == 4
    assert lib.hils_decode(*args, None, need, None) == 4
    bad = list(args)
    bad[8] = None  # cache_len
    assert lib.hils_decode(*bad, ALIGNED, need, None) == 1
    bad = list(args)
    bad[4] = -1  # C
    assert lib.hils_decode(*bad, ALIGNED, need, None) == 1


def test_workspace_sizes(lib):
    assert lib.hils_workspace_bytes(None, 0, 1, 1) == 0
    assert lib.hils_workspace_bytes(ctypes.byref(_p(d=80).c()), 0, 1, 1) == 0
    assert lib.hils_workspace_bytes(ctypes.byref(_p().c()), hils.HILS_CALL_ATTEND_PREFILL, 8192, 128) == 256
    # many queries: the status word alone
    assert lib.hils_workspace_bytes(ctypes.byref(_p().c()), hils.HILS_CALL_SELECT, 8192, 128) == 256


def test_status_strings(lib):
    for code in range(6):
        assert lib.hils_status_string(code)
    assert b"unknown" in lib.hils_status_string(99)
    assert lib.hils_last_cuda_error() is not None


def test_binding_refuses_a_missing_library(tmp_path):
    with pytest.raises(ImportError):
        hils._lib_saved = hils._lib
        hils._lib = None
        try:
            hils.load_library(str(tmp_path / "missing.so"))
        finally:
            hils._lib = hils._lib_saved


def test_binding_rejects_mismatched_shapes():
    """The binding checks every tensor against the parameters before the C call, so a
    mismatched buffer can never be read or written out of bounds."""
    import torch

    p = hils.Params(B=1, H=32, d=128, K=16, W=512, dtype=torch.bfloat16)
    Q = torch.zeros(2, 3, 1, 128, dtype=torch.bfloat16)
    Ksum = torch.zeros(2, 3, 10, 128, dtype=torch.bfloat16)
    Bsum = torch.zeros(2, 3, 10)
    idx = torch.zeros(2, 3, 1, 16, dtype=torch.int32)
    with pytest.raises(ValueError, match="shape"):
        hils.hils_select(p, Q, Ksum, Bsum, idx, idx.float(), idx[..., 0])
    p2 = hils.Params(B=2, H=3, d=128, K=16, W=512, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="dtype"):
        hils.hils_select(p2, Q.float(), Ksum, Bsum, idx, idx.float(), idx[..., 0])
    with pytest.raises(ValueError, match="CUDA"):
        hils.hils_select(p2, Q, Ksum, Bsum, idx, idx.float(), idx[..., 0])


def test_window_exclusion_flag_accepted(lib):
    """flags = HILS_FLAG_EXCLUDE_WINDOW_CHUNKS passes the parameter checks, other bits do
    not (hils_workspace_bytes runs the checks and returns 0 on a rejection; it launches
    nothing)."""
    p = _p(B=1, H=2)
    c = p.c()
    c.flags = hils.HILS_FLAG_EXCLUDE_WINDOW_CHUNKS
    assert lib.hils_workspace_bytes(ctypes.byref(c), hils.HILS_CALL_SELECT, 1, 8000) > 0
    c.flags = 2
    assert lib.hils_workspace_bytes(ctypes.byref(c), hils.HILS_CALL_SELECT, 1, 8000) == 0


class _OnDevice:
    """Stands in for a CUDA tensor in the binding's argument checks (shape, dtype and
    device are all they read before the C call)."""

    is_cuda = True

    def __init__(self, *shape, dtype=torch.bfloat16):
        self.shape = torch.Size(shape)
        self.dtype = dtype

    def is_contiguous(self):
        return True


def test_grouped_query_shapes_checked_by_the_binding():
    """With H_kv, the binding expects idx/nsel and K/V with the key-value heads and score
    with the query heads; a tensor with the wrong head count is refused before any C
    call."""
    D = _OnDevice
    p = hils.Params(B=1, H=8, d=128, K=4, W=64, dtype=torch.bfloat16, H_kv=2)
    assert p.Hk == 2
    Q, Ksum, Bsum = D(1, 8, 300, 128), D(1, 8, 4, 128), D(1, 8, 4, dtype=torch.float32)
    idx_ok, nsel = D(1, 2, 300, 4, dtype=torch.int32), D(1, 2, 300, dtype=torch.int32)
    score = D(1, 8, 300, 4, dtype=torch.float32)
    with pytest.raises(ValueError, match="idx has shape"):
        hils.hils_select(p, Q, Ksum, Bsum, D(1, 8, 300, 4, dtype=torch.int32), score, nsel)
    with pytest.raises(ValueError, match="score has shape"):
        hils.hils_select(p, Q, Ksum, Bsum, idx_ok, D(1, 2, 300, 4, dtype=torch.float32), nsel)
    with pytest.raises(ValueError, match="nsel has shape"):
        hils.hils_select(p, Q, Ksum, Bsum, idx_ok, score, D(1, 8, 300, dtype=torch.int32))
    with pytest.raises(ValueError, match="K has shape"):
        hils.hils_attend_prefill(p, Q, D(1, 8, 300, 128), D(1, 2, 300, 128), idx_ok, score, nsel, Q)
    with pytest.raises(ValueError, match="hils_summarize: K has shape"):
        hils.hils_summarize(p, D(1, 8, 300, 128), D(1, 8, 4, 128), Ksum, Bsum)
    with pytest.raises(ValueError, match="Kc has shape"):
        hils.hils_attend_decode(p, D(1, 8, 1, 128), D(1, 8, 5000, 128), D(1, 2, 5000, 128),
                                D(1, dtype=torch.int32), D(1, 2, 1, 4, dtype=torch.int32),
                                D(1, 8, 1, 4, dtype=torch.float32), D(1, 2, 1, dtype=torch.int32), D(1, 8, 1, 128))


def test_backward_binding_checks():
    """The backward calls want float32 dense gradients of the forward's shapes."""
    D = _OnDevice
    p = hils.Params(B=1, H=2, d=64, K=3, W=64, dtype=torch.bfloat16)
    N = 200
    Q = D(1, 2, N, 64)
    idx, nsel = D(1, 2, N, 3, dtype=torch.int32), D(1, 2, N, dtype=torch.int32)
    score, lse = D(1, 2, N, 3, dtype=torch.float32), D(1, 2, N, dtype=torch.float32)
    g = D(1, 2, N, 64, dtype=torch.float32)
    with pytest.raises(ValueError, match="dscore has shape"):
        hils.hils_attend_prefill_backward(p, Q, Q, Q, idx, score, nsel, Q, lse, g, g, g, g,
                                          D(1, 2, N, 4, dtype=torch.float32))
    with pytest.raises(ValueError, match="dQ has dtype"):
        hils.hils_attend_prefill_backward(p, Q, Q, Q, idx, score, nsel, Q, lse, g, D(1, 2, N, 64), g, g,
                                          D(1, 2, N, 3, dtype=torch.float32))
    with pytest.raises(ValueError, match="dKsum has shape"):
        hils.hils_select_backward(p, Q, D(1, 2, 3, 64), idx, nsel, score, g, D(1, 2, 4, 64, dtype=torch.float32),
                                  D(1, 2, 3, dtype=torch.float32))
    with pytest.raises(ValueError, match="dLQ has shape"):
        hils.hils_summarize_backward(p, Q, D(1, 2, 3, 64), D(1, 2, 3, 64, dtype=torch.float32),
                                     D(1, 2, 3, dtype=torch.float32), g, D(1, 2, 4, 64, dtype=torch.float32))


def test_backward_workspace_size(lib):
    """HILS_CALL_ATTEND_BACKWARD: a 256-byte status word, D_i per query, then per (b,
    group) chunk counts, starts, cursors and the inverted index; for bf16 with d = 128 (the
    tensor-core walk) also one 16-byte record per (query head, index entry), the chunk
    items (at most C + ceil(N K / 1024) per group, 16 bytes each) and their counts, and
    bf16 copies of dO and Q; each part rounded up to 256 bytes."""
    N = 8192
    C = N // 64

    def a256(x):
        return (x + 255) // 256 * 256

    base = 256 + a256(2 * 4 * N * 4) + a256(2 * 2 * C * 4) + a256(2 * 2 * (C + 1) * 4) + a256(2 * 2 * C * 4) + \
        a256(2 * 2 * N * 16 * 4)
    p = hils.Params(B=2, H=4, d=64, K=16, W=512, dtype=torch.bfloat16, H_kv=2)
    assert lib.hils_workspace_bytes(ctypes.byref(p.c()), hils.HILS_CALL_ATTEND_BACKWARD, N, 0) == base
    p = hils.Params(B=2, H=4, d=128, K=16, W=512, dtype=torch.float32, H_kv=2)
    assert lib.hils_workspace_bytes(ctypes.byref(p.c()), hils.HILS_CALL_ATTEND_BACKWARD, N, 0) == base
    p = hils.Params(B=2, H=4, d=128, K=16, W=512, dtype=torch.bfloat16, H_kv=2)
    items = C + (N * 16 + 1023) // 1024
    tc = a256(2 * 4 * N * 16 * 16) + a256(2 * 2 * items * 16) + a256(2 * 2 * 4) + 2 * a256(2 * 4 * N * 128 * 2)
    assert lib.hils_workspace_bytes(ctypes.byref(p.c()), hils.HILS_CALL_ATTEND_BACKWARD, N, 0) == base + tc


def test_decode_time_and_backward_entry_points_validate_first(lib):
    """hils_summarize_append and the three backward calls reject bad arguments with the
    documented codes before any launch: null arrays (1), negative sizes (1), misaligned
    views (3), a workspace smaller than hils_workspace_bytes (4), unsupported params (2)."""
    p = _p(B=1, H=2, d=128, K=4, W=64)
    c = ctypes.byref(p.c())
    v = T(ALIGNED, 4 * 8192 * 128, 8192 * 128, 128)   # [1, 2, 8192, 128] view
    s = T(ALIGNED, 2 * 128 * 128, 128 * 128, 128)     # [1, 2, 128, 128] table
    bad = T(ALIGNED + 8, 4 * 8192 * 128, 8192 * 128, 128)
    A = ALIGNED
    N, C = 8192, 128
    # hils_summarize_append(p, K, cache_len, LQ, Ksum, Bsum, C, stream)
    assert lib.hils_summarize_append(c, v, None, s, s, A, C, None) == 1
    assert lib.hils_summarize_append(c, v, A, s, s, A, -1, None) == 1
    assert lib.hils_summarize_append(c, bad, A, s, s, A, C, None) == 3
    assert lib.hils_summarize_append(ctypes.byref(_p(d=96).c()), v, A, s, s, A, C, None) == 2
    # hils_attend_prefill_backward(p, Q, K, V, N, idx, score, nsel, O, lse, dO, dQ, dK, dV, dscore, ws, n, stream)
    need = lib.hils_workspace_bytes(c, hils.HILS_CALL_ATTEND_BACKWARD, N, 0)
    assert need > 0
    args = [v, v, v, N, A, A, A, v, A, A, A, A, A, A]
    assert lib.hils_attend_prefill_backward(c, *args, A, need - 1, None) == 4
    assert lib.hils_attend_prefill_backward(c, *args, None, need, None) == 4
    assert lib.hils_attend_prefill_backward(c, *args[:9], None, *args[10:], A, need, None) == 1  # dO
    assert lib.hils_attend_prefill_backward(c, *args[:3], -1, *args[4:], A, need, None) == 1
    assert lib.hils_attend_prefill_backward(c, bad, *args[1:], A, need, None) == 3
    assert lib.hils_attend_prefill_backward(c, *args[:8], A + 2, *args[9:], A, need, None) == 3  # lse
    # hils_select_backward(p, Qcal, Lq, Ksum, C, idx, nsel, dscore, dQcal, dKsum, dBsum, stream)
    assert lib.hils_select_backward(c, v, N, s, C, A, A, None, A, A, A, None) == 1
    assert lib.hils_select_backward(c, v, -1, s, C, A, A, A, A, A, A, None) == 1
    assert lib.hils_select_backward(c, bad, N, s, C, A, A, A, A, A, A, None) == 3
    assert lib.hils_select_backward(ctypes.byref(_p(K=40).c()), v, N, s, C, A, A, A, A, A, A, None) == 2
    # hils_summarize_backward(p, K, N, LQ, dKsum, dBsum, dK, dLQ, stream)
    assert lib.hils_summarize_backward(c, v, N, s, A, A, None, A, None) == 1
    assert lib.hils_summarize_backward(c, v, -64, s, A, A, A, A, None) == 1
    assert lib.hils_summarize_backward(c, v, N, bad, A, A, A, A, None) == 3
    g = _p(H=4, H_kv=3)
    assert lib.hils_summarize_backward(ctypes.byref(g.c()), v, N, s, A, A, A, A, None) == 1


C_CALLER = r"""
#include <stdio.h>
#include <string.h>
#include "hils.h"

/* every entry point the header declares, taken by address: the program links only if
   the library defines each one with C linkage */
typedef void (*any_fn)(void);
static const any_fn entry_points[] = {
%(entries)s
};

int main(void) {
    hils_params p;
    size_t n;
    int i;
    memset(&p, 0, sizeof p);
    p.B = 1; p.H = 32; p.d = 128; p.S = 64; p.K = 16; p.W = 512; p.dtype = HILS_BF16;
    for (i = 0; i < (int)(sizeof entry_points / sizeof entry_points[0]); ++i)
        if (!entry_points[i]) return 10;
    for (i = HILS_OK; i <= HILS_ERR_CUDA; ++i)
        if (!hils_status_string(i) || !hils_status_string(i)[0]) return 11;
    n = hils_workspace_bytes(&p, HILS_CALL_DECODE, 1, 8191);
    printf("decode_ws %%zu\n", n);
    /* host checks run before anything is launched: no device is touched */
    printf("null_params %%d\n", hils_summarize(NULL, (hils_ctensor){0}, 64, (hils_ctensor){0},
                                              (hils_tensor){0}, NULL, 0));
    p.d = 80;
    printf("bad_d %%d\n", hils_summarize(&p, (hils_ctensor){0}, 64, (hils_ctensor){0},
                                        (hils_tensor){0}, NULL, 0));
    return 0;
}
"""


def test_header_is_plain_c_and_links_from_a_c_program(lib, tmp_path):
    """A C99 program (gcc, no C++) includes hils.h, takes the address of every declared
    entry point, links against libhils.so and runs on the host: the status strings, the
    decode chain's workspace size (equal to the value the binding sees) and two calls
    that the host checks reject before any launch."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    cuda_inc = "/usr/local/cuda/include"
    src = tmp_path / "caller.c"
    src.write_text(C_CALLER % {"entries": ",\n".join(f"    (any_fn)&{n}" for n in _declared())})
    exe = tmp_path / "caller"
    pkg = os.path.dirname(hils.LIB_PATH)
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), "-isystem", cuda_inc, str(src), "-o", str(exe),
           "-L", pkg, "-l:libhils.so", f"-Wl,-rpath,{pkg}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    got = dict(line.split() for line in r.stdout.strip().splitlines())
    p = _p(B=1, H=32, K=16, W=512)
    assert int(got["decode_ws"]) == lib.hils_workspace_bytes(ctypes.byref(p.c()), hils.HILS_CALL_DECODE, 1, 8191) > 0
    assert int(got["null_params"]) == 1  # HILS_ERR_INVALID_ARG
    assert int(got["bad_d"]) == 2  # HILS_ERR_UNSUPPORTED
