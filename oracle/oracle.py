"""Python access to the fp64 CPU oracle (``rsa_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the benchmark's
CPU-baseline leg may import this module; the library and its binding never do.

Every function takes numpy arrays of shape [B, H, L, d] (any float dtype; they are upcast to
fp64) and returns fp64 arrays. ``build()`` compiles ``rsa_oracle.c`` with gcc and OpenMP into
``_build/librsa_oracle.so`` next to this file.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "librsa_oracle.so")
_lib = None
_lock = threading.Lock()

_D = ctypes.POINTER(ctypes.c_double)
_LP = ctypes.POINTER(ctypes.c_long)
_l = ctypes.c_long
_i = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile the oracle shared library if it is missing or older than its source."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_SIGS = {
    "rsa_oracle_forward_plain": [_D, _D, _D, _l, _l, _l, _i, _D, _D],
    "rsa_oracle_probs_plain": [_D, _D, _l, _l, _l, _i, _D],
    "rsa_oracle_backward_plain": [_D, _D, _D, _D, _l, _l, _l, _i, _D, _D, _D],
    "rsa_oracle_forward_ring": [_D, _D, _D, _l, _l, _l, _l, _i, _D, _D],
    "rsa_oracle_backward_ring": [_D, _D, _D, _D, _l, _l, _l, _l, _i, _D, _D, _D],
    "rsa_oracle_forward_rows": [_D, _D, _D, _l, _l, _i, _LP, _l, _D, _D],
    "rsa_oracle_backward_rows": [_D, _D, _D, _D, _l, _l, _i, _LP, _l, _D],
    "rsa_oracle_backward_keys": [_D, _D, _D, _D, _l, _l, _i, _LP, _l, _D, _D],
    "rsa_oracle_linear": [_D, _D, _D, _D, _l, _l, _l, _i, _D],
}


def open_library(path: str):
    """Load an oracle shared library and declare its signatures."""
    lib = ctypes.CDLL(path)
    for name, args in _SIGS.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = _i
    lib.rsa_oracle_set_threads.argtypes = [_i]
    lib.rsa_oracle_set_threads.restype = None
    lib.rsa_oracle_max_threads.argtypes = []
    lib.rsa_oracle_max_threads.restype = _i
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = open_library(build())
    return _lib


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_D)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise RuntimeError(f"{what} failed with code {rc}")


def set_threads(n: int) -> None:
    _load().rsa_oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().rsa_oracle_max_threads())


def _shape(q):
    if q.ndim != 4:
        raise ValueError("expected [B, H, L, d]")
    B, H, L, d = q.shape
    return B, H, L, d


def forward(q, k, v, causal: bool = False):
    """Plain definition. Returns (O [B,H,L,d], lse [B,H,L])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, L, d = _shape(q)
    o = np.empty_like(q)
    lse = np.empty((B, H, L))
    _check(_load().rsa_oracle_forward_plain(_ptr(q), _ptr(k), _ptr(v), B * H, L, d,
                                            int(causal), _ptr(o), _ptr(lse)), "forward")
    return o, lse


def probs(q, k, causal: bool = False):
    """Softmax probabilities P [B,H,L,L] (small problems)."""
    q, k = _f64(q), _f64(k)
    B, H, L, d = _shape(q)
    p = np.empty((B, H, L, L))
    _check(_load().rsa_oracle_probs_plain(_ptr(q), _ptr(k), B * H, L, d, int(causal), _ptr(p)),
           "probs")
    return p


def backward(q, k, v, do, causal: bool = False):
    """Plain definition. Returns (dQ, dK, dV)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, L, d = _shape(q)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    _check(_load().rsa_oracle_backward_plain(_ptr(q), _ptr(k), _ptr(v), _ptr(do), B * H, L, d,
                                             int(causal), _ptr(dq), _ptr(dk), _ptr(dv)),
           "backward")
    return dq, dk, dv


def forward_ring(q, k, v, N: int, causal: bool = False):
    """Ring schedule with N chunks. Returns (O, lse)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, L, d = _shape(q)
    o = np.empty_like(q)
    lse = np.empty((B, H, L))
    _check(_load().rsa_oracle_forward_ring(_ptr(q), _ptr(k), _ptr(v), B * H, L, d, N,
                                           int(causal), _ptr(o), _ptr(lse)), "forward_ring")
    return o, lse


def backward_ring(q, k, v, do, N: int, causal: bool = False):
    """Ring schedule with N chunks. Returns (dQ, dK, dV)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, L, d = _shape(q)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    _check(_load().rsa_oracle_backward_ring(_ptr(q), _ptr(k), _ptr(v), _ptr(do), B * H, L, d, N,
                                            int(causal), _ptr(dq), _ptr(dk), _ptr(dv)),
           "backward_ring")
    return dq, dk, dv


def _head(x, b, h):
    return _f64(np.asarray(x)[b, h])


def _idx(rows):
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64))


def forward_rows(q, k, v, b: int, h: int, rows, causal: bool = False):
    """O and lse of the listed query rows of head (b, h). Returns (O [n,d], lse [n])."""
    qh, kh, vh = _head(q, b, h), _head(k, b, h), _head(v, b, h)
    L, d = qh.shape
    r = _idx(rows)
    o = np.empty((len(r), d))
    lse = np.empty(len(r))
    _check(_load().rsa_oracle_forward_rows(_ptr(qh), _ptr(kh), _ptr(vh), L, d, int(causal),
                                           r.ctypes.data_as(_LP), len(r), _ptr(o), _ptr(lse)),
           "forward_rows")
    return o, lse


def backward_rows(q, k, v, do, b: int, h: int, rows, causal: bool = False):
    """dQ of the listed query rows of head (b, h), shape [n, d]."""
    qh, kh, vh, doh = _head(q, b, h), _head(k, b, h), _head(v, b, h), _head(do, b, h)
    L, d = qh.shape
    r = _idx(rows)
    dq = np.empty((len(r), d))
    _check(_load().rsa_oracle_backward_rows(_ptr(qh), _ptr(kh), _ptr(vh), _ptr(doh), L, d,
                                            int(causal), r.ctypes.data_as(_LP), len(r), _ptr(dq)),
           "backward_rows")
    return dq


def backward_keys(q, k, v, do, b: int, h: int, keys, causal: bool = False):
    """dK and dV of the listed key rows of head (b, h), each [n, d]."""
    qh, kh, vh, doh = _head(q, b, h), _head(k, b, h), _head(v, b, h), _head(do, b, h)
    L, d = qh.shape
    r = _idx(keys)
    dk = np.empty((len(r), d))
    dv = np.empty((len(r), d))
    _check(_load().rsa_oracle_backward_keys(_ptr(qh), _ptr(kh), _ptr(vh), _ptr(doh), L, d,
                                            int(causal), r.ctypes.data_as(_LP), len(r), _ptr(dk),
                                            _ptr(dv)), "backward_keys")
    return dk, dv


def linear(x, w, b=None, r=None, gelu: bool = False):
    """Y = act(X W^T + b) + R on rows: X [M, K], W [N, K], b [N] or None, R [M, N] or None;
    act = exact GELU when `gelu`, else the identity. Returns Y [M, N] fp64."""
    x, w = _f64(x), _f64(w)
    if x.ndim != 2 or w.ndim != 2 or x.shape[1] != w.shape[1]:
        raise ValueError("expected X [M, K] and W [N, K]")
    M, K = x.shape
    N = w.shape[0]
    bb = _f64(b) if b is not None else None
    rr = _f64(r) if r is not None else None
    if bb is not None and bb.shape != (N,):
        raise ValueError("bias must be [N]")
    if rr is not None and rr.shape != (M, N):
        raise ValueError("residual must be [M, N]")
    y = np.empty((M, N))
    _check(_load().rsa_oracle_linear(_ptr(x), _ptr(w), _ptr(bb) if bb is not None else None,
                                     _ptr(rr) if rr is not None else None, M, N, K, int(gelu),
                                     _ptr(y)), "linear")
    return y


@contextlib.contextmanager
def using_library(lib):
    """Route this module's functions to another loaded oracle library for the duration of the
    block (the mutation tests load deliberately broken copies of the oracle this way)."""
    global _lib
    _load()
    with _lock:
        prev, _lib = _lib, lib
    try:
        yield
    finally:
        with _lock:
            _lib = prev
