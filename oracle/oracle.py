"""ctypes front end of the fp64 CPU oracle (test infrastructure only).

Each function takes numpy arrays in the layer's layouts and returns float64 results:

    x  [b, L, H, P]   dt [b, L, H]   A [H]   D [H]
    B  [b, L, G, N]   C  [b, L, G, N]         state [b, H, P, N]   ->   y [b, L, H, P]

`recurrence` is the sequential recurrence h_t = exp(dt_t A_h) h_{t-1} + dt_t x_t B_t^T,
y_t = C_t h_t + D_h x_t ("Engineering Hybrid State-Space Models", section 2, with the
scalar-per-head dynamics of "Compiler-First State Space Duality ...", abstract).
`quadratic` is the semiseparable form Y = (M o C B^T) X of the same section and `chunked`
the fixed-size-chunk form with an inter-chunk carry; both exist to pin `recurrence`.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _load(path: str = None):
    global _lib
    if path is not None:
        lib = ctypes.CDLL(path)
        _declare(lib)
        return lib
    if _lib is None:
        _lib = ctypes.CDLL(_build.build())
        _declare(_lib)
    return _lib


def _declare(lib):
    i64, dp, ci = ctypes.c_int64, ctypes.POINTER(ctypes.c_double), ctypes.c_int
    lib.ssd_oracle_recurrence.argtypes = [i64] * 6 + [dp] * 8 + [ci]
    lib.ssd_oracle_quadratic.argtypes = [i64] * 6 + [dp] * 9 + [ci]
    lib.ssd_oracle_chunked.argtypes = [i64] * 7 + [dp] * 9 + [ci]
    for f in (lib.ssd_oracle_recurrence, lib.ssd_oracle_quadratic, lib.ssd_oracle_chunked):
        f.restype = ci


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _dims(x, B):
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    return b, L, H, P, N, G


def recurrence(x, dt, A, B, C, D, state=None, nthreads=None, lib=None):
    """Sequential fp64 recurrence.  `state` is the initial state (zeros if None).

    Returns (y [b,L,H,P], final_state [b,H,P,N]).
    """
    lib = lib or _load()
    x, dt, A, B, C, D = map(_f64, (x, dt, A, B, C, D))
    b, L, H, P, N, G = _dims(x, B)
    st = np.zeros((b, H, P, N)) if state is None else _f64(state).copy()
    y = np.zeros((b, L, H, P))
    rc = lib.ssd_oracle_recurrence(b, L, H, P, N, G, _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                                   _ptr(C), _ptr(D), _ptr(st), _ptr(y),
                                   nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle recurrence rejected the arguments (code {rc})")
    return y, st


def quadratic(x, dt, A, B, C, D, state=None, nthreads=None, lib=None):
    """Quadratic semiseparable form; O(L^2) per head, tiny inputs only."""
    lib = lib or _load()
    x, dt, A, B, C, D = map(_f64, (x, dt, A, B, C, D))
    b, L, H, P, N, G = _dims(x, B)
    init = None if state is None else _f64(state)
    y = np.zeros((b, L, H, P))
    fin = np.zeros((b, H, P, N))
    rc = lib.ssd_oracle_quadratic(b, L, H, P, N, G, _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                                  _ptr(C), _ptr(D), _ptr(init), _ptr(y), _ptr(fin),
                                  nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle quadratic rejected the arguments (code {rc})")
    return y, fin


def chunked(x, dt, A, B, C, D, chunk, state=None, nthreads=None, lib=None):
    """Chunked form with chunk length `chunk` (the last chunk may be partial)."""
    lib = lib or _load()
    x, dt, A, B, C, D = map(_f64, (x, dt, A, B, C, D))
    b, L, H, P, N, G = _dims(x, B)
    init = None if state is None else _f64(state)
    y = np.zeros((b, L, H, P))
    fin = np.zeros((b, H, P, N))
    rc = lib.ssd_oracle_chunked(b, L, H, P, N, G, int(chunk), _ptr(x), _ptr(dt), _ptr(A),
                                _ptr(B), _ptr(C), _ptr(D), _ptr(init), _ptr(y), _ptr(fin),
                                nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle chunked rejected the arguments (code {rc})")
    return y, fin
