"""fp64 CPU oracle for the SSD layer -- test infrastructure only.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library in
``ssd_chunked_scan_02_b200`` and its binding) never imports it, and the two
share no code: the only thing both sides use is the seeded input generator,
which holds none of the method's arithmetic.

The arithmetic lives in ``ssd_oracle.c`` (plain C, double precision, OpenMP
over (batch, head) pairs): the sequential linear recurrence

    a_t = exp(dt_t * A_h);  S_t = a_t S_{t-1} + dt_t x_t B_t^T;  y_t = S_t C_t + D_h x_t

following "论文解读：Mamba: Linear-Time Sequence Modeling with Selective State
Spaces", section 状态空间模型 (discretise, then evaluate as a linear
recurrence) and "Transformers are SSMs" (CiteArk), AI research summary
(1-semiseparable selective SSM).  Every function is pinned by the ``not gpu``
tests in ``tests/test_oracle_pins.py`` against closed forms, the materialised
semiseparable matrix and brute-force expansions.  ``backward`` (the gradients
of the same recurrence, for the training use the pages name) is pinned in
``tests/test_oracle_backward.py`` against central finite differences of the
forward recurrence and closed forms.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "libssd_oracle.so")
_lib = None

_dbl_p = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile ssd_oracle.c into libssd_oracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC", "-std=c11",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _open(path):
    lib = ctypes.CDLL(path)
    lib.ssd_oracle_recurrence.restype = ctypes.c_int
    lib.ssd_oracle_recurrence.argtypes = [_i64] * 6 + [_dbl_p] * 9 + [ctypes.c_int]
    lib.ssd_oracle_step.restype = ctypes.c_int
    lib.ssd_oracle_step.argtypes = [_i64] * 5 + [_dbl_p] * 8
    lib.ssd_oracle_backward.restype = ctypes.c_int
    lib.ssd_oracle_backward.argtypes = [_i64] * 6 + [_dbl_p] * 16
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _open(_LIB)
    return _lib


def _f64(a):
    """Contiguous float64 copy of a numpy array or (CPU) torch tensor."""
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dbl_p)


def recurrence(x, dt, A, B, C, D, init=None, threads: int = 0, _lib_override=None):
    """Run the fp64 recurrence.  Shapes: x (b,L,H,P), dt (b,L,H), A (H),
    B/C (b,L,G,N), D (H), init (b,H,P,N) or None.  Returns (y, final) as
    float64 numpy arrays of shapes (b,L,H,P) and (b,H,P,N)."""
    x, dt, A, B, C, D, init = (_f64(v) for v in (x, dt, A, B, C, D, init))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert dt.shape == (b, L, H) and A.shape == (H,) and D.shape == (H,)
    assert B.shape == (b, L, G, N) and C.shape == (b, L, G, N)
    if init is not None:
        assert init.shape == (b, H, P, N)
    y = np.empty((b, L, H, P), dtype=np.float64)
    final = np.empty((b, H, P, N), dtype=np.float64)
    lib = _lib_override if _lib_override is not None else _load()
    rc = lib.ssd_oracle_recurrence(b, L, H, P, N, G, _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                                       _ptr(C), _ptr(D), _ptr(init), _ptr(y), _ptr(final),
                                       int(threads))
    if rc != 0:
        raise ValueError("ssd_oracle_recurrence rejected its arguments")
    return y, final


def recurrence_from(path):
    """A ``recurrence`` bound to another build of ssd_oracle.c (used by the
    mutation test, which compiles deliberately broken copies)."""
    lib = _open(path)

    def rec(x, dt, A, B, C, D, init=None, threads: int = 0):
        return recurrence(x, dt, A, B, C, D, init, threads, _lib_override=lib)
    return rec


def step(state, x, dt, A, B, C, D):
    """One fp64 decode step.  state (b,H,P,N) is NOT modified; returns
    (y (b,H,P), new_state (b,H,P,N))."""
    st = _f64(state).copy()
    x, dt, A, B, C, D = (_f64(v) for v in (x, dt, A, B, C, D))
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    assert st.shape == (b, H, P, N) and dt.shape == (b, H)
    y = np.empty((b, H, P), dtype=np.float64)
    rc = _load().ssd_oracle_step(b, H, P, N, G, _ptr(st), _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                                 _ptr(C), _ptr(D), _ptr(y))
    if rc != 0:
        raise ValueError("ssd_oracle_step rejected its arguments")
    return y, st


def backward(x, dt, A, B, C, D, init, dy, dfinal=None, _lib_override=None):
    """Gradients of the fp64 recurrence for a loss with dL/dy = dy (b,L,H,P)
    and dL/dfinal = dfinal (b,H,P,N) or None (zero).  init None means a zero
    initial state.  Returns a dict of float64 arrays: dx (b,L,H,P), ddt
    (b,L,H), dA (H), dB (b,L,G,N), dC (b,L,G,N), dD (H), dinit (b,H,P,N)."""
    x, dt, A, B, C, D, init, dy, dfinal = (_f64(v) for v in (x, dt, A, B, C, D, init, dy, dfinal))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert dy.shape == x.shape
    if dfinal is not None:
        assert dfinal.shape == (b, H, P, N)
    out = {"dx": np.empty((b, L, H, P)), "ddt": np.empty((b, L, H)), "dA": np.empty((H,)),
           "dB": np.empty((b, L, G, N)), "dC": np.empty((b, L, G, N)), "dD": np.empty((H,)),
           "dinit": np.empty((b, H, P, N))}
    lib = _lib_override if _lib_override is not None else _load()
    rc = lib.ssd_oracle_backward(b, L, H, P, N, G, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                                 _ptr(D), _ptr(init), _ptr(dy), _ptr(dfinal), _ptr(out["dx"]),
                                 _ptr(out["ddt"]), _ptr(out["dA"]), _ptr(out["dB"]),
                                 _ptr(out["dC"]), _ptr(out["dD"]), _ptr(out["dinit"]))
    if rc != 0:
        raise ValueError("ssd_oracle_backward rejected its arguments")
    return out


def backward_from(path):
    """A ``backward`` bound to another build of ssd_oracle.c (mutation tests)."""
    lib = _open(path)

    def bwd(x, dt, A, B, C, D, init, dy, dfinal=None):
        return backward(x, dt, A, B, C, D, init, dy, dfinal, _lib_override=lib)
    return bwd
