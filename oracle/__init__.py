"""fp64 CPU oracle for the Mamba-2 SSD layer (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
its Python binding) never does. The arithmetic lives in ``ssd_oracle.c``
(plain C, fp64, no shared code with the CUDA library); this module compiles it
with gcc on first use and marshals numpy arrays to it.

Pages followed (see ``ssd_oracle.c`` for the passage per routine):
"Mamba-2" (docsaid.org), sections "Writing the SSM as one matrix",
"Simplifying A to one number", "Computing with four tokens"; "Mamba paper
review" (youngju.dev), section 3.3; "Mamba-2 SSD note" (0h-n0.github.io),
section "SSD layer: equivalence under the scalar constraint".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libssd_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``ssd_oracle.c`` into ``oracle/_build/libssd_oracle.so``."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        compile_source(_SRC, tmp)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def compile_source(src_path: str, out_path: str) -> str:
    """Compile a C source with the oracle's flags (used by ``build`` and by the
    tests that plant a mistake in a copy of the oracle)."""
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
           "-fno-fast-math", "-std=c99", src_path, "-o", out_path, "-lm"]
    subprocess.run(cmd, check=True)
    return out_path


def bind(path: str):
    """Load a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    i = ctypes.c_int
    lib.ssd_oracle_forward.argtypes = [dp] * 9 + [i] * 7
    lib.ssd_oracle_mask.argtypes = [dp, i, dp]
    lib.ssd_oracle_quadratic.argtypes = [dp] * 7 + [i] * 6
    lib.ssd_oracle_scan_core.argtypes = [dp] * 7 + [i] * 3
    lib.ssd_oracle_step.argtypes = [dp] * 8 + [i] * 5
    for f in (lib.ssd_oracle_forward, lib.ssd_oracle_mask, lib.ssd_oracle_quadratic,
              lib.ssd_oracle_scan_core, lib.ssd_oracle_step):
        f.restype = ctypes.c_int
    return lib


_override = None


def use_library(lib) -> None:
    """Route the module functions to another compiled oracle (``None`` resets)."""
    global _override
    _override = lib


def _load():
    global _lib
    if _override is not None:
        return _override
    with _lock:
        if _lib is None:
            _lib = bind(build())
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: invalid arguments")


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def forward(x, dt, A, Bm, Cm, D=None, init_state=None, nthreads: int | None = None):
    """Sequential fp64 recurrence. Shapes: x[B,L,H,P], dt[B,L,H], A[H],
    Bm/Cm[B,L,G,N], D[H] or None, init_state[B,H,P,N] or None.
    Returns (y[B,L,H,P], final_state[B,H,P,N]) in fp64."""
    x, dt, A, Bm, Cm = map(_f64, (x, dt, A, Bm, Cm))
    D = None if D is None else _f64(D)
    init_state = None if init_state is None else _f64(init_state)
    Bsz, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    assert dt.shape == (Bsz, L, H) and A.shape == (H,)
    assert Bm.shape == (Bsz, L, G, N) and Cm.shape == Bm.shape
    y = np.empty((Bsz, L, H, P), np.float64)
    fs = np.empty((Bsz, H, P, N), np.float64)
    rc = _load().ssd_oracle_forward(_ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(D),
                                    _ptr(init_state), _ptr(y), _ptr(fs),
                                    Bsz, L, H, P, G, N, nthreads or default_threads())
    _check(rc, "ssd_oracle_forward")
    return y, fs


def mask(a):
    """L[j, i] = a_j ... a_{i+1} for j >= i, else 0 (literal products)."""
    a = _f64(a)
    L = a.shape[0]
    out = np.empty((L, L), np.float64)
    _check(_load().ssd_oracle_mask(_ptr(a), L, _ptr(out)), "ssd_oracle_mask")
    return out


def quadratic(x, dt, A, Bm, Cm, D=None):
    """Brute-force y = (L o C B^T)(dt o x) + D x; tiny inputs only."""
    x, dt, A, Bm, Cm = map(_f64, (x, dt, A, Bm, Cm))
    D = None if D is None else _f64(D)
    Bsz, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    y = np.empty((Bsz, L, H, P), np.float64)
    rc = _load().ssd_oracle_quadratic(_ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(D),
                                      _ptr(y), Bsz, L, H, P, G, N)
    _check(rc, "ssd_oracle_quadratic")
    return y


def scan_core(a, s, x, Bm, Cm):
    """One head: h = a_t h + s_t x_t B_t^T, y_t = h C_t. x[L,P], Bm/Cm[L,N].
    Returns (y[L,P], h_final[P,N])."""
    a, s, x, Bm, Cm = map(_f64, (a, s, x, Bm, Cm))
    L, P = x.shape
    N = Bm.shape[1]
    y = np.empty((L, P), np.float64)
    h = np.empty((P, N), np.float64)
    rc = _load().ssd_oracle_scan_core(_ptr(a), _ptr(s), _ptr(x), _ptr(Bm), _ptr(Cm), _ptr(y),
                                      _ptr(h), L, P, N)
    _check(rc, "ssd_oracle_scan_core")
    return y, h


def step(x, dt, A, Bm, Cm, D, state):
    """One decode step. x[B,H,P], dt[B,H], Bm/Cm[B,G,N], state[B,H,P,N].
    Returns (y[B,H,P], new_state[B,H,P,N]); the input state is not modified."""
    x, dt, A, Bm, Cm = map(_f64, (x, dt, A, Bm, Cm))
    D = None if D is None else _f64(D)
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    Bsz, H, P = x.shape
    G, N = Bm.shape[1], Bm.shape[2]
    y = np.empty((Bsz, H, P), np.float64)
    rc = _load().ssd_oracle_step(_ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(D),
                                 _ptr(st), _ptr(y), Bsz, H, P, G, N)
    _check(rc, "ssd_oracle_step")
    return y, st
