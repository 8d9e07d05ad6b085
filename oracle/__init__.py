"""fp64 CPU oracle for RetNet multi-scale retention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The CUDA product path shares no code with it and never
calls it.  The arithmetic lives in ``retnet_oracle.c`` (plain loops, fp64); this
module only marshals numpy arrays to it.

Sources: "阅读笔记：RetNet" (mzeromiko blog): §2.2 Recurrent Mode, §2.3 Parallel Mode,
§2.4 Chunkwise Recurrent Mode, §三.2 MSR, §三.3 Normalization.  The readings taken
where the page is silent are listed at the top of ``retnet_oracle.c``.

Pins: every function here is pinned by ``tests/test_oracle_pins.py`` against closed
forms, library special cases and the three-way agreement of the page's three forms.
"""
import ctypes
import os

import numpy as np

from . import build as _build

F_XPOS = 1
F_SCALE_SQRT_D = 2
F_NORM_D = 4
F_NORM_R = 8
F_ALL = F_XPOS | F_SCALE_SQRT_D | F_NORM_D | F_NORM_R


class _Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("heads", ctypes.c_int64),
                ("d_k", ctypes.c_int64), ("d_v", ctypes.c_int64)]


_lib = None


def _load():
    global _lib
    if _lib is None:
        # A test may point the wrapper at a deliberately broken copy of the oracle
        # (tests/test_oracle_mutants.py) to show that the pins catch the mistake.
        path = os.environ.get("RETNET_ORACLE_LIB_OVERRIDE") or _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_parallel.argtypes = [dp, dp, dp, dp, _Dims, dp, dp, ctypes.c_int64, ctypes.c_uint,
                                        ctypes.c_int]
        lib.oracle_recurrent.argtypes = [dp, dp, dp, dp, _Dims, dp, dp, ctypes.c_int64, ctypes.c_uint,
                                         dp, dp, dp, dp, ctypes.c_int]
        lib.oracle_chunkwise.argtypes = [dp, dp, dp, dp, _Dims, dp, dp, ctypes.c_int64, ctypes.c_uint,
                                         ctypes.c_int64, dp, dp, dp, dp, ctypes.c_int]
        lib.oracle_msr_epilogue.argtypes = [dp, dp, dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.c_double, ctypes.c_int]
        lib.oracle_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_backward.argtypes = [dp, dp, dp, dp, dp, dp, dp, _Dims, dp, dp, ctypes.c_int64, ctypes.c_uint,
                                        dp, dp, ctypes.c_int]
        for f in (lib.oracle_parallel, lib.oracle_recurrent, lib.oracle_chunkwise,
                  lib.oracle_msr_epilogue, lib.oracle_num_threads, lib.oracle_backward):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    """Contiguous fp64 copy of x (a numpy array or anything np.asarray accepts, e.g. a CPU tensor)."""
    if hasattr(x, "detach"):  # torch tensor: upcast exactly, then to numpy
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _dims(q, v):
    b, L, h, dk = q.shape
    dv = v.shape[-1]
    return _Dims(b, L, h, dk, dv)


def _theta_arr(theta, dk):
    if theta is None:
        return np.zeros(max(dk // 2, 1), dtype=np.float64)
    return _f64(theta)


def num_threads(nthreads: int = 0) -> int:
    """Threads the oracle's OpenMP loops use for a given request (0 = runtime default)."""
    return _load().oracle_num_threads(nthreads)


def parallel(q, k, v, gamma, theta=None, pos0=0, flags=F_ALL, nthreads=0):
    """Parallel form O = (QK^T (.) D)V with the normalisations (page §2.3, §三.3).

    q,k: (batch, L, heads, d_k); v: (batch, L, heads, d_v); returns o like v, fp64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    o = np.zeros(v.shape, dtype=np.float64)
    g, th = _f64(gamma), _theta_arr(theta, q.shape[-1])
    rc = _load().oracle_parallel(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _dims(q, v), _ptr(g), _ptr(th),
                                 int(pos0), int(flags), int(nthreads))
    assert rc == 0
    return o


def recurrent(q, k, v, gamma, theta=None, pos0=0, flags=F_ALL, state_in=None, z_in=None, nthreads=0):
    """Recurrent form S_n = gamma S_{n-1} + K_n^T V_n, o_n = Q_n S_n (page §2.2).

    Returns (o, state_out (batch, heads, d_k, d_v), z_out (batch, heads, d_k)), fp64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    b, L, h, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros(v.shape, dtype=np.float64)
    so = np.zeros((b, h, dk, dv), dtype=np.float64)
    zo = np.zeros((b, h, dk), dtype=np.float64)
    si = None if state_in is None else _f64(state_in)
    zi = None if z_in is None else _f64(z_in)
    g, th = _f64(gamma), _theta_arr(theta, dk)
    rc = _load().oracle_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _dims(q, v), _ptr(g), _ptr(th),
                                  int(pos0), int(flags), _ptr(si), _ptr(so), _ptr(zi), _ptr(zo),
                                  int(nthreads))
    assert rc == 0
    return o, so, zo


def chunkwise(q, k, v, gamma, chunk, theta=None, pos0=0, flags=F_ALL, state_in=None, z_in=None,
              nthreads=0):
    """Chunkwise recurrent form of page §2.4 with chunk length ``chunk``.

    Returns (o, state_out, z_out), fp64, like :func:`recurrent`.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    b, L, h, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros(v.shape, dtype=np.float64)
    so = np.zeros((b, h, dk, dv), dtype=np.float64)
    zo = np.zeros((b, h, dk), dtype=np.float64)
    si = None if state_in is None else _f64(state_in)
    zi = None if z_in is None else _f64(z_in)
    g, th = _f64(gamma), _theta_arr(theta, dk)
    rc = _load().oracle_chunkwise(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _dims(q, v), _ptr(g), _ptr(th),
                                  int(pos0), int(flags), int(chunk), _ptr(si), _ptr(so), _ptr(zi),
                                  _ptr(zo), int(nthreads))
    assert rc == 0
    return o, so, zo


def msr_epilogue(y, g, heads, eps=1e-5, nthreads=0):
    """GroupNorm over each head's d_v values, then swish(G) (.) Y (page §三.2).

    y, g: (..., heads*d_v) or (..., heads, d_v); returns out with y's shape, fp64.
    """
    y, g = _f64(y), _f64(g)
    shape = y.shape
    total = y.size
    dv = (shape[-1] // heads) if (len(shape) < 2 or shape[-2] != heads) else shape[-1]
    tokens = total // (heads * dv)
    out = np.zeros(shape, dtype=np.float64)
    rc = _load().oracle_msr_epilogue(_ptr(y), _ptr(g), _ptr(out), tokens, heads, dv, float(eps),
                                     int(nthreads))
    assert rc == 0
    return out


def backward(q, k, v, dout, gamma, theta=None, pos0=0, flags=F_ALL & ~F_NORM_R, state_in=None, nthreads=0):
    """Gradient of the retention output O (with an optional state_in before the first token)
    with respect to q, k, v and state_in, given dO (product rule on the definition; no R~).

    Returns (dq, dk, dv, dstate) in fp64; dstate is None without state_in.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    b, L, h, dk = q.shape
    dv = v.shape[-1]
    gq, gk, gv = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    si = None if state_in is None else _f64(state_in)
    ds = None if state_in is None else np.zeros((b, h, dk, dv))
    g, th = _f64(gamma), _theta_arr(theta, dk)
    rc = _load().oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(gq), _ptr(gk), _ptr(gv), _dims(q, v),
                                 _ptr(g), _ptr(th), int(pos0), int(flags), _ptr(si), _ptr(ds), int(nthreads))
    assert rc == 0, "the oracle's gradient does not cover R~"
    return gq, gk, gv, ds
