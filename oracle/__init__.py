"""CPU fp64 oracle for Lightning Attention-2 -- test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never does, and shares no code with it.

The arithmetic lives in ``la2_oracle.c`` (plain C, double precision, OpenMP
over independent sequences); this module compiles it with gcc and marshals
numpy arrays.  See the C file's header for what each function computes and
which passage of the pages it follows.

Arrays are ``[..., T, d]`` (queries/keys) and ``[..., T, e]`` (values,
outputs); the leading dimensions index independent sequences and ``lam`` holds
one decay per sequence (same leading shape).  Inputs of any float dtype are
upcast to float64 exactly; results are float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "la2_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libla2oracle.so")

_lib = None

# Sequences handed to the C code per call; bounds the float64 copies held at once.
_CHUNK_BYTES = 1 << 30


def build(force: bool = False) -> str:
    """Compile la2_oracle.c into oracle/_build/libla2oracle.so (gcc, OpenMP)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        lib.la2o_forward.argtypes = [i, i, i, i, dp, dp, dp, dp, dp, i]
        lib.la2o_backward.argtypes = [i, i, i, i, dp, dp, dp, dp, dp, dp, dp, dp, i]
        lib.la2o_forward_blocked.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, i]
        lib.la2o_backward_blocked.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, dp, dp, dp, i]
        lib.la2o_forward_state.argtypes = [i, i, i, i, dp, dp, dp, dp, dp, dp, dp, i]
        lib.la2o_decode_step.argtypes = [i, i, i, dp, dp, dp, dp, dp, dp]
        lib.la2o_backward_state.argtypes = [i, i, i, i, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp,
                                            dp, i]
        lib.la2o_dlambda.argtypes = [i, i, i, i, dp, dp, dp, dp, dp, dp, dp, dp, i]
        lib.la2o_forward_norm.argtypes = [i, i, i, i, dp, dp, dp, dp, dp, dp, i]
        lib.la2o_backward_norm.argtypes = [i, i, i, i, dp, dp, dp, dp, dp, dp, dp, dp, i]
        lib.la2o_max_threads.restype = i
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().la2o_max_threads())


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor on the CPU
        x = x.detach().float().numpy() if str(x.dtype) == "torch.bfloat16" else x.detach().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _prep(q, k, v, lam, extra=()):
    q = np.asarray(q) if not hasattr(q, "detach") else q
    lead = tuple(q.shape[:-2])
    T, d = int(q.shape[-2]), int(q.shape[-1])
    e = int(v.shape[-1])
    ns = int(np.prod(lead)) if lead else 1
    lam = np.broadcast_to(np.asarray(lam, dtype=np.float64), lead).reshape(ns)
    return lead, ns, T, d, e, np.ascontiguousarray(lam)


def _chunks(ns, T, width):
    per = max(1, _CHUNK_BYTES // max(1, 8 * T * width))
    for s in range(0, ns, per):
        yield s, min(ns, s + per)


def forward(q, k, v, lam, nthreads: int = 0) -> np.ndarray:
    """o_t = sum_{s<=t} lam^(t-s) (q_t . k_s) v_s by the serial recurrence."""
    lib = _load()
    lead, ns, T, d, e, lam = _prep(q, k, v, lam)
    qf, kf, vf = (x.reshape(ns, T, -1) for x in (q, k, v))
    out = np.empty((ns, T, e), dtype=np.float64)
    for a, b in _chunks(ns, T, 2 * d + 2 * e):
        qc, kc, vc = _f64(qf[a:b]), _f64(kf[a:b]), _f64(vf[a:b])
        oc = np.empty((b - a, T, e), dtype=np.float64)
        lib.la2o_forward(b - a, T, d, e, _ptr(lam[a:b]), _ptr(qc), _ptr(kc), _ptr(vc),
                         _ptr(oc), int(nthreads))
        out[a:b] = oc
    return out.reshape(*lead, T, e)


def forward_state(q, k, v, lam, s0=None, nthreads: int = 0):
    """(o, S_T): the forward recurrence started from the state s0 ([..., d, e];
    None = zero) instead of zero, and the state after the last position."""
    lib = _load()
    lead, ns, T, d, e, lam = _prep(q, k, v, lam)
    qc, kc, vc = (_f64(x).reshape(ns, T, -1) for x in (q, k, v))
    out = np.empty((ns, T, e), dtype=np.float64)
    sT = np.empty((ns, d, e), dtype=np.float64)
    s0p = None
    if s0 is not None:
        s0c = _f64(s0).reshape(ns, d, e)
        s0p = _ptr(s0c)
    lib.la2o_forward_state(ns, T, d, e, _ptr(lam), _ptr(qc), _ptr(kc), _ptr(vc), s0p, _ptr(out),
                           _ptr(sT), int(nthreads))
    return out.reshape(*lead, T, e), sT.reshape(*lead, d, e)


def decode_step(q, k, v, lam, state):
    """(o, S'): one new token per sequence, q, k [..., d], v [..., e], state
    [..., d, e]: S' = lam S + k v^T, o = S'^T q.  The input state is not modified."""
    lib = _load()
    q, v = _f64(q), _f64(v)
    lead = tuple(q.shape[:-1])
    d, e = int(q.shape[-1]), int(v.shape[-1])
    ns = int(np.prod(lead)) if lead else 1
    lamv = np.ascontiguousarray(np.broadcast_to(np.asarray(lam, dtype=np.float64), lead).reshape(ns))
    qc, kc, vc = q.reshape(ns, d), _f64(k).reshape(ns, d), _f64(v).reshape(ns, e)
    S = _f64(state).reshape(ns, d, e).copy()
    o = np.empty((ns, e), dtype=np.float64)
    lib.la2o_decode_step(ns, d, e, _ptr(lamv), _ptr(qc), _ptr(kc), _ptr(vc), _ptr(S), _ptr(o))
    return o.reshape(*lead, e), S.reshape(*lead, d, e)


def backward(q, k, v, lam, dout, nthreads: int = 0):
    """(dq, dk, dv) of L = sum_t dout_t . o_t, by the forward and reverse sweeps."""
    lib = _load()
    lead, ns, T, d, e, lam = _prep(q, k, v, lam)
    qf, kf, vf, gf = (x.reshape(ns, T, -1) for x in (q, k, v, dout))
    dq = np.empty((ns, T, d)); dk = np.empty((ns, T, d)); dv = np.empty((ns, T, e))
    for a, b in _chunks(ns, T, 4 * d + 4 * e):
        qc, kc, vc, gc = _f64(qf[a:b]), _f64(kf[a:b]), _f64(vf[a:b]), _f64(gf[a:b])
        n = b - a
        dqc = np.empty((n, T, d)); dkc = np.empty((n, T, d)); dvc = np.empty((n, T, e))
        lib.la2o_backward(n, T, d, e, _ptr(lam[a:b]), _ptr(qc), _ptr(kc), _ptr(vc), _ptr(gc),
                          _ptr(dqc), _ptr(dkc), _ptr(dvc), int(nthreads))
        dq[a:b], dk[a:b], dv[a:b] = dqc, dkc, dvc
    return dq.reshape(*lead, T, d), dk.reshape(*lead, T, d), dv.reshape(*lead, T, e)


def backward_state(q, k, v, lam, dout, s0=None, dsT=None, nthreads: int = 0):
    """(dq, dk, dv, dS0) of L = sum_t dout_t . o_t + <dsT, S_{T-1}> for the
    forward started from the state s0 ([..., d, e]; None = zero); dsT is the
    gradient arriving at the final state (None = zero)."""
    lib = _load()
    lead, ns, T, d, e, lam = _prep(q, k, v, lam)
    qc, kc, vc, gc = (_f64(x).reshape(ns, T, w) for x, w in ((q, d), (k, d), (v, e), (dout, e)))
    dq = np.empty((ns, T, d)); dk = np.empty((ns, T, d)); dv = np.empty((ns, T, e))
    ds0 = np.empty((ns, d, e))
    s0a = _f64(s0).reshape(ns, d, e) if s0 is not None else None
    gTa = _f64(dsT).reshape(ns, d, e) if dsT is not None else None
    lib.la2o_backward_state(ns, T, d, e, _ptr(lam), _ptr(qc), _ptr(kc), _ptr(vc), _ptr(gc),
                            _ptr(s0a) if s0a is not None else None,
                            _ptr(gTa) if gTa is not None else None,
                            _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ds0), int(nthreads))
    return (dq.reshape(*lead, T, d), dk.reshape(*lead, T, d), dv.reshape(*lead, T, e),
            ds0.reshape(*lead, d, e))


def dlambda(q, k, v, lam, dout, s0=None, dsT=None, nthreads: int = 0):
    """dL/dlam per sequence ([...]) for L = sum_t dout_t . o_t + <dsT, S_{T-1}>,
    the forward started from s0 (None = zero, dsT None = zero)."""
    lib = _load()
    lead, ns, T, d, e, lam = _prep(q, k, v, lam)
    qc, kc, vc, gc = (_f64(x).reshape(ns, T, w) for x, w in ((q, d), (k, d), (v, e), (dout, e)))
    s0a = _f64(s0).reshape(ns, d, e) if s0 is not None else None
    gTa = _f64(dsT).reshape(ns, d, e) if dsT is not None else None
    out = np.empty(ns)
    lib.la2o_dlambda(ns, T, d, e, _ptr(lam), _ptr(qc), _ptr(kc), _ptr(vc), _ptr(gc),
                     _ptr(s0a) if s0a is not None else None,
                     _ptr(gTa) if gTa is not None else None, _ptr(out), int(nthreads))
    return out.reshape(lead)


def forward_norm(q, k, v, lam, nthreads: int = 0):
    """(y, den): the normalised form y_t = (S_t^T q_t) / (q_t . z_t) with
    z_t = lam z_{t-1} + k_t (identity feature map)."""
    lib = _load()
    lead, ns, T, d, e, lam = _prep(q, k, v, lam)
    qc, kc, vc = (_f64(x).reshape(ns, T, w) for x, w in ((q, d), (k, d), (v, e)))
    y = np.empty((ns, T, e))
    den = np.empty((ns, T))
    lib.la2o_forward_norm(ns, T, d, e, _ptr(lam), _ptr(qc), _ptr(kc), _ptr(vc), _ptr(y), _ptr(den),
                          int(nthreads))
    return y.reshape(*lead, T, e), den.reshape(*lead, T)


def backward_norm(q, k, v, lam, dy, nthreads: int = 0):
    """(dq, dk, dv) of L = sum_t dy_t . y_t for y = forward_norm(...)[0]."""
    lib = _load()
    lead, ns, T, d, e, lam = _prep(q, k, v, lam)
    qc, kc, vc, gc = (_f64(x).reshape(ns, T, w) for x, w in ((q, d), (k, d), (v, e), (dy, e)))
    dq = np.empty((ns, T, d)); dk = np.empty((ns, T, d)); dv = np.empty((ns, T, e))
    lib.la2o_backward_norm(ns, T, d, e, _ptr(lam), _ptr(qc), _ptr(kc), _ptr(vc), _ptr(gc),
                           _ptr(dq), _ptr(dk), _ptr(dv), int(nthreads))
    return dq.reshape(*lead, T, d), dk.reshape(*lead, T, d), dv.reshape(*lead, T, e)


def forward_blocked(q, k, v, lam, block: int, nthreads: int = 0) -> np.ndarray:
    """The tiled forward (intra masked product + inter state product + carry)."""
    lib = _load()
    lead, ns, T, d, e, lam = _prep(q, k, v, lam)
    qc, kc, vc = (_f64(x).reshape(ns, T, -1) for x in (q, k, v))
    out = np.empty((ns, T, e), dtype=np.float64)
    lib.la2o_forward_blocked(ns, T, d, e, int(block), _ptr(lam), _ptr(qc), _ptr(kc), _ptr(vc),
                             _ptr(out), int(nthreads))
    return out.reshape(*lead, T, e)


def backward_blocked(q, k, v, lam, dout, block: int, nthreads: int = 0):
    """The tiled backward: dq by a forward scan, dk and dv by reverse scans."""
    lib = _load()
    lead, ns, T, d, e, lam = _prep(q, k, v, lam)
    qc, kc, vc, gc = (_f64(x).reshape(ns, T, -1) for x in (q, k, v, dout))
    dq = np.empty((ns, T, d)); dk = np.empty((ns, T, d)); dv = np.empty((ns, T, e))
    lib.la2o_backward_blocked(ns, T, d, e, int(block), _ptr(lam), _ptr(qc), _ptr(kc), _ptr(vc),
                              _ptr(gc), _ptr(dq), _ptr(dk), _ptr(dv), int(nthreads))
    return dq.reshape(*lead, T, d), dk.reshape(*lead, T, d), dv.reshape(*lead, T, e)
