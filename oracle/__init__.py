"""fp64 CPU oracle for the chunkwise linear-recurrence layer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the product library never
does.  It shares no code with the CUDA path.

The arithmetic lives in ``sf_oracle.c`` (a token-by-token fp64 loop, see its
header for the recurrence and the hand-derived backward).  This module only
compiles it with gcc, loads it with ctypes and marshals numpy arrays.

Layouts: q, k ``[B, T, H, dk]``; v, o ``[B, T, H, dv]``; g, beta ``[B, T, H]``;
states ``[B, H, dk, dv]``.  ``g=None`` means no decay (a_t = 1); ``beta=None``
means plain linear attention (no delta term).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sf_oracle.c")
_LIB = os.path.join(_HERE, "libsf_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile sf_oracle.c into libsf_oracle.so next to it (gcc, -O3, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c99", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        # SF_ORACLE_LIB: a build of a deliberately altered sf_oracle.c, which the tests
        # that plant a mistake load to check that the pins catch it
        path = os.environ.get("SF_ORACLE_LIB")
        if not path:
            path = build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.sfo_fwd.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, P, I]
        lib.sfo_fwd.restype = I
        lib.sfo_bwd.argtypes = [I, I, I, I, I] + [P] * 14 + [I, I]
        lib.sfo_bwd.restype = I
        lib.sfo_max_threads.argtypes = []
        lib.sfo_max_threads.restype = I
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().sfo_max_threads())


def _c64(x):
    if x is None:
        return None
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x):
    return None if x is None else x.ctypes.data


def _dims(q, v):
    B, T, H, dk = q.shape
    dv = v.shape[3]
    return B, T, H, dk, dv


def fwd(q, k, v, g=None, beta=None, S_in=None, nthreads: int | None = None):
    """Token-loop forward.  Returns ``(o, S_out)`` in fp64."""
    lib = _load()
    q, k, v, g, beta, S_in = map(_c64, (q, k, v, g, beta, S_in))
    B, T, H, dk, dv = _dims(q, v)
    assert k.shape == (B, T, H, dk) and v.shape == (B, T, H, dv)
    if g is not None:
        assert g.shape == (B, T, H)
    if beta is not None:
        assert beta.shape == (B, T, H)
    if S_in is not None:
        assert S_in.shape == (B, H, dk, dv)
    o = np.zeros((B, T, H, dv), np.float64)
    S_out = np.zeros((B, H, dk, dv), np.float64)
    nt = nthreads or max_threads()
    rc = lib.sfo_fwd(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S_in),
                     _ptr(o), _ptr(S_out), nt)
    if rc != 0:
        raise ValueError("oracle fwd rejected its arguments")
    return o, S_out


def bwd(q, k, v, g, beta, S_in, dO, dS_out=None, nthreads: int | None = None, seg: int = 64):
    """Hand-derived reverse of the token loop.

    Returns a dict with ``dq, dk, dv, dg, dbeta, dS_in`` (``dg``/``dbeta`` are
    None when ``g``/``beta`` are None).
    """
    lib = _load()
    q, k, v, g, beta, S_in, dO, dS_out = map(_c64, (q, k, v, g, beta, S_in, dO, dS_out))
    B, T, H, dk, dv = _dims(q, v)
    assert dO.shape == (B, T, H, dv)
    dq = np.zeros_like(q)
    dk_ = np.zeros_like(k)
    dv_ = np.zeros_like(v)
    dg = None if g is None else np.zeros((B, T, H), np.float64)
    db = None if beta is None else np.zeros((B, T, H), np.float64)
    dS_in = np.zeros((B, H, dk, dv), np.float64)
    nt = nthreads or max_threads()
    rc = lib.sfo_bwd(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S_in),
                     _ptr(dO), _ptr(dS_out), _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dg), _ptr(db),
                     _ptr(dS_in), seg, nt)
    if rc != 0:
        raise ValueError("oracle bwd rejected its arguments")
    return {"dq": dq, "dk": dk_, "dv": dv_, "dg": dg, "dbeta": db, "dS_in": dS_in}


def fwd_seq(lens, q, k, v, g=None, beta=None, S_in=None, nthreads=None):
    """Run the oracle sub-sequence by sub-sequence, carrying the state.

    This is the Sequence Accumulation schedule ("Sequence Accumulation and
    Beyond", Approach): sub-sequences one after another, the state of one the
    initial state of the next.  Returns ``(o, S_out, S_saved)`` where
    ``S_saved[i]`` is the state entering sub-sequence i.
    """
    B, T, H, dk, dv = _dims(np.asarray(q), np.asarray(v))
    assert sum(lens) == T
    S = np.zeros((B, H, dk, dv)) if S_in is None else np.array(S_in, np.float64)
    outs, saved, t0 = [], [], 0
    for L in lens:
        sl = slice(t0, t0 + L)
        saved.append(S.copy())
        o, S = fwd(q[:, sl], k[:, sl], v[:, sl], None if g is None else g[:, sl],
                   None if beta is None else beta[:, sl], S, nthreads)
        outs.append(o)
        t0 += L
    return np.concatenate(outs, axis=1), S, saved


def bwd_seq(lens, q, k, v, g, beta, S_saved, dO, dS_out=None, nthreads=None):
    """Backward sub-sequence by sub-sequence in reverse, carrying dS."""
    B, T, H, dk, dv = _dims(np.asarray(q), np.asarray(v))
    starts = np.cumsum([0] + list(lens))
    dS = None if dS_out is None else np.array(dS_out, np.float64)
    parts = [None] * len(lens)
    for i in reversed(range(len(lens))):
        sl = slice(int(starts[i]), int(starts[i + 1]))
        r = bwd(q[:, sl], k[:, sl], v[:, sl], None if g is None else g[:, sl],
                None if beta is None else beta[:, sl], S_saved[i], dO[:, sl], dS, nthreads)
        parts[i] = r
        dS = r["dS_in"]
    out = {}
    for key in ("dq", "dk", "dv", "dg", "dbeta"):
        out[key] = None if parts[0][key] is None else np.concatenate([p[key] for p in parts], axis=1)
    out["dS_in"] = dS
    return out
