"""Thin ctypes binding of libsf (the C ABI in include/sf.h), same entry-point names.

Argument marshalling only: tensors are passed as raw device pointers, streams
as raw ``cudaStream_t`` handles.  Every step of the layer runs in the CUDA
library; there is no fallback.  Importing this module loads ``lib/libsf.so``
and raises if it has not been built
(``python -m chunked_linear_recurrence_chunkwise_b200.build``).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libsf.so")

SF_OK, SF_ERR_INVALID, SF_ERR_UNSUPPORTED, SF_ERR_WORKSPACE, SF_ERR_CUDA, SF_ERR_TIMEOUT = range(6)
SF_F32, SF_BF16 = 0, 1
SF_OP_FWD, SF_OP_BWD = 0, 1


class sf_shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "T", "H", "dk", "dv", "chunk", "dtype", "ld_t")]


class sf_chunk_costs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_double) for n in ("intra_us", "output_us", "grad_us", "state_fwd_us",
                                               "state_bwd_us")] + [("sms", ctypes.c_int),
                                                                   ("min_chunks", ctypes.c_int)]


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libsf.so is not built ({LIB_PATH}); run "
                      "`python -m chunked_linear_recurrence_chunkwise_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
_S = ctypes.c_size_t
_SP = ctypes.POINTER(sf_shape)
_IP = ctypes.POINTER(ctypes.c_int)

_SIGS = {
    "sf_workspace_bytes": (_S, [_SP, _I]),
    "sf_seq_workspace_bytes": (_S, [_SP, _I, _IP, _I]),
    "sf_fwd": (_I, [_SP] + [_P] * 8 + [_P, _S, _P]),
    "sf_bwd": (_I, [_SP] + [_P] * 14 + [_P, _S, _P]),
    "sf_fwd_seq": (_I, [_SP, _I, _IP] + [_P] * 9 + [_P, _S, _P, _P]),
    "sf_bwd_seq": (_I, [_SP, _I, _IP] + [_P] * 14 + [_P, _S, _P, _P]),
    "sf_keep_bytes": (_S, [_SP, _I, _IP]),
    "sf_fwd_seq_keep": (_I, [_SP, _I, _IP] + [_P] * 8 + [_P, _S, _P, _S, _P, _P]),
    "sf_bwd_seq_keep": (_I, [_SP, _I, _IP] + [_P] * 5 + [_P, _S] + [_P] * 8 + [_P, _S, _P, _P]),
    "sf_fwd_noalloc": (_I, [_SP] + [_P] * 8 + [_P]),
    "sf_check_noalloc": (_I, [_P]),
    "sf_check": (_I, [_P, _P]),
    "sf_status_string": (ctypes.c_char_p, [_I]),
    "sf_timing_enable": (None, [_I]),
    "sf_timing_reset": (None, []),
    "sf_timing_read": (_I, [_I, ctypes.POINTER(ctypes.c_char_p), _IP,
                            ctypes.POINTER(ctypes.c_double)]),
    "sf_timing_trace": (_I, [_I, _IP, _IP, ctypes.POINTER(ctypes.c_double),
                             ctypes.POINTER(ctypes.c_double)]),
    "sf_model_seq_us": (ctypes.c_double, [_SP, _I, _IP, ctypes.POINTER(sf_chunk_costs)]),
    "sf_plan_cut": (_I, [_SP, _I, ctypes.POINTER(sf_chunk_costs), _IP]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTS = tuple(_SIGS)


class SfError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {sf_status_string(status)} (status {status})")


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int, what: str):
    if status != SF_OK:
        raise SfError(status, what)


def _lens(lens):
    arr = (ctypes.c_int * len(lens))(*[int(x) for x in lens])
    return arr


def sf_status_string(status: int) -> str:
    return _lib.sf_status_string(int(status)).decode()


def shape(B, T, H, dk, dv, dtype, ld_t=0, chunk=64) -> sf_shape:
    return sf_shape(B, T, H, dk, dv, chunk, dtype, ld_t)


def shape_of(q, v, ld_t=0) -> sf_shape:
    """sf_shape for token-major tensors q [B, T, H, dk] and v [B, T, H, dv]."""
    import torch
    B, T, H, dk = q.shape
    dt = SF_BF16 if q.dtype == torch.bfloat16 else SF_F32
    return shape(B, T, H, dk, v.shape[3], dt, ld_t)


def sf_workspace_bytes(sh: sf_shape, op: int) -> int:
    return int(_lib.sf_workspace_bytes(ctypes.byref(sh), op))


def sf_seq_workspace_bytes(sh: sf_shape, lens, op: int) -> int:
    return int(_lib.sf_seq_workspace_bytes(ctypes.byref(sh), len(lens), _lens(lens), op))


def sf_fwd(sh, q, k, v, g, beta, S_in, o, S_out, ws, ws_bytes=None, stream=None):
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.sf_fwd(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S_in),
                       _ptr(o), _ptr(S_out), _ptr(ws), ws_bytes, _stream(stream)), "sf_fwd")


def sf_bwd(sh, q, k, v, g, beta, S_in, dO, dS_out, dq, dk, dv, dg, dbeta, dS_in, ws,
           ws_bytes=None, stream=None):
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.sf_bwd(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S_in),
                       _ptr(dO), _ptr(dS_out), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dbeta),
                       _ptr(dS_in), _ptr(ws), ws_bytes, _stream(stream)), "sf_bwd")


def sf_fwd_seq(sh, lens, q, k, v, g, beta, S_in, o, S_out, S_saved, ws, ws_bytes=None,
               stream_main=None, stream_aux=None):
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    sm = _stream(stream_main)
    sa = sm if stream_aux is None else _stream(stream_aux)
    _check(_lib.sf_fwd_seq(ctypes.byref(sh), len(lens), _lens(lens), _ptr(q), _ptr(k), _ptr(v),
                           _ptr(g), _ptr(beta), _ptr(S_in), _ptr(o), _ptr(S_out), _ptr(S_saved),
                           _ptr(ws), ws_bytes, sm, sa), "sf_fwd_seq")


def sf_bwd_seq(sh, lens, q, k, v, g, beta, S_saved, dO, dS_out, dq, dk, dv, dg, dbeta, dS_in, ws,
               ws_bytes=None, stream_main=None, stream_aux=None):
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    sm = _stream(stream_main)
    sa = sm if stream_aux is None else _stream(stream_aux)
    _check(_lib.sf_bwd_seq(ctypes.byref(sh), len(lens), _lens(lens), _ptr(q), _ptr(k), _ptr(v),
                           _ptr(g), _ptr(beta), _ptr(S_saved), _ptr(dO), _ptr(dS_out), _ptr(dq),
                           _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dbeta), _ptr(dS_in), _ptr(ws),
                           ws_bytes, sm, sa), "sf_bwd_seq")


def sf_keep_bytes(sh: sf_shape, lens) -> int:
    return int(_lib.sf_keep_bytes(ctypes.byref(sh), len(lens), _lens(lens)))


def sf_fwd_seq_keep(sh, lens, q, k, v, g, beta, S_in, o, S_out, keep, ws, keep_bytes=None,
                    ws_bytes=None, stream_main=None, stream_aux=None):
    keep_bytes = keep.numel() * keep.element_size() if keep_bytes is None else keep_bytes
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    sm = _stream(stream_main)
    sa = sm if stream_aux is None else _stream(stream_aux)
    _check(_lib.sf_fwd_seq_keep(ctypes.byref(sh), len(lens), _lens(lens), _ptr(q), _ptr(k), _ptr(v),
                                _ptr(g), _ptr(beta), _ptr(S_in), _ptr(o), _ptr(S_out), _ptr(keep),
                                keep_bytes, _ptr(ws), ws_bytes, sm, sa), "sf_fwd_seq_keep")


def sf_bwd_seq_keep(sh, lens, q, k, v, g, beta, keep, dO, dS_out, dq, dk, dv, dg, dbeta, dS_in, ws,
                    keep_bytes=None, ws_bytes=None, stream_main=None, stream_aux=None):
    keep_bytes = keep.numel() * keep.element_size() if keep_bytes is None else keep_bytes
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    sm = _stream(stream_main)
    sa = sm if stream_aux is None else _stream(stream_aux)
    _check(_lib.sf_bwd_seq_keep(ctypes.byref(sh), len(lens), _lens(lens), _ptr(q), _ptr(k), _ptr(v),
                                _ptr(g), _ptr(beta), _ptr(keep), keep_bytes, _ptr(dO), _ptr(dS_out),
                                _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dbeta), _ptr(dS_in),
                                _ptr(ws), ws_bytes, sm, sa), "sf_bwd_seq_keep")


def sf_fwd_noalloc(sh, q, k, v, g, beta, S_in, o, S_out, stream=None):
    """sf_fwd with the library's built-in scratch instead of a caller workspace."""
    _check(_lib.sf_fwd_noalloc(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                               _ptr(S_in), _ptr(o), _ptr(S_out), _stream(stream)), "sf_fwd_noalloc")


def sf_check_noalloc(stream=None):
    """sf_check for sf_fwd_noalloc: the built-in scratch array's error word."""
    _check(_lib.sf_check_noalloc(_stream(stream)), "sf_check_noalloc")


def sf_check(ws, stream=None):
    _check(_lib.sf_check(_ptr(ws), _stream(stream)), "sf_check")


def sf_timing_enable(on: bool):
    _lib.sf_timing_enable(1 if on else 0)


def sf_timing_reset():
    _lib.sf_timing_reset()


def sf_timing_read() -> dict:
    """{kernel name: (launches, total ms)} accumulated since the last reset."""
    cap = 32
    names = (ctypes.c_char_p * cap)()
    launches = (ctypes.c_int * cap)()
    ms = (ctypes.c_double * cap)()
    n = _lib.sf_timing_read(cap, names, launches, ms)
    return {names[i].decode(): (launches[i], ms[i]) for i in range(n)}


def sf_timing_trace(cap: int = 4096) -> list:
    """[(kernel kind index, stream index, start ms, end ms)] of the recorded launches."""
    kinds = (ctypes.c_int * cap)()
    streams = (ctypes.c_int * cap)()
    t0 = (ctypes.c_double * cap)()
    t1 = (ctypes.c_double * cap)()
    n = _lib.sf_timing_trace(cap, kinds, streams, t0, t1)
    return [(kinds[i], streams[i], t0[i], t1[i]) for i in range(n)]


def raw_call(name: str, *args):
    """Calls a C entry point with already-marshalled arguments (tests of the error paths)."""
    return getattr(_lib, name)(*args)


def chunk_costs(intra_us, output_us, grad_us, state_fwd_us, state_bwd_us, sms,
                min_chunks=0) -> sf_chunk_costs:
    """Per-chunk kernel costs (microseconds for one 64-token chunk of all heads) for the planner."""
    return sf_chunk_costs(float(intra_us), float(output_us), float(grad_us), float(state_fwd_us),
                          float(state_bwd_us), int(sms), int(min_chunks))


def sf_model_seq_us(sh: sf_shape, lens, costs: sf_chunk_costs) -> float:
    us = float(_lib.sf_model_seq_us(ctypes.byref(sh), len(lens), _lens(lens), ctypes.byref(costs)))
    if us < 0:
        raise SfError(SF_ERR_INVALID, "sf_model_seq_us")
    return us


def sf_plan_cut(sh: sf_shape, n_sub: int, costs: sf_chunk_costs) -> list:
    out = (ctypes.c_int * int(n_sub))()
    _check(_lib.sf_plan_cut(ctypes.byref(sh), int(n_sub), ctypes.byref(costs), out), "sf_plan_cut")
    return [int(x) for x in out]
