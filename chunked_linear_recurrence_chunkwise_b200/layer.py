"""User-facing calls of the layer on torch tensors.

These allocate outputs and workspace with torch (device memory is the only
thing torch provides here) and call the C ABI through ``sf``; all arithmetic
runs in libsf's CUDA kernels.  Tensors: q, k ``[B, T, H, dk]``; v ``[B, T, H,
dv]`` (fp32 or bf16, contiguous, same device); g, beta ``[B, T, H]`` float32
or None; states ``[B, H, dk, dv]`` float32.
"""
from __future__ import annotations

import torch

from . import sf


def _ws(nbytes: int, device) -> torch.Tensor:
    if nbytes <= 0:
        raise sf.SfError(sf.SF_ERR_INVALID, "workspace size")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    ws[:min(nbytes, 256)].zero_()  # the device error word at its head starts clear
    return ws


def _check_inputs(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def forward(q, k, v, g=None, beta=None, S_in=None, lens=None, stream=None, aux_stream=None,
            ws=None):
    """Runs the layer forward.  Returns ``(o, S_out, S_saved)``.

    ``lens`` (list of ints summing to T) runs the sub-sequence driver and
    returns the state entering each piece in ``S_saved`` [n_sub, B, H, dk, dv];
    without it the whole sequence is one piece and ``S_saved`` is None.
    """
    _check_inputs(q, k, v, g, beta, S_in)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    sh = sf.shape_of(q, v)
    o = torch.empty_like(v)
    S_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    if lens is None:
        ws = _ws(sf.sf_workspace_bytes(sh, sf.SF_OP_FWD), q.device) if ws is None else ws
        sf.sf_fwd(sh, q, k, v, g, beta, S_in, o, S_out, ws, stream=stream)
        return o, S_out, None
    S_saved = torch.empty((len(lens), B, H, dk, dv), dtype=torch.float32, device=q.device)
    ws = _ws(sf.sf_seq_workspace_bytes(sh, lens, sf.SF_OP_FWD), q.device) if ws is None else ws
    sf.sf_fwd_seq(sh, lens, q, k, v, g, beta, S_in, o, S_out, S_saved, ws, stream_main=stream,
                  stream_aux=aux_stream)
    return o, S_out, S_saved


def backward(q, k, v, g, beta, dO, S_in=None, S_saved=None, dS_out=None, lens=None, stream=None,
             aux_stream=None, ws=None):
    """Gradients of the layer.  Returns a dict with dq, dk, dv, dg, dbeta, dS_in.

    Without ``lens`` the state entering the sequence is ``S_in``; with ``lens``
    the per-piece entering states ``S_saved`` from :func:`forward` are used.
    """
    _check_inputs(q, k, v, g, beta, dO, S_in, S_saved, dS_out)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    sh = sf.shape_of(q, v)
    dq = torch.empty_like(q)
    dk_ = torch.empty_like(k)
    dv_ = torch.empty_like(v)
    dg = None if g is None else torch.empty_like(g)
    db = None if beta is None else torch.empty_like(beta)
    dS_in = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    if lens is None:
        ws = _ws(sf.sf_workspace_bytes(sh, sf.SF_OP_BWD), q.device) if ws is None else ws
        sf.sf_bwd(sh, q, k, v, g, beta, S_in, dO, dS_out, dq, dk_, dv_, dg, db, dS_in, ws,
                  stream=stream)
    else:
        ws = _ws(sf.sf_seq_workspace_bytes(sh, lens, sf.SF_OP_BWD), q.device) if ws is None else ws
        sf.sf_bwd_seq(sh, lens, q, k, v, g, beta, S_saved, dO, dS_out, dq, dk_, dv_, dg, db, dS_in,
                      ws, stream_main=stream, stream_aux=aux_stream)
    return {"dq": dq, "dk": dk_, "dv": dv_, "dg": dg, "dbeta": db, "dS_in": dS_in}


def forward_keep(q, k, v, g=None, beta=None, S_in=None, lens=None, stream=None, aux_stream=None,
                 ws=None, keep=None):
    """Forward that keeps every piece's intermediates for :func:`backward_keep`
    (no activation recompute).  Returns ``(o, S_out, keep)``; ``lens`` defaults
    to one piece."""
    _check_inputs(q, k, v, g, beta, S_in)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    lens = [T] if lens is None else list(lens)
    sh = sf.shape_of(q, v)
    o = torch.empty_like(v)
    S_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    keep = _ws(sf.sf_keep_bytes(sh, lens), q.device) if keep is None else keep
    ws = _ws(sf.sf_seq_workspace_bytes(sh, lens, sf.SF_OP_FWD), q.device) if ws is None else ws
    sf.sf_fwd_seq_keep(sh, lens, q, k, v, g, beta, S_in, o, S_out, keep, ws, stream_main=stream,
                       stream_aux=aux_stream)
    return o, S_out, keep


def backward_keep(q, k, v, g, beta, dO, keep, dS_out=None, lens=None, stream=None, aux_stream=None,
                  ws=None):
    """Gradients from the intermediates :func:`forward_keep` kept (same inputs
    and ``lens``).  Returns a dict with dq, dk, dv, dg, dbeta, dS_in."""
    _check_inputs(q, k, v, g, beta, dO, dS_out)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    lens = [T] if lens is None else list(lens)
    sh = sf.shape_of(q, v)
    dq = torch.empty_like(q)
    dk_ = torch.empty_like(k)
    dv_ = torch.empty_like(v)
    dg = None if g is None else torch.empty_like(g)
    db = None if beta is None else torch.empty_like(beta)
    dS_in = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    ws = _ws(sf.sf_seq_workspace_bytes(sh, lens, sf.SF_OP_BWD), q.device) if ws is None else ws
    sf.sf_bwd_seq_keep(sh, lens, q, k, v, g, beta, keep, dO, dS_out, dq, dk_, dv_, dg, db, dS_in, ws,
                       stream_main=stream, stream_aux=aux_stream)
    return {"dq": dq, "dk": dk_, "dv": dv_, "dg": dg, "dbeta": db, "dS_in": dS_in}


def chunk_costs(timing: dict, steps: int, n_chunks: int, bh: int, sms: int, min_chunks=None):
    """Per-chunk kernel costs for the planner from a timing profile of the keep drivers.

    ``timing`` is ``sf.sf_timing_read()`` after ``steps`` fwd+bwd steps of the keep
    drivers run with both driver streams merged onto one stream, so that every kernel
    is timed alone.  The steps cover ``n_chunks`` 64-token chunks of ``bh`` heads
    (batch rows x heads).  The result holds microseconds per chunk of all heads.
    ``min_chunks`` defaults to the chunks whose kernels fill the GPU once at three
    CTAs per SM."""
    def us(prefix):
        return sum(v[1] for k_, v in timing.items() if k_.startswith(prefix)) * 1e3 / steps / n_chunks
    if min_chunks is None:
        min_chunks = -(-3 * sms // bh)
    return sf.chunk_costs(us("intra"), us("output"), us("grad") + us("dd_pre"),
                          us("state_fwd"), us("state_bwd"), sms, min_chunks)


def plan_cut(q, v, n_sub: int, costs) -> list:
    """The cut of q's sequence into ``n_sub`` pieces that ``sf.sf_plan_cut`` chooses for
    these costs (host computation; the tensors give the shape only)."""
    return sf.sf_plan_cut(sf.shape_of(q, v), n_sub, costs)
