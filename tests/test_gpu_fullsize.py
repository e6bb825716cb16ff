"""GPU parity at the workloads' full sizes, in the launch configuration bench.py
times (sub-sequence driver, two streams, the workload's cut).

Every output of two sampled heads (first and last (batch, head)) is compared
element by element with the fp64 oracle run over the whole sequence of those
heads (relative L2 per tensor: 1e-4 fp32, 2e-2 bf16).  The nonuniform-cut
workload must also equal the single pass over the whole sequence.
"""
import numpy as np
import pytest
import torch

import oracle
from chunked_linear_recurrence_chunkwise_b200 import inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_l2(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (n if n > 0 else 1.0))


def run_gpu(w, x, lens, stream_aux=True, keep=False):
    """The workload through the sub-sequence drivers: with activation recompute
    (keep=False) or with the forward's intermediates kept for the backward."""
    from chunked_linear_recurrence_chunkwise_b200 import layer
    aux = torch.cuda.Stream() if stream_aux else None
    if keep:
        o, S_out, kept = layer.forward_keep(x["q"], x["k"], x["v"], x["g"], x["beta"], lens=lens,
                                            aux_stream=aux)
    else:
        o, S_out, S_saved = layer.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], lens=lens,
                                          aux_stream=aux)
    gr = None
    if x["dO"] is not None:
        if keep:
            gr = layer.backward_keep(x["q"], x["k"], x["v"], x["g"], x["beta"], x["dO"], kept,
                                     lens=lens, aux_stream=aux)
        else:
            gr = layer.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["dO"], S_saved=S_saved,
                                lens=lens, aux_stream=aux)
    torch.cuda.synchronize()
    return o, S_out, gr


def sampled(t, heads, has_batch=True):
    """[B, T, H, ...] (or [B, H, ...] states) -> numpy of the sampled (b, h) pairs."""
    outs = []
    for b, h in heads:
        outs.append(t[b, :, h].float().cpu().numpy() if has_batch else t[b, h].float().cpu().numpy())
    return outs


# every workload with activation recompute; the kept-intermediates drivers (the
# bench's configuration) on the gated-delta-rule workloads
CASES = [(name, False) for name in inputs.WORKLOADS] + [
    (name, True) for name in inputs.WORKLOADS if inputs.WORKLOADS[name].variant == "gdn"]


@pytest.mark.parametrize("name,keep", CASES)
def test_full_size_sampled_heads_match_oracle(name, keep):
    w = inputs.WORKLOADS[name]
    lens = inputs.sub_lengths(w)
    heads = [(0, 0), (w.B - 1, w.H - 1)]
    x = inputs.to_torch(w, device="cuda", keep_heads=heads)
    o, S_out, gr = run_gpu(w, x, lens, keep=keep)
    tol = TOL[w.dtype]
    # both sampled heads as a batch of two single-head problems (the oracle runs them in parallel)
    cat = lambda key: (None if x["kept"][0][key] is None
                       else np.concatenate([kh[key] for kh in x["kept"]], axis=0))
    q, k, v, g, beta, dO = (cat(key) for key in ("q", "k", "v", "g", "beta", "dO"))
    o_ref, S_ref = oracle.fwd(q, k, v, g, beta)
    r = oracle.bwd(q, k, v, g, beta, None, dO) if gr is not None else None
    for i, (b, h) in enumerate(heads):
        errs = {"o": rel_l2(o[b, :, h].float().cpu().numpy(), o_ref[i, :, 0]),
                "S_out": rel_l2(S_out[b, h].cpu().numpy(), S_ref[i, 0])}
        if gr is not None:
            for key in ("dq", "dk", "dv"):
                errs[key] = rel_l2(gr[key][b, :, h].float().cpu().numpy(), r[key][i, :, 0])
            for key in ("dg", "dbeta"):
                if r[key] is not None:
                    errs[key] = rel_l2(gr[key][b, :, h].cpu().numpy(), r[key][i, :, 0])
            errs["dS_in"] = rel_l2(gr["dS_in"][b, h].cpu().numpy(), r["dS_in"][i, 0])
        bad = {k_: e for k_, e in errs.items() if not e <= tol}
        assert not bad, f"{name} head ({b},{h}): rel-L2 above {tol}: {bad} (all {errs})"


def test_nonuniform_cut_equals_single_pass():
    """The Dirichlet cut into 12 pieces gives the single-pass result (full size)."""
    w = inputs.WORKLOADS["gated_deltanet_bf16_h16_t256k_dirichlet12"]
    lens = inputs.sub_lengths(w)
    assert len(set(lens)) > 1
    x = inputs.to_torch(w, device="cuda")
    o1, S1, g1 = run_gpu(w, x, [w.T], stream_aux=False)
    o2, S2, g2 = run_gpu(w, x, lens)

    def rel(a, b):
        a = a.double()
        b = b.double()
        return float(torch.linalg.norm(a - b) / torch.linalg.norm(b))

    errs = {"o": rel(o2, o1), "S_out": rel(S2, S1)}
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dS_in"):
        errs[key] = rel(g2[key], g1[key])
    bad = {k_: e for k_, e in errs.items() if not e <= 1e-5}
    assert not bad, f"cut vs single pass: {bad} (all {errs})"
