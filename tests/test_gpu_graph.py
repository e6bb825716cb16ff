"""The sub-sequence drivers captured into a CUDA graph (stream capture of their main
stream; the aux and critical streams join the capture through the drivers' event
waits) replay the same kernels: the replayed step's outputs equal the eagerly launched
step's bit for bit, step after step, and the replay also matches the fp64 oracle."""
import zlib

import pytest
import torch

import oracle
from test_gpu_parity import TOL, make_case, rel_l2, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    ("bf16", 128, 128, [64, 100, 45], True),   # tensor-core path, keep drivers, ragged pieces
    ("bf16", 128, 128, [64] * 5 + [17], False),  # recompute drivers, more pieces than slots
    ("f32", 64, 64, [64, 100], True),           # SIMT path
]


@pytest.mark.parametrize("dtype,d,_d,lens,keep", CASES)
def test_graph_replay_equals_eager(dtype, d, _d, lens, keep):
    from chunked_linear_recurrence_chunkwise_b200 import sf
    from chunked_linear_recurrence_chunkwise_b200.layer import _ws
    B, T, H = 2, sum(lens), 2
    seed = zlib.crc32(repr((dtype, d, tuple(lens), keep)).encode()) % 997
    c = make_case(seed, B, T, H, d, d, True, True, dtype)
    x = to_dev(c, dtype)
    sh = sf.shape_of(x["q"], x["v"])
    dev = x["q"].device
    ws_f = _ws(sf.sf_seq_workspace_bytes(sh, lens, sf.SF_OP_FWD), dev)
    ws_b = _ws(sf.sf_seq_workspace_bytes(sh, lens, sf.SF_OP_BWD), dev)
    kept = _ws(sf.sf_keep_bytes(sh, lens), dev) if keep else None
    S_saved = torch.empty((len(lens), B, H, d, d), dtype=torch.float32, device=dev)
    outs = {"o": torch.empty_like(x["v"]), "S_out": torch.empty((B, H, d, d), device=dev),
            "dq": torch.empty_like(x["q"]), "dk": torch.empty_like(x["k"]), "dv": torch.empty_like(x["v"]),
            "dg": torch.empty_like(x["g"]), "db": torch.empty_like(x["beta"]),
            "dS_in": torch.empty((B, H, d, d), device=dev)}
    aux = torch.cuda.Stream()

    def step(sm):
        if keep:
            sf.sf_fwd_seq_keep(sh, lens, x["q"], x["k"], x["v"], x["g"], x["beta"], x["S_in"], outs["o"],
                               outs["S_out"], kept, ws_f, stream_main=sm, stream_aux=aux)
            sf.sf_bwd_seq_keep(sh, lens, x["q"], x["k"], x["v"], x["g"], x["beta"], kept, x["dO"],
                               x["dS_out"], outs["dq"], outs["dk"], outs["dv"], outs["dg"], outs["db"],
                               outs["dS_in"], ws_b, stream_main=sm, stream_aux=aux)
        else:
            sf.sf_fwd_seq(sh, lens, x["q"], x["k"], x["v"], x["g"], x["beta"], x["S_in"], outs["o"],
                          outs["S_out"], S_saved, ws_f, stream_main=sm, stream_aux=aux)
            sf.sf_bwd_seq(sh, lens, x["q"], x["k"], x["v"], x["g"], x["beta"], S_saved, x["dO"],
                          x["dS_out"], outs["dq"], outs["dk"], outs["dv"], outs["dg"], outs["db"],
                          outs["dS_in"], ws_b, stream_main=sm, stream_aux=aux)

    main = torch.cuda.Stream()
    step(main)  # eager first: creates the drivers' critical stream before any capture
    torch.cuda.synchronize()
    eager = {k: v.clone() for k, v in outs.items()}
    for v in outs.values():
        v.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=cap):
        step(cap)
    for _ in range(2):
        for v in outs.values():
            v.fill_(float("nan"))
        with torch.cuda.stream(main):
            g.replay()
        torch.cuda.synchronize()
        for k in outs:
            assert torch.equal(outs[k], eager[k]), f"{k}: graph replay differs from the eager step"
    sf.sf_check(ws_f)
    sf.sf_check(ws_b)
    # and the replay is the layer: against the fp64 oracle
    o_ref, S_ref, saved_ref = oracle.fwd_seq(lens, c["q"], c["k"], c["v"], c["g"], c["beta"], c["S_in"])
    r = oracle.bwd_seq(lens, c["q"], c["k"], c["v"], c["g"], c["beta"], saved_ref, c["dO"], c["dS_out"])
    tol = TOL[dtype]
    assert rel_l2(outs["o"].float().cpu().numpy(), o_ref) <= tol
    assert rel_l2(outs["dk"].float().cpu().numpy(), r["dk"]) <= tol
    assert rel_l2(outs["dS_in"].cpu().numpy(), r["dS_in"]) <= tol
