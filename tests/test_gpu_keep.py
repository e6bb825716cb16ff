"""GPU parity of the sub-sequence drivers that keep the forward's intermediates
for the backward (no activation recompute), through the C ABI.

Against the fp64 oracle element by element (relative L2 per tensor: 1e-4 fp32,
2e-2 bf16), over cuts with ragged pieces and every variant; and against the
recompute drivers on the same inputs, whose backward reads the same
intermediates recomputed: the gradients must agree to 1e-5 (fp32) and to
within the bf16 tolerance of each other's arithmetic (bf16).
"""
import numpy as np
import pytest
import torch

import oracle
from test_gpu_parity import TOL, VARIANTS, host, make_case, rel_l2, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layer():
    from chunked_linear_recurrence_chunkwise_b200 import layer as L
    return L


CASES = [
    # (dtype, dk, dv, lens): tensor-core path (bf16, d = 128) and SIMT paths
    ("bf16", 128, 128, [64, 100, 45]),
    ("bf16", 128, 128, [1, 64, 128, 16]),
    ("bf16", 128, 128, [64] * 9 + [100]),  # more pieces than workspace slots
    # long pieces (dozens of chunks per state pass), a ragged last chunk; one piece
    ("bf16", 128, 128, [64, 2048 + 17]),
    ("bf16", 128, 128, [4096 + 3 * 64]),
    ("bf16", 64, 64, [130, 70]),
    ("f32", 64, 64, [64, 100, 45]),
    ("f32", 128, 128, [200]),
]


@pytest.mark.parametrize("has_g,has_beta", VARIANTS)
@pytest.mark.parametrize("dtype,dk,dv,lens", CASES)
def test_keep_drivers_match_oracle(layer, dtype, dk, dv, lens, has_g, has_beta):
    B, T, H = 2, sum(lens), 2
    c = make_case(hash((dtype, dk, tuple(lens), has_g, has_beta)) % 997, B, T, H, dk, dv, has_g,
                  has_beta, dtype)
    d = to_dev(c, dtype)
    aux = torch.cuda.Stream()
    o, S_out, kept = layer.forward_keep(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"],
                                        lens=lens, aux_stream=aux)
    gr = layer.backward_keep(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], kept,
                             dS_out=d["dS_out"], lens=lens, aux_stream=aux)
    torch.cuda.synchronize()
    o_ref, S_ref, saved_ref = oracle.fwd_seq(lens, c["q"], c["k"], c["v"], c["g"], c["beta"],
                                             c["S_in"])
    g_ref = oracle.bwd_seq(lens, c["q"], c["k"], c["v"], c["g"], c["beta"], saved_ref, c["dO"],
                           c["dS_out"])
    tol = TOL[dtype]
    errs = {"o": rel_l2(host(o), o_ref), "S_out": rel_l2(host(S_out), S_ref)}
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dS_in"):
        if g_ref[key] is None:
            assert gr[key] is None
        else:
            errs[key] = rel_l2(host(gr[key]), g_ref[key])
    bad = {k_: e for k_, e in errs.items() if not e <= tol}
    assert not bad, f"rel-L2 above {tol}: {bad} (all: {errs})"


@pytest.mark.parametrize("dtype,dk,dv,lens", CASES)
def test_keep_equals_recompute(layer, dtype, dk, dv, lens):
    """Keeping the intermediates changes where they come from, not the gradients."""
    B, T, H = 1, sum(lens), 2
    c = make_case(23, B, T, H, dk, dv, True, True, dtype)
    d = to_dev(c, dtype)
    o1, S1, saved = layer.forward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], lens=lens)
    g1 = layer.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], S_saved=saved,
                        dS_out=d["dS_out"], lens=lens)
    o2, S2, kept = layer.forward_keep(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"],
                                      lens=lens)
    g2 = layer.backward_keep(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], kept,
                             dS_out=d["dS_out"], lens=lens)
    torch.cuda.synchronize()
    tol = 1e-5 if dtype == "f32" else TOL[dtype]
    assert rel_l2(host(o2), host(o1)) <= tol
    assert rel_l2(host(S2), host(S1)) <= tol
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dS_in"):
        assert rel_l2(host(g2[key]), host(g1[key])) <= tol, key


def test_keep_backward_is_repeatable(layer):
    """The backward only reads the kept buffer: running it twice gives the same bits."""
    lens = [64, 100, 45]
    c = make_case(31, 1, sum(lens), 2, 128, 128, True, True, "bf16")
    d = to_dev(c, "bf16")
    _, _, kept = layer.forward_keep(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], lens=lens)
    g1 = layer.backward_keep(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], kept, lens=lens)
    g2 = layer.backward_keep(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], kept, lens=lens)
    torch.cuda.synchronize()
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dS_in"):
        assert torch.equal(g1[key], g2[key]), key
    assert np.isfinite(host(g1["dq"])).all()


def test_planned_cut_gives_the_single_pass_result(layer):
    """The profile-guided cut (sf_plan_cut) is a cut like any other: the keep
    drivers on it give the single-pass result (fp32 state carry, chunk-aligned
    cuts: to 1e-5 on the bf16 tensor-core path, as for any cut)."""
    from chunked_linear_recurrence_chunkwise_b200 import sf
    B, T, H = 1, 2560 + 17, 4
    c = make_case(41, B, T, H, 128, 128, True, True, "bf16")
    d = to_dev(c, "bf16")
    sh = sf.shape_of(d["q"], d["v"])
    costs = sf.chunk_costs(65.7 / 64, 38.5 / 64, 160.4 / 64, 106.9 / 64, 136.1 / 64, 148, 2)
    plan = sf.sf_plan_cut(sh, 5, costs)
    assert len(set(plan)) > 1 and sum(plan) == T
    aux = torch.cuda.Stream()
    res = []
    for lens in ([T], plan):
        o, S_out, kept = layer.forward_keep(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"],
                                            lens=lens, aux_stream=aux)
        gr = layer.backward_keep(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], kept,
                                 dS_out=d["dS_out"], lens=lens, aux_stream=aux)
        torch.cuda.synchronize()
        res.append({"o": host(o), "S_out": host(S_out), **{k_: host(gr[k_]) for k_ in
                                                           ("dq", "dk", "dv", "dg", "dbeta", "dS_in")}})
    errs = {k_: rel_l2(res[1][k_], res[0][k_]) for k_ in res[0]}
    bad = {k_: e for k_, e in errs.items() if not e <= 1e-5}
    assert not bad, f"planned cut vs single pass: {bad} (all {errs})"
