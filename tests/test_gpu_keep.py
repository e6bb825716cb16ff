"""GPU parity of the sub-sequence drivers that keep the forward's intermediates
for the backward (no activation recompute), through the C ABI.

Against the fp64 oracle element by element (relative L2 per tensor: 1e-4 fp32,
2e-2 bf16), over cuts with ragged pieces and every variant; and against the
recompute drivers on the same inputs, whose backward reads the same
intermediates recomputed: the gradients must agree to 1e-5 (fp32) and to
within the bf16 tolerance of each other's arithmetic (bf16).
"""
import zlib

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
    # a seed fixed by the parameters (crc32, not hash(): str hashing is salted per process)
    seed = zlib.crc32(repr((dtype, dk, tuple(lens), has_g, has_beta)).encode()) % 997
    c = make_case(seed, B, T, H, dk, dv, has_g, has_beta, dtype)
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
    cuts: to 1e-5 on the bf16 tensor-core path, as for any cut), and both match
    the fp64 oracle within the bf16 tolerance."""
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
    o_ref, S_ref = oracle.fwd(c["q"], c["k"], c["v"], c["g"], c["beta"], c["S_in"])
    g_ref = oracle.bwd(c["q"], c["k"], c["v"], c["g"], c["beta"], c["S_in"], c["dO"], c["dS_out"])
    ref = {"o": o_ref, "S_out": S_ref, **{k_: g_ref[k_] for k_ in ("dq", "dk", "dv", "dg", "dbeta", "dS_in")}}
    errs = {k_: rel_l2(res[1][k_], ref[k_]) for k_ in ref}
    bad = {k_: e for k_, e in errs.items() if not e <= TOL["bf16"]}
    assert not bad, f"planned cut vs the oracle: {bad} (all {errs})"


def _cat(parts, dim=1):
    return torch.cat(parts, dim=dim)


@pytest.mark.parametrize("keep", [False, True])
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 64, 64)])
def test_resume_from_a_saved_piece_state_is_bit_identical(layer, keep, dtype, dk, dv):
    """Checkpoint / resume at a piece boundary (Sequence Accumulation, Approach: the
    backward pass runs over stored piece states).  The drivers stop after piece i; a
    fresh call restarts the remainder from the state saved there.  Forward: the
    remainder from S_saved[i]; backward: the remainder first, then the first part
    from the state gradient the remainder returned.  Every output must equal the
    uninterrupted run bit for bit."""
    lens = [64, 100, 192, 45, 128]
    i = 2
    B, T, H = 2, sum(lens), 2
    T1 = sum(lens[:i])
    c = make_case(57, B, T, H, dk, dv, True, True, dtype)
    d = to_dev(c, dtype)
    part = lambda t, a, b: None if t is None else t[:, a:b].contiguous()
    fwd = layer.forward_keep if keep else layer.forward

    # uninterrupted
    o, S_out, saved = fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], lens=lens)
    if keep:
        g_all = layer.backward_keep(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], saved,
                                    dS_out=d["dS_out"], lens=lens)
    else:
        g_all = layer.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], S_saved=saved,
                               dS_out=d["dS_out"], lens=lens)
    # stopped after piece i, then resumed from the state saved there
    xs = [{n: part(d[n], a, b) for n in ("q", "k", "v", "g", "beta", "dO")} for a, b in ((0, T1), (T1, T))]
    o1, S1, saved1 = fwd(xs[0]["q"], xs[0]["k"], xs[0]["v"], xs[0]["g"], xs[0]["beta"], d["S_in"],
                         lens=lens[:i])
    o2, S2, saved2 = fwd(xs[1]["q"], xs[1]["k"], xs[1]["v"], xs[1]["g"], xs[1]["beta"], S1, lens=lens[i:])
    if keep:
        g2 = layer.backward_keep(xs[1]["q"], xs[1]["k"], xs[1]["v"], xs[1]["g"], xs[1]["beta"], xs[1]["dO"],
                                 saved2, dS_out=d["dS_out"], lens=lens[i:])
        g1 = layer.backward_keep(xs[0]["q"], xs[0]["k"], xs[0]["v"], xs[0]["g"], xs[0]["beta"], xs[0]["dO"],
                                 saved1, dS_out=g2["dS_in"], lens=lens[:i])
    else:
        assert torch.equal(S1, saved[i])
        assert torch.equal(saved1, saved[:i]) and torch.equal(saved2, saved[i:])
        g2 = layer.backward(xs[1]["q"], xs[1]["k"], xs[1]["v"], xs[1]["g"], xs[1]["beta"], xs[1]["dO"],
                            S_saved=saved[i:], dS_out=d["dS_out"], lens=lens[i:])
        g1 = layer.backward(xs[0]["q"], xs[0]["k"], xs[0]["v"], xs[0]["g"], xs[0]["beta"], xs[0]["dO"],
                            S_saved=saved[:i], dS_out=g2["dS_in"], lens=lens[:i])
    torch.cuda.synchronize()
    assert torch.equal(_cat([o1, o2]), o)
    assert torch.equal(S2, S_out)
    for key in ("dq", "dk", "dv", "dg", "dbeta"):
        assert torch.equal(_cat([g1[key], g2[key]]), g_all[key]), key
    assert torch.equal(g1["dS_in"], g_all["dS_in"])
