"""GPU parity: libsf (through its C ABI) against the fp64 oracle, element by element.

Tolerances (relative L2 over each whole output tensor, ||x - ref|| / ||ref||):
1e-4 for fp32 inputs and 2e-2 for bf16 inputs; chunking invariance on the GPU
within 1e-5 in fp32.  bf16 cases feed the oracle the bf16-rounded inputs.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
VARIANTS = [(False, False), (True, False), (False, True), (True, True)]  # (gate, beta)


def rel_l2(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    n = np.linalg.norm(ref)
    return np.linalg.norm(x - ref) / (n if n > 0 else 1.0)


def make_case(seed, B, T, H, dk, dv, has_g, has_beta, dtype, s_in=True, ds_out=True):
    """Seeded small inputs with the workloads' distributions (q, k L2-normalised)."""
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, T, H, dk)).astype(np.float32)
    k = r.standard_normal((B, T, H, dk)).astype(np.float32)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((B, T, H, dv)).astype(np.float32)
    g = (-0.1 * np.logaddexp(0, r.standard_normal((B, T, H)))).astype(np.float32) if has_g else None
    beta = (1 / (1 + np.exp(-r.standard_normal((B, T, H))))).astype(np.float32) if has_beta else None
    dO = r.standard_normal((B, T, H, dv)).astype(np.float32)
    S_in = (0.1 * r.standard_normal((B, H, dk, dv))).astype(np.float32) if s_in else None
    dS_out = (0.1 * r.standard_normal((B, H, dk, dv))).astype(np.float32) if ds_out else None
    if dtype == "bf16":
        rb = lambda a: torch.from_numpy(a).to(torch.bfloat16).float().numpy()
        q, k, v, dO = rb(q), rb(k), rb(v), rb(dO)
    return dict(q=q, k=k, v=v, g=g, beta=beta, dO=dO, S_in=S_in, dS_out=dS_out)


def to_dev(c, dtype):
    io = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = {}
    for key, a in c.items():
        if a is None:
            out[key] = None
        elif key in ("q", "k", "v", "dO"):
            out[key] = torch.from_numpy(a).to("cuda", io).contiguous()
        else:
            out[key] = torch.from_numpy(a).to("cuda", torch.float32).contiguous()
    return out


def host(t):
    return None if t is None else t.float().cpu().numpy()


@pytest.fixture(scope="module")
def layer():
    from chunked_linear_recurrence_chunkwise_b200 import layer as L
    return L


SHAPES = [
    (2, 3 * 64 + 17, 3, 64, 64),  # several chunks and a ragged tail
    (1, 5 * 64, 2, 128, 128),     # whole chunks, full head size
    (1, 1, 2, 128, 128),          # one token
    (1, 150, 2, 48, 80),          # dk != dv, d_v tiles with a partial tile
]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("has_g,has_beta", VARIANTS)
@pytest.mark.parametrize("shape", SHAPES)
def test_single_piece_matches_oracle(layer, dtype, has_g, has_beta, shape):
    B, T, H, dk, dv = shape
    seed = zlib.crc32(repr((shape, has_g, has_beta)).encode()) % 1000  # fixed across processes
    c = make_case(seed, B, T, H, dk, dv, has_g, has_beta, dtype)
    d = to_dev(c, dtype)
    o, S_out, _ = layer.forward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"])
    gr = layer.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], S_in=d["S_in"],
                        dS_out=d["dS_out"])
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.fwd(c["q"], c["k"], c["v"], c["g"], c["beta"], c["S_in"])
    g_ref = oracle.bwd(c["q"], c["k"], c["v"], c["g"], c["beta"], c["S_in"], c["dO"], c["dS_out"])
    tol = TOL[dtype]
    errs = {"o": rel_l2(host(o), o_ref), "S_out": rel_l2(host(S_out), S_ref)}
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dS_in"):
        if g_ref[key] is None:
            assert gr[key] is None
        else:
            errs[key] = rel_l2(host(gr[key]), g_ref[key])
    bad = {k_: e for k_, e in errs.items() if not e <= tol}
    assert not bad, f"rel-L2 above {tol}: {bad} (all: {errs})"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("lens", [[64, 100, 45], [209], [1, 64, 128, 16]])
def test_sub_sequence_driver_matches_oracle(layer, dtype, lens):
    B, T, H, dk, dv = 2, sum(lens), 3, 64, 64
    c = make_case(7, B, T, H, dk, dv, True, True, dtype)
    d = to_dev(c, dtype)
    aux = torch.cuda.Stream()
    o, S_out, S_saved = layer.forward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"],
                                      lens=lens, aux_stream=aux)
    gr = layer.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], S_saved=S_saved,
                        dS_out=d["dS_out"], lens=lens, aux_stream=aux)
    torch.cuda.synchronize()
    o_ref, S_ref, saved_ref = oracle.fwd_seq(lens, c["q"], c["k"], c["v"], c["g"], c["beta"],
                                             c["S_in"])
    g_ref = oracle.bwd_seq(lens, c["q"], c["k"], c["v"], c["g"], c["beta"], saved_ref, c["dO"],
                           c["dS_out"])
    tol = TOL[dtype]
    assert rel_l2(host(o), o_ref) <= tol
    assert rel_l2(host(S_out), S_ref) <= tol
    for i, s in enumerate(saved_ref):
        assert rel_l2(host(S_saved[i]), s) <= tol
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dS_in"):
        assert rel_l2(host(gr[key]), g_ref[key]) <= tol, key


@pytest.mark.parametrize("has_g,has_beta", VARIANTS)
@pytest.mark.parametrize("lens", [[128, 192, 64], [100, 77, 207], [1] * 8 + [376]])
def test_chunking_invariance_fp32(layer, has_g, has_beta, lens):
    """Cutting the sequence into sub-sequences must not change the result (fp32, 1e-5)."""
    B, T, H, dk, dv = 1, sum(lens), 2, 128, 128
    c = make_case(11, B, T, H, dk, dv, has_g, has_beta, "f32")
    d = to_dev(c, "f32")
    o1, S1, _ = layer.forward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"])
    g1 = layer.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], S_in=d["S_in"],
                        dS_out=d["dS_out"])
    o2, S2, saved = layer.forward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], lens=lens,
                                  aux_stream=torch.cuda.Stream())
    g2 = layer.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], S_saved=saved,
                        dS_out=d["dS_out"], lens=lens, aux_stream=torch.cuda.Stream())
    torch.cuda.synchronize()
    assert rel_l2(host(o2), host(o1)) <= 1e-5
    assert rel_l2(host(S2), host(S1)) <= 1e-5
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dS_in"):
        if g1[key] is not None:
            assert rel_l2(host(g2[key]), host(g1[key])) <= 1e-5, key


def test_empty_sequence(layer):
    c = make_case(3, 1, 0, 2, 64, 64, True, True, "f32")
    d = to_dev(c, "f32")
    o, S_out, _ = layer.forward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"])
    gr = layer.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], S_in=d["S_in"],
                        dS_out=d["dS_out"])
    torch.cuda.synchronize()
    assert o.shape[1] == 0
    assert torch.equal(S_out, d["S_in"])
    assert torch.equal(gr["dS_in"], d["dS_out"])


def test_degenerate_zero_beta_and_strong_decay(layer):
    """beta = 0 only decays the state; g = -60 per token underflows the decay to 0 without NaN."""
    B, T, H, dk, dv = 1, 130, 2, 64, 64
    c = make_case(5, B, T, H, dk, dv, True, True, "f32")
    c["beta"] = np.zeros_like(c["beta"])
    c["g"][:, 70:] = -60.0
    d = to_dev(c, "f32")
    o, S_out, _ = layer.forward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"])
    gr = layer.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], S_in=d["S_in"],
                        dS_out=d["dS_out"])
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.fwd(c["q"], c["k"], c["v"], c["g"], c["beta"], c["S_in"])
    g_ref = oracle.bwd(c["q"], c["k"], c["v"], c["g"], c["beta"], c["S_in"], c["dO"], c["dS_out"])
    assert np.all(np.isfinite(host(o)))
    assert rel_l2(host(o), o_ref) <= 1e-4
    assert np.abs(host(S_out)).max() == 0.0 and np.abs(S_ref).max() < 1e-30
    for key in ("dq", "dk", "dv", "dbeta", "dS_in"):
        assert rel_l2(host(gr[key]), g_ref[key]) <= 1e-4, key
