"""Pins for the fp64 oracle (CPU only).

The pages print no worked example and no formula for the layer, so the oracle
is pinned by mathematics that does not go through its token loop:
  * the quadratic closed form of (gated) linear attention;
  * the UT/WY closed form of the delta rule over the whole sequence taken as
    one block, and the same form block by block with the state carried;
  * central finite differences of the forward for every input, which pins the
    hand-derived backward;
  * the invariant the StateFlow and Sequence Accumulation pages rest on: the
    result does not depend on how the sequence is cut into sub-sequences
    ("StateFlow ...", Abstract; "Sequence Accumulation and Beyond", Approach);
  * special cases: the delta rule with beta = 1 and unit keys writes v at key
    k; beta = 0 only decays the state; no gate and no beta is a prefix sum;
    one token worked by hand (tests/golden/gdn_t1_by_hand.json).
Shapes use dk != dv and B, H > 1 so a transposed operand or a wrong head or
batch index fails.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
VARIANTS = [(False, False), (True, False), (False, True), (True, True)]  # (has_g, has_beta)


def _inputs(seed, B=2, T=23, H=3, dk=3, dv=5, has_g=True, has_beta=True, s_in=True):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, T, H, dk))
    k = r.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((B, T, H, dv))
    g = -r.uniform(0.0, 0.7, (B, T, H)) if has_g else None
    beta = r.uniform(0.1, 1.0, (B, T, H)) if has_beta else None
    S_in = 0.5 * r.standard_normal((B, H, dk, dv)) if s_in else None
    return q, k, v, g, beta, S_in


def _head(x, b, h):
    return None if x is None else x[b, :, h]


def _cum(g, b, h, T):
    return np.zeros(T) if g is None else np.cumsum(g[b, :, h])


@pytest.mark.parametrize("has_g", [False, True])
def test_closed_form_linear_attention(has_g):
    """o = ((Q K^T) .* M) V + diag(exp(G)) Q S_in with M_ti = exp(G_t - G_i), i <= t."""
    q, k, v, g, _, S_in = _inputs(1, has_g=has_g, has_beta=False)
    B, T, H, dk = q.shape
    o, S_out = oracle.fwd(q, k, v, g, None, S_in)
    for b in range(B):
        for h in range(H):
            G = _cum(g, b, h, T)
            Q, K, V = q[b, :, h], k[b, :, h], v[b, :, h]
            M = np.tril(np.exp(G[:, None] - G[None, :]))
            o_ref = ((Q @ K.T) * M) @ V + np.exp(G)[:, None] * (Q @ S_in[b, h])
            S_ref = np.exp(G[-1]) * S_in[b, h] + (K * np.exp(G[-1] - G)[:, None]).T @ V
            np.testing.assert_allclose(o[b, :, h], o_ref, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(S_out[b, h], S_ref, rtol=1e-12, atol=1e-12)


def _ut_block(Q, K, V, beta, G, S):
    """Delta rule over one block in closed form (UT / WY representation).

    With the update written S_r = a_r S_{r-1} + k_r d_r^T and
    d_r = beta_r (v_r - a_r S_{r-1}^T k_r), the rows d_r solve
    (I + A) D = diag(beta) V - diag(beta * exp(G)) K S with
    A_ri = beta_r exp(G_r - G_i) k_r . k_i for i < r.
    """
    n = Q.shape[0]
    gam = np.exp(G)
    Gam = np.exp(G[:, None] - G[None, :])
    A = np.tril(beta[:, None] * Gam * (K @ K.T), -1)
    rhs = beta[:, None] * V - (beta * gam)[:, None] * (K @ S)
    D = np.linalg.solve(np.eye(n) + A, rhs)
    O = gam[:, None] * (Q @ S) + (np.tril(Q @ K.T) * np.tril(Gam)) @ D
    S_next = gam[-1] * S + (K * np.exp(G[-1] - G)[:, None]).T @ D
    return O, S_next


@pytest.mark.parametrize("has_g", [False, True])
def test_ut_whole_sequence_delta_rule(has_g):
    q, k, v, g, beta, S_in = _inputs(2, T=31, has_g=has_g, has_beta=True)
    B, T, H, _ = q.shape
    o, S_out = oracle.fwd(q, k, v, g, beta, S_in)
    for b in range(B):
        for h in range(H):
            O_ref, S_ref = _ut_block(q[b, :, h], k[b, :, h], v[b, :, h], beta[b, :, h],
                                     _cum(g, b, h, T), S_in[b, h])
            np.testing.assert_allclose(o[b, :, h], O_ref, rtol=1e-11, atol=1e-11)
            np.testing.assert_allclose(S_out[b, h], S_ref, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("C", [4, 8, 16])
def test_ut_blockwise_with_state_carry(C):
    """The same closed form applied block by block (block-local cumsum of g)."""
    q, k, v, g, beta, S_in = _inputs(3, T=37, has_g=True, has_beta=True)
    B, T, H, _ = q.shape
    o, S_out = oracle.fwd(q, k, v, g, beta, S_in)
    for b in range(B):
        for h in range(H):
            S = S_in[b, h].copy()
            outs = []
            for t0 in range(0, T, C):
                sl = slice(t0, min(T, t0 + C))
                G = np.cumsum(g[b, sl, h])
                O, S = _ut_block(q[b, sl, h], k[b, sl, h], v[b, sl, h], beta[b, sl, h], G, S)
                outs.append(O)
            np.testing.assert_allclose(o[b, :, h], np.concatenate(outs), rtol=1e-11, atol=1e-11)
            np.testing.assert_allclose(S_out[b, h], S, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("has_g,has_beta", VARIANTS)
def test_backward_matches_finite_differences(has_g, has_beta):
    """Central differences of L = <o, R_o> + <S_out, R_s> w.r.t. every input."""
    q, k, v, g, beta, S_in = _inputs(4, B=1, T=7, H=2, dk=3, dv=4, has_g=has_g, has_beta=has_beta)
    r = np.random.default_rng(5)
    Ro = r.standard_normal(v.shape)
    Rs = r.standard_normal(S_in.shape)
    names = ["q", "k", "v", "g", "beta", "S_in"]
    vals = dict(q=q, k=k, v=v, g=g, beta=beta, S_in=S_in)

    def loss(vv):
        o, S_out = oracle.fwd(vv["q"], vv["k"], vv["v"], vv["g"], vv["beta"], vv["S_in"], nthreads=1)
        return float(np.sum(o * Ro) + np.sum(S_out * Rs))

    grads = oracle.bwd(q, k, v, g, beta, S_in, Ro, Rs, nthreads=1)
    key = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "beta": "dbeta", "S_in": "dS_in"}
    h = 1e-6
    for n in names:
        if vals[n] is None:
            assert grads[key[n]] is None
            continue
        x = vals[n]
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            lp = loss(vals)
            x[idx] = old - h
            lm = loss(vals)
            x[idx] = old
            fd[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(grads[key[n]], fd, rtol=1e-6, atol=1e-7, err_msg=n)


@pytest.mark.parametrize("has_g,has_beta", VARIANTS)
def test_split_invariance(has_g, has_beta):
    """Any cut into sub-sequences with the state (and dS) carried equals one pass."""
    q, k, v, g, beta, S_in = _inputs(6, T=50, has_g=has_g, has_beta=has_beta)
    dO = np.random.default_rng(7).standard_normal(v.shape)
    dS_out = np.random.default_rng(8).standard_normal(S_in.shape)
    o1, S1 = oracle.fwd(q, k, v, g, beta, S_in)
    r1 = oracle.bwd(q, k, v, g, beta, S_in, dO, dS_out)
    for lens in ([7, 13, 30], [1] * 50, [49, 1], [25, 25]):
        o2, S2, saved = oracle.fwd_seq(lens, q, k, v, g, beta, S_in)
        np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(S2, S1, rtol=1e-12, atol=1e-12)
        r2 = oracle.bwd_seq(lens, q, k, v, g, beta, saved, dO, dS_out)
        for kk in ("dq", "dk", "dv", "dg", "dbeta", "dS_in"):
            if r1[kk] is None:
                assert r2[kk] is None
            else:
                np.testing.assert_allclose(r2[kk], r1[kk], rtol=1e-11, atol=1e-11, err_msg=kk)


@pytest.mark.parametrize("has_g", [False, True])
def test_delta_rule_writes_value_at_unit_key(has_g):
    """beta = 1, ||k|| = 1: after the update S_t^T k_t = v_t exactly, so q = k reads back v."""
    q, k, v, g, beta, S_in = _inputs(9, T=19, has_g=has_g, has_beta=True)
    beta = np.ones_like(beta)
    o, _ = oracle.fwd(k, k, v, g, beta, S_in)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)


def test_zero_beta_only_decays():
    q, k, v, g, beta, S_in = _inputs(10, T=17, has_g=True, has_beta=True)
    o, S_out = oracle.fwd(q, k, v, g, np.zeros_like(beta), S_in)
    G = np.cumsum(g, axis=1)  # [B, T, H]
    np.testing.assert_allclose(S_out, np.exp(G[:, -1])[:, :, None, None] * S_in, rtol=1e-13)
    o_ref = np.exp(G)[..., None] * np.einsum("bthi,bhij->bthj", q, S_in)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-13)


def test_ungated_linear_attention_is_a_prefix_sum():
    q, k, v, _, _, S_in = _inputs(11, T=29, has_g=False, has_beta=False)
    o, S_out = oracle.fwd(q, k, v, None, None, S_in)
    outer = np.einsum("bthi,bthj->bthij", k, v)
    S_t = S_in[:, None] + np.cumsum(outer, axis=1)  # [B, T, H, dk, dv]
    np.testing.assert_allclose(o, np.einsum("bthi,bthij->bthj", q, S_t), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S_out, S_t[:, -1], rtol=1e-12, atol=1e-12)


def test_one_token_worked_by_hand():
    gd = json.load(open(os.path.join(GOLDEN, "gdn_t1_by_hand.json")))
    i, e = gd["inputs"], gd["expected"]
    sh = lambda x: np.array(x, np.float64).reshape(1, 1, 1, -1)
    sc = lambda x: np.array(x, np.float64).reshape(1, 1, 1)
    S_in = np.array(i["S_in"]).reshape(1, 1, 2, 2)
    o, S_out = oracle.fwd(sh(i["q"]), sh(i["k"]), sh(i["v"]), sc(i["g"]), sc(i["beta"]), S_in)
    np.testing.assert_allclose(o.ravel(), e["o"], atol=1e-14)
    np.testing.assert_allclose(S_out.reshape(2, 2), e["S_out"], atol=1e-14)
    r = oracle.bwd(sh(i["q"]), sh(i["k"]), sh(i["v"]), sc(i["g"]), sc(i["beta"]), S_in, sh(i["dO"]))
    for key in ("dq", "dk", "dv"):
        np.testing.assert_allclose(r[key].ravel(), e[key], atol=1e-14, err_msg=key)
    np.testing.assert_allclose(r["dg"].item(), e["dg"], atol=1e-14)
    np.testing.assert_allclose(r["dbeta"].item(), e["dbeta"], atol=1e-14)
    np.testing.assert_allclose(r["dS_in"].reshape(2, 2), e["dS_in"], atol=1e-14)


def test_empty_sequence_passes_state_through():
    q, k, v, g, beta, S_in = _inputs(12, T=0)
    o, S_out = oracle.fwd(q, k, v, g, beta, S_in)
    assert o.shape[1] == 0
    np.testing.assert_array_equal(S_out, S_in)
    dS = np.random.default_rng(1).standard_normal(S_in.shape)
    r = oracle.bwd(q, k, v, g, beta, S_in, np.zeros(v.shape), dS)
    np.testing.assert_array_equal(r["dS_in"], dS)


@pytest.mark.parametrize("seg", [1, 5, 64])
def test_backward_checkpoint_segment_does_not_matter(seg):
    q, k, v, g, beta, S_in = _inputs(13, T=40)
    dO = np.random.default_rng(2).standard_normal(v.shape)
    a = oracle.bwd(q, k, v, g, beta, S_in, dO, seg=seg)
    b = oracle.bwd(q, k, v, g, beta, S_in, dO, seg=7)
    for key in a:
        np.testing.assert_allclose(a[key], b[key], rtol=1e-12, atol=1e-13, err_msg=key)
