"""sf_fwd_noalloc: the forward for callers that cannot allocate device memory.

Some callers are only handed their input and output buffers (a plugin inside a
framework that plans all memory before it runs, code running in an allocator
callback, loops that must not call cudaMalloc because it can synchronise the
device).  sf_fwd_noalloc serves them from a fixed scratch array inside the
library.  These checks call it through the C ABI twice in a row, on different
inputs, and compare each result with sf_fwd given an ordinary workspace and
with the fp64 oracle.  Before the checked calls, a call of another shape and
dtype fills the array with other data, and the sf_fwd reference runs on a
workspace filled with 0xFF bytes (NaN as floats), so that a read of a byte the
call has not written shows up in either result.  The file is named to be
collected last so that a stop-at-first-failure run has already run everything
else.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_l2(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (n if n > 0 else 1.0))


def host(t):
    return t.double().cpu().numpy()


def case(seed, B, T, H, d, dtype):
    g = torch.Generator().manual_seed(seed)
    io = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = torch.nn.functional.normalize(torch.randn(B, T, H, d, generator=g), dim=-1)
    k = torch.nn.functional.normalize(torch.randn(B, T, H, d, generator=g), dim=-1)
    v = torch.randn(B, T, H, d, generator=g)
    gg = -0.1 * torch.nn.functional.softplus(torch.randn(B, T, H, generator=g))
    beta = torch.sigmoid(torch.randn(B, T, H, generator=g))
    S_in = 0.1 * torch.randn(B, H, d, d, generator=g)
    dev = lambda t, dt=torch.float32: t.to("cuda", dt).contiguous()
    return dev(q, io), dev(k, io), dev(v, io), dev(gg), dev(beta), dev(S_in)


def fill_scratch_with_other_data(sf):
    """A call of another shape and dtype, so that the array holds its data."""
    q, k, v, g, beta, S_in = case(5, 1, 20 * 64, 3, 128, "bf16")
    o = torch.empty_like(v)
    S_out = torch.empty(1, 3, 128, 128, device="cuda")
    sf.sf_fwd_noalloc(sf.shape_of(q, v), q, k, v, g, beta, S_in, o, S_out)
    q, k, v, g, beta, S_in = case(6, 2, 9 * 64 + 5, 1, 64, "f32")
    o = torch.empty_like(v)
    S_out = torch.empty(2, 1, 64, 64, device="cuda")
    sf.sf_fwd_noalloc(sf.shape_of(q, v), q, k, v, g, beta, S_in, o, S_out)
    torch.cuda.synchronize()
    sf.sf_check_noalloc()


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_noalloc_forward_matches_sf_fwd_and_oracle_on_two_calls(dtype, d):
    from chunked_linear_recurrence_chunkwise_b200 import sf

    fill_scratch_with_other_data(sf)
    B, T, H = 2, 3 * 64 + 29, 2
    for call, seed in enumerate((11, 12)):
        q, k, v, g, beta, S_in = case(seed, B, T, H, d, dtype)
        sh = sf.shape_of(q, v)
        ws = torch.full((sf.sf_workspace_bytes(sh, sf.SF_OP_FWD),), 0xFF, dtype=torch.uint8, device="cuda")
        ws[:256].zero_()  # the error word starts at zero; every other byte reads as NaN
        o_ref = torch.empty_like(v)
        S_ref = torch.empty(B, H, d, d, device="cuda")
        sf.sf_fwd(sh, q, k, v, g, beta, S_in, o_ref, S_ref, ws)
        o = torch.full_like(v, float("nan"))
        S_out = torch.full((B, H, d, d), float("nan"), device="cuda")
        sf.sf_fwd_noalloc(sh, q, k, v, g, beta, S_in, o, S_out)
        torch.cuda.synchronize()
        sf.sf_check(ws)
        sf.sf_check_noalloc()
        assert rel_l2(host(o), host(o_ref)) <= TOL[dtype], (call, rel_l2(host(o), host(o_ref)))
        assert rel_l2(host(S_out), host(S_ref)) <= TOL[dtype], (call, rel_l2(host(S_out), host(S_ref)))
        # the fp64 oracle on the same (rounded) inputs
        o64, S64 = oracle.fwd(host(q), host(k), host(v), host(g), host(beta), host(S_in))
        assert rel_l2(host(o), o64) <= TOL[dtype], (call, rel_l2(host(o), o64))
        assert rel_l2(host(S_out), S64) <= TOL[dtype], (call, rel_l2(host(S_out), S64))


def test_noalloc_rejects_shapes_beyond_its_scratch():
    from chunked_linear_recurrence_chunkwise_b200 import sf

    sh = sf.shape(1, 1 << 20, 8, 128, 128, sf.SF_BF16)  # needs far more than the built-in 32 MiB
    with pytest.raises(sf.SfError) as exc:
        sf.sf_fwd_noalloc(sh, 16, 16, 16, None, None, None, 16, None)
    assert exc.value.status == sf.SF_ERR_WORKSPACE
