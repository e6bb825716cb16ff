"""Host-side checks of the seeded input generator (no GPU, no method arithmetic)."""
import numpy as np
import pytest

from chunked_linear_recurrence_chunkwise_b200 import inputs


def test_token_ranges_regenerate_identically():
    w = inputs.WORKLOADS["gated_deltanet_bf16_h32_t64k"].scaled(T=9000, H=3)
    full = inputs.generate(w)
    part = inputs.generate(w, 4000, 8300, heads=[2, 0])
    for key in ("q", "k", "v", "g", "beta", "dO"):
        np.testing.assert_array_equal(part[key], full[key][:, 4000:8300][:, :, [2, 0]])


def test_distributions_and_bf16_values():
    w = inputs.WORKLOADS["gated_deltanet_bf16_h32_t64k"].scaled(T=2048, H=2)
    x = inputs.generate(w)
    import torch
    for key in ("q", "k", "v", "dO"):
        t = torch.from_numpy(x[key])
        assert torch.equal(t.to(torch.bfloat16).float(), t), key  # exactly bf16 values
    n = np.linalg.norm(x["k"].astype(np.float64), axis=-1)
    assert np.all(np.abs(n - 1) < 1e-2)
    assert np.all((x["beta"] > 0) & (x["beta"] < 1))
    assert np.all(x["g"] < 0) and np.all(x["g"] > -2)


def test_gla_gate_is_logsigmoid_of_shifted_normal():
    w = inputs.WORKLOADS["gated_linear_attention_bf16_b2_h16_t32k"].scaled(T=4096, H=2)
    g = inputs.generate(w)["g"].astype(np.float64)
    # logsigmoid(N(2, 1)) has median logsigmoid(2) = -0.1269
    assert abs(np.median(g) + np.log1p(np.exp(-2.0))) < 0.01
    assert inputs.generate(w)["beta"] is None


@pytest.mark.parametrize("name", list(inputs.WORKLOADS))
def test_sub_lengths(name):
    w = inputs.WORKLOADS[name]
    lens = inputs.sub_lengths(w)
    assert len(lens) == w.n_sub and sum(lens) == w.T
    assert all(L % 64 == 0 and L >= 64 for L in lens)
    if w.cut == "dirichlet":
        assert len(set(lens)) > 1
        assert lens == inputs.sub_lengths(w)  # seeded


def test_kept_heads_match_the_device_copy():
    w = inputs.WORKLOADS["gated_deltanet_bf16_h32_t64k"].scaled(T=5000, H=3)
    x = inputs.to_torch(w, device="cpu", keep_heads=[(0, 2), (0, 0)])
    for (b, h), kept in zip([(0, 2), (0, 0)], x["kept"]):
        for key in ("q", "k", "v", "g", "beta", "dO"):
            np.testing.assert_array_equal(kept[key][0, :, 0], x[key][b, :, h].float().numpy())
