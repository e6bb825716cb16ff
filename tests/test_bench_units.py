"""Host logic of bench.py's accounting: the canonical flop counts and the layer's own
I/O bytes per token-head that the roofline fields are computed from."""
import bench
from chunked_linear_recurrence_chunkwise_b200 import inputs


def _gdn():
    return inputs.WORKLOADS["gated_deltanet_bf16_h32_t64k"]


def test_canonical_flops_add_up_to_the_layer_count():
    """Per token-head with C = 64, d = 128 (u = 2 C d, v = 2 d^2): forward 2.5 u + 3 v,
    backward 5 u + 6 v, 417792 flop in all for the gated delta rule."""
    w = _gdn()
    u, v = 2 * 64 * 128, 2 * 128 * 128
    per = lambda n: bench.canonical_flops(n, w) / 64
    fwd = per("intra_bwd") + per("state_fwd") + per("output_p")
    bwd = per("state_bwd") + per("grad_fused")
    assert fwd == 2.5 * u + 3 * v
    assert bwd == 5 * u + 6 * v
    assert fwd + bwd == 417792
    assert per("grad_fused") == 4.5 * u + 3 * v  # 172032, the gradient kernel's share
    # the recompute forward's output kernel forms P itself
    assert per("intra_fwd") + per("state_fwd") + per("output") == fwd


def test_linear_attention_counts_drop_the_delta_terms():
    w = inputs.WORKLOADS["gated_linear_attention_bf16_b2_h16_t32k"]
    u, v = 2 * 64 * 128, 2 * 128 * 128
    per = lambda n: bench.canonical_flops(n, w) / 64
    assert per("intra_bwd") + per("state_fwd") + per("output_p") == u + 2 * v
    assert per("state_bwd") + per("grad_attn") == 2 * u + 4 * v


def test_layer_io_bytes_per_token_head():
    """bf16 q, k, v, o, dO, dq, dk, dv (256 B each at d = 128), fp32 g, beta, dg, dbeta."""
    io = bench.layer_io_bytes_per_token_head(_gdn())
    assert io == {"fwd": 1032, "bwd": 1808, "total": 2840}


def test_gradient_kernel_io_is_the_backward_io():
    """The fused gradient kernel reads q, k, v, g, beta, dO and writes every gradient
    but dS: its algorithmic bytes are the backward's 1808 B per token-head."""
    w = _gdn()
    assert bench.kernel_units("grad_fused", w)["io_bytes"] == 1808 * 64


def test_step_roofline_of_the_bench_workload():
    w = _gdn()
    peaks = {"hbm_gbs": 6550.1, "bf16_tflops": 1589.5}
    s = bench.step_roofline(w, 5.0, peaks)
    th = w.B * w.T * w.H
    assert s["flops_per_token_head"] == 417792
    assert abs(s["tflops"] - 417792 * th / 5e-3 / 1e12) < 0.01
    assert abs(s["hbm_floor_ms"] - 2840 * th / 6550.1e9 * 1e3) < 1e-3
    assert abs(s["hbm_floor_frac"] - s["hbm_floor_ms"] / 5.0) < 1e-3


def test_source_hash_ignores_comments_only():
    import bench
    a = 'int x = 1; // one\n/* block\n comment */ const char* s = "a // b";\n'
    b = 'int   x = 1;\nconst char* s = "a // b";  // another note\n'
    c = 'int x = 2; const char* s = "a // b";'
    assert bench.code_of(a) == bench.code_of(b)
    assert bench.code_of(a) != bench.code_of(c)
    assert '"a // b"' in bench.code_of(a)  # string literals are kept whole
