"""The profile-guided cut (sf_plan_cut) and the schedule model it minimises
(sf_model_seq_us): host code of the C ABI, checked without a GPU.

The model replays the two streams of the drivers that keep the forward's
intermediates: the state passes on one stream (each holding one SM per
batch-head), the parallel kernels on the other, sharing the SMs left free.  The
pins below are schedules small enough to work out by hand.
"""
import pytest

# Per-chunk costs measured on a B200 for the 32-head, d = 128 gated-delta-rule
# workload (us for one 64-token chunk of all heads): intra, output, gradients on
# the whole GPU; forward and reverse state passes on one SM per head.
B200_COSTS = dict(intra_us=65.7 / 64, output_us=38.5 / 64, grad_us=160.4 / 64,
                  state_fwd_us=106.9 / 64, state_bwd_us=136.1 / 64, sms=148)


@pytest.fixture(scope="module")
def sf():
    from chunked_linear_recurrence_chunkwise_b200 import build
    build.build()
    from chunked_linear_recurrence_chunkwise_b200 import sf as sfm
    return sfm


def costs(sf, **kw):
    c = dict(B200_COSTS)
    c.update(kw)
    return sf.chunk_costs(c["intra_us"], c["output_us"], c["grad_us"], c["state_fwd_us"],
                          c["state_bwd_us"], c["sms"], c.get("min_chunks", 0))


def test_one_piece_runs_every_kernel_in_sequence(sf):
    # one piece: intra, state pass, output, then reverse pass and gradients, nothing overlaps
    sh = sf.shape(1, 640, 2, 128, 128, sf.SF_BF16)
    c = costs(sf, intra_us=1.0, output_us=2.0, grad_us=3.0, state_fwd_us=4.0, state_bwd_us=5.0, sms=4)
    assert sf.sf_model_seq_us(sh, [640], c) == pytest.approx(10 * (1 + 2 + 3 + 4 + 5))


def test_two_pieces_by_hand(sf):
    # 2 heads on 4 SMs: a running state pass leaves the parallel kernels half the GPU.
    # forward: intra0 [0,1]; state0 [1,3] beside intra1 (1 us of work at half rate) [1,3];
    # state1 [3,5] beside output0 [3,5]; output1 [5,6].  backward: reverse pass of
    # piece 1 [0,2]; reverse pass of piece 0 [2,4] beside the gradients of piece 1
    # (2 us of work: 1 done at half rate by 4, the rest alone) [2,5]; gradients of
    # piece 0 [5,7].  Total 6 + 7.
    sh = sf.shape(1, 128, 2, 128, 128, sf.SF_BF16)
    c = costs(sf, intra_us=1.0, output_us=1.0, grad_us=2.0, state_fwd_us=2.0, state_bwd_us=2.0, sms=4)
    assert sf.sf_model_seq_us(sh, [64, 64], c) == pytest.approx(13.0)


def test_state_passes_hold_every_sm_when_heads_outnumber_sms(sf):
    # 8 heads on 4 SMs: the state passes' costs, measured over all heads, already hold
    # their two waves of CTAs (they are not counted twice), and no SM is left free for
    # the parallel kernels beside them.  One piece: 1 + 3 + 1, then 5 + 1.
    sh = sf.shape(2, 64, 4, 128, 128, sf.SF_BF16)
    c = costs(sf, intra_us=1.0, output_us=1.0, grad_us=1.0, state_fwd_us=3.0, state_bwd_us=5.0, sms=4)
    assert sf.sf_model_seq_us(sh, [64], c) == pytest.approx(1 + 3 + 1 + 5 + 1)
    # two pieces, every cost 1: with no SM free, the parallel kernels advance only while
    # no state pass runs.  forward: intra0 [0,1]; state0 [1,2] (intra1 stalled); intra1
    # [2,3]; state1 [3,4] (output0 stalled); output0 [4,5]; output1 [5,6].  backward:
    # reverse pass of piece 1 [0,1]; reverse pass of piece 0 [1,2] (gradients of piece 1
    # stalled); gradients of piece 1 [2,3]; of piece 0 [3,4].  Total 6 + 4.
    c2 = costs(sf, intra_us=1.0, output_us=1.0, grad_us=1.0, state_fwd_us=1.0, state_bwd_us=1.0, sms=4)
    assert sf.sf_model_seq_us(sf.shape(2, 128, 4, 128, 128, sf.SF_BF16), [64, 64], c2) == pytest.approx(10.0)


def test_model_rejects_invalid_cuts(sf):
    sh = sf.shape(1, 256, 2, 128, 128, sf.SF_BF16)
    c = costs(sf)
    for lens in ([128, 64], [256, 0], [300, -44]):
        with pytest.raises(sf.SfError):
            sf.sf_model_seq_us(sh, lens, c)


@pytest.mark.parametrize("T,n_sub", [(65536, 16), (65536 + 17, 16), (262144, 12), (4096, 4), (640, 10)])
def test_plan_is_a_valid_cut_no_slower_than_the_even_one(sf, T, n_sub):
    sh = sf.shape(1, T, 32, 128, 128, sf.SF_BF16)
    c = costs(sf, min_chunks=14)
    plan = sf.sf_plan_cut(sh, n_sub, c)
    assert len(plan) == n_sub and sum(plan) == T and min(plan) > 0
    assert all(n % 64 == 0 for n in plan[:-1])
    chunks = -(-T // 64)
    even = [64 * (chunks // n_sub + (i < chunks % n_sub)) for i in range(n_sub)]
    even[-1] -= 64 * chunks - T
    assert sf.sf_model_seq_us(sh, plan, c) <= sf.sf_model_seq_us(sh, even, c) + 1e-9


def test_plan_shortens_the_pieces_the_backward_starts_with(sf):
    # measured costs: the backward opens with the last piece's reverse pass alone on 32
    # of 148 SMs, so the planned cut ramps down to a short last piece, no shorter than
    # min_chunks, and models faster than sixteen even pieces
    sh = sf.shape(1, 65536, 32, 128, 128, sf.SF_BF16)
    c = costs(sf, min_chunks=14)
    plan = sf.sf_plan_cut(sh, 16, c)
    assert plan[-1] < plan[0] and plan[-1] >= 14 * 64
    assert all(a >= b for a, b in zip(plan, plan[1:]))
    assert sf.sf_model_seq_us(sh, plan, c) < sf.sf_model_seq_us(sh, [4096] * 16, c)


def test_plan_keeps_the_even_cut_when_nothing_waits(sf):
    # with free state passes there is no bubble to remove: the even cut stays
    sh = sf.shape(1, 65536, 32, 128, 128, sf.SF_BF16)
    c = costs(sf, state_fwd_us=0.0, state_bwd_us=0.0)
    assert sf.sf_plan_cut(sh, 16, c) == [4096] * 16


def test_plan_rejects_invalid_arguments(sf):
    sh = sf.shape(1, 256, 2, 128, 128, sf.SF_BF16)
    with pytest.raises(sf.SfError):
        sf.sf_plan_cut(sh, 5, costs(sf))          # more pieces than chunks
    with pytest.raises(sf.SfError):
        sf.sf_plan_cut(sh, 2, costs(sf, sms=0))   # no SMs
    with pytest.raises(sf.SfError):
        sf.sf_plan_cut(sf.shape(1, 0, 2, 128, 128, sf.SF_BF16), 1, costs(sf))


def test_costs_from_a_timing_profile_and_the_layer_helpers(sf):
    import torch
    from chunked_linear_recurrence_chunkwise_b200 import layer
    # a serialized profile of 2 steps over 1024 chunks of 32 heads: kernel -> (launches, total ms)
    timing = {"intra_bwd": (32, 2 * 1.05), "state_fwd": (32, 2 * 1.7), "output": (32, 2 * 0.62),
              "state_bwd": (32, 2 * 2.18), "grad_fused": (32, 2 * 2.57), "intra_fwd": (0, 0.0)}
    c = layer.chunk_costs(timing, steps=2, n_chunks=1024, bh=32, sms=148)
    assert c.intra_us == pytest.approx(1.05e3 / 1024) and c.grad_us == pytest.approx(2.57e3 / 1024)
    assert c.state_fwd_us == pytest.approx(1.7e3 / 1024) and c.state_bwd_us == pytest.approx(2.18e3 / 1024)
    assert c.output_us == pytest.approx(0.62e3 / 1024)
    assert c.sms == 148 and c.min_chunks == 14  # ceil(3 * 148 / 32)
    q = torch.empty((1, 65536, 32, 128), dtype=torch.bfloat16)
    plan = layer.plan_cut(q, q, 16, c)
    assert sum(plan) == 65536 and len(plan) == 16 and plan[-1] < plan[0]
