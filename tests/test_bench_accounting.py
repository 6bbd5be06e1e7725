"""The work counts behind bench.py's throughputs and roofline, checked on the
CPU against brute-force counts: causal attention counts 4*D FLOPs for every
visible (query, key) pair, the backward 2.5x the forward, and the projections
2*K FLOPs per output element (a multiply and an add per term)."""
import pytest

import bench


@pytest.mark.parametrize("B,H,S,D", [(1, 1, 1, 64), (2, 3, 7, 128), (1, 2, 130, 64)])
def test_causal_flops_count_visible_pairs(B, H, S, D):
    visible = sum(1 for i in range(S) for j in range(S) if j <= i)
    assert bench.causal_flops(B, H, S, D) == 4.0 * D * B * H * visible


@pytest.mark.parametrize("causal", [False, True])
def test_backward_flops_are_five_matmuls_of_the_forward_two(causal):
    B, H, S, D = 2, 3, 9, 64
    fwd = bench.causal_flops(B, H, S, D) if causal else 4.0 * B * H * S * S * D
    assert bench.backward_flops(B, H, S, D, causal) == pytest.approx(fwd * 5 / 2)


def test_projection_flops_match_counted_multiply_adds():
    B, S, H, D, Dm = 2, 3, 2, 4, 5
    count_qkv = sum(1 for _row in range(B * S) for _col in range(3 * H * D) for _k in range(Dm))
    count_out = sum(1 for _row in range(B * S) for _col in range(Dm) for _k in range(H * D))
    assert bench.projection_flops(B, S, H, D, Dm) == (2.0 * count_qkv, 2.0 * count_out)


def test_max_over_ranks_single_rank_is_the_identity():
    assert bench.max_over_ranks([10.0, 2.5], 1) == [10.0, 2.5]


@pytest.mark.parametrize("S,world", [(32760, 2), (32760, 4), (32760, 8), (10007, 6), (9, 8)])
def test_multi_gpu_shards_cover_the_sequence_once(S, world):
    lens, ring_lens, subs = bench.multi_gpu_shards(S, world)
    assert sum(lens) == S and len(lens) == world and max(lens) - min(lens) <= 1
    # rank (i, j) = 2 i + j holds sub-shard j of ring chunk i: the same tokens
    flat = [n for chunk in subs for n in chunk]
    assert flat == lens
    assert ring_lens == [sum(c) for c in subs] and sum(ring_lens) == S


def test_ring_peak_choice_sustained_only_for_long_regions_with_the_figure():
    peaks = {"bf16_tflops": 1646.1, "bf16_tflops_sustained": 1450.0, "hbm_gbs": 6547.2}
    p, kind = bench.ring_peak_choice(peaks, "measured", 1.2)
    assert p == 1450.0 and kind.startswith("bf16_tflops_sustained, measured")
    p, kind = bench.ring_peak_choice(peaks, "measured", 0.4)
    assert p == 1646.1 and kind == "bf16_tflops burst, measured"
    no_sus = {"bf16_tflops": 1646.1, "hbm_gbs": 6547.2}
    p, kind = bench.ring_peak_choice(no_sus, "measured", 1.2)
    assert p == 1646.1 and "no sustained figure" in kind
