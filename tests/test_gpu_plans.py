"""Launch plans larger than one launch's parameter tables (8 problems, 64
groups, 128 segments, 512 K/V ranges): the planner splits them over several
launches, and the result must still match the oracle.  Also the largest ring
degree (512 chunks) and a 1000-shard kv_gather.  Through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from context_attention_long_b200 import api, build, inputs

from gpu_util import assert_close, f64_of, full_to_rank_buffers, rank_buffers_to_full, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _qkv(B, S, H, D, seed):
    q, k, v = inputs.make_qkv(B, S, H, D, seed, False)
    return (q, k, v), tuple(inputs.bf16_bits_to_f64(x) for x in (q, k, v)), tuple(to_dev(x) for x in (q, k, v))


def _no_timeouts():
    st, code = api.cpattn_device_status()
    assert st == 0 and code == 0, f"device wait expired: code {code:#x}"


@pytest.mark.parametrize("causal", [False, True])
def test_ring_with_more_segments_and_ranges_than_one_launch_holds(causal):
    # 3 batches x 48 shards = 144 segments (> 128); 48 ranges per segment, so
    # at most 10 segments fit the 512-range table of one launch.
    B, H, D, P = 3, 2, 64, 48
    lens = inputs.random_splits(960, P, 11)
    S = sum(lens)
    _, (q, k, v), (dq, dk, dv) = _qkv(B, S, H, D, 21)
    fn = api.cpattn_causal_ring_attention if causal else api.cpattn_ring_attention
    out, lse = fn(dq, dk, dv, P, lens)
    torch.cuda.synchronize()
    _no_timeouts()
    ref_o, ref_l = (oracle.causal_attention(q, k, v) if causal else oracle.attention(q, k, v))
    assert_close(f64_of(out), f64_of(lse), ref_o, ref_l, f"ring P={P} causal={causal}")


def test_ring_at_the_largest_degree():
    B, H, D, P = 1, 2, 64, 512
    S = 2 * P
    _, (q, k, v), (dq, dk, dv) = _qkv(B, S, H, D, 22)
    out, lse = api.cpattn_ring_attention(dq, dk, dv, P)
    torch.cuda.synchronize()
    _no_timeouts()
    assert_close(f64_of(out), f64_of(lse), *oracle.attention(q, k, v), "ring P=512")
    with pytest.raises(api.CpattnError):
        api.cpattn_ring_attention(dq, dk, dv, 513, [2] * 511 + [1, 1])


def test_kv_gather_with_a_thousand_shards():
    B, H, D, P = 1, 2, 64, 1000
    lens = [1] * P
    _, (q, k, v), (dq, dk, dv) = _qkv(B, P, H, D, 23)
    out, lse = api.cpattn_kv_gather_attention(dq, dk, dv, P, lens)
    torch.cuda.synchronize()
    _no_timeouts()
    assert_close(f64_of(out), f64_of(lse), *oracle.attention(q, k, v), "kv_gather P=1000")


@pytest.mark.parametrize("causal", [False, True])
def test_ulysses_with_more_problems_and_groups_than_one_launch_holds(causal):
    # 64 head ranks of one head each = 64 problems (> 8); with B = 2 that is
    # 128 groups (> 64).
    B, S, H, D, P = 2, 256, 64, 64, 64
    seq = inputs.random_splits(S, P, 12)
    (qb, kb, vb), (q, k, v), _ = _qkv(B, S, H, D, 24)
    flat = [to_dev(full_to_rank_buffers(x, seq)) for x in (qb, kb, vb)]
    fn = api.cpattn_causal_ulysses_attention if causal else api.cpattn_ulysses_attention
    out, lse = fn(*flat, B, S, H, D, P, seq)
    torch.cuda.synchronize()
    _no_timeouts()
    got = rank_buffers_to_full(f64_of(out), B, S, H, D, seq)
    ref_o, ref_l = (oracle.causal_attention(q, k, v) if causal else oracle.attention(q, k, v))
    assert_close(got, f64_of(lse), ref_o, ref_l, f"ulysses P={P} causal={causal}")
