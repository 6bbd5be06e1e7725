"""Attention over segments longer than one CTA's pair of Q tiles, against the
fp64 oracle through the C ABI (D = 128, non-causal): several whole units,
a partial last unit, lone-tile tails that become split units, several
segments and K/V ranges whose key counts are not multiples of 128, two batch
elements, several head groups of one launch, and the kv_gather, Ulysses and
ring-chunk entry points on the same kind of shapes; the same call twice gives
the same bytes."""
import numpy as np
import pytest
import torch

import oracle
from context_attention_long_b200 import api, build, inputs

from gpu_util import assert_close, f64_of, full_to_rank_buffers, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _no_timeouts():
    st, code = api.cpattn_device_status()
    assert st == 0 and code == 0, f"device wait expired: code {code:#x}"


def _qkv(B, S, H, seed):
    qb, kb, vb = inputs.make_qkv(B, S, H, 128, seed, True)
    return (qb, kb, vb), tuple(to_dev(x) for x in (qb, kb, vb)), tuple(inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb))


@pytest.mark.parametrize("B,H,S,P,lens", [
    (1, 2, 512, 1, None),                  # two whole units
    (2, 2, 800, 1, None),                  # three units, the last with 32 rows (a split unit)
    (1, 3, 1300, 2, None),                 # 650-row shards: units and a 138-row tail
    (2, 2, 2100, 3, [1030, 333, 737]),     # uneven shards, tails of 6, 77 and 225 rows
    (1, 2, 1031, 2, [1000, 31]),           # 31 keys in the second chunk
])
def test_ring_over_long_segments_matches_oracle(B, H, S, P, lens):
    _, (q, k, v), (qf, kf, vf) = _qkv(B, S, H, 2000 + S)
    out, lse = api.cpattn_ring_attention(q, k, v, P, lens)
    torch.cuda.synchronize()
    _no_timeouts()
    ref_o, ref_l = oracle.ring_attention(qf, kf, vf, P, lens)
    assert_close(f64_of(out), f64_of(lse), ref_o, ref_l, f"ring B{B} H{H} S{S} P{P}")
    # the same call twice gives the same bytes
    out2, lse2 = api.cpattn_ring_attention(q, k, v, P, lens)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16)) and torch.equal(lse, lse2)


def test_kv_gather_and_ulysses_over_long_segments_match_oracle():
    B, H, S = 2, 4, 1536
    (qb, kb, vb), (q, k, v), (qf, kf, vf) = _qkv(B, S, H, 2100)
    ref_o, ref_l = oracle.attention(qf, kf, vf)
    o, l = api.cpattn_kv_gather_attention(q, k, v, 2, [1000, 536])
    torch.cuda.synchronize()
    assert_close(f64_of(o), f64_of(l), ref_o, ref_l, "kv_gather")
    seq, heads = [700, 836], [3, 1]
    rq, rk, rv = (to_dev(full_to_rank_buffers(x, seq)) for x in (qb, kb, vb))
    o, l = api.cpattn_ulysses_attention(rq, rk, rv, B, S, H, 128, 2, seq, heads)
    torch.cuda.synchronize()
    assert_close(f64_of(o), f64_of(l), full_to_rank_buffers(ref_o, seq), ref_l, "ulysses (two head groups)")
    _no_timeouts()


def test_ring_chunk_single_step_in_bf16_matches_oracle():
    """A one-chunk ring step written straight to bf16 (no previous state)."""
    B, H, Sq, Skv = 1, 2, 900, 700
    S = Sq + Skv
    (qb, kb, vb), (q, k, v), (qf, kf, vf) = _qkv(B, S, H, 2200)
    q0 = q[:, :Sq].contiguous()
    kc, vc = k[:, Sq:].contiguous(), v[:, Sq:].contiguous()
    out = torch.empty_like(q0)
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device="cuda")
    api.cpattn_ring_chunk_attention(q0, kc, vc, Skv, out, lse)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.attention(qf[:, :Sq], kf[:, Sq:], vf[:, Sq:])
    assert_close(f64_of(out), f64_of(lse), ref_o, ref_l, "ring chunk")
    _no_timeouts()
