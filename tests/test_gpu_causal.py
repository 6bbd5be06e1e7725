"""Parity of the causal entry points (through the C ABI) with the fp64 oracle.

Causal masking by sequence positions (the Ulysses Sequence Parallelism
article, section 7): key j is visible to query i iff j <= i.  Cases span
several tiles with ragged tails, chunks shorter than a tile, empty chunks,
split lone tiles, D = 64, S = 1, the ring steps whose chunk lies after the
shard (exact zero output and -inf LSE), the Ulysses and unified flows, and the
image-DiT workload in full."""
import numpy as np
import pytest
import torch

import oracle
from context_attention_long_b200 import api, build, inputs

from gpu_util import (assert_close, bits_of, f64_of, full_to_rank_buffers, rank_buffers_to_full,
                      sample_positions, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _qkv(B, S, H, D, seed, rms=True):
    q, k, v = inputs.make_qkv(B, S, H, D, seed, rms)
    return (q, k, v), tuple(inputs.bf16_bits_to_f64(x) for x in (q, k, v)), tuple(to_dev(x) for x in (q, k, v))


def _no_timeouts():
    st, code = api.cpattn_device_status()
    assert st == 0 and code == 0, f"device wait expired: code {code:#x}"


CAUSAL_RING_CASES = [
    # B, H, S, D, degree, lens
    (1, 2, 256, 64, 4, None),
    (1, 2, 300, 128, 1, None),              # one shard: a pair and a split lone tile
    (2, 3, 300, 128, 3, [100, 0, 200]),     # ragged, an empty chunk
    (1, 1, 1, 64, 1, None),                 # single token
    (1, 2, 129, 128, 2, [1, 128]),          # one-token chunk
    (2, 2, 1000, 128, 4, [250, 250, 250, 250]),
    (1, 4, 777, 64, 5, [7, 300, 0, 270, 200]),
    (1, 3, 640, 128, 8, [64, 100, 36, 128, 129, 0, 120, 63]),
    (1, 2, 1100, 128, 2, [700, 400]),       # several pairs per shard, lone tiles at both ends
]


@pytest.mark.parametrize("B,H,S,D,P,lens", CAUSAL_RING_CASES)
def test_causal_ring_attention_matches_oracle(B, H, S, D, P, lens):
    _, (q, k, v), (dq, dk, dv) = _qkv(B, S, H, D, 700 + S + P, rms=(D == 128))
    out, lse = api.cpattn_causal_ring_attention(dq, dk, dv, P, lens)
    torch.cuda.synchronize()
    _no_timeouts()
    ref_o, ref_l = oracle.ring_attention(q, k, v, P, lens, causal=True)
    assert_close(f64_of(out), f64_of(lse), ref_o, ref_l, f"causal ring B{B} H{H} S{S} D{D} P{P}")


@pytest.mark.parametrize("B,H,S,D,P,lens", [(1, 2, 512, 128, 4, None), (2, 3, 300, 128, 3, [100, 0, 200]),
                                             (1, 2, 777, 64, 5, [7, 300, 0, 270, 200])])
def test_causal_ring_steps_and_merge_match_oracle(B, H, S, D, P, lens):
    _, (q, k, v), (dq, dk, dv) = _qkv(B, S, H, D, 800 + S, rms=(D == 128))
    lens_l = lens or [S // P] * P
    off = oracle.offsets(lens_l)
    parts_o, parts_l = [], []
    for t in range(P):
        po, pl = api.cpattn_causal_ring_step(dq, dk, dv, P, t, lens)
        ro, rl = oracle.ring_step_partials(q, k, v, P, t, lens, causal=True)
        assert_close(f64_of(po), f64_of(pl), ro, rl, f"causal step {t}")
        for r in range(P):
            c = oracle.ring_order(r, P)[t]
            if lens_l[r] > 0 and (c > r or lens_l[c] == 0):   # invisible or empty chunk: the neutral partial
                assert torch.all(po[:, off[r]:off[r + 1]] == 0)
                assert torch.all(torch.isneginf(pl[:, :, off[r]:off[r + 1]]))
        parts_o.append(po)
        parts_l.append(pl)
    _, b16, lse = api.cpattn_lse_merge(torch.stack(parts_o), torch.stack(parts_l))
    torch.cuda.synchronize()
    _no_timeouts()
    ref_o, ref_l = oracle.ring_attention(q, k, v, P, lens, causal=True)
    assert_close(f64_of(b16), f64_of(lse), ref_o, ref_l, "causal merged")


@pytest.mark.parametrize("B,S,H,D,P,seq,heads", [
    (1, 256, 4, 64, 2, None, None),
    (2, 300, 7, 128, 3, [100, 50, 150], [3, 2, 2]),
    (1, 1000, 6, 128, 4, [250, 250, 250, 250], [2, 2, 1, 1]),
])
def test_causal_ulysses_attention_matches_oracle(B, S, H, D, P, seq, heads):
    (qb, kb, vb), (q, k, v), _ = _qkv(B, S, H, D, 900 + S, rms=(D == 128))
    seq_l = seq or [S // P] * P
    flat = [to_dev(full_to_rank_buffers(x, seq_l)) for x in (qb, kb, vb)]
    out, lse = api.cpattn_causal_ulysses_attention(*flat, B, S, H, D, P, seq, heads)
    torch.cuda.synchronize()
    _no_timeouts()
    got = rank_buffers_to_full(f64_of(out), B, S, H, D, seq_l)
    qf, kf, vf = (full_to_rank_buffers(x, seq_l) for x in (q, k, v))
    ref_flat, ref_l = oracle.ulysses_attention(qf, kf, vf, B, S, H, D, P, seq, heads, causal=True)
    ref = rank_buffers_to_full(ref_flat, B, S, H, D, seq_l)
    assert_close(got, f64_of(lse), ref, ref_l, "causal ulysses")
    # the head-sharded step alone, on the permuted buffers
    yq, yk, yv = (api.cpattn_ulysses_permute(x, B, S, H, D, P, seq, heads) for x in flat)
    yo, l2 = api.cpattn_causal_head_sharded_attention(yq, yk, yv, B, S, H, D, P, heads)
    o2 = api.cpattn_ulysses_unpermute(yo, B, S, H, D, P, seq, heads)
    torch.cuda.synchronize()
    assert torch.equal(o2.view(torch.int16), out.view(torch.int16))
    assert torch.equal(l2, lse)


@pytest.mark.parametrize("B,S,H,D,R,U,ring_lens,heads", [
    (1, 256, 4, 64, 2, 2, None, None),
    (2, 500, 4, 128, 3, 2, [200, 0, 300], [3, 1]),
])
def test_causal_unified_attention_matches_oracle(B, S, H, D, R, U, ring_lens, heads):
    _, (q, k, v), (dq, dk, dv) = _qkv(B, S, H, D, 950 + S, rms=(D == 128))
    out, lse = api.cpattn_causal_unified_attention(dq, dk, dv, R, U, ring_lens, heads)
    torch.cuda.synchronize()
    _no_timeouts()
    ref_o, ref_l = oracle.unified_attention(q, k, v, R, U, ring_lens, heads, causal=True)
    assert_close(f64_of(out), f64_of(lse), ref_o, ref_l, "causal unified")


def test_causal_first_token_is_its_value_and_runs_are_deterministic():
    (qb, kb, vb), _, (dq, dk, dv) = _qkv(1, 640, 4, 128, 77)
    o1, l1 = api.cpattn_causal_ring_attention(dq, dk, dv, 4)
    o2, l2 = api.cpattn_causal_ring_attention(dq, dk, dv, 4)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)
    # token 0 sees only key 0: out = v_0 exactly (P = 1, one bf16 value per element)
    assert np.array_equal(bits_of(o1)[:, 0], vb[:, 0])


def test_dit_workload_causal_ring_and_ulysses_full():
    cfg, qb, kb, vb = inputs.config_inputs("dit")
    B, S, H, D = qb.shape
    q, k, v = (inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb))
    dq, dk, dv = (to_dev(x) for x in (qb, kb, vb))
    ref_o, ref_l = oracle.causal_attention(q, k, v)
    o, l = api.cpattn_causal_ring_attention(dq, dk, dv, cfg["ring_degree"])
    assert_close(f64_of(o), f64_of(l), ref_o, ref_l, "dit causal ring")
    o, l = api.cpattn_causal_ulysses_attention(dq.reshape(-1), dk.reshape(-1), dv.reshape(-1), B, S, H, D,
                                               cfg["ulysses_degree"])
    assert_close(f64_of(o).reshape(B, S, H, D), f64_of(l), ref_o, ref_l, "dit causal ulysses")
    _no_timeouts()


def test_hires_workload_causal_ring_sampled():
    cfg, qb, kb, vb = inputs.config_inputs("hires")
    B, S, H, D = qb.shape
    P = cfg["ring_degree"]
    pos = sample_positions(S, list(range(0, S + 1, S // P)), 24, 3)
    o, l = api.cpattn_causal_ring_attention(*(to_dev(x) for x in (qb, kb, vb)), P)
    got_o, got_l = f64_of(o)[:, pos], f64_of(l)[:, :, pos]
    ref_o = np.zeros((B, len(pos), H, D))
    ref_l = np.zeros((B, H, len(pos)))
    kpos = np.arange(S)
    for b in range(B):
        for h in range(H):
            ro, rl = oracle.causal_attention_rows(inputs.bf16_bits_to_f64(qb[b, pos, h]),
                                                  inputs.bf16_bits_to_f64(kb[b, :, h]),
                                                  inputs.bf16_bits_to_f64(vb[b, :, h]), pos, kpos)
            ref_o[b, :, h] = ro
            ref_l[b, h] = rl
    assert_close(got_o, got_l, ref_o, ref_l, "hires causal ring (sampled)")
    _no_timeouts()
