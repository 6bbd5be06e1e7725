"""Seeded random configurations for every attention path against the oracle:
batch, heads, sequence length, head dimension, degrees and uneven splits
(zeros and one-token chunks included) are drawn from a fixed seed, so a
failure is reproducible from its case number.  Small sizes keep the oracle
fast; many cases exercise the planner's segment/tile/split logic."""
import numpy as np
import pytest
import torch

import oracle
from context_attention_long_b200 import api, build, inputs

from gpu_util import assert_close, f64_of, full_to_rank_buffers, rank_buffers_to_full, to_dev

pytestmark = pytest.mark.gpu

N_CASES = 64


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _case(i):
    rng = np.random.Generator(np.random.PCG64(9000 + i))
    B = int(rng.integers(1, 3))
    H = int(rng.integers(1, 6))
    S = int(rng.integers(1, 700))
    D = int(rng.choice([64, 128]))
    P = int(rng.integers(1, min(8, S) + 1))
    lens = inputs.random_splits(S, P, 9100 + i) if rng.random() < 0.7 else None
    if lens is None and S % P:
        lens = inputs.random_splits(S, P, 9200 + i)
    causal = bool(rng.random() < 0.5)
    return B, H, S, D, P, lens, causal


@pytest.mark.parametrize("i", range(N_CASES))
def test_fuzz_ring_paths(i):
    B, H, S, D, P, lens, causal = _case(i)
    qb, kb, vb = inputs.make_qkv(B, S, H, D, 9300 + i, D == 128)
    q, k, v = (inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb))
    dq, dk, dv = (to_dev(x) for x in (qb, kb, vb))
    what = f"case {i}: B{B} H{H} S{S} D{D} P{P} lens={lens} causal={causal}"
    ref_o, ref_l = oracle.ring_attention(q, k, v, P, lens, causal=causal)
    fused = api.cpattn_causal_ring_attention if causal else api.cpattn_ring_attention
    o, l = fused(dq, dk, dv, P, lens)
    step = api.cpattn_causal_ring_step if causal else api.cpattn_ring_step
    parts = [step(dq, dk, dv, P, t, lens) for t in range(P)]
    _, mo, ml = api.cpattn_lse_merge(torch.stack([x[0] for x in parts]), torch.stack([x[1] for x in parts]))
    torch.cuda.synchronize()
    st, code = api.cpattn_device_status()
    assert st == 0, f"{what}: device wait expired {code:#x}"
    assert_close(f64_of(o), f64_of(l), ref_o, ref_l, what + " fused")
    assert_close(f64_of(mo), f64_of(ml), ref_o, ref_l, what + " steps+merge")
    if not causal:
        go, gl = api.cpattn_kv_gather_attention(dq, dk, dv, P, lens)
        torch.cuda.synchronize()
        assert_close(f64_of(go), f64_of(gl), ref_o, ref_l, what + " kv_gather")


@pytest.mark.parametrize("i", range(N_CASES))
def test_fuzz_ulysses_and_unified(i):
    B, H, S, D, P, lens, causal = _case(i)
    rng = np.random.Generator(np.random.PCG64(9400 + i))
    U = int(rng.integers(1, min(H, 4) + 1))
    seq = inputs.random_splits(S, U, 9500 + i)
    heads = inputs.random_splits(H, U, 9600 + i)
    qb, kb, vb = inputs.make_qkv(B, S, H, D, 9700 + i, D == 128)
    q, k, v = (inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb))
    what = f"case {i}: B{B} H{H} S{S} D{D} U{U} seq={seq} heads={heads} causal={causal}"
    ref_o, ref_l = (oracle.causal_attention(q, k, v) if causal else oracle.attention(q, k, v))
    flat = [to_dev(full_to_rank_buffers(x, seq)) for x in (qb, kb, vb)]
    fn = api.cpattn_causal_ulysses_attention if causal else api.cpattn_ulysses_attention
    uo, ul = fn(*flat, B, S, H, D, U, seq, heads)
    # unified: the ring lengths of this case (or an equal split) over U head groups
    R = P if P <= 64 else 1
    ring_lens = lens or [S // R] * R
    dq, dk, dv = (to_dev(x) for x in (qb, kb, vb))
    fu = api.cpattn_causal_unified_attention if causal else api.cpattn_unified_attention
    fo, fl = fu(dq, dk, dv, R, U, ring_lens, heads)
    torch.cuda.synchronize()
    st, code = api.cpattn_device_status()
    assert st == 0, f"{what}: device wait expired {code:#x}"
    assert_close(rank_buffers_to_full(f64_of(uo), B, S, H, D, seq), f64_of(ul), ref_o, ref_l, what + " ulysses")
    assert_close(f64_of(fo), f64_of(fl), ref_o, ref_l, what + f" unified R{R} ring_lens={ring_lens}")


def _bwd_case(i):
    rng = np.random.Generator(np.random.PCG64(9500 + i))
    B = int(rng.integers(1, 3))
    H = int(rng.integers(1, 5))
    S = int(rng.integers(1, 700))
    D = int(rng.choice([64, 128]))
    causal = bool(rng.random() < 0.5)
    return B, H, S, D, causal


@pytest.mark.parametrize("i", range(32))
def test_fuzz_backward(i):
    """The attention backward on seeded random shapes (walks of 1 to 6 tiles,
    shorter than and past the three-stage load ring, ragged tails) against
    the fp64 backward oracle, each gradient relative to its largest entry."""
    B, H, S, D, causal = _bwd_case(i)
    qb, kb, vb = inputs.make_qkv(B, S, H, D, 9600 + i, D == 128)
    rng = np.random.Generator(np.random.PCG64(9700 + i))
    dob = inputs.f32_to_bf16_bits(rng.standard_normal((B, S, H, D)).astype(np.float32))
    dq_, dk_, dv_, do_ = (to_dev(x) for x in (qb, kb, vb, dob))
    fwd = api.cpattn_causal_ring_attention if causal else api.cpattn_ring_attention
    out, lse = fwd(dq_, dk_, dv_, 1)
    grads = api.cpattn_attention_backward(dq_, dk_, dv_, out, lse, do_, causal=causal)
    torch.cuda.synchronize()
    st, code = api.cpattn_device_status()
    what = f"case {i}: B{B} H{H} S{S} D{D} causal={causal}"
    assert st == 0, f"{what}: device wait expired {code:#x}"
    refs = oracle.attention_backward(*(inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb, dob)), causal=causal)
    dmax = np.abs(inputs.bf16_bits_to_f64(dob)).max()
    for name, got, ref in zip(("dq", "dk", "dv"), grads, refs):
        # floored at 2^-10 of max|dO|: a single visible key makes dQ = dK = 0 exactly
        g = max(np.max(np.abs(ref)), 2.0 ** -10 * dmax, 1e-30)
        err = np.abs(f64_of(got) - ref)
        assert np.all(np.isfinite(f64_of(got))), f"{what} {name}: non-finite"
        assert err.max() <= 2e-2 * g and err.mean() <= 2e-3 * g, f"{what} {name}: max-abs {err.max():.3e} vs {g:.3e}"


@pytest.mark.parametrize("i", range(16))
def test_fuzz_ulysses_backward(i):
    """The backward of the Ulysses flow on seeded random shapes, sequence
    splits and head splits (ranks without tokens or heads included), causal
    and not: the gradients stored straight into the sequence-sharded rank
    buffers against the fp64 backward oracle; the path (dQ GEMM with every
    head at once, in groups of one head, or the dQ kernel) rotates with i."""
    B, H, S, D, causal = _bwd_case(200 + i)
    rng = np.random.Generator(np.random.PCG64(9900 + i))
    U = int(rng.integers(2, min(H, 4) + 1)) if H >= 2 else 1
    seq = inputs.random_splits(S, U, 9910 + i)
    heads = inputs.random_splits(H, U, 9920 + i)
    qb, kb, vb = inputs.make_qkv(B, S, H, D, 9930 + i, D == 128)
    dob = inputs.f32_to_bf16_bits(rng.standard_normal((B, S, H, D)).astype(np.float32))
    q, k, v, do = (to_dev(full_to_rank_buffers(x, seq)) for x in (qb, kb, vb, dob))
    fwd = api.cpattn_causal_ulysses_attention if causal else api.cpattn_ulysses_attention
    out, lse = fwd(q, k, v, B, S, H, D, U, seq, heads)
    budget = [None, api.cpattn_attention_backward_ds_bytes(B, S, causal), 0][i % 3]
    grads = api.cpattn_ulysses_attention_backward(q, k, v, out, lse, do, B, S, H, D, U, seq, heads, causal,
                                                  ds_budget=budget)
    torch.cuda.synchronize()
    st, code = api.cpattn_device_status()
    what = f"case {i}: B{B} H{H} S{S} D{D} U{U} seq={seq} heads={heads} causal={causal} budget={budget}"
    assert st == 0, f"{what}: device wait expired {code:#x}"
    refs = oracle.attention_backward(*(inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb, dob)), causal=causal)
    dmax = np.abs(inputs.bf16_bits_to_f64(dob)).max()
    for name, got, ref in zip(("dq", "dk", "dv"), grads, refs):
        full = rank_buffers_to_full(f64_of(got), B, S, H, D, seq)
        g = max(np.max(np.abs(ref)), 2.0 ** -10 * dmax, 1e-30)   # a single visible key makes dQ = dK = 0 exactly
        err = np.abs(full - ref)
        assert np.all(np.isfinite(full)), f"{what} {name}: non-finite"
        assert err.max() <= 2e-2 * g and err.mean() <= 2e-3 * g, f"{what} {name}: max-abs {err.max():.3e} vs {g:.3e}"
