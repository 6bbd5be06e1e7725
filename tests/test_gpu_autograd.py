"""The autograd functions (context_attention_long_b200.autograd) on the GPU:
the forward equals the library's forward byte for byte, and the gradients
that autograd delivers to Q, K and V match the fp64 backward oracle for a
seeded upstream gradient (the same bar as tests/test_gpu_backward.py),
through the fused ring (even and uneven shards, causal and not) and the
Ulysses flow on rank buffers."""
import numpy as np
import pytest
import torch

import oracle
from context_attention_long_b200 import api, autograd, build, inputs

from gpu_util import f64_of, full_to_rank_buffers, rank_buffers_to_full, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _grad_close(got, ref, what, dout_max=1.0):
    # floored at 2^-10 of max|dO|: a single visible key makes dQ = dK = 0 exactly
    g = max(np.max(np.abs(ref)), 2.0 ** -10 * dout_max, 1e-30)
    err = np.abs(np.asarray(got, dtype=np.float64) - ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    assert err.max() <= 2e-2 * g, f"{what}: max-abs {err.max():.3e} vs {g:.3e}"
    assert err.mean() <= 2e-3 * g, f"{what}: mean-abs {err.mean():.3e} vs {g:.3e}"


def _inputs(B, S, H, D, seed):
    qb, kb, vb = inputs.make_qkv(B, S, H, D, seed, D == 128)
    rng = np.random.Generator(np.random.PCG64(seed + 1))
    dob = inputs.f32_to_bf16_bits(rng.standard_normal((B, S, H, D)).astype(np.float32))
    return qb, kb, vb, dob


@pytest.mark.parametrize("B,S,H,D,P,lens,causal", [
    (1, 512, 2, 128, 4, None, False),
    (2, 300, 3, 64, 3, [100, 37, 163], True),
    (1, 640, 2, 128, 2, None, True),
])
def test_ring_attention_autograd_matches_oracle(B, S, H, D, P, lens, causal):
    qb, kb, vb, dob = _inputs(B, S, H, D, 400 + S)
    q, k, v = (to_dev(x).requires_grad_(True) for x in (qb, kb, vb))
    out = autograd.ring_attention(q, k, v, P, causal, lens)
    fwd = api.cpattn_causal_ring_attention if causal else api.cpattn_ring_attention
    ref_out, _ = fwd(q.detach(), k.detach(), v.detach(), P, lens)
    assert torch.equal(out.detach().view(torch.int16), ref_out.view(torch.int16))
    out.backward(to_dev(dob))
    torch.cuda.synchronize()
    refs = oracle.attention_backward(*(inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb, dob)), causal=causal)
    for name, t, ref in zip(("dq", "dk", "dv"), (q, k, v), refs):
        _grad_close(f64_of(t.grad), ref, f"ring {name} S{S} P{P} causal={causal}",
                    np.abs(inputs.bf16_bits_to_f64(dob)).max())
    st, code = api.cpattn_device_status()
    assert st == 0 and code == 0


@pytest.mark.parametrize("B,S,H,D,P,seq,heads,causal", [
    (1, 512, 4, 128, 4, None, None, False),
    (2, 300, 6, 64, 3, [100, 50, 150], [3, 2, 1], True),
])
def test_ulysses_attention_autograd_matches_oracle(B, S, H, D, P, seq, heads, causal):
    seq_l = seq or [S // P] * P
    qb, kb, vb, dob = _inputs(B, S, H, D, 450 + S)
    q, k, v = (to_dev(full_to_rank_buffers(x, seq_l)).requires_grad_(True) for x in (qb, kb, vb))
    out = autograd.ulysses_attention(q, k, v, B, S, H, D, P, seq, heads, causal)
    out.backward(to_dev(full_to_rank_buffers(dob, seq_l)))
    torch.cuda.synchronize()
    refs = oracle.attention_backward(*(inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb, dob)), causal=causal)
    for name, t, ref in zip(("dq", "dk", "dv"), (q, k, v), refs):
        _grad_close(rank_buffers_to_full(f64_of(t.grad), B, S, H, D, seq_l), ref,
                    f"ulysses {name} S{S} P{P} causal={causal}", np.abs(inputs.bf16_bits_to_f64(dob)).max())
    st, code = api.cpattn_device_status()
    assert st == 0 and code == 0
