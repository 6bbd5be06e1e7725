"""Parity of the attention backward (through the C ABI) with the fp64
backward oracle: dQ, dK and dV for seeded inputs and a seeded upstream
gradient, causal and not, over tile-spanning and ragged shapes, D = 64 and
128, S = 1, and the image-DiT workload on sampled rows.  The forward output
and LSE come from the library's own forward.  Each small case runs on the
backward's three paths: dS stored by the dK/dV kernel and read by the dQ GEMM
with every head in one group, the same in groups of one head (a workspace
with one head's dS scratch), and the dQ kernel that recomputes S and dP (no
scratch).

Tolerance: every gradient is compared relative to its largest reference
entry g = max|ref|: max-abs error <= 2e-2 * g and mean-abs error <= 2e-3 * g.
P and dS are rounded to bf16 (relative 2^-9) before their MMAs and the
gradients are stored in bf16, as the forward's output is, so the bar is the
forward's bar scaled to the gradient's size."""
import numpy as np
import pytest
import torch

import oracle
from context_attention_long_b200 import api, build, inputs

from gpu_util import f64_of, full_to_rank_buffers, rank_buffers_to_full, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _no_timeouts():
    st, code = api.cpattn_device_status()
    assert st == 0 and code == 0, f"device wait expired: code {code:#x}"


def assert_grad_close(got, ref, what, dout_max=1.0):
    """Relative to the largest reference entry g, floored at 2^-10 of the
    upstream gradient's largest entry: a query with a single visible key has
    dQ = dK = 0 exactly (the softmax of one score is constant), and the fp32
    sums dO.V and rowsum(dO*O) then leave rounding residues far below the
    bf16 resolution of any gradient entry of dO's order."""
    got, ref = np.asarray(got, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    g = max(np.max(np.abs(ref)) if ref.size else 0.0, 2.0 ** -10 * dout_max, 1e-30)
    err = np.abs(got - ref)
    assert err.max() <= 2e-2 * g, f"{what}: max-abs {err.max():.3e} vs {g:.3e}"
    assert err.mean() <= 2e-3 * g, f"{what}: mean-abs {err.mean():.3e} vs {g:.3e}"


# ds_budget of each path (None: the binding's default, every head at once here;
# "one": one head's dS scratch, so the heads run in groups of one)
PATHS = {"gemm": None, "gemm_groups": "one", "dq_kernel": 0}


def _budget(path, B, S, causal):
    b = PATHS[path]
    return api.cpattn_attention_backward_ds_bytes(B, S, causal) if b == "one" else b


def _run(B, S, H, D, causal, seed, path="gemm"):
    qb, kb, vb = inputs.make_qkv(B, S, H, D, seed, D == 128)
    rng = np.random.Generator(np.random.PCG64(seed + 1))
    dob = inputs.f32_to_bf16_bits(rng.standard_normal((B, S, H, D)).astype(np.float32))
    q, k, v, do = (to_dev(x) for x in (qb, kb, vb, dob))
    fwd = api.cpattn_causal_ring_attention if causal else api.cpattn_ring_attention
    out, lse = fwd(q, k, v, 1)
    dq, dk, dv = api.cpattn_attention_backward(q, k, v, out, lse, do, causal=causal,
                                               ds_budget=_budget(path, B, S, causal))
    torch.cuda.synchronize()
    _no_timeouts()
    return (qb, kb, vb, dob), (dq, dk, dv)


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,S,H,D", [(1, 256, 2, 64), (2, 300, 3, 128), (1, 129, 2, 128), (1, 1, 1, 64),
                                     (1, 640, 2, 128)])
def test_backward_matches_oracle(B, S, H, D, causal, path):
    bits, grads = _run(B, S, H, D, causal, 31 + S, path)
    q, k, v, do = (inputs.bf16_bits_to_f64(x) for x in bits)
    refs = oracle.attention_backward(q, k, v, do, causal=causal)
    for name, got, ref in zip(("dq", "dk", "dv"), grads, refs):
        assert_grad_close(f64_of(got), ref, f"{name} B{B} S{S} H{H} D{D} causal={causal}", np.abs(do).max())


@pytest.mark.parametrize("causal", [False, True])
def test_backward_dit_workload_sampled_heads(causal):
    """Image-DiT shapes (B1 H24 S4608 D128) in full on the GPU; the oracle
    checks three heads in full (its cost grows with S^2 per head)."""
    cfg, qb, kb, vb = inputs.config_inputs("dit")
    B, S, H, D = qb.shape
    rng = np.random.Generator(np.random.PCG64(77))
    dob = inputs.f32_to_bf16_bits(rng.standard_normal((B, S, H, D)).astype(np.float32))
    q, k, v, do = (to_dev(x) for x in (qb, kb, vb, dob))
    fwd = api.cpattn_causal_ring_attention if causal else api.cpattn_ring_attention
    out, lse = fwd(q, k, v, cfg["ring_degree"])
    dq, dk, dv = api.cpattn_attention_backward(q, k, v, out, lse, do, causal=causal)
    torch.cuda.synchronize()
    _no_timeouts()
    pos = np.arange(S) if causal else None
    for h in (0, 11, 23):
        ref = oracle.attention_backward_rows(*(inputs.bf16_bits_to_f64(x[0, :, h]) for x in (qb, kb, vb, dob)),
                                             pos, pos)
        for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            assert_grad_close(f64_of(got)[0, :, h], r, f"dit {name} head {h} causal={causal}",
                              np.abs(inputs.bf16_bits_to_f64(dob)).max())


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,S,H,D", [(2, 300, 5, 128), (1, 520, 3, 64)])
def test_backward_paths_agree(B, S, H, D, causal):
    """dK and dV come from the same dK/dV kernel on every path: the same
    bytes.  dQ from the GEMM reads the same stored dS tiles whatever the
    grouping of the heads: the same bytes too.  The dQ kernel forms its own dS
    (checked against the oracle above)."""
    runs = {path: _run(B, S, H, D, causal, 300 + S, path)[1] for path in PATHS}
    two = api.cpattn_attention_backward_ds_bytes(B, S, causal) * 2

    def bits(t):
        return t.view(torch.int16)

    for path, (dq, dk, dv) in runs.items():
        assert torch.equal(bits(dk), bits(runs["gemm"][1])), f"dk {path}"
        assert torch.equal(bits(dv), bits(runs["gemm"][2])), f"dv {path}"
    assert torch.equal(bits(runs["gemm_groups"][0]), bits(runs["gemm"][0]))
    # groups of two heads (the last group holds one when H is odd)
    qb, kb, vb = inputs.make_qkv(B, S, H, D, 300 + S, D == 128)
    rng = np.random.Generator(np.random.PCG64(301 + S))
    dob = inputs.f32_to_bf16_bits(rng.standard_normal((B, S, H, D)).astype(np.float32))
    q, k, v, do = (to_dev(x) for x in (qb, kb, vb, dob))
    fwd = api.cpattn_causal_ring_attention if causal else api.cpattn_ring_attention
    out, lse = fwd(q, k, v, 1)
    g2 = api.cpattn_attention_backward(q, k, v, out, lse, do, causal=causal, ds_budget=two)
    torch.cuda.synchronize()
    _no_timeouts()
    for a, b in zip(g2, runs["gemm"]):
        assert torch.equal(bits(a), bits(b))


@pytest.mark.parametrize("causal", [False, True])
def test_backward_video_workload_sampled(causal):
    """Video shapes (B1 H40 S32760 D128), the largest configuration, on the
    default path: the bindings' dS budget holds 4 of the 40 heads (7 under
    the causal mask), so the backward runs in 10 (6) head groups.  The oracle
    checks sampled rows (tile edges, the ends, seeded interior rows) of heads
    0 and 39, in the first and the last group."""
    cfg, qb, kb, vb = inputs.config_inputs("video")
    B, S, H, D = qb.shape
    per = api.cpattn_attention_backward_ds_bytes(B, S, causal)
    assert api.BACKWARD_DS_BUDGET // per < H        # several head groups
    rng = np.random.Generator(np.random.PCG64(78))
    dob = inputs.f32_to_bf16_bits(rng.standard_normal((B, S, H, D)).astype(np.float32))
    q, k, v, do = (to_dev(x) for x in (qb, kb, vb, dob))
    fwd = api.cpattn_causal_ring_attention if causal else api.cpattn_ring_attention
    out, lse = fwd(q, k, v, cfg["ring_degree"])
    dq, dk, dv = api.cpattn_attention_backward(q, k, v, out, lse, do, causal=causal)
    torch.cuda.synchronize()
    _no_timeouts()
    rows = sorted({0, 1, 127, 128, 4095, 4096, S // 2, S - 129, S - 128, S - 2, S - 1} |
                  {int(x) for x in rng.integers(0, S, size=8)})
    dmax = np.abs(inputs.bf16_bits_to_f64(dob)).max()
    for h in (0, H - 1):
        ref = oracle.attention_backward_sampled(*(inputs.bf16_bits_to_f64(x[0, :, h]) for x in (qb, kb, vb, dob)),
                                                rows, rows, causal=causal)
        for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            assert_grad_close(f64_of(got[0, rows, h]), r, f"video {name} head {h} causal={causal}", dmax)


def test_backward_is_deterministic_and_validates():
    bits, g1 = _run(1, 384, 2, 128, True, 5)
    _, g2 = _run(1, 384, 2, 128, True, 5)
    for a, b in zip(g1, g2):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    lib = api._native.load()
    F = g1[0].data_ptr()
    assert lib.cpattn_attention_backward(F, F, F, F, None, F, F, F, F, 1, 2, 384, 128, 0, F, 1 << 20, None) == 1
    assert lib.cpattn_attention_backward(F, F, F, F, F, F, F, F, F, 1, 2, 384, 128, 0, F, 16, None) == 8


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("B,S,H,D,P,seq,heads,causal", [
    (1, 256, 4, 64, 2, None, None, False),
    (2, 300, 7, 128, 3, [100, 50, 150], [3, 2, 2], True),
    (1, 1000, 6, 128, 4, [250, 250, 250, 250], [2, 2, 1, 1], False),
    (1, 320, 10, 64, 10, None, None, True),     # 10 head ranks: more problems than one launch holds
])
def test_ulysses_backward_matches_oracle(B, S, H, D, P, seq, heads, causal, path):
    """The backward of the Ulysses flow on sequence-sharded rank buffers, with
    the forward's output and LSE from the Ulysses forward, on each path."""
    seq_l = seq or [S // P] * P
    qb, kb, vb = inputs.make_qkv(B, S, H, D, 90 + S, D == 128)
    rng = np.random.Generator(np.random.PCG64(91 + S))
    dob = inputs.f32_to_bf16_bits(rng.standard_normal((B, S, H, D)).astype(np.float32))
    q, k, v, do = (to_dev(full_to_rank_buffers(x, seq_l)) for x in (qb, kb, vb, dob))
    fwd = api.cpattn_causal_ulysses_attention if causal else api.cpattn_ulysses_attention
    out, lse = fwd(q, k, v, B, S, H, D, P, seq, heads)
    dq, dk, dv = api.cpattn_ulysses_attention_backward(q, k, v, out, lse, do, B, S, H, D, P, seq, heads, causal,
                                                       ds_budget=_budget(path, B, S, causal))
    torch.cuda.synchronize()
    _no_timeouts()
    refs = oracle.attention_backward(*(inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb, dob)), causal=causal)
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        full = rank_buffers_to_full(f64_of(got), B, S, H, D, seq_l)
        assert_grad_close(full, ref, f"ulysses {name} B{B} S{S} H{H} P{P} causal={causal}",
                          np.abs(inputs.bf16_bits_to_f64(dob)).max())
