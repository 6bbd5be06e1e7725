"""Parity of the fused Ulysses projections (through the C ABI) with the fp64
oracle: the Q/K/V projection whose epilogue stores the head-sharded layout
(the first all-to-all folded in) and the output projection that reads the
head-sharded attention output in place (the second all-to-all folded in).

Tolerance: each output is an fp32 sum of K bf16 products rounded once to bf16,
so it lies within half a bf16 ulp (2^-9 relative) of the exact value, plus
the fp32 rounding of a K <= 3072 term sum (orders of magnitude smaller).  The
bar is 2^-8 |ref| + 1e-3 max|ref| per element and a mean error below
2e-3 mean|ref|; a wrong head, token or weight row is off by O(1).

Cases span several 128 x 256 tiles, ragged rows (B*S not a multiple of 128)
and columns (3*H*D or Dm not a multiple of 256), uneven and empty ranks,
D = 64 and 128, degree 1..4, and the image-DiT projections (Dm = 3072) on
sampled tokens."""
import numpy as np
import pytest
import torch

import oracle
from context_attention_long_b200 import api, build, inputs

from gpu_util import bits_of, f64_of, sample_positions, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def assert_proj_close(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-3 * np.abs(ref).max()
    bad = np.argwhere(err > bound)
    if bad.size:
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} elements out of bound, first at {i}: got {got[i]}, ref {ref[i]}")
    assert err.mean() <= 2e-3 * np.abs(ref).mean(), f"{what}: mean-abs {err.mean():.3e}"


def _no_timeouts():
    st, code = api.cpattn_device_status()
    assert st == 0 and code == 0, f"device wait expired: code {code:#x}"


CASES = [
    # B, S, H, D, Dm, degree, seq_splits, head_splits
    (1, 256, 4, 128, 512, 2, None, None),
    (2, 300, 6, 64, 384, 3, [100, 50, 150], [3, 2, 1]),
    (1, 1000, 5, 128, 640, 4, [250, 0, 500, 250], [2, 0, 2, 1]),
    (1, 129, 3, 64, 64, 1, None, None),
    (3, 77, 2, 128, 1024, 2, [40, 37], [1, 1]),
]


def _splits(total, degree, splits):
    return list(splits) if splits is not None else [total // degree] * degree


@pytest.mark.parametrize("B,S,H,D,Dm,P,seq,heads", CASES)
def test_qkv_projection_matches_oracle(B, S, H, D, Dm, P, seq, heads):
    xb, wb, _ = inputs.make_projection_inputs(B, S, H, D, Dm, 500 + S)
    ys = api.cpattn_ulysses_qkv_projection(to_dev(xb), to_dev(wb), B, S, H, D, Dm, P, seq, heads)
    torch.cuda.synchronize()
    _no_timeouts()
    refs = oracle.ulysses_qkv_projection(inputs.bf16_bits_to_f64(xb).reshape(-1), inputs.bf16_bits_to_f64(wb),
                                         B, S, H, D, Dm, P, seq, heads)
    for t, (y, ref) in enumerate(zip(ys, refs)):
        assert_proj_close(f64_of(y), ref, f"qkv projection tensor {t} B{B} S{S} H{H} D{D} Dm{Dm} P{P}")


@pytest.mark.parametrize("B,S,H,D,Dm,P,seq,heads", CASES)
def test_output_projection_matches_oracle(B, S, H, D, Dm, P, seq, heads):
    _, _, wob = inputs.make_projection_inputs(B, S, H, D, Dm, 600 + S)
    yob, _, _ = inputs.make_qkv(B, S, H, D, 700 + S, False)   # any head-side bf16 values
    yob = yob.reshape(-1)
    out = api.cpattn_ulysses_output_projection(to_dev(yob), to_dev(wob), B, S, H, D, Dm, P, seq, heads)
    torch.cuda.synchronize()
    _no_timeouts()
    ref = oracle.ulysses_output_projection(inputs.bf16_bits_to_f64(yob), inputs.bf16_bits_to_f64(wob),
                                           B, S, H, D, Dm, P, seq, heads)
    assert_proj_close(f64_of(out), ref, f"output projection B{B} S{S} H{H} D{D} Dm{Dm} P{P}")


@pytest.mark.parametrize("B,S,H,D,Dm,P,seq,heads", CASES[1:3])
def test_fused_stores_move_values_only(B, S, H, D, Dm, P, seq, heads):
    """The permuted stores change where a value goes, never the value: the
    fused projection followed by the (bit-exact) unpermute equals the degree-1
    projection bit for bit, and the output projection of permuted input equals
    the degree-1 output projection bit for bit."""
    xb, wb, wob = inputs.make_projection_inputs(B, S, H, D, Dm, 800 + S)
    x, w = to_dev(xb), to_dev(wb)
    seq_l = _splits(S, P, seq)
    # degree 1 reads x in token order; the sharded call reads rank buffers
    x_tok = oracle.token_order_rows(xb.reshape(-1), B, S, Dm, seq_l)
    plain = api.cpattn_ulysses_qkv_projection(to_dev(x_tok), w, B, S, H, D, Dm, 1)
    fused = api.cpattn_ulysses_qkv_projection(x, w, B, S, H, D, Dm, P, seq, heads)
    for t in range(3):
        back = api.cpattn_ulysses_unpermute(fused[t], B, S, H, D, P, seq, heads)   # sequence side, rank buffers
        back_tok = oracle.token_order_rows(bits_of(back), B, S, H * D, seq_l)
        assert np.array_equal(back_tok.reshape(-1), bits_of(plain[t])), f"tensor {t}"
    yob, _, _ = inputs.make_qkv(B, S, H, D, 900 + S, False)
    yo_tok = to_dev(yob.reshape(-1))                       # degree-1 head side = token order
    # head side for degree P: permute the token-order tensor cut into sequence-side rank buffers
    cuts = np.cumsum([0] + seq_l)
    seq_side = to_dev(np.concatenate([np.ascontiguousarray(yob[:, cuts[r]:cuts[r + 1]]).reshape(-1)
                                      for r in range(P)]))
    yo_heads = api.cpattn_ulysses_permute(seq_side, B, S, H, D, P, seq, heads)
    wo = to_dev(wob)
    o_plain = api.cpattn_ulysses_output_projection(yo_tok, wo, B, S, H, D, Dm, 1)
    o_fused = api.cpattn_ulysses_output_projection(yo_heads, wo, B, S, H, D, Dm, P, seq, heads)
    torch.cuda.synchronize()
    _no_timeouts()
    o_tok = oracle.token_order_rows(bits_of(o_fused), B, S, Dm, seq_l)
    assert np.array_equal(o_tok.reshape(-1), bits_of(o_plain))


def test_dit_projections_sampled():
    """Image-DiT sizes: B1 S4608 H24 D128, model width 3072, Ulysses degree 4;
    every head of sampled tokens (shard edges and random) against the oracle's
    projection of those rows."""
    B, S, H, D, Dm, P = 1, 4608, 24, 128, 3072, 4
    xb, wb, wob = inputs.make_projection_inputs(B, S, H, D, Dm, 1235)
    yq, yk, yv = api.cpattn_ulysses_qkv_projection(to_dev(xb), to_dev(wb), B, S, H, D, Dm, P)
    pos = sample_positions(S, list(range(0, S + 1, S // P)), 24, 5)
    x_rows = inputs.bf16_bits_to_f64(xb)[pos]                      # B = 1: sequence side = token order
    ref = oracle.project_rows(x_rows, inputs.bf16_bits_to_f64(wb)).reshape(len(pos), 3, H, D)
    Hu = H // P
    for t, y in enumerate((yq, yk, yv)):
        full = np.concatenate([f64_of(y).reshape(P, B, S, Hu, D)[u] for u in range(P)], axis=2)   # (B, S, H, D)
        assert_proj_close(full[0, pos], ref[:, t], f"dit qkv projection tensor {t}")
    # output projection of the head-side Q, read in place
    out = api.cpattn_ulysses_output_projection(yq, to_dev(wob), B, S, H, D, Dm, P)
    torch.cuda.synchronize()
    _no_timeouts()
    o_heads = np.concatenate([f64_of(yq).reshape(P, B, S, Hu, D)[u] for u in range(P)], axis=2)
    ref_o = oracle.project_rows(o_heads[0, pos].reshape(len(pos), H * D), inputs.bf16_bits_to_f64(wob))
    assert_proj_close(f64_of(out).reshape(S, Dm)[pos], ref_o, "dit output projection")
