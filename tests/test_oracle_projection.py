"""Pins of the projection oracle (oracle/projection.py) to things other than
itself: brute-force matrix products, identity weights that reduce the fused
step to the bare all-to-all, a head-side layout read off element by element,
and the unsharded composition X W_q^T W_o^T.  A planted mistake (Q and K
blocks swapped; the weight used untransposed) fails the element-wise pin."""
import numpy as np
import pytest

import oracle
from oracle.projection import project_rows, token_order_rows

from context_attention_long_b200 import inputs

CASES = [
    # B, S, H, D, Dm, degree, seq_splits, head_splits
    (1, 8, 2, 4, 8, 2, None, None),
    (2, 7, 3, 4, 12, 3, [3, 0, 4], [1, 2, 0]),
    (2, 9, 5, 2, 6, 4, [2, 3, 0, 4], [2, 1, 1, 1]),
    (1, 5, 4, 3, 10, 1, None, None),
]


def _weights(B, S, H, D, Dm, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.integers(-3, 4, size=(B * S, Dm)).astype(np.float64)
    w_qkv = rng.integers(-2, 3, size=(3 * H * D, Dm)).astype(np.float64)
    w_o = rng.integers(-2, 3, size=(Dm, H * D)).astype(np.float64)
    return x, w_qkv, w_o


def _splits(total, degree, splits):
    return list(splits) if splits is not None else [total // degree] * degree


def test_project_rows_is_the_matrix_product():
    rng = np.random.Generator(np.random.PCG64(5))
    x = rng.integers(-4, 5, size=(6, 5)).astype(np.float64)
    w = rng.integers(-4, 5, size=(3, 5)).astype(np.float64)
    y = project_rows(x, w)
    for i in range(6):
        for j in range(3):
            assert y[i, j] == sum(x[i, k] * w[j, k] for k in range(5))


def _head_side_matches(ys, x, w_qkv, B, S, H, D, Dm, P, seq, heads):
    """yq/yk/yv rank u buffer (B, S, H_u, D) at (b, s, hl, d) holds
    sum_k x[token (b, s), k] * w_qkv[t*H*D + (hoff_u + hl)*D + d, k], with the
    sequence-side rows of x in rank-buffer order."""
    seq_l, heads_l = _splits(S, P, seq), _splits(H, P, heads)
    x_tok = token_order_rows(x.reshape(-1), B, S, Dm, seq_l).reshape(B, S, Dm)
    hoff = np.concatenate([[0], np.cumsum(heads_l)])
    for t in range(3):
        pos = 0
        for u in range(P):
            Hu = heads_l[u]
            buf = ys[t][pos:pos + B * S * Hu * D].reshape(B, S, Hu, D)
            pos += B * S * Hu * D
            for b in range(B):
                for s in range(S):
                    for hl in range(Hu):
                        h = hoff[u] + hl
                        for d in range(D):
                            row = w_qkv[t * H * D + h * D + d]
                            if buf[b, s, hl, d] != float(sum(x_tok[b, s, k] * row[k] for k in range(Dm))):
                                return False
    return True


@pytest.mark.parametrize("B,S,H,D,Dm,P,seq,heads", CASES)
def test_qkv_projection_head_side_element_by_element(B, S, H, D, Dm, P, seq, heads):
    x, w_qkv, _ = _weights(B, S, H, D, Dm, 11 + S)
    ys = oracle.ulysses_qkv_projection(x.reshape(-1), w_qkv, B, S, H, D, Dm, P, seq, heads)
    assert _head_side_matches(ys, x, w_qkv, B, S, H, D, Dm, P, seq, heads)


@pytest.mark.parametrize("B,S,H,D,Dm,P,seq,heads", CASES)
def test_identity_weights_reduce_to_the_permute(B, S, H, D, Dm, P, seq, heads):
    """With W_qkv = [I; 2I; 3I] (Dm = H*D) the step is the bare first
    all-to-all (times 1, 2, 3); with W_o = I the output step is the bare
    second all-to-all."""
    Dm = H * D
    rng = np.random.Generator(np.random.PCG64(21))
    x = rng.integers(-5, 6, size=B * S * Dm).astype(np.float64)
    eye = np.eye(Dm)
    yq, yk, yv = oracle.ulysses_qkv_projection(x, np.concatenate([eye, 2 * eye, 3 * eye]), B, S, H, D, Dm, P,
                                               seq, heads)
    perm = oracle.ulysses_permute(x, B, S, H, D, P, seq, heads)
    assert np.array_equal(yq, perm) and np.array_equal(yk, 2 * perm) and np.array_equal(yv, 3 * perm)
    out = oracle.ulysses_output_projection(perm, eye, B, S, H, D, Dm, P, seq, heads)
    assert np.array_equal(out, x)


@pytest.mark.parametrize("B,S,H,D,Dm,P,seq,heads", CASES)
def test_projection_round_trip_is_the_unsharded_composition(B, S, H, D, Dm, P, seq, heads):
    """Output projection of the head-side Q equals X W_q^T W_o^T token by
    token, with no exchange at all."""
    x, w_qkv, w_o = _weights(B, S, H, D, Dm, 31 + S)
    seq_l = _splits(S, P, seq)
    yq, _, _ = oracle.ulysses_qkv_projection(x.reshape(-1), w_qkv, B, S, H, D, Dm, P, seq, heads)
    out = oracle.ulysses_output_projection(yq, w_o, B, S, H, D, Dm, P, seq, heads)
    x_tok = token_order_rows(x.reshape(-1), B, S, Dm, seq_l)
    ref = x_tok @ w_qkv[:H * D].T @ w_o.T
    assert np.array_equal(token_order_rows(out, B, S, Dm, seq_l), ref)


def test_token_order_rows_reorders_rank_buffers():
    # B = 2, splits [1, 2]: rank 0 holds (b0 s0), (b1 s0); rank 1 holds (b0 s1), (b0 s2), (b1 s1), (b1 s2)
    flat = np.array([0, 3, 1, 2, 4, 5], dtype=np.float64)
    got = token_order_rows(flat, 2, 3, 1, [1, 2]).reshape(-1)
    assert np.array_equal(got, [0, 1, 2, 3, 4, 5])


def test_planted_mistakes_fail_the_element_pin(monkeypatch):
    """The element-wise pin rejects plausible slips planted in the oracle: Q
    and K blocks swapped, the weight used untransposed, heads taken in the
    wrong rank order."""
    import oracle.projection as proj
    B, S, H, D, Dm, P, seq, heads = 2, 7, 3, 4, 12, 3, [3, 0, 4], [1, 2, 0]
    x, w_qkv, _ = _weights(B, S, H, D, Dm, 7)
    good = proj.ulysses_qkv_projection(x.reshape(-1), w_qkv, B, S, H, D, Dm, P, seq, heads)
    assert _head_side_matches(good, x, w_qkv, B, S, H, D, Dm, P, seq, heads)
    swapped = np.concatenate([w_qkv[H * D:2 * H * D], w_qkv[:H * D], w_qkv[2 * H * D:]])
    bad = proj.ulysses_qkv_projection(x.reshape(-1), swapped, B, S, H, D, Dm, P, seq, heads)
    assert not _head_side_matches(bad, x, w_qkv, B, S, H, D, Dm, P, seq, heads)
    # untransposed weight: x (rows, Dm) times W (N, Dm) read as (Dm, N) -- planted on a square-free shape
    monkeypatch.setattr(proj, "project_rows",
                        lambda a, w: np.asarray(a, np.float64) @ np.asarray(w, np.float64).reshape(-1, w.shape[0]))
    bad = proj.ulysses_qkv_projection(x.reshape(-1), w_qkv, B, S, H, D, Dm, P, seq, heads)
    assert not _head_side_matches(bad, x, w_qkv, B, S, H, D, Dm, P, seq, heads)
    monkeypatch.undo()
    bad = proj.ulysses_qkv_projection(x.reshape(-1), w_qkv, B, S, H, D, Dm, P, seq, list(reversed(heads)))
    assert not _head_side_matches(bad, x, w_qkv, B, S, H, D, Dm, P, seq, heads)


def test_projection_inputs_are_seeded_bf16():
    a = inputs.make_projection_inputs(1, 8, 2, 64, 128, 3)
    b = inputs.make_projection_inputs(1, 8, 2, 64, 128, 3)
    assert all(np.array_equal(p, q) for p, q in zip(a, b))
    x, w_qkv, w_o = a
    assert x.shape == (8, 128) and w_qkv.shape == (384, 128) and w_o.shape == (128, 128)
    assert x.dtype == np.uint16
    # weights scaled by 1/sqrt(fan_in): rms near 1/sqrt(128)
    assert 0.07 < np.sqrt(np.mean(inputs.bf16_bits_to_f64(w_qkv) ** 2)) < 0.1
