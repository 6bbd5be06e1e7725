"""Pins for the backward oracle: torch autograd in float64 (an independent
library routine), central finite differences of <dO, O>, closed forms, and a
planted mistake.  CPU only."""
import math

import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed, scale=1.0):
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.standard_normal(size=shape) * scale


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,S,H,D", [(1, 7, 2, 8), (2, 33, 3, 16)])
def test_backward_matches_torch_autograd_float64(B, S, H, D, causal):
    q, k, v, do = (_rand((B, S, H, D), s) for s in (1, 2, 3, 4))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, causal=causal)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3).clone().requires_grad_(True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
    o.backward(torch.from_numpy(do).permute(0, 2, 1, 3))
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.max(np.abs(mine - ref.permute(0, 2, 1, 3).numpy())) < 1e-11


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_central_differences(causal):
    B, S, H, D = 1, 5, 1, 4
    q, k, v, do = (_rand((B, S, H, D), s) for s in (5, 6, 7, 8))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, causal=causal)
    fwd = oracle.causal_attention if causal else oracle.attention

    def loss(q_, k_, v_):
        return float((fwd(q_, k_, v_)[0] * do).sum())

    h = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for idx in np.ndindex(B, S, H, D):
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            num = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(num - grad[idx]) < 1e-7, (which, idx, num, grad[idx])


def test_constant_values_give_no_query_or_key_gradient():
    """v_j = c for all keys: O = c whatever P is, so dP - Delta = 0 row by
    row and dQ = dK = 0; dV = P^T dO."""
    B, S, H, D = 1, 12, 2, 8
    q, k, do = _rand((B, S, H, D), 9, 2.0), _rand((B, S, H, D), 10, 2.0), _rand((B, S, H, D), 11)
    v = np.broadcast_to(_rand((1, 1, H, D), 12), (B, S, H, D)).copy()
    dq, dk, dv = oracle.attention_backward(q, k, v, do)
    assert np.max(np.abs(dq)) < 1e-13 and np.max(np.abs(dk)) < 1e-13
    # dV column sums: sum_j dV_j = sum_j sum_i P_ij dO_i = sum_i dO_i (rows of P sum to 1)
    assert np.max(np.abs(dv.sum(axis=1) - do.sum(axis=1))) < 1e-12


def test_causal_first_token_has_no_query_gradient():
    """Token 0 sees only key 0: P = 1, O_0 = v_0, so dS_00 = dO_0.(v_0 - O_0) = 0."""
    B, S, H, D = 2, 9, 2, 4
    q, k, v, do = (_rand((B, S, H, D), s) for s in (13, 14, 15, 16))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, causal=True)
    assert np.max(np.abs(dq[:, 0])) < 1e-14
    # the last key is seen only by the last token: dV_{S-1} = P_{S-1,S-1} dO_{S-1}
    s_last = np.einsum("bhd,bjhd->bhj", q[:, -1], k) / math.sqrt(D)
    p_last = np.exp(s_last - s_last.max(axis=-1, keepdims=True))
    p_last /= p_last.sum(axis=-1, keepdims=True)
    assert np.max(np.abs(dv[:, -1] - p_last[:, :, -1][..., None] * do[:, -1])) < 1e-13


def test_planted_missing_scale_is_caught(monkeypatch):
    import importlib
    ob = importlib.import_module("oracle.backward")
    good = ob.attention_backward_rows

    def no_scale(q, k, v, dout, q_pos=None, k_pos=None):
        dq, dk, dv = good(q, k, v, dout, q_pos, k_pos)
        return dq / oracle.softmax_scale(q.shape[1]), dk, dv

    monkeypatch.setattr(ob, "attention_backward_rows", no_scale)
    with pytest.raises(AssertionError):
        test_backward_matches_torch_autograd_float64(1, 7, 2, 8, False)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S,D,block", [(37, 8, 8), (300, 16, 128)])
def test_sampled_backward_matches_torch_autograd_float64(S, D, block, causal):
    """The sampled-row form of the gradient (a blockwise forward for the row
    statistics, then single rows and key columns) against torch autograd in
    float64, over blocks smaller than S with a ragged last block; first,
    last and interior rows, keys and queries sampled separately."""
    q, k, v, do = (_rand((S, D), s) for s in (11, 12, 13, 14))
    q_rows = [0, 1, S // 2, S - 1]
    k_rows = [0, S // 3, S - 2, S - 1]
    dq, dk, dv = oracle.attention_backward_sampled(q, k, v, do, q_rows, k_rows, causal=causal, block=block)
    tq, tk, tv = (torch.from_numpy(x)[None, None].clone().requires_grad_(True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
    o.backward(torch.from_numpy(do)[None, None])
    assert np.max(np.abs(dq - tq.grad[0, 0].numpy()[q_rows])) < 1e-11
    assert np.max(np.abs(dk - tk.grad[0, 0].numpy()[k_rows])) < 1e-11
    assert np.max(np.abs(dv - tv.grad[0, 0].numpy()[k_rows])) < 1e-11
    # and the full-matrix form, row for row
    pos = np.arange(S) if causal else None
    fq, fk, fv = oracle.attention_backward_rows(q, k, v, do, pos, pos)
    assert np.max(np.abs(dq - fq[q_rows])) < 1e-12 and np.max(np.abs(dk - fk[k_rows])) < 1e-12
    assert np.max(np.abs(dv - fv[k_rows])) < 1e-12
