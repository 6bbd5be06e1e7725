"""Oracle: the gradient of softmax attention (test infrastructure only, float64).

The pages train with Ulysses over long contexts ([USP] sections 1 and 7:
training with million-token contexts, causal masking by position ids), so the
hot path has a backward pass.  The pages print no backward formulas; the
gradient is the plain derivative of the forward definition in
``oracle.attention``, written out per (batch, head) with S = Q K^T * scale,
P = softmax(S) (rows masked by position when causal), O = P V and an upstream
gradient dO of O:
    dV    = P^T dO
    dP    = dO V^T
    Delta = rowsum(dO * O)                 (= rowsum(P * dP))
    dS    = P * (dP - Delta)               (the softmax Jacobian applied to dP)
    dQ    = dS K * scale,   dK = dS^T Q * scale
Rows that see no key (possible only with positions) have P = 0 and give no
gradient.
"""
from __future__ import annotations

import numpy as np

from .attention import softmax_scale


def attention_backward_rows(q, k, v, dout, q_pos=None, k_pos=None):
    """Gradient for one (batch, head): q (n, D), k and v (m, D), dout (n, D).
    Returns dq (n, D), dk (m, D), dv (m, D)."""
    n, D = q.shape
    m = k.shape[0]
    scale = softmax_scale(D)
    s = (q @ k.T) * scale
    if q_pos is not None:
        visible = np.asarray(k_pos)[None, :] <= np.asarray(q_pos)[:, None]
    else:
        visible = np.ones((n, m), dtype=bool)
    s = np.where(visible, s, -np.inf)
    seen = visible.any(axis=1)
    row_max = np.where(seen, s.max(axis=1, initial=-np.inf), 0.0)[:, None]
    e = np.where(visible, np.exp(s - row_max), 0.0)
    ell = e.sum(axis=1, keepdims=True)
    p = np.where(ell > 0, e / np.where(ell > 0, ell, 1.0), 0.0)
    o = p @ v
    dv = p.T @ dout
    dp = dout @ v.T
    delta = (dout * o).sum(axis=1, keepdims=True)
    ds = p * (dp - delta)
    dq = (ds @ k) * scale
    dk = (ds.T @ q) * scale
    return dq, dk, dv


def attention_backward(q, k, v, dout, causal=False):
    """Gradient of attention over full (B, S, H, D) tensors with respect to q,
    k and v, given the upstream gradient dout of the output; causal: the
    position mask of ``oracle.causal_attention`` (token i sees keys 0..i).
    The ring, Ulysses and unified paths compute the same attention, so this is
    their gradient too."""
    B, S, H, D = q.shape
    dq = np.zeros_like(q, dtype=np.float64)
    dk = np.zeros_like(k, dtype=np.float64)
    dv = np.zeros_like(v, dtype=np.float64)
    pos = np.arange(S) if causal else None
    for b in range(B):
        for h in range(H):
            g = attention_backward_rows(q[b, :, h], k[b, :, h], v[b, :, h], dout[b, :, h], pos, pos)
            dq[b, :, h], dk[b, :, h], dv[b, :, h] = g
    return dq, dk, dv


def attention_backward_sampled(q, k, v, dout, q_rows, k_rows, causal=False, block=1024):
    """The same gradient for one (batch, head) of a long sequence, at sampled
    rows only: q, k, v, dout (S, D); returns dq[q_rows], dk[k_rows] and
    dv[k_rows] without forming the S x S matrices.  A forward over blocks of
    query rows gives every row's log-sum-exp L_i, output O_i and
    Delta_i = dO_i . O_i.  Then, by the definition above, a query row i has
    P_i = exp(S_i - L_i), dS_i = P_i * (dO_i V^T - Delta_i) and
    dQ_i = dS_i K * scale; a key row j has the column P_:j = exp(S_:j - L),
    dV_j = P_:j^T dO, dS_:j = P_:j * (dO v_j - Delta) and dK_j = dS_:j^T Q * scale.
    Causal: key j is visible to query i iff j <= i."""
    q, k, v, dout = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dout))
    S, D = q.shape
    scale = softmax_scale(D)
    lse = np.empty(S)
    delta = np.empty(S)
    keys = np.arange(S)
    for i0 in range(0, S, block):
        i1 = min(S, i0 + block)
        s = (q[i0:i1] @ k.T) * scale
        if causal:
            s = np.where(keys[None, :] <= np.arange(i0, i1)[:, None], s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        ell = e.sum(axis=1, keepdims=True)
        lse[i0:i1] = (m + np.log(ell))[:, 0]
        o = (e / ell) @ v
        delta[i0:i1] = (dout[i0:i1] * o).sum(axis=1)
    q_rows, k_rows = np.asarray(q_rows), np.asarray(k_rows)
    dq = np.empty((len(q_rows), D))
    for n, i in enumerate(q_rows):
        s = (k @ q[i]) * scale
        p = np.exp(s - lse[i])
        if causal:
            p = np.where(keys <= i, p, 0.0)
        ds = p * (v @ dout[i] - delta[i])
        dq[n] = (ds @ k) * scale
    dk = np.empty((len(k_rows), D))
    dv = np.empty((len(k_rows), D))
    for n, j in enumerate(k_rows):
        s = (q @ k[j]) * scale
        p = np.exp(s - lse)
        if causal:
            p = np.where(keys >= j, p, 0.0)
        dv[n] = p @ dout
        ds = p * (dout @ v[j] - delta)
        dk[n] = (ds @ q) * scale
    return dq, dk, dv
