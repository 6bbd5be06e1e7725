"""Oracle: attention, chunk partials, the LSE merge, ring and kv_gather.

Test infrastructure only (see the package docstring).  float64 throughout;
inputs are float64 arrays in (batch, seq, heads, head_dim) layout.
"""
from __future__ import annotations

import numpy as np


def softmax_scale(D: int) -> float:
    """Softmax scale head_dim**-0.5 ([PR], Gemma 3 attention ``self.scaling``)."""
    return 1.0 / np.sqrt(float(D))


def attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray):
    """Attention of query rows against one set of keys, for a single (batch, head).

    q: (n, D), k and v: (m, D), float64.  Returns (out (n, D), lse (n,)) with
        s_ij   = (q_i . k_j) * D**-0.5
        lse_i  = log sum_j exp(s_ij)                      (natural log)
        out_i  = sum_j exp(s_ij - lse_i) v_j
    The maximum is subtracted before exponentiating only for range safety; it
    cancels exactly.  An empty key set (m == 0) gives out = 0, lse = -inf, the
    neutral element of the merge below.
    """
    n, D = q.shape
    m = k.shape[0]
    if m == 0 or n == 0:
        return np.zeros((n, v.shape[1] if v.ndim == 2 else D)), np.full((n,), -np.inf)
    s = (q @ k.T) * softmax_scale(D)
    row_max = s.max(axis=1, keepdims=True)
    e = np.exp(s - row_max)
    ell = e.sum(axis=1, keepdims=True)
    out = (e @ v) / ell
    lse = (row_max + np.log(ell))[:, 0]
    return out, lse


def causal_attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, q_pos, k_pos):
    """Attention of query rows against keys under a causal mask given by
    sequence positions, for a single (batch, head).

    [USP] section 7: for causal masking over long sequences, Ulysses and ring
    attention use position ids instead of a materialised 4-D attention mask.
    Written out: key j is visible to query i iff k_pos[j] <= q_pos[i]; over
    the visible keys the result is attention_rows' formula.  A query that sees
    no key gets out = 0, lse = -inf (the neutral element of the LSE merge).
    """
    q_pos = np.asarray(q_pos, dtype=np.int64)
    k_pos = np.asarray(k_pos, dtype=np.int64)
    n, D = q.shape
    m = k.shape[0]
    dv = v.shape[1] if v.ndim == 2 else D
    out = np.zeros((n, dv))
    lse = np.full((n,), -np.inf)
    if m == 0 or n == 0:
        return out, lse
    visible = k_pos[None, :] <= q_pos[:, None]                     # (n, m)
    s = np.where(visible, (q @ k.T) * softmax_scale(D), -np.inf)
    seen = visible.any(axis=1)
    row_max = np.where(seen, s.max(axis=1), 0.0)[:, None]
    e = np.where(visible, np.exp(s - row_max), 0.0)
    ell = e.sum(axis=1, keepdims=True)
    out[seen] = (e[seen] @ v) / ell[seen]
    lse[seen] = (row_max + np.log(np.where(ell > 0, ell, 1.0)))[seen, 0]
    return out, lse


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, q_pos=None, k_pos=None):
    """Monolithic softmax attention softmax(Q K^T / sqrt(D)) V, non-causal
    unless sequence positions are given.

    q: (B, Sq, H, D); k, v: (B, Sk, H, D).  Returns out (B, Sq, H, D) and
    lse (B, H, Sq), natural log.  Heads are independent ([USP] section 3).
    With q_pos (Sq,) and k_pos (Sk,) the causal mask of causal_attention_rows
    applies.
    """
    B, Sq, H, D = q.shape
    out = np.zeros((B, Sq, H, v.shape[3]))
    lse = np.full((B, H, Sq), -np.inf)
    for b in range(B):
        for h in range(H):
            if q_pos is None:
                o, l = attention_rows(q[b, :, h, :], k[b, :, h, :], v[b, :, h, :])
            else:
                o, l = causal_attention_rows(q[b, :, h, :], k[b, :, h, :], v[b, :, h, :], q_pos, k_pos)
            out[b, :, h, :] = o
            lse[b, h, :] = l
    return out, lse


def causal_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray):
    """Monolithic causal attention over one sequence: token i (position i)
    sees keys 0..i.  q, k, v: (B, S, H, D)."""
    S = q.shape[1]
    pos = np.arange(S)
    return attention(q, k, v, pos, pos)


def lse_merge(outs, lses):
    """Merge partial attention results computed over disjoint key sets.

    outs[p]: (B, Sq, H, D) partial outputs, each normalised over its own keys;
    lses[p]: (B, H, Sq) their log-sum-exps ([API] ``convert_to_fp32``: partial
    output and LSE are kept in float32 by the method; here float64).
    The online-softmax / LSE merge named in [SP] "Numerics across node
    boundaries", written out:
        M   = max_p LSE_p
        LSE = M + log sum_p exp(LSE_p - M)
        out = sum_p exp(LSE_p - LSE) * out_p
    Partials with LSE = -inf (empty chunks) get weight 0.  If every partial is
    empty the result is out = 0, LSE = -inf.
    """
    L = np.stack([np.asarray(x, dtype=np.float64) for x in lses])      # (P, B, H, Sq)
    M = L.max(axis=0)
    finite = np.isfinite(M)
    M0 = np.where(finite, M, 0.0)
    with np.errstate(invalid="ignore"):
        w = np.where(np.isfinite(L), np.exp(L - M0[None]), 0.0)          # (P, B, H, Sq)
    total = w.sum(axis=0)
    with np.errstate(divide="ignore"):
        lse = np.where(total > 0, M0 + np.log(np.where(total > 0, total, 1.0)), -np.inf)
    coef = np.where(total[None] > 0, w / np.where(total > 0, total, 1.0)[None], 0.0)
    coef = np.transpose(coef, (0, 1, 3, 2))[..., None]                  # (P, B, Sq, H, 1)
    out = np.zeros_like(np.asarray(outs[0], dtype=np.float64))
    for p in range(len(outs)):
        out = out + coef[p] * np.asarray(outs[p], dtype=np.float64)
    return out, lse


def equal_splits(total: int, parts: int) -> list[int]:
    """Standard (non-'anything') split: requires total % parts == 0 ([CP]
    variants table: the sequence length must be divisible by the degree)."""
    if parts < 1 or total % parts != 0:
        raise ValueError(f"{total} is not divisible by degree {parts}")
    return [total // parts] * parts


def offsets(lens) -> list[int]:
    """Prefix sums [0, l0, l0+l1, ...]."""
    out = [0]
    for x in lens:
        out.append(out[-1] + int(x))
    return out


def ring_order(rank: int, degree: int) -> list[int]:
    """Chunks visited by `rank` in ring order: at step t it holds the K/V chunk
    that started at rank (rank - t) mod P, since each GPU passes its block to
    the next GPU after computing on it ([CP] "Ring Attention")."""
    return [(rank - t) % degree for t in range(degree)]


def _chunk_lens(S: int, degree: int, chunk_lens):
    if chunk_lens is None:
        return equal_splits(S, degree)
    lens = [int(x) for x in chunk_lens]
    if len(lens) != degree or any(x < 0 for x in lens) or sum(lens) != S:
        raise ValueError("chunk_lens must be `degree` non-negative lengths summing to S")
    return lens


def _positions(off, r):
    """Sequence positions of chunk r's tokens."""
    return np.arange(off[r], off[r + 1])


def ring_step_partials(q, k, v, degree: int, step: int, chunk_lens=None, causal=False):
    """One ring step for every rank: rank r attends its Q shard to the K/V chunk
    it holds at `step`, c = (r - step) mod P.  Returns the partial output
    (B, S, H, D) and LSE (B, H, S) over all Q rows (shard r's rows hold rank
    r's partial).  causal: the position mask of causal_attention_rows, with
    every token's position its index in the full sequence (a chunk after the
    rank's own shard gives out = 0, lse = -inf)."""
    B, S, H, D = q.shape
    lens = _chunk_lens(S, degree, chunk_lens)
    off = offsets(lens)
    out = np.zeros((B, S, H, v.shape[3]))
    lse = np.full((B, H, S), -np.inf)
    for r in range(degree):
        c = ring_order(r, degree)[step]
        qs = slice(off[r], off[r + 1])
        ks = slice(off[c], off[c + 1])
        if causal:
            o, l = attention(q[:, qs], k[:, ks], v[:, ks], _positions(off, r), _positions(off, c))
        else:
            o, l = attention(q[:, qs], k[:, ks], v[:, ks])
        out[:, qs] = o
        lse[:, :, qs] = l
    return out, lse


def ring_attention(q, k, v, degree: int, chunk_lens=None, causal=False):
    """Ring attention emulated on one host ([CP] "Ring Attention", "Ring Anything
    Attention"; [API] ring_degree, convert_to_fp32, rotate_method).

    The sequence is cut into `degree` shards (equal, or `chunk_lens` for Ring
    Anything; the padding to the longest local length that Ring Anything applies
    before its all-gather is sliced away again before attention, so it does not
    enter the result).  Rank r holds shard r of Q, K and V.  For t = 0..P-1 it
    computes the partial attention of its Q shard against chunk (r - t) mod P,
    keeping partial output and LSE, and merges all P partials with the LSE rule.
    Returns out (B, S, H, D) and lse (B, H, S).  causal: every partial takes
    the position mask of causal_attention_rows ([USP] section 7), positions
    being indices in the full sequence.
    """
    B, S, H, D = q.shape
    lens = _chunk_lens(S, degree, chunk_lens)
    off = offsets(lens)
    out = np.zeros((B, S, H, v.shape[3]))
    lse = np.full((B, H, S), -np.inf)
    for r in range(degree):
        qs = slice(off[r], off[r + 1])
        outs, lses = [], []
        for c in ring_order(r, degree):
            ks = slice(off[c], off[c + 1])
            if causal:
                o, l = attention(q[:, qs], k[:, ks], v[:, ks], _positions(off, r), _positions(off, c))
            else:
                o, l = attention(q[:, qs], k[:, ks], v[:, ks])
            outs.append(o)
            lses.append(l)
        o, l = lse_merge(outs, lses)
        out[:, qs] = o
        lse[:, :, qs] = l
    return out, lse


def kv_gather_attention(q, k, v, degree: int, q_lens=None):
    """kv_gather exchange ([SP] "Choosing The Attention Exchange"): Q and the
    output stay sequence-sharded; K and V are all-gathered, and each rank
    computes its own rows directly against the full K/V.  Non-causal, ring
    degree 1.  Shard r covers rows off_r .. off_r + len_r of every batch."""
    B, S, H, D = q.shape
    lens = _chunk_lens(S, degree, q_lens)
    off = offsets(lens)
    out = np.zeros((B, S, H, v.shape[3]))
    lse = np.full((B, H, S), -np.inf)
    for r in range(degree):
        qs = slice(off[r], off[r + 1])
        o, l = attention(q[:, qs], k, v)
        out[:, qs] = o
        lse[:, :, qs] = l
    return out, lse
