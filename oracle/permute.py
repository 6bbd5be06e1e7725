"""Oracle: the Ulysses exchange and the attention flows built on it.

Test infrastructure only (see the package docstring).

Layouts (in-memory emulation of P ranks on one host):
  * sequence-sharded side: the P rank buffers concatenated in rank order,
    rank r holding (B, S_r, H, D) -- its own tokens, all heads.  With B = 1 this
    is exactly the full (B, S, H, D) tensor.
  * head-sharded side: the P rank buffers concatenated in rank order, rank r'
    holding (B, S, H_r', D) -- every token, its own heads.
Both are passed around as flat 1-D arrays of B*S*H*D elements, any dtype.
"""
from __future__ import annotations

import numpy as np

from .attention import attention, equal_splits, lse_merge, offsets, ring_order


def _splits(total, degree, splits, what):
    if splits is None:
        return equal_splits(total, degree)
    s = [int(x) for x in splits]
    if len(s) != degree or any(x < 0 for x in s) or sum(s) != total:
        raise ValueError(f"{what} splits must be {degree} non-negative values summing to {total}")
    return s


def seq_rank_views(x_flat, B, H, D, seq_splits):
    """Views (B, S_r, H, D) of the sequence-sharded rank buffers in a flat array."""
    views, pos = [], 0
    for n in seq_splits:
        size = B * n * H * D
        views.append(x_flat[pos:pos + size].reshape(B, n, H, D))
        pos += size
    return views


def head_rank_views(y_flat, B, S, D, head_splits):
    """Views (B, S, H_r', D) of the head-sharded rank buffers in a flat array."""
    views, pos = [], 0
    for n in head_splits:
        size = B * S * n * D
        views.append(y_flat[pos:pos + size].reshape(B, S, n, D))
        pos += size
    return views


def ulysses_permute(x_flat, B, S, H, D, degree, seq_splits=None, head_splits=None):
    """Sequence-sharded -> head-sharded, the first all-to-all of Ulysses
    ([CP] "Ulysses Attention": the data is regrouped so that each GPU holds
    every token for a subset of attention heads; [USP] section 4).

        y_{r'}[b, s, h - hoff_{r'}, :] = x_{r(s)}[b, s - off_{r(s)}, h, :]

    for every b, token s (owned by sequence rank r(s)) and head h (owned by
    head rank r').  `seq_splits` / `head_splits` default to the equal split,
    which requires S and H divisible by the degree ([CP] variants table);
    explicit uneven splits are Ulysses Anything ([CP] "Ulysses Anything
    Attention").  Written block by block: the block (sequence rank r, head
    rank r') is the set of elements the formula moves from x_r to y_{r'}.
    """
    seq = _splits(S, degree, seq_splits, "sequence")
    heads = _splits(H, degree, head_splits, "head")
    soff, hoff = offsets(seq), offsets(heads)
    x_flat = np.asarray(x_flat).reshape(-1)
    y_flat = np.empty_like(x_flat)
    xs = seq_rank_views(x_flat, B, H, D, seq)
    ys = head_rank_views(y_flat, B, S, D, heads)
    for r in range(degree):
        for rp in range(degree):
            ys[rp][:, soff[r]:soff[r + 1], :, :] = xs[r][:, :, hoff[rp]:hoff[rp + 1], :]
    return y_flat


def ulysses_unpermute(y_flat, B, S, H, D, degree, seq_splits=None, head_splits=None):
    """Head-sharded -> sequence-sharded, the second all-to-all of Ulysses, which
    regroups the attention results by token ([CP] "Ulysses Attention"):

        x_r[b, s - off_r, h, :] = y_{r'(h)}[b, s, h - hoff_{r'(h)}, :]

    the exact inverse of `ulysses_permute`."""
    seq = _splits(S, degree, seq_splits, "sequence")
    heads = _splits(H, degree, head_splits, "head")
    soff, hoff = offsets(seq), offsets(heads)
    y_flat = np.asarray(y_flat).reshape(-1)
    x_flat = np.empty_like(y_flat)
    xs = seq_rank_views(x_flat, B, H, D, seq)
    ys = head_rank_views(y_flat, B, S, D, heads)
    for r in range(degree):
        for rp in range(degree):
            xs[r][:, :, hoff[rp]:hoff[rp + 1], :] = ys[rp][:, soff[r]:soff[r + 1], :, :]
    return x_flat


def ulysses_attention(q_flat, k_flat, v_flat, B, S, H, D, degree,
                      seq_splits=None, head_splits=None, causal=False):
    """Ulysses attention ([USP] section 4; [CP] "Ulysses Attention"): all-to-all
    to the head-sharded layout, local attention of every rank over all S tokens
    of its heads, inverse all-to-all of the output.

    q/k/v_flat: float64, sequence-sharded rank buffers.  Returns
    (out_flat in the sequence-sharded layout, lse (B, H, S) indexed by the
    global head and token).  causal: the local attention takes the position
    mask of causal_attention_rows; after the first all-to-all every rank holds
    all S tokens, so a token's position is its index s ([USP] section 7)."""
    heads = _splits(H, degree, head_splits, "head")
    hoff = offsets(heads)
    yq = ulysses_permute(q_flat, B, S, H, D, degree, seq_splits, heads)
    yk = ulysses_permute(k_flat, B, S, H, D, degree, seq_splits, heads)
    yv = ulysses_permute(v_flat, B, S, H, D, degree, seq_splits, heads)
    yo = np.zeros(B * S * H * D)
    lse = np.full((B, H, S), -np.inf)
    qv = head_rank_views(yq, B, S, D, heads)
    kv = head_rank_views(yk, B, S, D, heads)
    vv = head_rank_views(yv, B, S, D, heads)
    ov = head_rank_views(yo, B, S, D, heads)
    pos = np.arange(S) if causal else None
    for rp in range(degree):
        o, l = attention(qv[rp], kv[rp], vv[rp], pos, pos)
        ov[rp][...] = o
        lse[:, hoff[rp]:hoff[rp + 1], :] = l
    out = ulysses_unpermute(yo, B, S, H, D, degree, seq_splits, heads)
    return out, lse


def unified_attention(q, k, v, ring_degree, ulysses_degree, ring_lens=None,
                      head_splits=None, sub_splits=None, causal=False):
    """Unified (ring x Ulysses) attention ([CP] "Unified Attention"): an
    all-to-all that redistributes heads and tokens, ring attention on the
    result, and the inverse all-to-all.  The GPUs form a ring_degree x
    ulysses_degree grid; each belongs to one Ulysses group and one ring group.

    q, k, v: full (B, S, H, D) float64.  Reading used here: ring chunks are the
    outer split of the sequence (rows off_i .. off_i + len_i of every batch,
    equal or `ring_lens`); inside ring chunk i the Ulysses group's ranks hold
    sub-shards of it (`sub_splits[i]`, default the front-loaded split); heads
    are split by `head_splits`.  Steps:
      1. within every ring group i: Ulysses permute of the group's sub-shards
         -> for head group u, the chunk-i tokens of heads u, (B, len_i, H_u, D);
      2. for every head group u: ring attention over the chunks (ring order,
         LSE merge), Q shard i against K/V chunks (i - t) mod R;
      3. within every ring group: the inverse permute of the output.
    Returns out (B, S, H, D) and lse (B, H, S).  causal: step 2 takes the
    position mask of causal_attention_rows, chunk i's tokens sitting at
    positions off_i .. off_i + len_i - 1 ([USP] section 7)."""
    B, S, H, D = q.shape
    R, U = ring_degree, ulysses_degree
    rl = equal_splits(S, R) if ring_lens is None else [int(x) for x in ring_lens]
    if len(rl) != R or sum(rl) != S or min(rl) < 0:
        raise ValueError("bad ring_lens")
    heads = _splits(H, U, head_splits, "head")
    roff, hoff = offsets(rl), offsets(heads)
    if sub_splits is None:
        sub_splits = [[n // U + (1 if j < n % U else 0) for j in range(U)] for n in rl]

    def to_group_heads(x):
        # step 1 for one tensor: per group i the seq rank buffers of its sub-shards
        per = []
        for i in range(R):
            chunk = x[:, roff[i]:roff[i + 1]]
            so = offsets(sub_splits[i])
            flat = np.concatenate([chunk[:, so[j]:so[j + 1]].reshape(-1) for j in range(U)])
            y = ulysses_permute(flat, B, rl[i], H, D, U, sub_splits[i], heads)
            per.append(head_rank_views(y, B, rl[i], D, heads))   # per[i][u]
        return per

    Yq, Yk, Yv = to_group_heads(q), to_group_heads(k), to_group_heads(v)
    out = np.zeros((B, S, H, D))
    lse = np.full((B, H, S), -np.inf)
    Yo = [[None] * U for _ in range(R)]
    for u in range(U):
        for i in range(R):
            outs, lses = [], []
            for c in ring_order(i, R):
                if causal:
                    o, l = attention(Yq[i][u], Yk[c][u], Yv[c][u],
                                     np.arange(roff[i], roff[i + 1]), np.arange(roff[c], roff[c + 1]))
                else:
                    o, l = attention(Yq[i][u], Yk[c][u], Yv[c][u])
                outs.append(o)
                lses.append(l)
            o, l = lse_merge(outs, lses)
            Yo[i][u] = o
            lse[:, hoff[u]:hoff[u + 1], roff[i]:roff[i + 1]] = l
    for i in range(R):
        yflat = np.concatenate([Yo[i][u].reshape(-1) for u in range(U)])
        xflat = ulysses_unpermute(yflat, B, rl[i], H, D, U, sub_splits[i], heads)
        so = offsets(sub_splits[i])
        views = seq_rank_views(xflat, B, H, D, sub_splits[i])
        for j in range(U):
            out[:, roff[i] + so[j]:roff[i] + so[j + 1]] = views[j]
    return out, lse
