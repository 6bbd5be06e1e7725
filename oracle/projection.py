"""Oracle: the Ulysses projections around the two all-to-alls.

Test infrastructure only (see the package docstring).

The Ulysses flow of the "Ulysses Sequence Parallelism" article, section 4:
each rank computes the Q, K and V projections of its own sequence chunk, the
first all-to-all regroups them by head, local attention runs, the second
all-to-all regroups the output by token, and each rank applies the output
projection to its own chunk.  These functions are the two projection steps
composed with their all-to-all, written in that order:

  qkv:  per sequence rank r, QKV_r = X_r W_qkv^T, split into Q | K | V of
        (B, S_r, H, D) each, then `ulysses_permute` of each;
  out:  `ulysses_unpermute` of the head-side output, then per sequence rank r,
        out_r = O_r W_o^T with O_r viewed as (B, S_r, H*D).

W follows the nn.Linear layout (out_features, in_features); the rows of W_qkv
are [Q heads | K heads | V heads], head h of each at rows [h*D, (h+1)*D).  No
bias (the pages name the projections and nothing more).  Arithmetic in
float64; the inputs are whatever the caller passes (bf16 values widened).
"""
from __future__ import annotations

import numpy as np

from .attention import offsets
from .permute import _splits, seq_rank_views, ulysses_permute, ulysses_unpermute


def project_rows(x, w):
    """x W^T in float64: the projection of every row of x (a plain matrix product)."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T


def ulysses_qkv_projection(x_flat, w_qkv, B, S, H, D, Dm, degree, seq_splits=None, head_splits=None):
    """Q, K, V projections of the sequence-side activations (rank buffers
    (B, S_r, Dm) concatenated, flat) followed by the first all-to-all; returns
    the head-side (yq, yk, yv), flat float64 arrays of B*S*H*D."""
    seq = _splits(S, degree, seq_splits, "sequence")
    x_flat = np.asarray(x_flat, dtype=np.float64).reshape(-1)
    w_qkv = np.asarray(w_qkv, dtype=np.float64).reshape(3 * H * D, Dm)
    seq_side = [np.empty(B * S * H * D) for _ in range(3)]
    pos_x = pos_y = 0
    for n in seq:
        x_r = x_flat[pos_x:pos_x + B * n * Dm].reshape(B * n, Dm)
        qkv_r = project_rows(x_r, w_qkv)                       # (B*S_r, 3*H*D)
        for t in range(3):
            seq_side[t][pos_y:pos_y + B * n * H * D] = qkv_r[:, t * H * D:(t + 1) * H * D].reshape(-1)
        pos_x += B * n * Dm
        pos_y += B * n * H * D
    return tuple(ulysses_permute(y, B, S, H, D, degree, seq, head_splits) for y in seq_side)


def ulysses_output_projection(yo_flat, w_o, B, S, H, D, Dm, degree, seq_splits=None, head_splits=None):
    """The second all-to-all of the head-side attention output followed by the
    output projection; returns the sequence side (rank buffers (B, S_r, Dm)
    concatenated), a flat float64 array of B*S*Dm."""
    seq = _splits(S, degree, seq_splits, "sequence")
    o_seq = ulysses_unpermute(np.asarray(yo_flat, dtype=np.float64), B, S, H, D, degree, seq, head_splits)
    w_o = np.asarray(w_o, dtype=np.float64).reshape(Dm, H * D)
    out = np.empty(B * S * Dm)
    pos = 0
    for o_r, n in zip(seq_rank_views(o_seq, B, H, D, seq), seq):
        out[pos:pos + B * n * Dm] = project_rows(o_r.reshape(B * n, H * D), w_o).reshape(-1)
        pos += B * n * Dm
    return out


def token_order_rows(flat, B, S, width, seq_splits):
    """Rows of a sequence-side buffer (rank buffers (B, S_r, width)) in plain
    token order (b, s): a (B*S, width) float64 array.  Used by the tests to
    compare with unsharded references."""
    flat = np.asarray(flat).reshape(-1)
    off = offsets(seq_splits)
    out = np.empty((B, S, width), dtype=flat.dtype)
    pos = 0
    for r, n in enumerate(seq_splits):
        out[:, off[r]:off[r + 1]] = flat[pos:pos + B * n * width].reshape(B, n, width)
        pos += B * n * width
    return out.reshape(B * S, width)
