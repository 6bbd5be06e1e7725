"""torch.autograd functions over this library's attention kernels, for
training with context-parallel attention (the Ulysses Sequence Parallelism
article, sections 1 and 7: long-context training, causal masking by position).

Each function's forward is one of the library's forward entry points and its
backward the matching backward entry point (the derivative of the forward's
definition: dQ, dK and dV from the forward's output, its log-sum-exp and the
upstream gradient).  Like api.py, this module only marshals arguments: both
passes run in the library's kernels, and nothing here computes.
"""
from __future__ import annotations

import torch

from . import api


class RingAttentionFunction(torch.autograd.Function):
    """Attention of (B, S, H, D) bf16 Q, K, V whose sequence is cut into
    `ring_degree` shards (the fused ring kernel; `chunk_lens` for uneven
    shards), causal or not.  The gradient does not depend on the sharding:
    it is the attention backward over the full tensors."""

    @staticmethod
    def forward(ctx, q, k, v, ring_degree, causal, chunk_lens):
        fn = api.cpattn_causal_ring_attention if causal else api.cpattn_ring_attention
        out, lse = fn(q, k, v, ring_degree, chunk_lens)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.causal = bool(causal)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        dq, dk, dv = api.cpattn_attention_backward(q, k, v, out, lse, dout.contiguous(), ctx.causal)
        return dq, dk, dv, None, None, None


class UlyssesAttentionFunction(torch.autograd.Function):
    """The Ulysses flow on sequence-sharded rank buffers (flat bf16: the
    `degree` ranks' (B, S_r, H, D) buffers concatenated), even or uneven
    `seq_splits` / `head_splits`, causal or not.  The backward runs the
    Ulysses flow's backward on the same layout."""

    @staticmethod
    def forward(ctx, q, k, v, B, S, H, D, degree, seq_splits, head_splits, causal):
        fn = api.cpattn_causal_ulysses_attention if causal else api.cpattn_ulysses_attention
        out, lse = fn(q, k, v, B, S, H, D, degree, seq_splits, head_splits)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.args = (B, S, H, D, degree, seq_splits, head_splits, bool(causal))
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        B, S, H, D, degree, seq_splits, head_splits, causal = ctx.args
        dq, dk, dv = api.cpattn_ulysses_attention_backward(q, k, v, out, lse, dout.contiguous(), B, S, H, D,
                                                           degree, seq_splits, head_splits, causal)
        return (dq, dk, dv) + (None,) * 8


def ring_attention(q, k, v, ring_degree=1, causal=False, chunk_lens=None):
    """Differentiable fused ring attention; returns out (B, S, H, D) bf16."""
    return RingAttentionFunction.apply(q, k, v, ring_degree, causal, chunk_lens)


def ulysses_attention(q, k, v, B, S, H, D, degree, seq_splits=None, head_splits=None, causal=False):
    """Differentiable Ulysses attention on rank buffers; returns out in the
    same rank-buffer layout."""
    return UlyssesAttentionFunction.apply(q, k, v, B, S, H, D, degree, seq_splits, head_splits, causal)
