"""Oracle for the context-parallel attention hot path.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  A plain, slow, obviously
correct CPU restatement, in float64, of what the hot path computes:

* monolithic non-causal softmax attention (the plain definition), and the
  causal variant masked by sequence positions,
* per-chunk partial attention with its log-sum-exp, and the LSE merge of
  partials (ring attention; Ring Anything chunk lengths),
* the kv_gather exchange (each Q shard against the full K/V),
* the gradient of attention with respect to Q, K and V (causal or not),
* the Ulysses sequence-sharded <-> head-sharded permutation and its inverse
  (including the uneven Ulysses Anything splits), and the Ulysses and unified
  (ring x Ulysses) attention flows composed from the pieces above,
* the Ulysses Q/K/V and output projections composed with their all-to-all.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
reference leg of ``bench.py`` may import this package.  It shares no code with
the CUDA path (``context_attention_long_b200``) and imports nothing from it;
inputs reach it as numpy arrays.

Sources (web pages, cited by title and section):
  [CP]   diffusers v0.43.0 docs, "Context parallelism" -- variants table,
         sections "Ring Attention", "Ulysses Attention", "Unified Attention",
         "Ulysses Anything Attention", "Ring Anything Attention".
  [SP]   SGLang Diffusion docs, "Sequence Parallelism" -- "Choosing The
         Attention Exchange", "Numerics across node boundaries".
  [USP]  "Ulysses Sequence Parallelism: training with million-token contexts"
         (article summary) -- sections 1, 2, 3, 4, 5, 7.
  [API]  diffusers docs, "parallel" -- ContextParallelConfig parameters.
  [PR]   sglang PR #30086 analysis -- Gemma 3 attention (B, S, H, D) view and
         head_dim**-0.5 scale.

Parity status: every function here is pinned by ``tests/test_oracle.py``
against brute force, closed forms, invariants or an independent library
routine; none is "parity unpinned".
"""
from .attention import (
    softmax_scale,
    attention,
    attention_rows,
    causal_attention,
    causal_attention_rows,
    lse_merge,
    equal_splits,
    offsets,
    ring_order,
    ring_attention,
    ring_step_partials,
    kv_gather_attention,
)
from .backward import attention_backward, attention_backward_rows, attention_backward_sampled
from .projection import (
    project_rows,
    ulysses_qkv_projection,
    ulysses_output_projection,
    token_order_rows,
)
from .permute import (
    ulysses_permute,
    ulysses_unpermute,
    ulysses_attention,
    unified_attention,
)

__all__ = [
    "softmax_scale", "attention", "attention_rows", "causal_attention",
    "causal_attention_rows", "lse_merge", "equal_splits",
    "offsets", "ring_order", "ring_attention", "ring_step_partials",
    "kv_gather_attention", "ulysses_permute", "ulysses_unpermute",
    "ulysses_attention", "unified_attention", "attention_backward", "attention_backward_rows",
    "attention_backward_sampled",
    "project_rows", "ulysses_qkv_projection", "ulysses_output_projection", "token_order_rows",
]
