"""Context-parallel attention driven by one configuration object, with the
semantics of diffusers' ContextParallelConfig (diffusers "parallel": the
ring_degree, ulysses_degree, convert_to_fp32, rotate_method, ulysses_anything,
ring_anything and mesh arguments; "Context parallelism": the variants table
and its requirements), dispatched to this library's exchanges
(context_attention_long_b200.exchange).

    ring_degree > 1                 Ring Attention; S divisible by ring_degree
    ulysses_degree > 1              Ulysses Attention; S and H divisible by
                                    ulysses_degree
    both > 1                        Unified Attention on a ring x Ulysses grid
                                    of ring_degree * ulysses_degree >= 4 ranks
    ulysses_anything                uneven S and H; ring_degree must be 1
    ring_anything                   uneven S; ulysses_degree must be 1, and
                                    inference only

This module checks arguments and dispatches; torch.distributed moves the data
and the library's kernels compute.  It has no compute of its own.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Any, Optional

import torch

from . import exchange


@dataclass(frozen=True)
class ContextParallelConfig:
    """The degrees and modes of context parallelism.

    convert_to_fp32 is accepted for compatibility: every variant here keeps
    the partial outputs and LSEs in float32 (on chip in the fused ring) and
    writes bf16 once.  rotate_method "allgather" gathers the ring's K/V chunks
    first (diffusers' default); "p2p" pipelines a point-to-point rotation
    against the attention of the chunk already held (SGLang "Sequence
    Parallelism", "Cross-Node Sequence Parallelism").  The two give
    byte-identical results.  mesh: a DeviceMesh with "ring" and "ulysses"
    dimensions of the configured sizes, whose groups are used instead of new
    ones."""

    ring_degree: int = 1
    ulysses_degree: int = 1
    convert_to_fp32: bool = True
    rotate_method: str = "allgather"
    ulysses_anything: bool = False
    ring_anything: bool = False
    mesh: Optional[Any] = None

    def __post_init__(self):
        for name in ("ring_degree", "ulysses_degree"):
            d = getattr(self, name)
            if not isinstance(d, int) or isinstance(d, bool) or d < 1:
                raise ValueError(f"{name} must be an integer >= 1, got {d!r}")
        if self.rotate_method not in ("allgather", "p2p"):
            raise ValueError(f"rotate_method must be 'allgather' or 'p2p', got {self.rotate_method!r}")
        if self.ulysses_anything and not (self.ulysses_degree > 1 and self.ring_degree == 1):
            raise ValueError("ulysses_anything needs ulysses_degree > 1 and ring_degree == 1")
        if self.ring_anything and not (self.ring_degree > 1 and self.ulysses_degree == 1):
            raise ValueError("ring_anything needs ring_degree > 1 and ulysses_degree == 1")
        if self.mesh is not None:
            names = tuple(getattr(self.mesh, "mesh_dim_names", None) or ())
            if "ring" not in names or "ulysses" not in names:
                raise ValueError("mesh must have 'ring' and 'ulysses' dimensions")
            if (self.mesh.size(names.index("ring")) != self.ring_degree or
                    self.mesh.size(names.index("ulysses")) != self.ulysses_degree):
                raise ValueError("the mesh's 'ring' and 'ulysses' sizes must equal ring_degree and ulysses_degree")

    @property
    def world_size(self) -> int:
        return self.ring_degree * self.ulysses_degree

    @property
    def variant(self) -> str:
        if self.ring_degree > 1 and self.ulysses_degree > 1:
            return "unified"
        if self.ring_degree > 1:
            return "ring"
        if self.ulysses_degree > 1:
            return "ulysses"
        return "none"

    def check(self, S: int, H: int, training: bool = False) -> None:
        """The variants table's requirements for a sequence of S tokens (all
        ranks together) and H heads; raises ValueError."""
        R, U = self.ring_degree, self.ulysses_degree
        if training and self.ring_anything:
            raise ValueError("ring_anything is inference only")
        if self.variant == "ring" and not self.ring_anything and S % R:
            raise ValueError(f"sequence length {S} is not divisible by ring_degree {R} (ring_anything lifts this)")
        if self.variant == "ulysses" and not self.ulysses_anything and (S % U or H % U):
            raise ValueError(f"sequence length {S} and heads {H} must be divisible by ulysses_degree {U} "
                             "(ulysses_anything lifts this)")
        if self.variant == "unified" and (S % (R * U) or H % U):
            raise ValueError(f"unified attention needs S % (ring_degree * ulysses_degree) == 0 and "
                             f"H % ulysses_degree == 0, got S={S}, H={H}")


class ContextParallel:
    """A configuration bound to process groups.  Every rank of the job
    constructs it (group creation is collective), then calls attention() with
    its own shard."""

    def __init__(self, config: ContextParallelConfig, kernels=None):
        import torch.distributed as dist
        self.config = config
        self.kernels = kernels
        world = dist.get_world_size()
        if world != config.world_size:
            raise ValueError(f"ring_degree * ulysses_degree = {config.world_size} but the job has {world} ranks")
        self.ring_group = self.ulysses_group = None
        if config.mesh is not None:
            self.ring_group = config.mesh.get_group("ring")
            self.ulysses_group = config.mesh.get_group("ulysses")
        elif config.variant == "unified":
            self.ring_group, self.ulysses_group = exchange.unified_groups(config.ring_degree, config.ulysses_degree)

    @staticmethod
    def _gather(value, group=None) -> list:
        """`value` of every rank of `group`, in the group's rank order (a
        small host-side exchange of metadata, before any data moves)."""
        import torch.distributed as dist
        out = [None] * dist.get_world_size(group)
        dist.all_gather_object(out, value, group=group)
        return out

    def _lengths(self, n: int):
        """The shard lengths the variant's exchange takes: the ring's or the
        Ulysses group's lengths in group order, or for the unified grid the
        sub-shard lengths of every (ring chunk i, Ulysses rank j)."""
        import torch.distributed as dist
        cfg = self.config
        if cfg.variant in ("none", "ring"):
            return [int(x) for x in self._gather(int(n), self.ring_group)]
        if cfg.variant == "ulysses":
            return [int(x) for x in self._gather(int(n), self.ulysses_group)]
        i, j = dist.get_rank(self.ring_group), dist.get_rank(self.ulysses_group)
        subs = [[0] * cfg.ulysses_degree for _ in range(cfg.ring_degree)]
        for ii, jj, nn in self._gather((i, j, int(n))):
            subs[ii][jj] = nn
        return subs

    def attention(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                  head_splits=None, return_lse: bool = False):
        """Attention of this rank's shard: q, k, v are contiguous bf16
        (B, S_r, H, D); the shards of all ranks in rank order are the full
        sequence.  Returns out (B, S_r, H, D) bf16, and with return_lse the
        float32 LSE that the variant's exchange returns (ring: (B, H, S_r);
        Ulysses: (B, H_r, S) of this rank's heads; unified: (B, H_j, S_i) of
        this rank's head group over its ring chunk).  head_splits: the heads
        of each Ulysses rank under ulysses_anything (None: front-loaded).
        When q, k or v requires a gradient, the output is differentiable
        across the ranks: the Ulysses exchange runs its all-to-alls
        backwards, and the ring and unified forwards take their gradient on
        the head side of a Ulysses all-to-all (one extra forward there)."""
        cfg = self.config
        B, Sr, H, D = q.shape
        training = torch.is_grad_enabled() and any(t.requires_grad for t in (q, k, v))
        lens = self._lengths(Sr)
        S = sum(sum(x) for x in lens) if cfg.variant == "unified" else sum(lens)
        cfg.check(S, H, training=training)
        if training:
            # Gradients cross GPUs through a Ulysses all-to-all: the Ulysses
            # exchange runs its all-to-alls backwards; the ring and unified
            # forwards take their gradient on the head side of a Ulysses
            # all-to-all over a group whose rank order is the sequence order.
            if return_lse:
                raise NotImplementedError("return_lse is for inference")
            if cfg.variant in ("none", "ulysses"):
                heads = None
                if cfg.ulysses_anything:
                    heads = list(head_splits) if head_splits is not None else exchange.front_loaded_splits(
                        H, cfg.ulysses_degree)
                return exchange.ulysses_attention_trainable(q, k, v, self.ulysses_group, lens, heads, causal,
                                                            kernels=self.kernels)
            if cfg.variant == "ring":
                return exchange.ring_attention_trainable(q, k, v, self.ring_group, lens, causal, cfg.rotate_method,
                                                         kernels=self.kernels)
            if cfg.mesh is not None:
                raise NotImplementedError("unified training with a custom mesh (its rank order need not be the "
                                          "sequence order)")
            kern = self.kernels or exchange.CudaKernels()
            fwd = lambda a, b, c: exchange.unified_attention(a, b, c, self.ring_group, self.ulysses_group, None,
                                                             lens, None, causal, cfg.rotate_method, kern)[0]
            seq = [n for chunk in lens for n in chunk]       # grid rank i * U + j holds sub-shard j of chunk i
            return exchange.HeadSideBackwardFunction.apply(q, k, v, fwd, None, seq, causal, kern)
        if cfg.variant in ("none", "ring"):
            out, lse = exchange.ring_attention(q, k, v, self.ring_group, lens, causal, cfg.rotate_method,
                                               kernels=self.kernels)
        elif cfg.variant == "ulysses":
            heads = None
            if cfg.ulysses_anything:
                heads = list(head_splits) if head_splits is not None else exchange.front_loaded_splits(
                    H, cfg.ulysses_degree)
            out, lse = exchange.ulysses_attention(q, k, v, self.ulysses_group, lens, heads, causal,
                                                  kernels=self.kernels)
        else:
            out, lse = exchange.unified_attention(q, k, v, self.ring_group, self.ulysses_group, None, lens, None,
                                                  causal, cfg.rotate_method, kernels=self.kernels)
        return (out, lse) if return_lse else out
