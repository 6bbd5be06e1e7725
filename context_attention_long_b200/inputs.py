"""Seeded synthetic inputs for the context-parallel attention hot path.

This module is shared by the CUDA path's tests and benchmark and by the
oracle's tests.  It holds none of the attention arithmetic: only random draws
(numpy PCG64), the per-head RMS normalisation that shapes the synthetic Q/K the
way a QK-normed diffusion transformer produces them, bf16 round-to-nearest-even,
and the split-length recipes used by the workload definitions.

Layout of every Q/K/V tensor: (batch, seq, heads, head_dim) contiguous, the
``view(B, S, H, D)`` layout of the attention module shown in the sglang
PR #30086 analysis page (Gemma 3 encoder ``forward``).  Tensors are returned as
bf16 bit patterns in ``numpy.uint16`` arrays so that the GPU path and the oracle
consume byte-identical inputs.
"""
from __future__ import annotations

import numpy as np

# Workloads.  Shapes follow the DiT-style workloads the pages benchmark
# (FLUX.1-dev / Qwen-Image / Wan / LTX in the diffusers "Context parallelism"
# tables and the SGLang "Sequence Parallelism" tables); data is synthetic.
CONFIGS = {
    # tiny check: everything the oracle can do in seconds.
    "tiny": dict(B=1, H=2, S=256, D=64, ring_degree=4, ulysses_degree=2,
                 rms_qk=False, seed=1234),
    # image DiT: 4096 latent-patch tokens + 512 text tokens.
    "dit": dict(B=1, H=24, S=4608, D=128, ring_degree=4, ulysses_degree=4,
                rms_qk=True, seed=1235),
    # high-res image: 96x96 latent patches, CFG pair as batch 2.
    "hires": dict(B=2, H=24, S=9216, D=128, ring_degree=8, kv_gather_degree=8,
                  ulysses_degree=8, rms_qk=True, seed=1236),
    # uneven "anything" splits: S prime, H not divisible by the Ulysses degree.
    "anything": dict(B=1, H=30, S=10007, D=128, ring_degree=6, ulysses_degree=4,
                     rms_qk=True, seed=1237),
    # video DiT: 21 latent frames x 30x52 patches; ring 8 x Ulysses 2.
    "video": dict(B=1, H=40, S=32760, D=128, ring_degree=8, ulysses_degree=2,
                  rms_qk=True, seed=1238),
}

RMS_EPS = 1e-6


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); return the bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return bf16_bits_to_f32(bits).astype(np.float64)


def _rms_normalise(x: np.ndarray) -> np.ndarray:
    """x / sqrt(mean(x^2 over head_dim) + eps), float32, no learned weight."""
    ms = np.mean(np.square(x, dtype=np.float32), axis=-1, keepdims=True, dtype=np.float32)
    return (x / np.sqrt(ms + np.float32(RMS_EPS))).astype(np.float32)


def make_qkv(B: int, S: int, H: int, D: int, seed: int, rms_qk: bool):
    """Draw Q, K, V ~ N(0, 1) in float32 from PCG64(seed) in that order, optionally
    RMS-normalise Q and K per (token, head), and round all three to bf16.

    Returns three uint16 arrays of shape (B, S, H, D) holding bf16 bits.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    out = []
    for name in ("q", "k", "v"):
        x = rng.standard_normal(size=(B, S, H, D), dtype=np.float32)
        if rms_qk and name in ("q", "k"):
            x = _rms_normalise(x)
        out.append(f32_to_bf16_bits(x))
        del x
    return out[0], out[1], out[2]


def make_projection_inputs(B: int, S: int, H: int, D: int, Dm: int, seed: int):
    """Activations and weights of the Ulysses projections, as bf16 bits.

    From PCG64(seed), in this order: x ~ N(0, 1) of (B*S, Dm) (the
    sequence-side rank buffers concatenated, any split: the rows are just
    tokens), w_qkv ~ N(0, 1/Dm) of (3*H*D, Dm) and w_o ~ N(0, 1/(H*D)) of
    (Dm, H*D), so that every projection output has unit scale.  The
    nn.Linear weight layout (out_features, in_features).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    x = f32_to_bf16_bits(rng.standard_normal(size=(B * S, Dm), dtype=np.float32))
    w_qkv = f32_to_bf16_bits(rng.standard_normal(size=(3 * H * D, Dm), dtype=np.float32) / np.float32(np.sqrt(Dm)))
    w_o = f32_to_bf16_bits(rng.standard_normal(size=(Dm, H * D), dtype=np.float32) / np.float32(np.sqrt(H * D)))
    return x, w_qkv, w_o


def config_inputs(name: str):
    """(cfg, q, k, v) for a named workload."""
    cfg = dict(CONFIGS[name])
    q, k, v = make_qkv(cfg["B"], cfg["S"], cfg["H"], cfg["D"], cfg["seed"], cfg["rms_qk"])
    return cfg, q, k, v


def front_loaded_splits(total: int, parts: int) -> list[int]:
    """Uneven split used by the 'anything' workloads: the first (total mod parts)
    parts get ceil(total/parts), the rest floor(total/parts).  30 heads over 4
    ranks gives 8/8/7/7; 10007 tokens over 4 ranks gives 2502/2502/2502/2501."""
    base, rem = divmod(total, parts)
    return [base + 1 if i < rem else base for i in range(parts)]


def ring_anything_lens(total: int, parts: int, seed: int) -> list[int]:
    """Seeded floor/ceil chunk lengths for the Ring Anything workload: every
    chunk gets ceil(total/parts) except (parts - total mod parts) chunks of
    floor(total/parts), placed cyclically from position seed mod parts.
    S=10007 over 6 chunks: five chunks of 1668 and one of 1667."""
    base, rem = divmod(total, parts)
    if rem == 0:
        return [base] * parts
    lens = [base + 1] * parts
    for i in range(parts - rem):
        lens[(seed + i) % parts] = base
    return lens


def random_splits(total: int, parts: int, seed: int, allow_zero: bool = True) -> list[int]:
    """Seeded random composition of `total` into `parts` non-negative integers
    (strictly positive when allow_zero is False)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    if allow_zero:
        cuts = np.sort(rng.integers(0, total + 1, size=parts - 1))
    else:
        if total < parts:
            raise ValueError("total < parts with allow_zero=False")
        cuts = np.sort(rng.choice(np.arange(1, total), size=parts - 1, replace=False))
    edges = np.concatenate([[0], cuts, [total]])
    return [int(x) for x in np.diff(edges)]


def iota_rows(B: int, S: int, H: int, D: int) -> np.ndarray:
    """A (B, S, H, D) uint16 array whose every element is distinct modulo 2^16
    as long as B*S*H*D <= 65536; used for permutation checks."""
    n = B * S * H * D
    return (np.arange(n, dtype=np.uint64) % 65536).astype(np.uint16).reshape(B, S, H, D)
