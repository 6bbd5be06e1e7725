"""Helpers shared by the GPU tests: moving the seeded bf16 inputs to the device,
comparing against the oracle with the stated tolerances, layout conversions
between full (B, S, H, D) tensors and sequence-side rank buffers."""
import numpy as np
import torch

from context_attention_long_b200 import inputs

# Attention parity bar (bf16 in, fp32 accumulate): output max-abs / mean-abs,
# LSE max-abs.
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> bf16 CUDA tensor (same bytes)."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bits_of(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64_of(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return inputs.bf16_bits_to_f64(bits_of(t))
    return t.detach().double().cpu().numpy()


def assert_close(out, lse, ref_out, ref_lse, what=""):
    out = np.asarray(out, dtype=np.float64)
    ref_out = np.asarray(ref_out, dtype=np.float64)
    err = np.abs(out - ref_out)
    assert np.all(np.isfinite(out)), f"{what}: non-finite output"
    assert err.max() <= OUT_MAX_ABS, f"{what}: out max-abs {err.max():.3e}"
    assert err.mean() <= OUT_MEAN_ABS, f"{what}: out mean-abs {err.mean():.3e}"
    if lse is not None:
        lse = np.asarray(lse, dtype=np.float64)
        ref_lse = np.asarray(ref_lse, dtype=np.float64)
        fin = np.isfinite(ref_lse)
        assert np.array_equal(fin, np.isfinite(lse)), f"{what}: LSE finiteness differs"
        if fin.any():
            lerr = np.abs(lse[fin] - ref_lse[fin])
            assert lerr.max() <= LSE_MAX_ABS, f"{what}: lse max-abs {lerr.max():.3e}"
    return err.max(), err.mean()


def full_to_rank_buffers(x: np.ndarray, seq) -> np.ndarray:
    """(B, S, H, D) -> flat concatenation of rank buffers (B, S_r, H, D)."""
    off = np.concatenate([[0], np.cumsum(seq)])
    return np.concatenate([np.ascontiguousarray(x[:, off[r]:off[r + 1]]).reshape(-1) for r in range(len(seq))])


def rank_buffers_to_full(flat: np.ndarray, B, S, H, D, seq) -> np.ndarray:
    off = np.concatenate([[0], np.cumsum(seq)])
    out = np.empty((B, S, H, D), dtype=flat.dtype)
    pos = 0
    for r, n in enumerate(seq):
        size = B * n * H * D
        out[:, off[r]:off[r + 1]] = flat[pos:pos + size].reshape(B, n, H, D)
        pos += size
    return out


def sample_positions(S, boundaries, n_random, seed):
    """Sequence positions: first/last row of every shard/chunk plus random rows."""
    pos = set()
    for a, b in zip(boundaries[:-1], boundaries[1:]):
        if b > a:
            pos.update([a, b - 1, min(a + 1, b - 1), max(a, b - 2)])
    rng = np.random.Generator(np.random.PCG64(seed))
    pos.update(int(x) for x in rng.integers(0, S, size=n_random))
    return np.array(sorted(pos), dtype=np.int64)


def oracle_rows(oracle_mod, q_bits, k_bits, v_bits, positions, b_list=None):
    """Monolithic attention (the oracle's definition) at sampled positions, all heads.
    Returns out (B, n, H, D) and lse (B, H, n)."""
    B, S, H, D = q_bits.shape
    bs = range(B) if b_list is None else b_list
    out = np.zeros((B, len(positions), H, D))
    lse = np.zeros((B, H, len(positions)))
    for b in bs:
        for h in range(H):
            qh = inputs.bf16_bits_to_f64(q_bits[b, positions, h, :])
            kh = inputs.bf16_bits_to_f64(k_bits[b, :, h, :])
            vh = inputs.bf16_bits_to_f64(v_bits[b, :, h, :])
            o, l = oracle_mod.attention_rows(qh, kh, vh)
            out[b, :, h, :] = o
            lse[b, h, :] = l
    return out, lse
