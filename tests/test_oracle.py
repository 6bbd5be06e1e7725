"""Pins for the oracle: each check compares it with something other than itself
(hand-worked values, brute force, closed forms, an independent library routine,
or invariants the method fixes).  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from context_attention_long_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.standard_normal(size=shape) * scale


def _tiny_f64():
    cfg, q, k, v = inputs.config_inputs("tiny")
    return cfg, inputs.bf16_bits_to_f64(q), inputs.bf16_bits_to_f64(k), inputs.bf16_bits_to_f64(v)


# ----------------------------------------------------------------- attention

def test_attention_matches_scalar_brute_force():
    """Brute force with scalar loops, math.exp and no max subtraction."""
    B, Sq, Sk, H, D = 2, 5, 7, 3, 4
    q, k, v = _rand((B, Sq, H, D), 1), _rand((B, Sk, H, D), 2), _rand((B, Sk, H, D), 3)
    out, lse = oracle.attention(q, k, v)
    for b in range(B):
        for h in range(H):
            for i in range(Sq):
                w = []
                for j in range(Sk):
                    dot = sum(q[b, i, h, d] * k[b, j, h, d] for d in range(D))
                    w.append(math.exp(dot / math.sqrt(D)))
                z = sum(w)
                assert abs(lse[b, h, i] - math.log(z)) < 1e-12
                for d in range(D):
                    ref = sum(w[j] * v[b, j, h, d] for j in range(Sk)) / z
                    assert abs(out[b, i, h, d] - ref) < 1e-12


def test_attention_matches_torch_sdpa_float64():
    """Independent library routine: torch SDPA (float64, CPU) on the tiny workload."""
    cfg, q, k, v = _tiny_f64()
    out, lse = oracle.attention(q, k, v)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))   # (B, H, S, D)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(0, 2, 1, 3).numpy()
    assert np.max(np.abs(out - ref)) < 1e-12
    scores = torch.matmul(tq, tk.transpose(-1, -2)) / math.sqrt(cfg["D"])
    ref_lse = torch.logsumexp(scores, dim=-1).numpy()
    assert np.max(np.abs(lse - ref_lse)) < 1e-12


def test_constant_v_yields_v():
    B, S, H, D = 1, 33, 2, 8
    q, k = _rand((B, S, H, D), 4, 3.0), _rand((B, S, H, D), 5, 3.0)
    v = np.full((B, S, H, D), 0.375)
    out, _ = oracle.attention(q, k, v)
    assert np.max(np.abs(out - 0.375)) < 1e-14


def test_zero_keys_give_uniform_softmax():
    B, S, H, D = 2, 19, 3, 16
    q, v = _rand((B, 7, H, D), 6), _rand((B, S, H, D), 7)
    out, lse = oracle.attention(q, np.zeros((B, S, H, D)), v)
    assert np.max(np.abs(lse - math.log(S))) < 1e-13
    assert np.max(np.abs(out - v.mean(axis=1, keepdims=True))) < 1e-13


def test_one_hot_key_selects_value():
    """q_i = a e_0, k_j* = b e_0, other keys 0, a*b/sqrt(D) = 100."""
    B, S, H, D = 1, 64, 1, 64
    a, b, jstar = 32.0, 25.0, 17
    q = np.zeros((B, 4, H, D)); q[..., 0] = a
    k = np.zeros((B, S, H, D)); k[0, jstar, 0, 0] = b
    v = _rand((B, S, H, D), 8)
    out, lse = oracle.attention(q, k, v)
    assert np.max(np.abs(out - v[:, jstar:jstar + 1])) < 1e-40 + S * math.exp(-100) * 10
    assert np.max(np.abs(lse - (100.0 + math.log1p((S - 1) * math.exp(-100.0))))) < 1e-12


def test_softmax_rows_sum_to_one():
    """With V = identity (v_j = e_j) the output rows are the softmax rows."""
    B, S, H = 1, 24, 2
    q, k = _rand((B, 9, H, S), 9, 2.0), _rand((B, S, H, S), 10, 2.0)
    v = np.broadcast_to(np.eye(S)[None, :, None, :], (B, S, H, S)).copy()
    out, _ = oracle.attention(q, k, v)
    assert np.min(out) > 0.0
    assert np.max(np.abs(out.sum(axis=-1) - 1.0)) < 1e-13


def test_empty_key_set_is_neutral():
    q = _rand((1, 3, 1, 4), 11)
    out, lse = oracle.attention(q, np.zeros((1, 0, 1, 4)), np.zeros((1, 0, 1, 4)))
    assert np.all(out == 0) and np.all(np.isneginf(lse))


# ----------------------------------------------------------------- LSE merge

def test_merge_two_partials_by_hand():
    """LSE_1 = 0, LSE_2 = ln 3: LSE = ln 4, weights 1/4 and 3/4."""
    o1 = np.full((1, 1, 1, 2), 2.0); o2 = np.full((1, 1, 1, 2), -1.0)
    out, lse = oracle.lse_merge([o1, o2], [np.zeros((1, 1, 1)), np.full((1, 1, 1), math.log(3.0))])
    assert abs(lse[0, 0, 0] - math.log(4.0)) < 1e-15
    assert np.max(np.abs(out - (0.25 * 2.0 + 0.75 * -1.0))) < 1e-15


def test_merge_of_zero_key_chunks_closed_form():
    """K = 0: chunk c has LSE = ln len_c and out = mean of its V; merged LSE = ln S."""
    lens = [5, 0, 11, 3]
    S, D = sum(lens), 6
    q = _rand((1, 4, 1, D), 12); v = _rand((1, S, 1, D), 13)
    off = oracle.offsets(lens)
    outs, lses = [], []
    for c, n in enumerate(lens):
        o, l = oracle.attention(q, np.zeros((1, n, 1, D)), v[:, off[c]:off[c + 1]])
        outs.append(o); lses.append(l)
        if n:
            assert np.max(np.abs(l - math.log(n))) < 1e-14
    out, lse = oracle.lse_merge(outs, lses)
    assert np.max(np.abs(lse - math.log(S))) < 1e-14
    assert np.max(np.abs(out - v.mean(axis=1, keepdims=True))) < 1e-14


def test_merge_with_all_empty_partials():
    o = np.zeros((1, 2, 1, 3))
    out, lse = oracle.lse_merge([o, o], [np.full((1, 1, 2), -np.inf)] * 2)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


# ----------------------------------------------------------------- ring / kv_gather

def test_ring_order_by_hand():
    # rank 2 of 4 starts with its own chunk, then receives from rank 1, 0, 3.
    assert oracle.ring_order(2, 4) == [2, 1, 0, 3]
    assert oracle.ring_order(0, 3) == [0, 2, 1]


@pytest.mark.parametrize("degree", [1, 2, 3, 4, 5, 6, 7, 8])
def test_ring_equals_monolithic_equal_chunks(degree):
    B, H, D = 2, 2, 8
    S = 8 * 3 * 5 * 7
    q, k, v = (_rand((B, S, H, D), s, 1.5) for s in (20, 21, 22))
    ref_o, ref_l = oracle.attention(q, k, v)
    o, l = oracle.ring_attention(q, k, v, degree)
    assert np.max(np.abs(o - ref_o)) < 1e-12 and np.max(np.abs(l - ref_l)) < 1e-12


@pytest.mark.parametrize("lens", [[1668, 1667, 1668], [0, 7, 0, 30], [37], [1, 1, 1, 50, 0, 2]])
def test_ring_equals_monolithic_uneven_chunks(lens):
    S = sum(lens)
    q, k, v = (_rand((1, S, 2, 4), s, 2.0) for s in (23, 24, 25))
    ref_o, ref_l = oracle.attention(q, k, v)
    o, l = oracle.ring_attention(q, k, v, len(lens), lens)
    assert np.max(np.abs(o - ref_o)) < 1e-12
    fin = np.isfinite(ref_l)
    assert np.array_equal(fin, np.isfinite(l)) and np.max(np.abs(l[fin] - ref_l[fin])) < 1e-12


def test_ring_step_partials_merge_to_ring():
    lens = [9, 4, 0, 12]
    S = sum(lens)
    q, k, v = (_rand((2, S, 3, 4), s) for s in (26, 27, 28))
    parts = [oracle.ring_step_partials(q, k, v, 4, t, lens) for t in range(4)]
    o, l = oracle.lse_merge([p[0] for p in parts], [p[1] for p in parts])
    ref_o, ref_l = oracle.attention(q, k, v)
    assert np.max(np.abs(o - ref_o)) < 1e-12 and np.max(np.abs(l - ref_l)) < 1e-12


def test_ring_rejects_indivisible_without_lens():
    q = np.zeros((1, 10, 1, 4))
    with pytest.raises(ValueError):
        oracle.ring_attention(q, q, q, 3)


@pytest.mark.parametrize("q_lens", [None, [3, 13, 0, 8]])
def test_kv_gather_equals_monolithic(q_lens):
    S = 24
    q, k, v = (_rand((2, S, 2, 8), s) for s in (29, 30, 31))
    ref_o, ref_l = oracle.attention(q, k, v)
    o, l = oracle.kv_gather_attention(q, k, v, 4, q_lens)
    assert np.max(np.abs(o - ref_o)) < 1e-12 and np.max(np.abs(l - ref_l)) < 1e-12


# ----------------------------------------------------------------- permutes

def test_permute_hand_worked_cases():
    with open(os.path.join(GOLDEN, "ulysses_permute_tiny.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        x = np.array(c["x_seq_sharded"], dtype=np.int64)
        y = oracle.ulysses_permute(x, c["B"], c["S"], c["H"], c["D"], c["degree"],
                                   c["seq_splits"], c["head_splits"])
        assert y.tolist() == c["y_head_sharded"]
        back = oracle.ulysses_unpermute(y, c["B"], c["S"], c["H"], c["D"], c["degree"],
                                        c["seq_splits"], c["head_splits"])
        assert back.tolist() == c["x_seq_sharded"]


def _brute_force_permute(x, B, S, H, D, seq, heads):
    """Element loop over every (b, s, h, d) with explicit rank lookup."""
    P = len(seq)
    so, ho = oracle.offsets(seq), oracle.offsets(heads)
    y = np.empty_like(x)
    for b in range(B):
        for s in range(S):
            r = max(i for i in range(P) if so[i] <= s and seq[i] > 0 and s < so[i + 1])
            for h in range(H):
                rp = max(i for i in range(P) if ho[i] <= h and heads[i] > 0 and h < ho[i + 1])
                for d in range(D):
                    src = B * so[r] * H * D + ((b * seq[r] + (s - so[r])) * H + h) * D + d
                    dst = B * S * ho[rp] * D + ((b * S + s) * heads[rp] + (h - ho[rp])) * D + d
                    y[dst] = x[src]
    return y


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_permute_matches_element_loop(seed):
    B, S, H, D, P = 2, 11, 7, 3, 3
    seq = inputs.random_splits(S, P, seed + 100)
    heads = inputs.random_splits(H, P, seed + 200)
    x = np.arange(B * S * H * D, dtype=np.int64)
    y = oracle.ulysses_permute(x, B, S, H, D, P, seq, heads)
    assert np.array_equal(y, _brute_force_permute(x, B, S, H, D, seq, heads))


@pytest.mark.parametrize("P", [1, 2, 4, 8])
def test_permute_even_split_equals_reshape_transpose(P):
    """Textbook form for B = 1, even splits: y = x.reshape(S, P, H/P, D).transpose(1, 0, 2, 3)."""
    B, S, H, D = 1, 16, 8, 5
    x = np.arange(B * S * H * D, dtype=np.int64)
    y = oracle.ulysses_permute(x, B, S, H, D, P)
    ref = x.reshape(S, P, H // P, D).transpose(1, 0, 2, 3).reshape(-1)
    assert np.array_equal(y, ref)


def test_degree_one_is_identity():
    x = np.arange(2 * 5 * 3 * 4, dtype=np.int64)
    assert np.array_equal(oracle.ulysses_permute(x, 2, 5, 3, 4, 1), x)


@pytest.mark.parametrize("seed", range(6))
def test_permute_round_trip_and_bijection(seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    P = int(rng.integers(1, 9))
    B, S, H, D = int(rng.integers(1, 3)), int(rng.integers(1, 40)), int(rng.integers(1, 12)), 4
    seq = inputs.random_splits(S, P, seed + 7)
    heads = inputs.random_splits(H, P, seed + 8)
    x = np.arange(B * S * H * D, dtype=np.int64)
    y = oracle.ulysses_permute(x, B, S, H, D, P, seq, heads)
    assert np.array_equal(np.sort(y), x)                      # every element exactly once
    assert np.array_equal(oracle.ulysses_unpermute(y, B, S, H, D, P, seq, heads), x)


def test_permute_rejects_indivisible_without_splits():
    with pytest.raises(ValueError):
        oracle.ulysses_permute(np.zeros(30), 1, 5, 6, 1, 4)


# ----------------------------------------------------------------- flows

def _seq_rank_buffers_from_full(x, seq):
    off = oracle.offsets(seq)
    return np.concatenate([x[:, off[r]:off[r + 1]].reshape(-1) for r in range(len(seq))])


@pytest.mark.parametrize("B,seq,heads", [(1, [6, 6], [2, 2]), (2, [5, 0, 7], [3, 1, 0]), (2, [3, 4, 5, 0], [1, 1, 1, 1])])
def test_ulysses_attention_equals_monolithic(B, seq, heads):
    S, H, D = sum(seq), sum(heads), 4
    q, k, v = (_rand((B, S, H, D), s) for s in (40, 41, 42))
    ref_o, ref_l = oracle.attention(q, k, v)
    qf, kf, vf = (_seq_rank_buffers_from_full(x, seq) for x in (q, k, v))
    o, l = oracle.ulysses_attention(qf, kf, vf, B, S, H, D, len(seq), seq, heads)
    assert np.max(np.abs(o - _seq_rank_buffers_from_full(ref_o, seq))) < 1e-12
    assert np.max(np.abs(l - ref_l)) < 1e-12


@pytest.mark.parametrize("B,R,U,ring_lens,heads", [(1, 2, 2, None, None), (2, 3, 2, [5, 0, 9], [3, 1]), (1, 4, 3, [4, 4, 3, 5], [2, 2, 1])])
def test_unified_equals_monolithic(B, R, U, ring_lens, heads):
    S = 16 if ring_lens is None else sum(ring_lens)
    H = 4 if heads is None else sum(heads)
    q, k, v = (_rand((B, S, H, 4), s) for s in (43, 44, 45))
    ref_o, ref_l = oracle.attention(q, k, v)
    o, l = oracle.unified_attention(q, k, v, R, U, ring_lens, heads)
    assert np.max(np.abs(o - ref_o)) < 1e-12 and np.max(np.abs(l - ref_l)) < 1e-12


# ----------------------------------------------------------------- causal

def test_causal_attention_matches_scalar_brute_force():
    """Scalar loops over the visible keys j <= i only, math.exp, no max."""
    B, S, H, D = 2, 6, 2, 4
    q, k, v = _rand((B, S, H, D), 50), _rand((B, S, H, D), 51), _rand((B, S, H, D), 52)
    out, lse = oracle.causal_attention(q, k, v)
    for b in range(B):
        for h in range(H):
            for i in range(S):
                w = [math.exp(sum(q[b, i, h, d] * k[b, j, h, d] for d in range(D)) / math.sqrt(D)) for j in range(i + 1)]
                z = sum(w)
                assert abs(lse[b, h, i] - math.log(z)) < 1e-12
                for d in range(D):
                    assert abs(out[b, i, h, d] - sum(w[j] * v[b, j, h, d] for j in range(i + 1)) / z) < 1e-12


def test_causal_matches_torch_sdpa_float64():
    """Independent library routine: torch SDPA with is_causal=True (float64, CPU)."""
    cfg, q, k, v = _tiny_f64()
    out, lse = oracle.causal_attention(q, k, v)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True).permute(0, 2, 1, 3).numpy()
    assert np.max(np.abs(out - ref)) < 1e-12
    S = q.shape[1]
    scores = torch.matmul(tq, tk.transpose(-1, -2)) / math.sqrt(cfg["D"])
    scores = scores.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    assert np.max(np.abs(lse - torch.logsumexp(scores, dim=-1).numpy())) < 1e-12


def test_causal_zero_keys_closed_form():
    """K = 0: query i sees i + 1 equal scores, so lse_i = ln(i + 1) and out_i is
    the running mean of v_0..v_i (an off-by-one in the mask changes both)."""
    B, S, H, D = 2, 23, 3, 8
    q, v = _rand((B, S, H, D), 53), _rand((B, S, H, D), 54)
    out, lse = oracle.causal_attention(q, np.zeros((B, S, H, D)), v)
    n = np.arange(1, S + 1)
    assert np.max(np.abs(lse - np.log(n)[None, None, :])) < 1e-13
    running_mean = np.cumsum(v, axis=1) / n[None, :, None, None]
    assert np.max(np.abs(out - running_mean)) < 1e-13


def test_causal_first_token_returns_its_value():
    B, S, H, D = 1, 9, 2, 4
    q, k, v = _rand((B, S, H, D), 55, 3.0), _rand((B, S, H, D), 56, 3.0), _rand((B, S, H, D), 57)
    out, lse = oracle.causal_attention(q, k, v)
    assert np.max(np.abs(out[:, 0] - v[:, 0])) < 1e-15
    s00 = np.einsum("bhd,bhd->bh", q[:, 0], k[:, 0]) / math.sqrt(D)
    assert np.max(np.abs(lse[:, :, 0] - s00)) < 1e-13


def test_causal_query_without_visible_key_is_neutral():
    q, k, v = _rand((1, 2, 1, 4), 58), _rand((1, 3, 1, 4), 59), _rand((1, 3, 1, 4), 60)
    out, lse = oracle.attention(q, k, v, np.array([4, 7]), np.array([6, 7, 9]))
    assert np.all(out[0, 0] == 0) and np.isneginf(lse[0, 0, 0])
    o1, l1 = oracle.attention(q[:, 1:], k[:, :2], v[:, :2])        # query 7 sees keys 6 and 7
    assert np.max(np.abs(out[:, 1:] - o1)) < 1e-14 and np.max(np.abs(lse[:, :, 1:] - l1)) < 1e-14


@pytest.mark.parametrize("degree,lens", [(1, None), (4, None), (3, [5, 0, 9]), (5, [1, 7, 0, 3, 6]), (2, [13, 1])])
def test_causal_ring_equals_monolithic(degree, lens):
    S = 16 if lens is None else sum(lens)
    B, H, D = 2, 3, 4
    q, k, v = (_rand((B, S, H, D), s) for s in (61, 62, 63))
    ref_o, ref_l = oracle.causal_attention(q, k, v)
    o, l = oracle.ring_attention(q, k, v, degree, lens, causal=True)
    assert np.max(np.abs(o - ref_o)) < 1e-12 and np.max(np.abs(l - ref_l)) < 1e-12


def test_causal_ring_steps_after_the_shard_are_empty_and_merge_to_ring():
    B, S, H, D, P = 1, 12, 2, 4, 3
    q, k, v = (_rand((B, S, H, D), s) for s in (64, 65, 66))
    parts = [oracle.ring_step_partials(q, k, v, P, t, causal=True) for t in range(P)]
    off = oracle.offsets([4, 4, 4])
    for t, (o, l) in enumerate(parts):
        for r in range(P):
            c = (r - t) % P
            rows = slice(off[r], off[r + 1])
            if c > r:
                assert np.all(o[:, rows] == 0) and np.all(np.isneginf(l[:, :, rows]))
            else:
                assert np.all(np.isfinite(l[:, :, rows]))
    o, l = oracle.lse_merge([p[0] for p in parts], [p[1] for p in parts])
    ref_o, ref_l = oracle.causal_attention(q, k, v)
    assert np.max(np.abs(o - ref_o)) < 1e-12 and np.max(np.abs(l - ref_l)) < 1e-12


@pytest.mark.parametrize("B,seq,heads", [(1, [6, 6], [2, 2]), (2, [5, 0, 7], [3, 1, 0])])
def test_causal_ulysses_equals_monolithic(B, seq, heads):
    S, H, D = sum(seq), sum(heads), 4
    q, k, v = (_rand((B, S, H, D), s) for s in (67, 68, 69))
    ref_o, ref_l = oracle.causal_attention(q, k, v)
    qf, kf, vf = (_seq_rank_buffers_from_full(x, seq) for x in (q, k, v))
    o, l = oracle.ulysses_attention(qf, kf, vf, B, S, H, D, len(seq), seq, heads, causal=True)
    assert np.max(np.abs(o - _seq_rank_buffers_from_full(ref_o, seq))) < 1e-12
    assert np.max(np.abs(l - ref_l)) < 1e-12


@pytest.mark.parametrize("B,R,U,ring_lens,heads", [(1, 2, 2, None, None), (2, 3, 2, [5, 0, 9], [3, 1])])
def test_causal_unified_equals_monolithic(B, R, U, ring_lens, heads):
    S = 16 if ring_lens is None else sum(ring_lens)
    H = 4 if heads is None else sum(heads)
    q, k, v = (_rand((B, S, H, 4), s) for s in (70, 71, 72))
    ref_o, ref_l = oracle.causal_attention(q, k, v)
    o, l = oracle.unified_attention(q, k, v, R, U, ring_lens, heads, causal=True)
    assert np.max(np.abs(o - ref_o)) < 1e-12 and np.max(np.abs(l - ref_l)) < 1e-12


# ----------------------------------------------------------------- planted mistakes

def _pins_pass(fn):
    try:
        fn()
        return True
    except AssertionError:
        return False


def test_planted_mistakes_are_caught(monkeypatch):
    """Plant plausible mistakes in the oracle; at least one pin must fail for each."""
    import importlib
    oa = importlib.import_module("oracle.attention")
    op = importlib.import_module("oracle.permute")
    good_rows, good_merge, good_permute = oa.attention_rows, oa.lse_merge, op.ulysses_permute

    def no_scale(q, k, v):
        s = q @ k.T
        m = s.max(1, keepdims=True); e = np.exp(s - m); l = e.sum(1, keepdims=True)
        return (e @ v) / l, (m + np.log(l))[:, 0]

    def log2_lse(q, k, v):
        o, l = good_rows(q, k, v)
        return o, l / math.log(2.0)

    def merge_flipped(outs, lses):
        o, l = good_merge(outs, [-x for x in lses])
        return o, -l

    def permute_off_by_one(x, B, S, H, D, degree, seq_splits=None, head_splits=None):
        y = good_permute(x, B, S, H, D, degree, seq_splits, head_splits)
        return np.roll(y, 1)

    cases = [
        ("attention_rows", no_scale, [test_attention_matches_torch_sdpa_float64]),
        ("attention_rows", log2_lse, [test_zero_keys_give_uniform_softmax]),
        ("lse_merge", merge_flipped, [test_merge_two_partials_by_hand]),
    ]
    for name, bad, pins in cases:
        good = {"attention_rows": good_rows, "lse_merge": good_merge}[name]
        monkeypatch.setattr(oa, name, bad)
        if hasattr(oracle, name):
            monkeypatch.setattr(oracle, name, bad)
        assert not all(_pins_pass(p) for p in pins), f"planted mistake in {name} not caught"
        monkeypatch.setattr(oa, name, good)
        if hasattr(oracle, name):
            monkeypatch.setattr(oracle, name, good)
    good_causal = oa.causal_attention_rows

    def causal_strict(q, k, v, q_pos, k_pos):
        return good_causal(q, k, v, np.asarray(q_pos) - 1, k_pos)   # key j visible iff j < i

    monkeypatch.setattr(oa, "causal_attention_rows", causal_strict)
    assert not _pins_pass(test_causal_zero_keys_closed_form), "planted strict causal mask not caught"
    monkeypatch.setattr(oa, "causal_attention_rows", good_causal)
    monkeypatch.setattr(op, "ulysses_permute", permute_off_by_one)
    monkeypatch.setattr(oracle, "ulysses_permute", permute_off_by_one)
    assert not _pins_pass(test_permute_hand_worked_cases)
