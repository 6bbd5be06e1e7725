"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on seeded
inputs: small shapes that span several tiles and a ragged tail (full
comparison), edge cases (S=1, chunks shorter than a tile, empty chunks, D=64),
bit-exact permutes, and the named workloads (full or sampled rows)."""
import numpy as np
import pytest
import torch

import oracle
from context_attention_long_b200 import api, build, inputs

from gpu_util import (assert_close, bits_of, f64_of, full_to_rank_buffers, oracle_rows,
                      rank_buffers_to_full, sample_positions, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _qkv(B, S, H, D, seed, rms=True):
    q, k, v = inputs.make_qkv(B, S, H, D, seed, rms)
    return (q, k, v), tuple(inputs.bf16_bits_to_f64(x) for x in (q, k, v)), tuple(to_dev(x) for x in (q, k, v))


def _no_timeouts():
    st, code = api.cpattn_device_status()
    assert st == 0 and code == 0, f"device wait expired: code {code:#x}"


# ------------------------------------------------------------------ ring

RING_CASES = [
    # B, H, S, D, degree, lens
    (1, 2, 256, 64, 4, None),               # tiny workload shape
    (1, 2, 256, 64, 1, None),
    (2, 3, 300, 128, 3, [100, 0, 200]),     # ragged, an empty chunk
    (1, 1, 1, 64, 1, None),                 # single token
    (1, 2, 129, 128, 2, [1, 128]),          # one-token chunk
    (2, 2, 1000, 128, 4, [250, 250, 250, 250]),
    (1, 4, 777, 64, 5, [7, 300, 0, 270, 200]),
    (1, 3, 640, 128, 8, [64, 100, 36, 128, 129, 0, 120, 63]),
]


@pytest.mark.parametrize("B,H,S,D,P,lens", RING_CASES)
def test_ring_attention_matches_oracle(B, H, S, D, P, lens):
    _, (q, k, v), (dq, dk, dv) = _qkv(B, S, H, D, 100 + S + P, rms=(D == 128))
    out, lse = api.cpattn_ring_attention(dq, dk, dv, P, lens)
    torch.cuda.synchronize()
    _no_timeouts()
    ref_o, ref_l = oracle.ring_attention(q, k, v, P, lens)
    assert_close(f64_of(out), f64_of(lse), ref_o, ref_l, f"ring B{B} H{H} S{S} D{D} P{P}")


@pytest.mark.parametrize("B,H,S,D,P,lens", [RING_CASES[0], RING_CASES[2], RING_CASES[6]])
def test_ring_steps_and_merge_match_oracle(B, H, S, D, P, lens):
    _, (q, k, v), (dq, dk, dv) = _qkv(B, S, H, D, 200 + S, rms=(D == 128))
    parts_o, parts_l = [], []
    for t in range(P):
        po, pl = api.cpattn_ring_step(dq, dk, dv, P, t, lens)
        ro, rl = oracle.ring_step_partials(q, k, v, P, t, lens)
        assert_close(f64_of(po), f64_of(pl), ro, rl, f"step {t}")
        # empty chunk: exactly zero output and -inf LSE
        if lens is not None:
            off = oracle.offsets(lens)
            for r in range(P):
                if lens[oracle.ring_order(r, P)[t]] == 0 and lens[r] > 0:
                    assert torch.all(po[:, off[r]:off[r + 1]] == 0)
                    assert torch.all(torch.isneginf(pl[:, :, off[r]:off[r + 1]]))
        parts_o.append(po)
        parts_l.append(pl)
    f32, b16, lse = api.cpattn_lse_merge(torch.stack(parts_o), torch.stack(parts_l), want_f32=True)
    torch.cuda.synchronize()
    _no_timeouts()
    ref_o, ref_l = oracle.ring_attention(q, k, v, P, lens)
    assert_close(f64_of(b16), f64_of(lse), ref_o, ref_l, "merged bf16")
    assert_close(f64_of(f32), None, ref_o, None, "merged f32")


@pytest.mark.parametrize("P,D", [(1, 64), (2, 128), (3, 64), (5, 128), (8, 128), (13, 64), (20, 128)])
def test_lse_merge_matches_oracle(P, D):
    B, S, H = 2, 37, 3
    rng = np.random.Generator(np.random.PCG64(P * 7 + D))
    po = rng.standard_normal((P, B, S, H, D)).astype(np.float32)
    pl = (rng.standard_normal((P, B, H, S)) * 5).astype(np.float32)
    pl[rng.random(pl.shape) < 0.2] = -np.inf            # empty partials
    pl[:, 0, 0, :3] = -np.inf                           # rows with no keys at all
    f32, b16, lse = api.cpattn_lse_merge(torch.from_numpy(po).cuda(), torch.from_numpy(pl).cuda(), want_f32=True)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.lse_merge(list(po.astype(np.float64)), list(pl.astype(np.float64)))
    got = f64_of(f32)
    assert np.max(np.abs(got - ref_o)) < 1e-5
    gl = f64_of(lse)
    fin = np.isfinite(ref_l)
    assert np.array_equal(fin, np.isfinite(gl))
    assert np.max(np.abs(gl[fin] - ref_l[fin])) < 1e-5
    assert np.all(got[0, :3, 0, :] == 0)
    assert np.max(np.abs(f64_of(b16) - ref_o)) <= 2.0 ** -8 * np.max(np.abs(ref_o)) + 1e-6


def test_lse_merge_in_place_alias():
    P, B, S, H, D = 4, 1, 64, 2, 128
    rng = np.random.Generator(np.random.PCG64(3))
    po = rng.standard_normal((P, B, S, H, D)).astype(np.float32)
    pl = rng.standard_normal((P, B, H, S)).astype(np.float32)
    dpo, dpl = torch.from_numpy(po).cuda(), torch.from_numpy(pl).cuda()
    api.cpattn_lse_merge(dpo, dpl, out_f32=dpo[0], lse_out=dpl[0], want_bf16=False)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.lse_merge(list(po.astype(np.float64)), list(pl.astype(np.float64)))
    assert np.max(np.abs(f64_of(dpo[0]) - ref_o)) < 1e-5
    assert np.max(np.abs(f64_of(dpl[0]) - ref_l)) < 1e-5


# ------------------------------------------------------------------ kv_gather

@pytest.mark.parametrize("B,H,S,D,P,lens", [(2, 3, 600, 128, 8, None), (1, 2, 333, 64, 3, [0, 300, 33]),
                                            (1, 2, 256, 64, 4, None)])
def test_kv_gather_matches_oracle(B, H, S, D, P, lens):
    if lens is None and S % P:
        pytest.skip("indivisible")
    _, (q, k, v), (dq, dk, dv) = _qkv(B, S, H, D, 300 + S, rms=(D == 128))
    out, lse = api.cpattn_kv_gather_attention(dq, dk, dv, P, lens)
    torch.cuda.synchronize()
    _no_timeouts()
    ref_o, ref_l = oracle.kv_gather_attention(q, k, v, P, lens)
    assert_close(f64_of(out), f64_of(lse), ref_o, ref_l, "kv_gather")


# ------------------------------------------------------------------ permutes

PERMUTE_CASES = [
    # B, S, H, D, degree, seq, heads, dtype
    (1, 256, 2, 64, 2, None, None, torch.bfloat16),
    (2, 37, 7, 64, 3, [10, 0, 27], [3, 3, 1], torch.bfloat16),
    (2, 50, 6, 128, 4, [20, 10, 10, 10], [0, 2, 2, 2], torch.float32),
    (1, 9, 5, 8, 2, [4, 5], [2, 3], torch.uint8),       # 8-byte rows: rejected (not a multiple of 16)
    (3, 19, 8, 16, 8, [1, 2, 3, 4, 0, 0, 4, 5], [1] * 8, torch.float32),
    (1, 33, 3, 16, 3, [11, 11, 11], [1, 1, 1], torch.uint8),   # 16-byte rows of bytes
    (2, 41, 5, 12, 3, [13, 0, 28], [2, 1, 2], torch.float32),  # 48-byte rows: 3 vectors, lanes cross rows
    (1, 17, 3, 1000, 2, [9, 8], [2, 1], torch.float32),        # 4000-byte rows: 250 vectors per row
    (1, 10007, 30, 128, 4, [2502, 2502, 2502, 2501], [8, 8, 7, 7], torch.bfloat16),
]


@pytest.mark.parametrize("B,S,H,D,P,seq,heads,dtype", PERMUTE_CASES)
def test_permute_bit_exact_and_round_trip(B, S, H, D, P, seq, heads, dtype):
    n = B * S * H * D
    esz = torch.tensor([], dtype=dtype).element_size()
    if (D * esz) % 16:
        with pytest.raises(api.CpattnError):
            api.cpattn_ulysses_permute(torch.zeros(n, dtype=dtype, device="cuda"), B, S, H, D, P, seq, heads)
        return
    rng = np.random.Generator(np.random.PCG64(n))
    raw = rng.integers(0, 256, size=n * esz, dtype=np.uint8)
    x = torch.from_numpy(raw).cuda().view(dtype)
    y = api.cpattn_ulysses_permute(x, B, S, H, D, P, seq, heads)
    back = api.cpattn_ulysses_unpermute(y, B, S, H, D, P, seq, heads)
    torch.cuda.synchronize()
    xb = raw.view({1: np.uint8, 2: np.uint16, 4: np.uint32}[esz])
    ref = oracle.ulysses_permute(xb, B, S, H, D, P, seq, heads)
    assert np.array_equal(y.cpu().view(torch.uint8).numpy().view(ref.dtype), ref)
    assert torch.equal(back.view(torch.uint8), x.view(torch.uint8))


@pytest.mark.parametrize("B,S,H,D,P,seq,heads", [
    (1, 4608, 24, 128, 4, None, None),                    # image-DiT Ulysses 4
    (2, 300, 7, 64, 3, [100, 0, 200], [3, 2, 2]),        # uneven, an empty sequence shard
])
def test_permute_qkv_equals_three_permutes(B, S, H, D, P, seq, heads):
    """The one-launch Q/K/V permute is bit-identical to the oracle's permute of
    each tensor."""
    n = B * S * H * D
    rng = np.random.Generator(np.random.PCG64(n + 5))
    raws = [rng.integers(0, 1 << 16, size=n, dtype=np.uint16) for _ in range(3)]
    xs = [torch.from_numpy(r.view(np.int16)).cuda().view(torch.bfloat16) for r in raws]
    ys = api.cpattn_ulysses_permute_qkv(*xs, B, S, H, D, P, seq, heads)
    torch.cuda.synchronize()
    for raw, y in zip(raws, ys):
        ref = oracle.ulysses_permute(raw, B, S, H, D, P, seq, heads)
        assert np.array_equal(bits_of(y).reshape(-1), ref)


# ------------------------------------------------------------------ Ulysses / unified

@pytest.mark.parametrize("B,S,H,D,P,seq,heads", [
    (1, 256, 2, 64, 2, None, None),                       # tiny workload
    (2, 300, 7, 128, 3, [100, 50, 150], [3, 2, 2]),       # uneven, B = 2
    (1, 200, 5, 64, 4, [60, 0, 70, 70], [2, 1, 2, 0]),    # empty rank
])
def test_ulysses_attention_matches_oracle(B, S, H, D, P, seq, heads):
    (qb, kb, vb), (q, k, v), _ = _qkv(B, S, H, D, 400 + S, rms=(D == 128))
    seq_l = seq or [S // P] * P
    flat = [to_dev(full_to_rank_buffers(x, seq_l)) for x in (qb, kb, vb)]
    out, lse = api.cpattn_ulysses_attention(*flat, B, S, H, D, P, seq, heads)
    torch.cuda.synchronize()
    _no_timeouts()
    got = rank_buffers_to_full(f64_of(out), B, S, H, D, seq_l)
    qf, kf, vf = (full_to_rank_buffers(x, seq_l) for x in (q, k, v))
    ref_flat, ref_l = oracle.ulysses_attention(qf, kf, vf, B, S, H, D, P, seq, heads)
    ref = rank_buffers_to_full(ref_flat, B, S, H, D, seq_l)
    assert_close(got, f64_of(lse), ref, ref_l, "ulysses")


@pytest.mark.parametrize("B,S,H,D,R,U,ring_lens,heads", [
    (1, 256, 4, 64, 2, 2, None, None),
    (2, 500, 4, 128, 3, 2, [200, 0, 300], [3, 1]),
    (1, 390, 6, 128, 4, 3, [90, 100, 100, 100], [2, 2, 2]),
])
def test_unified_attention_matches_oracle(B, S, H, D, R, U, ring_lens, heads):
    _, (q, k, v), (dq, dk, dv) = _qkv(B, S, H, D, 500 + S, rms=(D == 128))
    out, lse = api.cpattn_unified_attention(dq, dk, dv, R, U, ring_lens, heads)
    torch.cuda.synchronize()
    _no_timeouts()
    ref_o, ref_l = oracle.unified_attention(q, k, v, R, U, ring_lens, heads)
    assert_close(f64_of(out), f64_of(lse), ref_o, ref_l, "unified")


# ------------------------------------------------------------------ named workloads

def test_tiny_workload_all_paths():
    cfg, qb, kb, vb = inputs.config_inputs("tiny")
    q, k, v = (inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb))
    dq, dk, dv = (to_dev(x) for x in (qb, kb, vb))
    ref_o, ref_l = oracle.attention(q, k, v)
    o, l = api.cpattn_ring_attention(dq, dk, dv, cfg["ring_degree"])
    assert_close(f64_of(o), f64_of(l), *oracle.ring_attention(q, k, v, cfg["ring_degree"]), "tiny ring")
    o, l = api.cpattn_kv_gather_attention(dq, dk, dv, cfg["ring_degree"])
    assert_close(f64_of(o), f64_of(l), ref_o, ref_l, "tiny kv_gather")
    B, S, H, D = qb.shape
    o, l = api.cpattn_ulysses_attention(dq.reshape(-1), dk.reshape(-1), dv.reshape(-1), B, S, H, D,
                                        cfg["ulysses_degree"])
    assert_close(f64_of(o).reshape(B, S, H, D), f64_of(l), ref_o, ref_l, "tiny ulysses")
    _no_timeouts()


def test_dit_workload_ring_and_ulysses_full():
    cfg, qb, kb, vb = inputs.config_inputs("dit")
    B, S, H, D = qb.shape
    q, k, v = (inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb))
    dq, dk, dv = (to_dev(x) for x in (qb, kb, vb))
    ref_o, ref_l = oracle.ring_attention(q, k, v, cfg["ring_degree"])
    o, l = api.cpattn_ring_attention(dq, dk, dv, cfg["ring_degree"])
    assert_close(f64_of(o), f64_of(l), ref_o, ref_l, "dit ring")
    o, l = api.cpattn_ulysses_attention(dq.reshape(-1), dk.reshape(-1), dv.reshape(-1), B, S, H, D,
                                        cfg["ulysses_degree"])
    assert_close(f64_of(o).reshape(B, S, H, D), f64_of(l), ref_o, ref_l, "dit ulysses")
    _no_timeouts()


def _sampled_check(out, lse, qb, kb, vb, positions, what):
    ref_o, ref_l = oracle_rows(oracle, qb, kb, vb, positions)
    got_o = f64_of(out)[:, positions]
    got_l = f64_of(lse)[:, :, positions]
    assert_close(got_o, got_l, ref_o, ref_l, what)


def test_hires_workload_sampled():
    cfg, qb, kb, vb = inputs.config_inputs("hires")
    B, S, H, D = qb.shape
    P = cfg["ring_degree"]
    dq, dk, dv = (to_dev(x) for x in (qb, kb, vb))
    pos = sample_positions(S, list(range(0, S + 1, S // P)), 24, 1)
    o, l = api.cpattn_ring_attention(dq, dk, dv, P)
    _sampled_check(o, l, qb, kb, vb, pos, "hires ring")
    o, l = api.cpattn_kv_gather_attention(dq, dk, dv, cfg["kv_gather_degree"])
    _sampled_check(o, l, qb, kb, vb, pos, "hires kv_gather")
    # Ulysses on rank buffers of the same tensors (B = 2: rank buffers differ from BSHD)
    Pu = cfg["ulysses_degree"]
    seq = [S // Pu] * Pu
    flat = [to_dev(full_to_rank_buffers(x, seq)) for x in (qb, kb, vb)]
    o, l = api.cpattn_ulysses_attention(*flat, B, S, H, D, Pu)
    o_full = torch.from_numpy(rank_buffers_to_full(bits_of(o), B, S, H, D, seq).view(np.int16)).view(torch.bfloat16)
    _sampled_check(o_full, l, qb, kb, vb, pos, "hires ulysses")
    _no_timeouts()


def test_anything_workload_sampled():
    cfg, qb, kb, vb = inputs.config_inputs("anything")
    B, S, H, D = qb.shape
    dq, dk, dv = (to_dev(x) for x in (qb, kb, vb))
    lens = inputs.ring_anything_lens(S, cfg["ring_degree"], cfg["seed"])
    pos = sample_positions(S, oracle.offsets(lens), 24, 2)
    o, l = api.cpattn_ring_attention(dq, dk, dv, cfg["ring_degree"], lens)
    _sampled_check(o, l, qb, kb, vb, pos, "anything ring")
    seq = inputs.front_loaded_splits(S, cfg["ulysses_degree"])
    heads = inputs.front_loaded_splits(H, cfg["ulysses_degree"])
    assert heads == [8, 8, 7, 7]
    o, l = api.cpattn_ulysses_attention(dq.reshape(-1), dk.reshape(-1), dv.reshape(-1), B, S, H, D,
                                        cfg["ulysses_degree"], seq, heads)
    _sampled_check(o.reshape(B, S, H, D), l, qb, kb, vb, sample_positions(S, oracle.offsets(seq), 8, 3),
                   "anything ulysses")
    # the standard modes refuse the uneven workload (diffusers variants table)
    with pytest.raises(api.CpattnError):
        api.cpattn_ring_attention(dq, dk, dv, cfg["ring_degree"])
    with pytest.raises(api.CpattnError):
        api.cpattn_ulysses_attention(dq.reshape(-1), dk.reshape(-1), dv.reshape(-1), B, S, H, D,
                                     cfg["ulysses_degree"])
    _no_timeouts()


def test_video_workload_unified_sampled():
    cfg, qb, kb, vb = inputs.config_inputs("video")
    B, S, H, D = qb.shape
    R, U = cfg["ring_degree"], cfg["ulysses_degree"]
    dq, dk, dv = (to_dev(x) for x in (qb, kb, vb))
    pos = sample_positions(S, list(range(0, S + 1, S // R)), 16, 4)
    o, l = api.cpattn_unified_attention(dq, dk, dv, R, U)
    _sampled_check(o, l, qb, kb, vb, pos, "video unified")
    _no_timeouts()


# ------------------------------------------------------------------ invariants

def test_same_call_twice_is_byte_identical():
    """SGLang 'Numerics across node boundaries': the same deployment run twice
    must give byte-identical output."""
    cfg, qb, kb, vb = inputs.config_inputs("dit")
    dq, dk, dv = (to_dev(x) for x in (qb, kb, vb))
    o1, l1 = api.cpattn_ring_attention(dq, dk, dv, cfg["ring_degree"])
    o2, l2 = api.cpattn_ring_attention(dq, dk, dv, cfg["ring_degree"])
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)


def test_constant_v_and_zero_k_closed_forms():
    B, S, H, D = 1, 300, 2, 128
    qb, kb, vb = inputs.make_qkv(B, S, H, D, 9, True)
    dq, dk = to_dev(qb), to_dev(kb)
    v_const = torch.full((B, S, H, D), 0.375, dtype=torch.bfloat16, device="cuda")
    o, _ = api.cpattn_ring_attention(dq, dk, v_const, 3)
    assert torch.max(torch.abs(o.float() - 0.375)).item() <= 2.0 ** -9
    zk = torch.zeros_like(dk)
    o, l = api.cpattn_ring_attention(dq, zk, to_dev(vb), 3)
    assert torch.max(torch.abs(l - np.log(S))).item() < 1e-4
    mean_v = inputs.bf16_bits_to_f64(vb).mean(axis=1, keepdims=True)
    assert np.max(np.abs(f64_of(o) - mean_v)) < 1e-2
    _no_timeouts()


@pytest.mark.parametrize("D", [64, 128])
def test_one_hot_key_selects_its_value(D):
    """One-hot selection closed form: K = 0 except key j* = b e_0 and every query
    q_i = a e_0 (a, b exact in bf16), so each row has one logit s* = a b D**-0.5
    and S - 1 logits 0: out_i = v_j* up to e^-s* (S - 1), far below bf16's
    resolution, and LSE_i = ln(e^s* + S - 1).  Pinned for the ring (uneven
    chunks, j* in the middle chunk), kv_gather and the Ulysses flow."""
    B, S, H = 1, 333, 3
    a, b = 32.0, (25.0 if D == 64 else 36.0)      # D = 64: s* = 32 * 25 / 8 = 100 exactly
    s_star = a * b / np.sqrt(D)
    j_star = 170
    q = torch.zeros((B, S, H, D), dtype=torch.bfloat16, device="cuda")
    q[..., 0] = a
    k = torch.zeros_like(q)
    k[:, j_star, :, 0] = b
    _, _, (_, _, v) = _qkv(B, S, H, D, 77, rms=False)
    want_o = v[:, j_star:j_star + 1].expand(B, S, H, D)
    want_l = s_star + np.log1p((S - 1) * np.exp(-s_star))
    lens = [100, 133, 100]
    ws = torch.empty(api.cpattn_ulysses_workspace_bytes(B, H, S, D), dtype=torch.uint8, device="cuda")
    results = {
        "ring": api.cpattn_ring_attention(q, k, v, 3, lens),
        "kv_gather": api.cpattn_kv_gather_attention(q, k, v, 3, lens),
        "ulysses": api.cpattn_ulysses_attention(q.reshape(-1), k.reshape(-1), v.reshape(-1), B, S, H, D, 3,
                                                lens, [1, 1, 1], workspace=ws),
    }
    torch.cuda.synchronize()
    _no_timeouts()
    for name, (o, l) in results.items():
        o = o.view(B, S, H, D)
        assert torch.equal(o.view(torch.int16), want_o.contiguous().view(torch.int16)), f"{name}: not v_j*"
        assert np.max(np.abs(f64_of(l) - want_l)) <= 1e-3, f"{name}: LSE {f64_of(l).ravel()[:3]} vs {want_l}"


def test_lse_merge_dit_size_p4_full():
    """The merge of the ring-step partials of the image-DiT workload (P = 4),
    every row, against the oracle's merge of the same float32 partials."""
    cfg, qb, kb, vb = inputs.config_inputs("dit")
    B, S, H, D = qb.shape
    P = cfg["ring_degree"]
    dq, dk, dv = (to_dev(x) for x in (qb, kb, vb))
    po = torch.empty((P, B, S, H, D), dtype=torch.float32, device="cuda")
    pl = torch.empty((P, B, H, S), dtype=torch.float32, device="cuda")
    for t in range(P):
        api.cpattn_ring_step(dq, dk, dv, P, t, part_out=po[t], part_lse=pl[t])
    f32, b16, lse = api.cpattn_lse_merge(po, pl, want_f32=True)
    torch.cuda.synchronize()
    _no_timeouts()
    ref_o, ref_l = oracle.lse_merge(list(f64_of(po)), list(f64_of(pl)))
    assert np.max(np.abs(f64_of(f32) - ref_o)) < 1e-5
    assert np.max(np.abs(f64_of(lse) - ref_l)) < 1e-5
    assert np.max(np.abs(f64_of(b16) - ref_o)) <= 2.0 ** -8 * np.max(np.abs(ref_o)) + 1e-6


def test_lse_merge_video_size_p8_sampled():
    """The 8-way merge at the video workload's size (B1 S32760 H40 D128, the
    partials the bench times: 5.4 GB of float32), on sampled rows: the merge
    is independent per (b, h, s) row, so rows can be checked one by one."""
    B, S, H, D, P = 1, 32760, 40, 128, 8
    gen = torch.Generator(device="cuda").manual_seed(11)
    po = torch.randn((P, B, S, H, D), generator=gen, device="cuda", dtype=torch.float32)
    pl = torch.randn((P, B, H, S), generator=gen, device="cuda", dtype=torch.float32) * 4
    pl[1, :, :, ::7] = float("-inf")                 # empty partials
    pl[:, :, 3, 5] = float("-inf")                   # a row with no keys at all
    b16 = torch.empty((B, S, H, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    api.cpattn_lse_merge(po, pl, out_bf16=b16, lse_out=lse, want_f32=False)
    torch.cuda.synchronize()
    _no_timeouts()
    pos = np.unique(np.concatenate([[0, 5, 7, S - 1], sample_positions(S, [0, S], 60, 12)]))
    pt = torch.from_numpy(pos).cuda()
    ref_o, ref_l = oracle.lse_merge(list(f64_of(po[:, :, pt])), list(f64_of(pl[:, :, :, pt])))
    got_l = f64_of(lse[:, :, pt])
    fin = np.isfinite(ref_l)
    assert np.array_equal(fin, np.isfinite(got_l))
    assert np.max(np.abs(got_l[fin] - ref_l[fin])) < 1e-5
    assert np.max(np.abs(f64_of(b16[:, pt]) - ref_o)) <= 2.0 ** -8 * np.max(np.abs(ref_o)) + 1e-6
    assert np.all(f64_of(b16[:, 5, 3]) == 0)
    del po, pl
    torch.cuda.empty_cache()


def test_bounded_wait_reports_timeout_and_context_survives():
    api.cpattn_debug_wait_timeout(2000)
    st, code = api.cpattn_device_status()
    assert st == 7 and code != 0
    st, code = api.cpattn_device_status()
    assert st == 0 and code == 0
    # the context is still usable
    cfg, qb, kb, vb = inputs.config_inputs("tiny")
    o, l = api.cpattn_ring_attention(to_dev(qb), to_dev(kb), to_dev(vb), 4)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
