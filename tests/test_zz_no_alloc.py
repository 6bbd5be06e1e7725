"""The no-allocation Ulysses entry point, for callers that cannot allocate
device memory when they call (a plug-in inside a framework that owns every
device allocation, a service that reserves all GPU memory at start-up).

It must give the same results as the workspace entry point
(cpattn_ulysses_attention) -- the same kernels on the same plans, so the same
bytes -- and match the fp64 oracle's Ulysses attention within the attention
tolerance used by the other GPU tests, on two calls in a row (the second call
finds the first call's data still in the library's scratch).  A problem that
fills the scratch almost to its end must write exactly its outputs, and a
problem whose scratch would not fit is rejected before anything is launched.
Calls go through the C ABI.  Runs alone in a fresh process or after the rest
of the suite; this file is named so that pytest collects it last."""
import numpy as np
import pytest
import torch

import oracle
from context_attention_long_b200 import _native, api, build, inputs

from gpu_util import (assert_close, f64_of, full_to_rank_buffers, oracle_rows, rank_buffers_to_full,
                      sample_positions, to_dev)

pytestmark = pytest.mark.gpu
GUARD = 4096


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _inputs(B, S, H, D, seed):
    return inputs.make_qkv(B, S, H, D, seed, D == 128)


def _guarded(numel, dtype):
    n = numel * torch.tensor([], dtype=dtype).element_size()
    raw = torch.full((GUARD + n + GUARD,), 0xA5, dtype=torch.uint8, device="cuda")
    return raw, raw[GUARD:GUARD + n].view(dtype)


def _guards_intact(raw):
    return bool(torch.all(raw[:GUARD] == 0xA5)) and bool(torch.all(raw[-GUARD:] == 0xA5))


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("want_lse", [True, False])
def test_noalloc_matches_workspace_entry_point_on_two_calls(D, want_lse):
    B, S, H, P = 2, 300, 7, 3
    seq, heads = [100, 50, 150], [3, 2, 2]
    assert api.cpattn_ulysses_workspace_bytes(B, H, S, D) <= api.NOALLOC_SCRATCH_BYTES
    for call, seed in enumerate((71, 72)):          # two calls in a row, different inputs
        q, k, v = (to_dev(full_to_rank_buffers(x, seq)) for x in _inputs(B, S, H, D, seed))
        ref_o, ref_l = api.cpattn_ulysses_attention(q, k, v, B, S, H, D, P, seq, heads)
        out = torch.empty_like(q)
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device) if want_lse else None
        api.cpattn_ulysses_attention_noalloc(q, k, v, B, S, H, D, P, seq, heads, out=out, lse=lse,
                                             want_lse=want_lse)
        torch.cuda.synchronize()
        st, code = api.cpattn_device_status()
        assert st == 0, f"device wait expired: {code:#x}"
        assert torch.equal(out.view(torch.int16), ref_o.view(torch.int16)), f"call {call}: output bytes differ"
        if want_lse:
            assert torch.equal(lse, ref_l), f"call {call}: LSE differs"


@pytest.mark.parametrize("B,S,H,D,P,seq,heads", [
    (1, 256, 4, 64, 2, None, None),                      # the standard (even) Ulysses split
    (2, 333, 10, 128, 4, [100, 0, 150, 83], [3, 3, 2, 2]),  # Ulysses Anything: uneven, one empty rank
])
def test_noalloc_matches_oracle_on_two_calls(B, S, H, D, P, seq, heads):
    seq_l = seq or [S // P] * P
    for call, seed in enumerate((81, 82)):
        qb, kb, vb = _inputs(B, S, H, D, seed)
        q, k, v = (to_dev(full_to_rank_buffers(x, seq_l)) for x in (qb, kb, vb))
        out, lse = api.cpattn_ulysses_attention_noalloc(q, k, v, B, S, H, D, P, seq, heads)
        torch.cuda.synchronize()
        st, code = api.cpattn_device_status()
        assert st == 0, f"device wait expired: {code:#x}"
        ref_o, ref_l = oracle.ulysses_attention(
            *(inputs.bf16_bits_to_f64(full_to_rank_buffers(x, seq_l)) for x in (qb, kb, vb)),
            B, S, H, D, P, seq, heads)
        assert_close(f64_of(out), f64_of(lse), ref_o, ref_l, f"no-alloc vs oracle, call {call}")


def test_noalloc_near_full_scratch_writes_only_its_outputs():
    # 8 * B*S*H*D = 67 100 672 bytes: the last of the four scratch buffers
    # ends 8 KiB before the end of the 64 MiB array.
    B, S, H, D, P = 1, 8191, 8, 128, 2
    need = api.cpattn_ulysses_workspace_bytes(B, H, S, D)
    assert api.NOALLOC_SCRATCH_BYTES - 16384 < need <= api.NOALLOC_SCRATCH_BYTES
    seq, heads = [4096, 4095], [5, 3]
    qb, kb, vb = _inputs(B, S, H, D, 91)
    q, k, v = (to_dev(full_to_rank_buffers(x, seq)) for x in (qb, kb, vb))
    n = B * S * H * D
    out_raw, out = _guarded(n, torch.bfloat16)
    lse_raw, lse = _guarded(B * H * S, torch.float32)
    for _ in range(2):
        api.cpattn_ulysses_attention_noalloc(q, k, v, B, S, H, D, P, seq, heads, out=out,
                                             lse=lse.view(B, H, S))
    ref_o, ref_l = api.cpattn_ulysses_attention(q, k, v, B, S, H, D, P, seq, heads)
    torch.cuda.synchronize()
    st, code = api.cpattn_device_status()
    assert st == 0, f"device wait expired: {code:#x}"
    assert _guards_intact(out_raw) and _guards_intact(lse_raw)
    assert torch.equal(out.view(torch.int16), ref_o.view(torch.int16))
    assert torch.equal(lse.view(B, H, S), ref_l)
    # sampled rows against the oracle's attention definition (Ulysses is
    # monolithic attention in exact arithmetic)
    pos = sample_positions(S, [0, 4096, S], 24, 5)
    ro, rl = oracle_rows(oracle, qb, kb, vb, pos)
    full = rank_buffers_to_full(f64_of(out), B, S, H, D, seq)
    assert_close(full[:, pos], f64_of(lse.view(B, H, S))[:, :, pos], ro, rl, "near-full scratch, sampled rows")


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = _native.load()
    # 8 * B*S*H*D bytes of scratch: 1 x 8192 x 16 x 128 needs 128 MiB > 64 MiB.
    B, S, H, D = 1, 8192, 16, 128
    assert api.cpattn_ulysses_workspace_bytes(B, H, S, D) > api.NOALLOC_SCRATCH_BYTES
    fake = 1 << 20   # never dereferenced: the size check comes before any launch
    st = lib.cpattn_ulysses_attention_noalloc(fake, fake, fake, fake, None, B, H, S, D, 4, None, None, None)
    assert st == 8   # CPATTN_ERR_WORKSPACE
    # one element over the limit: 1 x 8192 x 8 x 128 needs exactly 64 MiB and fits;
    # 1 x 8193 x 8 x 128 does not.
    st = lib.cpattn_ulysses_attention_noalloc(fake, fake, fake, fake, None, 1, 8, 8193, 128, 1, None, None, None)
    assert st == 8
