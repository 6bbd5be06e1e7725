"""Out-of-bounds checks: every output tensor is placed between 4 KiB guard
regions filled with 0xA5; the kernels must write exactly their output and
nothing around it (ragged tiles, uneven and empty chunks, split units, LSE
omitted), and an omitted LSE must not change the output."""
import numpy as np
import pytest
import torch

from context_attention_long_b200 import api, build, inputs

from gpu_util import to_dev

pytestmark = pytest.mark.gpu
GUARD = 4096


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def guarded(shape, dtype):
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    raw = torch.full((GUARD + n + GUARD,), 0xA5, dtype=torch.uint8, device="cuda")
    view = raw[GUARD:GUARD + n].view(dtype).view(shape)
    return raw, view


def guards_intact(raw):
    head = raw[:GUARD]
    tail = raw[-GUARD:]
    return bool(torch.all(head == 0xA5)) and bool(torch.all(tail == 0xA5))


@pytest.mark.parametrize("B,H,S,D,P,lens", [
    (1, 3, 333, 128, 3, [100, 0, 233]),
    (2, 2, 129, 64, 2, [1, 128]),
    (1, 2, 1152 * 2, 128, 2, None),        # shards with a lone tile: split units
])
def test_ring_writes_only_its_outputs(B, H, S, D, P, lens):
    q, k, v = (to_dev(x) for x in inputs.make_qkv(B, S, H, D, 7 + S, D == 128))
    out_raw, out = guarded((B, S, H, D), torch.bfloat16)
    lse_raw, lse = guarded((B, H, S), torch.float32)
    api.cpattn_ring_attention(q, k, v, P, lens, out=out, lse=lse)
    ref, ref_lse = api.cpattn_ring_attention(q, k, v, P, lens)
    no_lse_out, none = api.cpattn_ring_attention(q, k, v, P, lens, want_lse=False)
    torch.cuda.synchronize()
    assert none is None
    assert guards_intact(out_raw) and guards_intact(lse_raw)
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(lse, ref_lse)
    assert torch.equal(no_lse_out.view(torch.int16), ref.view(torch.int16))


def test_ring_step_and_merge_write_only_their_outputs():
    B, H, S, D, P, lens = 1, 2, 300, 128, 3, [100, 0, 200]
    q, k, v = (to_dev(x) for x in inputs.make_qkv(B, S, H, D, 11, True))
    po_raw, po = guarded((B, S, H, D), torch.float32)
    pl_raw, pl = guarded((B, H, S), torch.float32)
    api.cpattn_ring_step(q, k, v, P, 1, lens, part_out=po, part_lse=pl)
    parts = [api.cpattn_ring_step(q, k, v, P, t, lens) for t in range(P)]
    ob_raw, ob = guarded((B, S, H, D), torch.bfloat16)
    of_raw, of = guarded((B, S, H, D), torch.float32)
    lo_raw, lo = guarded((B, H, S), torch.float32)
    api.cpattn_lse_merge(torch.stack([x[0] for x in parts]), torch.stack([x[1] for x in parts]),
                         out_f32=of, out_bf16=ob, lse_out=lo)
    torch.cuda.synchronize()
    for raw in (po_raw, pl_raw, ob_raw, of_raw, lo_raw):
        assert guards_intact(raw)


def test_permute_and_flows_write_only_their_outputs():
    B, S, H, D, P = 2, 37, 7, 64, 3
    seq, heads = [10, 0, 27], [3, 3, 1]
    x = torch.randint(0, 255, (B * S * H * D * 2,), dtype=torch.uint8, device="cuda").view(torch.bfloat16)
    y_raw, y = guarded((B * S * H * D,), torch.bfloat16)
    api.cpattn_ulysses_permute(x, B, S, H, D, P, seq, heads, y=y)
    x2_raw, x2 = guarded((B * S * H * D,), torch.bfloat16)
    api.cpattn_ulysses_unpermute(y, B, S, H, D, P, seq, heads, x=x2)
    torch.cuda.synchronize()
    assert guards_intact(y_raw) and guards_intact(x2_raw)
    assert torch.equal(x2.view(torch.int16), x.view(torch.int16))
    # Ulysses flow with a guarded workspace and output
    D = 128
    qb, kb, vb = inputs.make_qkv(1, S, H, D, 13, True)
    q, k, v = (to_dev(t).reshape(-1) for t in (qb, kb, vb))
    ws_raw, ws = guarded((api.cpattn_ulysses_workspace_bytes(1, H, S, D),), torch.uint8)
    o_raw, o = guarded((S * H * D,), torch.bfloat16)
    api.cpattn_ulysses_attention(q, k, v, 1, S, H, D, P, seq, heads, out=o, workspace=ws)
    # unified with guarded workspace
    qf, kf, vf = (t.view(1, S, H, D) for t in (q, k, v))
    wu_raw, wu = guarded((api.cpattn_unified_workspace_bytes(1, H, S, D),), torch.uint8)
    ou_raw, ou = guarded((1, S, H, D), torch.bfloat16)
    api.cpattn_unified_attention(qf, kf, vf, 3, 2, [10, 20, 7], [4, 3], out=ou, workspace=wu)
    torch.cuda.synchronize()
    for raw in (ws_raw, o_raw, wu_raw, ou_raw):
        assert guards_intact(raw)


@pytest.mark.parametrize("B,H,S,D,P,lens", [
    (1, 3, 333, 128, 3, [100, 0, 233]),
    (1, 2, 1152 * 2, 128, 2, None),
])
def test_causal_paths_write_only_their_outputs(B, H, S, D, P, lens):
    q, k, v = (to_dev(x) for x in inputs.make_qkv(B, S, H, D, 17 + S, True))
    out_raw, out = guarded((B, S, H, D), torch.bfloat16)
    lse_raw, lse = guarded((B, H, S), torch.float32)
    api.cpattn_causal_ring_attention(q, k, v, P, lens, out=out, lse=lse)
    po_raw, po = guarded((B, S, H, D), torch.float32)
    pl_raw, pl = guarded((B, H, S), torch.float32)
    api.cpattn_causal_ring_step(q, k, v, P, P - 1, lens, part_out=po, part_lse=pl)
    seq = lens or [S // P] * P
    qf, kf, vf = (t.reshape(-1) for t in (q, k, v))
    ws_raw, ws = guarded((api.cpattn_ulysses_workspace_bytes(B, H, S, D),), torch.uint8)
    ou_raw, ou = guarded((B * S * H * D,), torch.bfloat16)
    api.cpattn_causal_ulysses_attention(qf, kf, vf, B, S, H, D, P, seq, [H - 1] + [1] * (P - 2) + [0] if P > 2 else None,
                                        out=ou, workspace=ws)
    torch.cuda.synchronize()
    for raw in (out_raw, lse_raw, po_raw, pl_raw, ws_raw, ou_raw):
        assert guards_intact(raw)
