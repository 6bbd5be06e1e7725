"""The no-allocation Ulysses entry point, for callers that cannot allocate
device memory when they call (a plug-in inside a framework that owns every
device allocation, a service that reserves all GPU memory at start-up).

It must give the same results as the workspace entry point
(cpattn_ulysses_attention) within the attention tolerance used by the other
GPU tests, on two calls in a row -- the second call finds the first call's
data still in the library's scratch -- and must reject a problem whose scratch
would not fit, before launching anything.  Calls go through the C ABI.
Runs alone in a fresh process or after the rest of the suite; this file is
named so that pytest collects it last."""
import numpy as np
import pytest
import torch

from context_attention_long_b200 import _native, api, build, inputs

from gpu_util import assert_close, f64_of, full_to_rank_buffers, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _rank_buffers(B, S, H, D, seq, seed):
    qb, kb, vb = inputs.make_qkv(B, S, H, D, seed, True)
    return [to_dev(full_to_rank_buffers(x, seq)) for x in (qb, kb, vb)]


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    B, S, H, D, P = 2, 300, 7, 128, 3
    seq, heads = [100, 50, 150], [3, 2, 2]
    needed = api.cpattn_ulysses_workspace_bytes(B, H, S, D)
    assert needed <= api.NOALLOC_SCRATCH_BYTES
    for call, seed in enumerate((71, 72)):          # two calls in a row, different inputs
        q, k, v = _rank_buffers(B, S, H, D, seq, seed)
        ref_o, ref_l = api.cpattn_ulysses_attention(q, k, v, B, S, H, D, P, seq, heads)
        out = torch.empty_like(q)
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
        api.cpattn_ulysses_attention_noalloc(q, k, v, B, S, H, D, P, seq, heads, out=out, lse=lse)
        torch.cuda.synchronize()
        st, code = api.cpattn_device_status()
        assert st == 0, f"device wait expired: {code:#x}"
        assert_close(f64_of(out), f64_of(lse), f64_of(ref_o), f64_of(ref_l), f"no-alloc call {call}")


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = _native.load()
    # 8 * B*S*H*D bytes of scratch: 1 x 8192 x 16 x 128 needs 128 MiB > 64 MiB.
    B, S, H, D = 1, 8192, 16, 128
    assert api.cpattn_ulysses_workspace_bytes(B, H, S, D) > api.NOALLOC_SCRATCH_BYTES
    fake = 1 << 20   # never dereferenced: the size check comes before any launch
    st = lib.cpattn_ulysses_attention_noalloc(fake, fake, fake, fake, None, B, H, S, D, 4, None, None, None)
    assert st == 8   # CPATTN_ERR_WORKSPACE
