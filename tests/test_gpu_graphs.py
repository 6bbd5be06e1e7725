"""The library's calls can be captured in a CUDA graph: nothing on their launch
path synchronises or allocates, and every kernel takes its launch plan by
value.  A captured ring + Ulysses step and a captured backward, replayed on
new inputs copied into the same buffers, give the bytes eager calls give."""
import numpy as np
import pytest
import torch

from context_attention_long_b200 import api, build, inputs

from gpu_util import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def test_captured_forward_and_backward_replay_equal_eager():
    B, S, H, D, P, U = 1, 640, 4, 128, 4, 2
    q, k, v = (to_dev(x) for x in inputs.make_qkv(B, S, H, D, 61, True))
    do = to_dev(inputs.f32_to_bf16_bits(
        np.random.Generator(np.random.PCG64(62)).standard_normal((B, S, H, D)).astype(np.float32)))
    out_r, out_u = torch.empty_like(q), torch.empty_like(q).reshape(-1)
    lse_r = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    lse_u = torch.empty_like(lse_r)
    ws = torch.empty(api.cpattn_ulysses_workspace_bytes(B, H, S, D), dtype=torch.uint8, device="cuda")
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    wsb = torch.empty(api.cpattn_attention_backward_workspace_bytes(B, H, S), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()

    def step():
        api.cpattn_ring_attention(q, k, v, P, out=out_r, lse=lse_r, stream=stream)
        api.cpattn_ulysses_attention(q.reshape(-1), k.reshape(-1), v.reshape(-1), B, S, H, D, U, out=out_u,
                                     lse=lse_u, workspace=ws, stream=stream)
        api.cpattn_attention_backward(q, k, v, out_r, lse_r, do, False, dq, dk, dv, wsb, stream=stream)

    with torch.cuda.stream(stream):
        step()                                   # warm-up outside capture (one-time attribute setup)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    # new inputs into the captured buffers, then replay
    q2, k2, v2 = (to_dev(x) for x in inputs.make_qkv(B, S, H, D, 63, True))
    q.copy_(q2); k.copy_(k2); v.copy_(v2)
    graph.replay()
    torch.cuda.synchronize()
    got = [t.clone() for t in (out_r, lse_r, out_u, dq, dk, dv)]
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    want = (out_r, lse_r, out_u, dq, dk, dv)
    for g, w in zip(got, want):
        assert torch.equal(g.view(torch.uint8) if g.dtype != torch.float32 else g,
                           w.view(torch.uint8) if w.dtype != torch.float32 else w)
    st, code = api.cpattn_device_status()
    assert st == 0, f"device status {code:#x}"
    del graph


def test_captured_projection_flow_replay_equals_eager():
    """The fused projections launch in clusters of two CTAs (cudaLaunchKernelEx);
    captured together with the head-sharded attention between them, a replay
    on new activations gives the bytes eager calls give."""
    B, S, H, D, U = 1, 512, 4, 128, 2
    Dm = H * D
    xb, wb, wob = inputs.make_projection_inputs(B, S, H, D, Dm, 71)
    x, w, wo = to_dev(xb), to_dev(wb), to_dev(wob)
    n = B * S * H * D
    yq, yk, yv, yo = (torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    out = torch.empty(B * S * Dm, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    stream = torch.cuda.Stream()

    def step():
        api.cpattn_ulysses_qkv_projection(x, w, B, S, H, D, Dm, U, yq=yq, yk=yk, yv=yv, stream=stream)
        api.cpattn_head_sharded_attention(yq, yk, yv, B, S, H, D, U, yo=yo, lse=lse, stream=stream)
        api.cpattn_ulysses_output_projection(yo, wo, B, S, H, D, Dm, U, out=out, stream=stream)

    with torch.cuda.stream(stream):
        step()                                   # warm-up outside capture (one-time attribute setup)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    x.copy_(to_dev(inputs.make_projection_inputs(B, S, H, D, Dm, 72)[0]))
    graph.replay()
    torch.cuda.synchronize()
    got = [t.clone() for t in (yq, yo, out)]
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    for g, want in zip(got, (yq, yo, out)):
        assert torch.equal(g.view(torch.int16), want.view(torch.int16))
    st, code = api.cpattn_device_status()
    assert st == 0, f"device status {code:#x}"
