"""The local-compute entry points of the multi-GPU exchanges on one GPU,
through the C ABI: a rank's ring steps over separate chunk buffers with the
running LSE merge in the kernel epilogue (cpattn_ring_chunk_attention), the
attention against padded all-gathered chunks (cpattn_gathered_kv_attention),
and attention over the rank-buffer layout an all-to-all delivers
(cpattn_rank_buffer_attention), each against the fp64 oracle; and the CUDA
kernels against the CPU stand-in that the gloo tests of the exchanges use, on
the same inputs, so that both sides of those tests honour one contract."""
import numpy as np
import pytest
import torch

import oracle
from context_attention_long_b200 import api, build, exchange, inputs

from exchange_standin import OracleKernels
from gpu_util import assert_close, f64_of, full_to_rank_buffers, oracle_rows, sample_positions, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _no_timeouts():
    st, code = api.cpattn_device_status()
    assert st == 0 and code == 0, f"device wait expired: code {code:#x}"


def _emulated_ring_rank(q, k, v, lens, r, causal, padded):
    """Rank r's ring steps, one kernel call per chunk in ring order, the
    running float32 state merged in the epilogue, the last step in bf16."""
    B, S, H, D = q.shape
    P = len(lens)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(int)
    Smax = max(lens)
    qr = q[:, off[r]:off[r + 1]].contiguous()
    order = [(r - t) % P for t in range(P)]
    steps = [t for t in range(P) if lens[order[t]] > 0 and (not causal or order[t] <= r)]
    out = torch.empty_like(qr)
    lse = torch.empty((B, H, lens[r]), dtype=torch.float32, device="cuda")
    state = torch.empty((B, lens[r], H, D), dtype=torch.float32, device="cuda")
    for t in steps:
        c = order[t]
        if padded:
            kc = torch.zeros((B, Smax, H, D), dtype=q.dtype, device="cuda")
            vc = torch.zeros_like(kc)
            kc[:, :lens[c]] = k[:, off[c]:off[c + 1]]
            vc[:, :lens[c]] = v[:, off[c]:off[c + 1]]
        else:
            kc, vc = k[:, off[c]:off[c + 1]].contiguous(), v[:, off[c]:off[c + 1]].contiguous()
        last = t == steps[-1]
        api.cpattn_ring_chunk_attention(qr, kc, vc, lens[c], out if last else state, lse,
                                        prev_out=None if t == steps[0] else state, q_pos0=int(off[r]),
                                        kv_pos0=int(off[c]), causal=causal)
    return out, lse


@pytest.mark.parametrize("B,H,D,lens,causal", [
    (2, 3, 128, [100, 0, 200, 60], False),
    (1, 2, 64, [129, 128], False),
    (1, 3, 128, [300, 257, 44], True),       # lone tiles: split units merge three states
    (2, 2, 64, [64, 33, 0, 100], True),
])
def test_ring_chunk_steps_match_oracle(B, H, D, lens, causal):
    S = sum(lens)
    qb, kb, vb = inputs.make_qkv(B, S, H, D, 900 + S, D == 128)
    q, k, v = (to_dev(x) for x in (qb, kb, vb))
    qf, kf, vf = (inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb))
    ref_o, ref_l = oracle.causal_attention(qf, kf, vf) if causal else oracle.attention(qf, kf, vf)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(int)
    for r in range(len(lens)):
        if lens[r] == 0:
            continue
        o, l = _emulated_ring_rank(q, k, v, lens, r, causal, padded=False)
        op, lp = _emulated_ring_rank(q, k, v, lens, r, causal, padded=True)
        torch.cuda.synchronize()
        _no_timeouts()
        assert_close(f64_of(o), f64_of(l), ref_o[:, off[r]:off[r + 1]], ref_l[:, :, off[r]:off[r + 1]],
                     f"rank {r} of {lens}")
        # a chunk padded to the longest one (the all-gather layout) gives the same bytes
        assert torch.equal(o.view(torch.int16), op.view(torch.int16)) and torch.equal(l, lp)


@pytest.mark.parametrize("causal", [False, True])
def test_ring_chunk_steps_video_size_sampled(causal):
    """One rank of the video workload's 8-way ring (B1 H40 S32760 D128) in the
    launch sequence of the multi-GPU bench: one cpattn_ring_chunk_attention
    per 4095-row chunk in ring order, the running float32 state merged in the
    epilogue, the last step in bf16.  Sampled query rows (the shard's edges and
    random rows) against the oracle over all 32760 keys."""
    cfg, qb, kb, vb = inputs.config_inputs("video")
    B, S, H, D = qb.shape
    P, r = 8, 5
    lens = [S // P] * P
    off = np.concatenate([[0], np.cumsum(lens)]).astype(int)
    q, k, v = (to_dev(x) for x in (qb, kb, vb))
    o, l = _emulated_ring_rank(q, k, v, lens, r, causal, padded=False)
    torch.cuda.synchronize()
    _no_timeouts()
    local = sample_positions(lens[r], [0, lens[r]], 12, 21 + int(causal))
    pos = local + off[r]
    if causal:
        ref_o = np.zeros((B, len(pos), H, D))
        ref_l = np.zeros((B, H, len(pos)))
        for h in range(H):
            ro, rl = oracle.causal_attention_rows(inputs.bf16_bits_to_f64(qb[0, pos, h]),
                                                  inputs.bf16_bits_to_f64(kb[0, :, h]),
                                                  inputs.bf16_bits_to_f64(vb[0, :, h]), pos, np.arange(S))
            ref_o[0, :, h], ref_l[0, h] = ro, rl
    else:
        ref_o, ref_l = oracle_rows(oracle, qb, kb, vb, pos)
    lc = l.cpu().numpy()[:, :, local]
    assert_close(f64_of(o)[:, local], lc, ref_o, ref_l, f"video ring rank {r} causal {causal}")


@pytest.mark.parametrize("B,H,D,lens,causal", [
    (2, 3, 128, [100, 20, 0, 161], False),
    (1, 2, 64, [256, 256], False),
    (1, 2, 128, [130, 61, 200], True),
])
def test_gathered_kv_matches_oracle(B, H, D, lens, causal):
    S = sum(lens)
    qb, kb, vb = inputs.make_qkv(B, S, H, D, 950 + S, D == 128)
    qf, kf, vf = (inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb))
    ref_o, ref_l = oracle.causal_attention(qf, kf, vf) if causal else oracle.attention(qf, kf, vf)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(int)
    P, Smax = len(lens), max(lens)
    gk = torch.zeros((P, B, Smax, H, D), dtype=torch.bfloat16, device="cuda")
    gv = torch.zeros_like(gk)
    k, v = to_dev(kb), to_dev(vb)
    for c in range(P):
        gk[c, :, :lens[c]] = k[:, off[c]:off[c + 1]]
        gv[c, :, :lens[c]] = v[:, off[c]:off[c + 1]]
    for r in range(P):
        if lens[r] == 0:
            continue
        q = to_dev(np.ascontiguousarray(qb[:, off[r]:off[r + 1]]))
        o, l = api.cpattn_gathered_kv_attention(q, gk, gv, P, r, lens, causal=causal)
        torch.cuda.synchronize()
        _no_timeouts()
        assert_close(f64_of(o), f64_of(l), ref_o[:, off[r]:off[r + 1]], ref_l[:, :, off[r]:off[r + 1]],
                     f"gathered rank {r} of {lens}")


@pytest.mark.parametrize("B,H,D,seq,causal", [
    (2, 3, 128, [100, 0, 150, 83], False),
    (1, 4, 64, [128, 128], True),
    (2, 2, 64, [77, 200, 33], True),
])
def test_rank_buffer_attention_matches_oracle(B, H, D, seq, causal):
    S = sum(seq)
    qb, kb, vb = inputs.make_qkv(B, S, H, D, 990 + S, D == 128)
    qf, kf, vf = (inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb))
    ref_o, ref_l = oracle.causal_attention(qf, kf, vf) if causal else oracle.attention(qf, kf, vf)
    q, k, v = (to_dev(full_to_rank_buffers(x, seq)) for x in (qb, kb, vb))
    o, l = api.cpattn_rank_buffer_attention(q, k, v, B, S, H, D, len(seq), seq, causal=causal)
    torch.cuda.synchronize()
    _no_timeouts()
    assert_close(f64_of(o), f64_of(l), full_to_rank_buffers(ref_o, seq), ref_l, f"rank buffers {seq}")


def test_cuda_kernels_and_cpu_standin_honour_one_contract():
    """Each method of exchange.CudaKernels against tests/exchange_standin's
    OracleKernels on the same bf16 inputs: attention within the tolerance,
    permutes bit-exact."""
    cu, st = exchange.CudaKernels(), OracleKernels()
    B, H, D = 2, 3, 64
    lens = [70, 90, 41]
    S = sum(lens)
    qb, kb, vb = inputs.make_qkv(B, S, H, D, 1234 + S, False)
    host = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) for x in (qb, kb, vb)]
    dev = [t.cuda() for t in host]
    off = np.concatenate([[0], np.cumsum(lens)]).astype(int)
    # ring steps of rank 1: first (own chunk), middle, last (bf16), causal and not
    for causal in (False, True):
        res = {}
        for name, K, (q, k, v), loc in (("cuda", cu, dev, "cuda"), ("standin", st, host, "cpu")):
            qr = q[:, off[1]:off[2]].contiguous()
            out = torch.empty_like(qr)
            lse = torch.empty((B, H, lens[1]), dtype=torch.float32, device=loc)
            state = torch.empty((B, lens[1], H, D), dtype=torch.float32, device=loc)
            for i, c in enumerate((1, 0, 2)):
                kc, vc = k[:, off[c]:off[c + 1]].contiguous(), v[:, off[c]:off[c + 1]].contiguous()
                K.ring_chunk(qr, kc, vc, lens[c], out if i == 2 else state, lse, None if i == 0 else state,
                             int(off[1]), int(off[c]), causal, lens[c])
            res[name] = (out, lse)
        torch.cuda.synchronize()
        assert_close(f64_of(res["cuda"][0]), f64_of(res["cuda"][1]), f64_of(res["standin"][0]),
                     f64_of(res["standin"][1]), f"ring_chunk causal {causal}")
    # gathered, rank 2
    gk = [torch.zeros((3, B, 90, H, D), dtype=torch.bfloat16, device=d) for d in ("cuda", "cpu")]
    gv = [torch.zeros((3, B, 90, H, D), dtype=torch.bfloat16, device=d) for d in ("cuda", "cpu")]
    for i, (k, v) in enumerate(((dev[1], dev[2]), (host[1], host[2]))):
        for c in range(3):
            gk[i][c, :, :lens[c]] = k[:, off[c]:off[c + 1]]
            gv[i][c, :, :lens[c]] = v[:, off[c]:off[c + 1]]
    a = cu.gathered(dev[0][:, off[2]:].contiguous(), gk[0], gv[0], 3, 2, lens, False)
    b = st.gathered(host[0][:, off[2]:].contiguous(), gk[1], gv[1], 3, 2, lens, False)
    torch.cuda.synchronize()
    assert_close(f64_of(a[0]), f64_of(a[1]), f64_of(b[0]), f64_of(b[1]), "gathered")
    # rank buffers and the permutes (flat rank-buffer layout of the same tensors)
    flat_d = [to_dev(full_to_rank_buffers(x, lens)) for x in (qb, kb, vb)]
    flat_h = [t.cpu() for t in flat_d]
    a = cu.rank_buffer(*flat_d, B, S, H, D, 3, lens, True)
    b = st.rank_buffer(*flat_h, B, S, H, D, 3, lens, True)
    torch.cuda.synchronize()
    assert_close(f64_of(a[0]), f64_of(a[1]), f64_of(b[0]), f64_of(b[1]), "rank_buffer")
    heads = [2, 0, 1]
    pa = cu.permute_qkv(*flat_d, B, S, H, D, 3, lens, heads)
    pb = st.permute_qkv(*flat_h, B, S, H, D, 3, lens, heads)
    for x, y in zip(pa, pb):
        assert torch.equal(x.cpu().view(torch.int16), y.view(torch.int16))
    ua = cu.unpermute(pa[0], B, S, H, D, 3, lens, heads)
    ub = st.unpermute(pb[0], B, S, H, D, 3, lens, heads)
    assert torch.equal(ua.cpu().view(torch.int16), ub.view(torch.int16))
    assert torch.equal(ua.cpu().view(torch.int16), flat_h[0].view(torch.int16))
    _no_timeouts()


def test_exchange_module_runs_its_cuda_path_on_one_rank():
    """The exchange functions on a one-rank NCCL group: every call goes through
    CudaKernels (the collectives are trivial) and equals the single-GPU
    entry points' results."""
    import datetime
    import os
    import socket
    import torch.distributed as dist
    if dist.is_initialized():
        pytest.skip("a process group already exists")
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        B, S, H, D = 1, 300, 4, 128
        qb, kb, vb = inputs.make_qkv(B, S, H, D, 77, True)
        q, k, v = (to_dev(x) for x in (qb, kb, vb))
        ref_o, ref_l = api.cpattn_ring_attention(q, k, v, 1)
        for causal in (False, True):
            ro, rl = (api.cpattn_causal_ring_attention if causal else api.cpattn_ring_attention)(q, k, v, 1)
            for method in ("p2p", "allgather"):
                o, l = exchange.ring_attention(q, k, v, causal=causal, rotate_method=method)
                assert_close(f64_of(o), f64_of(l), f64_of(ro), f64_of(rl), f"ring {method}")
            o, l = exchange.ulysses_attention(q, k, v, causal=causal)
            assert_close(f64_of(o), f64_of(l), f64_of(ro), f64_of(rl), "ulysses")
        o, l = exchange.kv_gather_attention(q, k, v)
        assert_close(f64_of(o), f64_of(l), f64_of(ref_o), f64_of(ref_l), "kv_gather")
        rg, ug = exchange.unified_groups(1, 1)
        o, l = exchange.unified_attention(q, k, v, rg, ug)
        assert_close(f64_of(o), f64_of(l), f64_of(ref_o), f64_of(ref_l), "unified")
        # the differentiable Ulysses exchange: its gradients against the
        # single-GPU backward of the same tensors
        rng = np.random.Generator(np.random.PCG64(78))
        dout = to_dev(inputs.f32_to_bf16_bits(rng.standard_normal((B, S, H, D)).astype(np.float32)))
        for causal, trainable in ((False, exchange.ulysses_attention_trainable),
                                  (True, exchange.ulysses_attention_trainable),
                                  (True, exchange.ring_attention_trainable)):
            qq, kk, vv = (x.clone().requires_grad_(True) for x in (q, k, v))
            o = trainable(qq, kk, vv, causal=causal)
            o.backward(dout)
            ro, rl = (api.cpattn_causal_ring_attention if causal else api.cpattn_ring_attention)(q, k, v, 1)
            refs = api.cpattn_attention_backward(q, k, v, ro, rl, dout, causal)
            for name, got, ref in zip(("dq", "dk", "dv"), (qq.grad, kk.grad, vv.grad), refs):
                gref = f64_of(ref)
                err = np.abs(f64_of(got) - gref)
                assert err.max() <= 2e-2 * np.abs(gref).max(), f"trainable {name} causal={causal}"
        # the configuration object's dispatch (ContextParallelConfig semantics)
        from context_attention_long_b200.parallel import ContextParallel, ContextParallelConfig
        for method in ("allgather", "p2p"):
            o, l = ContextParallel(ContextParallelConfig(rotate_method=method)).attention(q, k, v, return_lse=True)
            assert_close(f64_of(o), f64_of(l), f64_of(ref_o), f64_of(ref_l), f"config {method}")
        torch.cuda.synchronize()
        _no_timeouts()
    finally:
        dist.destroy_process_group()
