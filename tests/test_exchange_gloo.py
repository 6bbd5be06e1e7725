"""The multi-GPU exchanges (context_attention_long_b200.exchange) on CPU ranks:
2, 3 and 4 gloo processes run ring (point-to-point and all-gather rotation),
Ulysses, kv_gather and unified attention on their shards of one seeded
sequence, with the oracle-backed kernel stand-in (tests/exchange_standin.py)
for the local compute, and every rank checks its rows against the oracle's
monolithic attention.  This covers who sends what to whom, the layouts, the
splits (even, uneven, empty), the ring order, the per-step merge and causal
masking; the CUDA kernels behind each local step are checked on the GPU
against the same contract (tests/test_gpu_exchange_kernels.py).  SGLang
"Sequence Parallelism", "Cross-Node Sequence Parallelism": the pipelined
rotation returns results byte-identical to the blocking one."""
import multiprocessing as mp
import os
import socket
import sys
import traceback

import pytest

REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bf16(bits):
    import numpy as np
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _check(out, lse, ref_o, ref_l, what):
    import numpy as np
    o = out.double().numpy()
    err = np.abs(o - ref_o)
    assert err.size == 0 or (err.max() <= 2e-2 and err.mean() <= 2e-3), f"{what}: out error {err.max():.3e}"
    l = lse.double().numpy()
    fin = np.isfinite(ref_l)
    assert np.array_equal(fin, np.isfinite(l)), f"{what}: LSE finiteness"
    if fin.any():
        assert np.abs(l[fin] - ref_l[fin]).max() <= 1e-3, f"{what}: LSE error"


def _cases(world, rank):
    """(name, fn) pairs run on every rank in the same order."""
    import numpy as np
    import torch
    import oracle
    from context_attention_long_b200 import exchange, inputs
    from exchange_standin import OracleKernels

    K = OracleKernels()
    out = []

    def ring_case(B, H, D, lens, causal):
        S = sum(lens)
        qb, kb, vb = inputs.make_qkv(B, S, H, D, 500 + S + world, D == 128)
        qf, kf, vf = (inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb))
        ref_o, ref_l = oracle.causal_attention(qf, kf, vf) if causal else oracle.attention(qf, kf, vf)
        off = np.concatenate([[0], np.cumsum(lens)]).astype(int)
        a, b = off[rank], off[rank + 1]
        q, k, v = (_bf16(x[:, a:b]) for x in (qb, kb, vb))
        res = {}
        for method in ("p2p", "allgather"):
            o, l = exchange.ring_attention(q, k, v, None, lens, causal, method, kernels=K)
            _check(o, l, ref_o[:, a:b], ref_l[:, :, a:b], f"ring {method} lens {lens} causal {causal}")
            res[method] = (o, l)
        assert torch.equal(res["p2p"][0].view(torch.int16), res["allgather"][0].view(torch.int16))
        assert torch.equal(res["p2p"][1], res["allgather"][1])

    def ulysses_case(B, H, D, seq, heads, causal):
        S = sum(seq)
        qb, kb, vb = inputs.make_qkv(B, S, H, D, 600 + S + world, D == 128)
        qf, kf, vf = (inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb))
        ref_o, ref_l = oracle.causal_attention(qf, kf, vf) if causal else oracle.attention(qf, kf, vf)
        off = np.concatenate([[0], np.cumsum(seq)]).astype(int)
        hoff = np.concatenate([[0], np.cumsum(heads if heads is not None else [H // world] * world)]).astype(int)
        a, b = off[rank], off[rank + 1]
        q, k, v = (_bf16(x[:, a:b]) for x in (qb, kb, vb))
        o, l = exchange.ulysses_attention(q, k, v, None, seq, heads, causal, kernels=K)
        _check(o, l, ref_o[:, a:b], ref_l[:, hoff[rank]:hoff[rank + 1]], f"ulysses {seq} {heads} causal {causal}")

    def kv_gather_case(B, H, D, lens):
        S = sum(lens)
        qb, kb, vb = inputs.make_qkv(B, S, H, D, 700 + S + world, D == 128)
        qf, kf, vf = (inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb))
        ref_o, ref_l = oracle.attention(qf, kf, vf)
        off = np.concatenate([[0], np.cumsum(lens)]).astype(int)
        a, b = off[rank], off[rank + 1]
        q, k, v = (_bf16(x[:, a:b]) for x in (qb, kb, vb))
        o, l = exchange.kv_gather_attention(q, k, v, None, lens, kernels=K)
        _check(o, l, ref_o[:, a:b], ref_l[:, :, a:b], f"kv_gather {lens}")

    if world == 3:
        out += [("ring anything", lambda: ring_case(1, 2, 64, [100, 37, 64], False)),
                ("ring causal", lambda: ring_case(2, 2, 128, [50, 50, 50], True)),
                ("ulysses anything", lambda: ulysses_case(1, 4, 64, [31, 64, 40], [2, 1, 1], False)),
                ("kv_gather", lambda: kv_gather_case(1, 3, 64, [10, 70, 0]))]
    elif world == 2:
        out += [("ring even", lambda: ring_case(2, 3, 64, [96, 96], False)),
                ("ring uneven causal", lambda: ring_case(1, 2, 128, [130, 61], True)),
                ("ulysses even", lambda: ulysses_case(2, 4, 64, [80, 80], [2, 2], False)),
                ("ulysses anything causal", lambda: ulysses_case(1, 3, 64, [77, 50], [2, 1], True)),
                ("kv_gather", lambda: kv_gather_case(2, 2, 64, [100, 60]))]
    else:
        out += [("ring anything", lambda: ring_case(2, 2, 64, [70, 0, 90, 41], False)),
                ("ring anything causal", lambda: ring_case(1, 3, 64, [64, 33, 0, 100], True)),
                ("ulysses anything", lambda: ulysses_case(2, 5, 64, [40, 0, 33, 50], [2, 1, 2, 0], False)),
                ("ulysses causal", lambda: ulysses_case(1, 4, 128, [32, 32, 32, 32], None, True)),
                ("kv_gather uneven", lambda: kv_gather_case(1, 3, 64, [50, 20, 0, 61]))]

        def unified_case(B, H, D, ring_lens, subs, heads, causal):
            import torch.distributed as dist
            rg, ug = exchange.unified_groups(2, 2)
            S = sum(ring_lens)
            qb, kb, vb = inputs.make_qkv(B, S, H, D, 800 + S, D == 128)
            qf, kf, vf = (inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb))
            ref_o, ref_l = oracle.causal_attention(qf, kf, vf) if causal else oracle.attention(qf, kf, vf)
            i, j = dist.get_rank() // 2, dist.get_rank() % 2
            coff = int(sum(ring_lens[:i]))
            a = coff + int(sum(subs[i][:j]))
            b = a + subs[i][j]
            hj = heads if heads is not None else [H // 2, H // 2]
            h0 = int(sum(hj[:j]))
            q, k, v = (_bf16(x[:, a:b]) for x in (qb, kb, vb))
            o, l = exchange.unified_attention(q, k, v, rg, ug, ring_lens, subs, heads, causal, kernels=K)
            _check(o, l, ref_o[:, a:b], ref_l[:, h0:h0 + hj[j], coff:coff + ring_lens[i]],
                   f"unified {ring_lens} {subs} causal {causal}")

        out += [("unified", lambda: unified_case(2, 4, 64, [90, 70], [[45, 45], [40, 30]], None, False)),
                ("unified uneven causal", lambda: unified_case(1, 3, 64, [64, 101], [[33, 31], [51, 50]], [2, 1],
                                                              True))]
    return out


def _worker(rank, world, port, q):
    import datetime
    sys.path.insert(0, REPO)
    sys.path.insert(0, TESTS)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    done = []
    try:
        for name, fn in _cases(world, rank):
            fn()
            done.append(name)
        q.put((rank, "ok", done))
    except Exception:  # noqa: BLE001
        q.put((rank, traceback.format_exc(), done))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
def test_exchanges_on_gloo_ranks_match_the_oracle(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = []
    try:
        for _ in range(world):
            rank, status, done = q.get(timeout=600)
            results.append((rank, status, done))
            assert status == "ok", f"rank {rank} after {done}:\n{status}"
    finally:
        failed = len(results) < world or any(r[1] != "ok" for r in results)
        for p in procs:       # a failed rank leaves the others waiting in a collective
            if failed and p.is_alive():
                p.terminate()
        for p in procs:
            p.join(60)
    assert all(p.exitcode == 0 for p in procs)
