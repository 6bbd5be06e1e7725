"""context_attention_long_b200.parallel: the configuration object's rules
(diffusers "parallel", ContextParallelConfig's arguments; "Context
parallelism", the variants table and its requirements), and its dispatch to
the exchanges on 2 and 4 gloo ranks on CPU with the oracle-backed kernel
stand-in (tests/exchange_standin.py), every rank's rows checked against the
oracle's monolithic attention."""
import multiprocessing as mp
import os
import socket
import sys
import traceback

import pytest

REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, REPO)

from context_attention_long_b200.parallel import ContextParallelConfig  # noqa: E402


def test_variants_follow_the_degrees():
    assert ContextParallelConfig().variant == "none"
    assert ContextParallelConfig(ring_degree=4).variant == "ring"
    assert ContextParallelConfig(ulysses_degree=2).variant == "ulysses"
    c = ContextParallelConfig(ring_degree=2, ulysses_degree=2)
    assert c.variant == "unified" and c.world_size == 4


@pytest.mark.parametrize("kwargs", [
    dict(ring_degree=0),
    dict(ulysses_degree=-1),
    dict(ring_degree=2.0),
    dict(rotate_method="alltoall"),
    dict(ulysses_anything=True),                                  # needs ulysses_degree > 1
    dict(ulysses_degree=2, ring_degree=2, ulysses_anything=True),  # not with unified
    dict(ring_anything=True),                                     # needs ring_degree > 1
    dict(ring_degree=2, ulysses_degree=2, ring_anything=True),     # not with unified
])
def test_invalid_configurations_are_refused(kwargs):
    with pytest.raises(ValueError):
        ContextParallelConfig(**kwargs)


def test_divisibility_rules_of_the_variants_table():
    ContextParallelConfig(ring_degree=4).check(4096, 24)
    with pytest.raises(ValueError):
        ContextParallelConfig(ring_degree=4).check(4097, 24)
    ContextParallelConfig(ring_degree=4, ring_anything=True).check(4097, 24)
    with pytest.raises(ValueError):                 # Ring Anything: inference only
        ContextParallelConfig(ring_degree=4, ring_anything=True).check(4097, 24, training=True)
    with pytest.raises(ValueError):
        ContextParallelConfig(ulysses_degree=4).check(4096, 30)
    with pytest.raises(ValueError):
        ContextParallelConfig(ulysses_degree=4).check(4098, 24)
    ContextParallelConfig(ulysses_degree=4, ulysses_anything=True).check(10007, 30)
    ContextParallelConfig(ring_degree=2, ulysses_degree=2).check(4096, 24)
    with pytest.raises(ValueError):
        ContextParallelConfig(ring_degree=2, ulysses_degree=2).check(4098, 24)


class _Mesh:
    """A stand-in with the DeviceMesh attributes the config reads."""

    def __init__(self, names, sizes):
        self.mesh_dim_names = names
        self._sizes = sizes

    def size(self, dim):
        return self._sizes[dim]


def test_mesh_must_name_and_size_both_dimensions():
    ContextParallelConfig(ring_degree=2, ulysses_degree=1, mesh=_Mesh(("ring", "ulysses", "fsdp"), (2, 1, 4)))
    with pytest.raises(ValueError):
        ContextParallelConfig(ring_degree=2, mesh=_Mesh(("ring", "fsdp"), (2, 4)))
    with pytest.raises(ValueError):
        ContextParallelConfig(ring_degree=2, mesh=_Mesh(("ring", "ulysses"), (4, 1)))


# ------------------------------------------------------------ gloo ranks

def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cases(world, rank):
    import numpy as np
    import torch
    import oracle
    from context_attention_long_b200 import inputs
    from context_attention_long_b200.parallel import ContextParallel
    from exchange_standin import OracleKernels

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)

    def run(cfg, B, H, D, lens, causal, seed, head_splits=None, expect_error=False):
        S = sum(lens)
        qb, kb, vb = inputs.make_qkv(B, S, H, D, seed, D == 128)
        off = np.concatenate([[0], np.cumsum(lens)]).astype(int)
        a, b = off[rank], off[rank + 1]
        q, k, v = (bf16(x[:, a:b]) for x in (qb, kb, vb))
        cp = ContextParallel(cfg, kernels=OracleKernels())
        if expect_error:
            with pytest.raises(ValueError):
                cp.attention(q, k, v, causal=causal)
            return
        out = cp.attention(q, k, v, causal=causal, head_splits=head_splits)
        qf, kf, vf = (inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb))
        ref_o, _ = oracle.causal_attention(qf, kf, vf) if causal else oracle.attention(qf, kf, vf)
        err = np.abs(out.double().numpy() - ref_o[:, a:b])
        assert err.size == 0 or (err.max() <= 2e-2 and err.mean() <= 2e-3), f"{cfg}: {err.max():.3e}"

    def train(cfg, B, H, D, lens, causal, seed, head_splits=None):
        """The gradients autograd delivers to this rank's shard against the
        oracle's backward over the full sequence."""
        S = sum(lens)
        qb, kb, vb = inputs.make_qkv(B, S, H, D, seed, D == 128)
        rng = np.random.Generator(np.random.PCG64(seed + 1))
        dob = inputs.f32_to_bf16_bits(rng.standard_normal((B, S, H, D)).astype(np.float32))
        off = np.concatenate([[0], np.cumsum(lens)]).astype(int)
        a, b = off[rank], off[rank + 1]
        q, k, v = (bf16(x[:, a:b]).requires_grad_(True) for x in (qb, kb, vb))
        cp = ContextParallel(cfg, kernels=OracleKernels())
        out = cp.attention(q, k, v, causal=causal, head_splits=head_splits)
        out.backward(bf16(dob[:, a:b]))
        refs = oracle.attention_backward(*(inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb, dob)), causal=causal)
        for name, t, ref in zip(("dq", "dk", "dv"), (q, k, v), refs):
            r = ref[:, a:b]
            g = max(np.max(np.abs(ref)), 1e-30)
            err = np.abs(t.grad.double().numpy() - r)
            assert err.size == 0 or (err.max() <= 2e-2 * g and err.mean() <= 2e-3 * g), f"{name} {cfg}"

    def refuse_training(cfg, B, H, D, lens, error):
        """Ring Anything is inference only (the pages' variants table)."""
        qb, kb, vb = inputs.make_qkv(B, sum(lens), H, D, 19, D == 128)
        a, b = sum(lens[:rank]), sum(lens[:rank + 1])
        q, k, v = (bf16(x[:, a:b]).requires_grad_(True) for x in (qb, kb, vb))
        with pytest.raises(error):
            ContextParallel(cfg, kernels=OracleKernels()).attention(q, k, v)

    C = ContextParallelConfig
    if world == 2:
        return [
            ("ring allgather", lambda: run(C(ring_degree=2), 1, 3, 64, [96, 96], False, 11)),
            ("ring p2p causal", lambda: run(C(ring_degree=2, rotate_method="p2p"), 2, 2, 128, [80, 80], True, 12)),
            ("ring anything", lambda: run(C(ring_degree=2, ring_anything=True), 1, 2, 64, [130, 61], False, 13)),
            ("ring uneven refused", lambda: run(C(ring_degree=2), 1, 2, 64, [130, 61], False, 14, expect_error=True)),
            ("ulysses", lambda: run(C(ulysses_degree=2), 2, 4, 64, [64, 64], True, 15)),
            ("ulysses anything", lambda: run(C(ulysses_degree=2, ulysses_anything=True), 1, 3, 64, [77, 50], False,
                                             16, head_splits=[2, 1])),
            ("ulysses training", lambda: train(C(ulysses_degree=2), 2, 4, 64, [48, 48], True, 17)),
            ("ulysses anything training", lambda: train(C(ulysses_degree=2, ulysses_anything=True), 1, 3, 64, [40, 29],
                                                       False, 18, head_splits=[2, 1])),
            ("ring training", lambda: train(C(ring_degree=2), 2, 3, 64, [40, 40], True, 25)),
            ("ring training, p2p, one head", lambda: train(C(ring_degree=2, rotate_method="p2p"), 1, 1, 128, [33, 33],
                                                          False, 26)),
            ("ring anything training refused", lambda: refuse_training(C(ring_degree=2, ring_anything=True), 1, 2, 64,
                                                                      [40, 23], ValueError)),
        ]
    return [
        ("unified 2x2", lambda: run(C(ring_degree=2, ulysses_degree=2), 1, 4, 64, [40, 40, 40, 40], False, 21)),
        ("unified 2x2 causal p2p", lambda: run(C(ring_degree=2, ulysses_degree=2, rotate_method="p2p"), 2, 2, 64,
                                               [32, 32, 32, 32], True, 22)),
        ("ring 4", lambda: run(C(ring_degree=4, rotate_method="p2p"), 1, 2, 128, [50, 50, 50, 50], True, 23)),
        ("ulysses 4 training, an empty head rank", lambda: train(C(ulysses_degree=4, ulysses_anything=True), 2, 3, 64,
                                                               [20, 0, 30, 25], True, 24, head_splits=[1, 1, 0, 1])),
        ("unified 2x2 training", lambda: train(C(ring_degree=2, ulysses_degree=2), 2, 4, 64, [24, 24, 24, 24], True,
                                               27)),
        ("ring 4 training, 3 heads over 4 ranks", lambda: train(C(ring_degree=4, rotate_method="p2p"), 1, 3, 64,
                                                                [20, 20, 20, 20], False, 28)),
    ]


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


@pytest.mark.parametrize("world", [2, 4])
def test_config_dispatch_on_gloo_ranks_matches_the_oracle(world):
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
        for p in procs:        # a failed rank leaves the others waiting in a collective
            if failed and p.is_alive():
                p.terminate()
        for p in procs:
            p.join(60)
    assert all(p.exitcode == 0 for p in procs)
