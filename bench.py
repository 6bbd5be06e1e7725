#!/usr/bin/env python
"""Benchmark of the context-parallel attention hot path on B200.

One step = one pass of the whole hot path over the video-DiT workload
(B=1, H=40, S=32760, D=128, seeded synthetic bf16, RMS-normalised Q/K), the
largest single-GPU workload:
  * ring attention, ring_degree 8 (fused: one kernel walks the K/V chunks in
    ring order and merges them with the LSE rule on chip),
  * unified ring 8 x Ulysses 2 attention: permute Q, K, V to the head groups
    (one launch), ring attention per head group whose epilogue stores the
    output back in the token layout (the inverse permute, fused; one launch).
Metric: attention TFLOP/s = (4*B*H*S^2*D per attention pass) * passes / time.
The HBM-bound kernels (the Q/K/V permute, the standalone unpermute and the
8-way LSE merge) are timed beside the step on the same sizes and reported
inside `roofline` with the attention kernel.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--extras]

N > 1 (torchrun, one process per GPU, NCCL): the sequence is sharded over the
GPUs and the exchanges are real collectives (context_attention_long_b200.exchange):
ring over all N GPUs and unified (N/2 ring) x (Ulysses 2); the same total work
as one GPU's step (strong scaling), timed as the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

REPO = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, REPO)

METRIC = "attention TFLOP/s (4·B·H·S²·D) & % BF16 peak; permute/merge GB/s & % HBM"
WORKLOAD = "video"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
# Link bandwidth fed to the exchange-selection model (--extras) unless
# --link-gbs is given: NVLink 5's nominal 900 GB/s per direction per GPU, an
# assumption taken from the vendor's specification, not a measurement.
NOMINAL_LINK_GBS = 900.0


def ring_peak_choice(peaks, peaks_kind, region_s):
    """Denominator of the step's ring-kernel roofline: the sustained bf16
    figure when the timed region lasts a second or more (the kernel then runs
    under the power cap) and the peaks file holds one, else the burst figure.
    Returns (peak TFLOP/s, label)."""
    burst = float(peaks["bf16_tflops"])
    if region_s >= 1.0 and "bf16_tflops_sustained" in peaks:
        return (float(peaks["bf16_tflops_sustained"]),
                f"bf16_tflops_sustained, {peaks_kind} (timed region {region_s:.1f} s of back-to-back steps)")
    note = "" if "bf16_tflops_sustained" in peaks else " (the peaks file holds no sustained figure)"
    return burst, f"bf16_tflops burst, {peaks_kind}{note}"


def load_peaks():
    path = os.path.join(REPO, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash():
    """Hash of the attention kernel sources; a stored ncu traffic figure is only
    reported while it matches the current kernel."""
    h = hashlib.sha256()
    csrc = os.path.join(REPO, "context_attention_long_b200", "csrc")
    for name in ("attn_kernel.cuh", "cpattn_ptx.cuh", "cpattn_internal.h"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel_key):
    path = os.path.join(REPO, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("bytes_per_launch")


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML (read-only) in a
    background thread; keeps the samples whose timestamps fall in a window."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x10: "sync_boost", 0x1: "gpu_idle"}

    def __init__(self, torch_dev):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            p = torch.cuda.get_device_properties(torch_dev)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                sm = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                reasons = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), sm, reasons))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "error": getattr(self, "err", "")}
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        if not win:   # region shorter than the sampling period: nearest samples
            win = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
        mask = 0
        for s in win:
            mask |= s[2]
        reasons = sorted(name for bit, name in self.REASONS.items() if mask & bit and name != "gpu_idle")
        return {"sm_mhz": float(statistics.median(s[1] for s in win)) if win else None,
                "sm_max_mhz": float(self.max_mhz), "reasons": reasons, "samples": len(win)}


def max_over_ranks(values, world, dist=None, device="cpu"):
    """Every rank's device-timed figures -> their maximum over the ranks (the
    job takes as long as its slowest rank)."""
    import torch
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def multi_gpu_shards(S, world, ulysses_degree=2):
    """The sequence split of the multi-GPU step: every rank's tokens (front-
    loaded split of S over the ranks), and the unified grid's view of the same
    shards: rank (i, j) = i * ulysses_degree + j holds sub-shard j of ring
    chunk i.  Returns (lens, ring_lens, subs)."""
    base, extra = divmod(S, world)
    lens = [base + (1 if r < extra else 0) for r in range(world)]
    R = world // ulysses_degree
    subs = [[lens[ulysses_degree * i + j] for j in range(ulysses_degree)] for i in range(R)]
    return lens, [sum(x) for x in subs], subs


# ----------------------------------------------------------------- reference arm (the oracle)
def flush_l2(flush):
    """Evicts L2: writes a buffer larger than L2, then reads it back, so that
    L2 holds clean lines of the flush buffer (a write alone would leave dirty
    lines that the next kernel must write back to HBM before it can use L2)."""
    import torch
    flush.zero_()
    torch.sum(flush.view(torch.int64))   # reads the 256 MiB in place (no widened copy)


def median_event_ms(fn, flush, stream, reps=10, warmup=1):
    """Median CUDA-event time of fn() on `stream`, each rep after an L2 flush
    (flush_l2) outside the timed events."""
    import torch
    for _ in range(warmup):
        fn()
    times = []
    for _ in range(reps):
        flush_l2(flush)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        times.append(a.elapsed_time(b))
    return float(np.median(times))


def oracle_sample_step(cfg, q, k, v, rows_per_shard, seed):
    """The oracle's step on a bounded sample of query rows: for every ring
    shard, sampled rows attend every K/V chunk in ring order (partials + LSE
    merge) -- the ring pass -- and the same rows attend all S keys of their
    head -- the unified pass, whose head groups run that attention per head in
    exact arithmetic.  Each head's K/V is widened to float64 once per step.
    Returns the attention FLOPs processed (4 * rows * S * D per head and pass)."""
    import oracle
    from context_attention_long_b200 import inputs as inp
    B, S, H, D = q.shape
    P = cfg["ring_degree"]
    lens = [S // P] * P
    off = oracle.offsets(lens)
    rng = np.random.Generator(np.random.PCG64(seed))
    rows = [off[r] + rng.integers(0, lens[r], size=rows_per_shard) for r in range(P)]
    flops = 0
    for b in range(B):
        for h in range(H):
            kh = inp.bf16_bits_to_f64(k[b, :, h, :])
            vh = inp.bf16_bits_to_f64(v[b, :, h, :])
            for r in range(P):
                qh = inp.bf16_bits_to_f64(q[b, rows[r], h, :])
                outs, lses = [], []
                for c in oracle.ring_order(r, P):
                    o, l = oracle.attention_rows(qh, kh[off[c]:off[c + 1]], vh[off[c]:off[c + 1]])
                    outs.append(o[None, :, None, :])
                    lses.append(l[None, None, :])
                oracle.lse_merge(outs, lses)
                oracle.attention_rows(qh, kh, vh)   # unified: attention of the head over all S keys
                flops += 2 * 4 * len(rows[r]) * S * D
    return flops


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from context_attention_long_b200 import inputs
    import torch
    cfg, q, k, v = inputs.config_inputs(WORKLOAD)
    threads = torch.get_num_threads()
    rows = 1
    for _ in range(args.warmup):
        oracle_sample_step(cfg, q, k, v, rows, 0)
    t0 = time.perf_counter()
    flops = 0
    for i in range(args.steps):
        flops += oracle_sample_step(cfg, q, k, v, rows, i + 1)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    B, S, H, D = q.shape
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1), RMS-normalised Q/K, bf16-rounded)",
        "config": config_block(cfg, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"per step {rows} query row per ring shard x {H} heads, ring + unified passes "
                                   f"vs all S={S} keys (fp64 numpy oracle)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def config_block(cfg, world=1):
    """The `config` of the bench line for `world` GPUs (both arms print it)."""
    B, H, S, D = cfg["B"], cfg["H"], cfg["S"], cfg["D"]
    if world == 1:
        return {"workload": f"video-DiT B{B} H{H} S{S} D{D}: ring {cfg['ring_degree']} (fused) + unified ring "
                            f"{cfg['ring_degree']} x Ulysses {cfg['ulysses_degree']}",
                "B": B, "H": H, "S": S, "D": D, "ring_degree": cfg["ring_degree"],
                "ulysses_degree": cfg["ulysses_degree"], "parallelism": "1 GPU, shards emulated in memory",
                "l2": "inputs larger than L2 (335 MB each) and an L2 flush (256 MiB written, then read) before every timed step"}
    return {"workload": f"video-DiT B{B} H{H} S{S} D{D}: ring {world} (NCCL P2P rotation) + unified ring "
                        f"{world // 2} x Ulysses 2 (NCCL all-to-all), sequence sharded over {world} GPUs",
            "B": B, "H": H, "S": S, "D": D, "ring_degree": world, "ulysses_degree": 2,
            "parallelism": f"context parallel over {world} GPUs",
            "l2": "an L2 flush (256 MiB written, then read) on every rank before every timed step"}


def cpu_baseline(cfg, q, k, v, budget_s=12.0):
    """The oracle, as it stands, on a bounded sample of the same workload."""
    import torch
    t0 = time.perf_counter()
    flops, i, rows = 0, 0, 2
    while time.perf_counter() - t0 < budget_s:
        flops += oracle_sample_step(cfg, q, k, v, rows, 1000 + i)
        i += 1
    dt = time.perf_counter() - t0
    B, S, H, D = q.shape
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": torch.get_num_threads(), "kind": "oracle",
            "sample": f"{i} x ({rows} rows per ring shard x {H} heads, ring + unified passes vs S={S} keys), "
                      f"{dt:.1f} s"}


def hbm_entry(name, nbytes, ms, peak_gbs, peaks_kind):
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"kernel": name, "bound": "hbm", "achieved": round(gbs, 1), "unit": "GB/s", "peak": peak_gbs,
            "frac": round(gbs / peak_gbs, 4), "bytes": int(nbytes), "ms": round(ms, 4), "peak_kind": peaks_kind}


def tensor_entry(name, flops, ms, peak_tf):
    tf = flops / (ms * 1e-3) / 1e12
    return {"kernel": name, "bound": "tensor", "achieved": round(tf, 1), "unit": "TFLOP/s",
            "frac": round(tf / peak_tf, 4), "flops": flops, "ms": round(ms, 4)}


# ----------------------------------------------------------------- our arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--extras", action="store_true",
                    help="also time the causal, backward and projection paths on the image-DiT workload and the "
                         "exchange-selection model; printed as a second JSON line")
    ap.add_argument("--link-gbs", type=float, default=NOMINAL_LINK_GBS,
                    help="interconnect bandwidth per direction fed to the exchange-selection model (--extras); "
                         "default: NVLink 5 nominal, an assumption")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="time every workload's paths (one JSON line per path) instead of the step")
    ap.add_argument("--kernel", default=None, choices=["ring", "causal_ring", "head_sharded", "permute", "permute_qkv",
                                                       "unpermute", "merge", "ring_step", "backward",
                                                       "qkv_projection", "output_projection", "unified"],
                    help="profiling mode: run only this kernel (warmup + steps launches) on --workload")
    ap.add_argument("--workload", default="dit", help="workload of --kernel mode")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
        return
    if args.kernel is not None:
        run_single_kernel(args)
        return
    if args.sweep:
        run_sweep(args)
        return

    import torch
    import torch.distributed as dist
    from context_attention_long_b200 import api, build, inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)     # before NCCL sees the process group
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
        run_multi_gpu(args, world, rank, dev)
        return

    cfg, qb, kb, vb = inputs.config_inputs(WORKLOAD)
    B, S, H, D = qb.shape
    P, U = cfg["ring_degree"], cfg["ulysses_degree"]

    def host_bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory()

    hq, hk, hv = host_bf16(qb), host_bf16(kb), host_bf16(vb)
    q, k, v = (t.to(dev) for t in (hq, hk, hv))
    out_r = torch.empty_like(q)
    lse_r = torch.empty((B, H, S), dtype=torch.float32, device=dev)
    out_u = torch.empty_like(q)
    lse_u = torch.empty((B, H, S), dtype=torch.float32, device=dev)
    ws = torch.empty(api.cpattn_unified_workspace_bytes(B, H, S, D), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    attn_flops = 4.0 * B * H * S * S * D      # one attention pass
    step_flops = 2 * attn_flops               # ring + unified
    launches_per_step = 3                     # ring; unified: Q/K/V permute, attention (unpermute fused)
    n_ev = 3
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]

    def step_on(qx, kx, vx, orx, oux, e=None):
        if e: e[0].record(stream)
        api.cpattn_ring_attention(qx, kx, vx, P, out=orx, lse=lse_r, stream=stream)
        if e: e[1].record(stream)
        api.cpattn_unified_attention(qx, kx, vx, P, U, out=oux, lse=lse_u, workspace=ws, stream=stream)
        if e: e[2].record(stream)

    for _ in range(args.warmup):
        flush_l2(flush)
        step_on(q, k, v, out_r, out_u)
    torch.cuda.synchronize()
    st, code = api.cpattn_device_status()
    if st != 0:
        raise RuntimeError(f"device wait expired during warm-up: {code:#x}")

    clocks = ClockSampler(dev)
    clocks.start()
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    for i in range(args.steps):
        flush_l2(flush)               # evict L2 (outside the timed events)
        step_on(q, k, v, out_r, out_u, ev[i])
    torch.cuda.synchronize()
    t_wall1 = time.perf_counter()
    clocks.stop()

    per = np.array([[ev[i][j].elapsed_time(ev[i][j + 1]) for j in range(n_ev - 1)] for i in range(args.steps)])
    step_ms = per.sum(axis=1)
    ms_per_step = float(step_ms.sum()) / args.steps
    value = step_flops / (ms_per_step * 1e-3) / 1e12

    peaks, peaks_kind = load_peaks()
    peak_tf = float(peaks["bf16_tflops"])
    hbm = float(peaks["hbm_gbs"])
    ring_ms = float(per[:, 0].mean())
    ring_tflops = attn_flops / (ring_ms * 1e-3) / 1e12
    uni_ms = float(per[:, 1].mean())
    tensor_bytes = B * S * H * D * 2

    # HBM-bound kernels of the step's unified flow at the same sizes, each rep
    # after an L2 flush: the first all-to-all (Q, K and V in one launch; for
    # B = 1 the unified flow's head-group layout is the Ulysses head-side
    # layout), the second all-to-all, and the 8-way merge of float32 partials.
    yq, yk, yv = (torch.empty_like(q) for _ in range(3))
    ms_pq = median_event_ms(lambda: api.cpattn_ulysses_permute_qkv(q, k, v, B, S, H, D, U, yq=yq, yk=yk, yv=yv,
                                                                   stream=stream), flush, stream, reps=7)
    ms_up = median_event_ms(lambda: api.cpattn_ulysses_unpermute(yq, B, S, H, D, U, x=yk, stream=stream),
                            flush, stream, reps=7)
    del yq, yk, yv
    po = torch.randn((P, B, S, H, D), device=dev, dtype=torch.float32)
    pl = torch.randn((P, B, H, S), device=dev, dtype=torch.float32)
    ob = torch.empty((B, S, H, D), device=dev, dtype=torch.bfloat16)
    lo = torch.empty((B, H, S), device=dev, dtype=torch.float32)
    ms_mg = median_event_ms(lambda: api.cpattn_lse_merge(po, pl, out_bf16=ob, lse_out=lo, want_f32=False,
                                                         stream=stream), flush, stream, reps=7)
    del po, pl, ob, lo
    torch.cuda.empty_cache()
    merge_bytes = B * H * S * (P * (4 * D + 4) + 2 * D + 4)
    hbm_kernels = [
        hbm_entry(f"permute_kernel: Q/K/V to {U} head groups, one launch", 6 * tensor_bytes, ms_pq, hbm, peaks_kind),
        hbm_entry(f"permute_kernel: output back from {U} head groups (standalone; fused in the flows)",
                  2 * tensor_bytes, ms_up, hbm, peaks_kind),
        hbm_entry(f"lse_merge_kernel<128,8>: P={P} fp32 partials -> bf16", merge_bytes, ms_mg, hbm, peaks_kind),
    ]
    causal_ms = median_event_ms(lambda: api.cpattn_causal_ring_attention(q, k, v, P, out=out_u, lse=lse_u,
                                                                         stream=stream), flush, stream, reps=5)
    # The ring kernel runs inside a step that repeats for the whole timed
    # region; when that region lasts a second or more the kernel runs under
    # the power cap, and the denominator is the sustained bf16 figure (a
    # seconds-long cuBLAS loop), else the burst figure.
    region_s = t_wall1 - t_wall0
    ring_peak, ring_peak_kind = ring_peak_choice(peaks, peaks_kind, region_s)
    tensor_kernels = [
        tensor_entry(f"unified ring {P} x Ulysses {U} (in the step; 2 launches)", attn_flops, uni_ms, ring_peak),
        tensor_entry(f"causal ring fused P={P} (visible pairs)", causal_flops(B, H, S, D), causal_ms, peak_tf),
    ]
    roofline = {"bound": "tensor", "kernel": f"attn_fwd_kernel<128,bf16> (ring fused, P={P}, in the step)",
                "achieved": ring_tflops, "peak": ring_peak, "unit": "TFLOP/s", "frac": ring_tflops / ring_peak,
                "peak_kind": ring_peak_kind,
                "frac_of_burst": ring_tflops / peak_tf,
                "traffic": stored_traffic("attn_fwd_ring_video"),
                "algorithmic_flops_per_launch": attn_flops,
                "tensor_kernels": tensor_kernels, "hbm_kernels": hbm_kernels}

    # ---- end to end through the public API with host buffers
    # Every step uploads its Q, K, V from pinned host memory and downloads
    # both attention outputs.  Uploads, compute and downloads run on three
    # streams with two device copies of the inputs and outputs, so step i+1's
    # upload and step i-1's download overlap step i's kernels (PCIe is full
    # duplex); the kernels of consecutive steps stay in order on one stream.
    hout_r = torch.empty_like(out_r, device="cpu").pin_memory()
    hout_u = torch.empty_like(out_u, device="cpu").pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    bufs = [(q, k, v, out_r, out_u),
            (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(out_r),
             torch.empty_like(out_u))]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def pipeline(n, e_start=None, e_end=None):
        if e_start is not None:
            e_start.record(s_in)
        for i in range(n):
            bi = i % 2
            qx, kx, vx, orx, oux = bufs[bi]
            if i >= 2:
                s_in.wait_event(ev_comp[bi])          # step i-2 has finished reading these inputs
            with torch.cuda.stream(s_in):
                qx.copy_(hq, non_blocking=True); kx.copy_(hk, non_blocking=True); vx.copy_(hv, non_blocking=True)
            ev_in[bi].record(s_in)
            stream.wait_event(ev_in[bi])
            if i >= 2:
                stream.wait_event(ev_out[bi])         # step i-2's outputs are on the host
            step_on(qx, kx, vx, orx, oux)
            ev_comp[bi].record(stream)
            s_out.wait_event(ev_comp[bi])
            with torch.cuda.stream(s_out):
                hout_r.copy_(orx, non_blocking=True); hout_u.copy_(oux, non_blocking=True)
            ev_out[bi].record(s_out)
        if e_end is not None:
            s_out.wait_event(ev_comp[(n - 1) % 2])
            e_end.record(s_out)

    pipeline(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pipeline(e2e_steps, e0, e1)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    # every step computes the same deterministic result: the downloaded
    # outputs must equal the device outputs
    if not (torch.equal(hout_r.view(torch.int16), out_r.cpu().view(torch.int16)) and
            torch.equal(hout_u.view(torch.int16), out_u.cpu().view(torch.int16))):
        raise RuntimeError("end-to-end pipeline: downloaded outputs differ from the device results")
    e2e = {"value": step_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
           "h2d_bytes_per_step": 3 * tensor_bytes, "d2h_bytes_per_step": 2 * tensor_bytes,
           "note": "pinned host Q/K/V in, both outputs out, every step; 3 streams, 2 device buffers"}
    del bufs

    # Mean absolute difference of the sharded paths' outputs from unsharded
    # attention (the fused kernel with one shard), in the MAE style of the
    # pages' sharded-vs-unsharded check; the paths differ only in rounding order.
    mono, _ = api.cpattn_ring_attention(q, k, v, 1, want_lse=False, stream=stream)
    torch.cuda.synchronize()
    mae = {"ring": float((out_r.float() - mono.float()).abs().mean()),
           "unified": float((out_u.float() - mono.float()).abs().mean())}
    del mono

    st, code = api.cpattn_device_status()
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1), RMS-normalised Q/K, bf16)",
        "config": config_block(cfg), "roofline": roofline, "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(t_wall0, t_wall1), "e2e": e2e, "device_status": code,
        "mae_vs_unsharded": mae,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, qb, kb, vb)
    extras = None
    if args.extras:
        del q, k, v, out_r, out_u, ws, hq, hk, hv
        torch.cuda.empty_cache()
        extras = dit_extras(api, torch, dev, flush, peaks, inputs, args.link_gbs)
    if extras is not None:
        print(json.dumps({"extras": extras}))
    print(json.dumps(line))


def run_multi_gpu(args, world, rank, dev):
    """N > 1 GPUs (one process each, NCCL): the video workload's sequence is
    sharded over the ranks and the exchanges are real collectives
    (context_attention_long_b200.exchange): ring attention over all N ranks
    with the point-to-point K/V rotation overlapped with each step's kernel,
    and unified attention on an (N/2 ring) x (Ulysses 2) grid.  The total work
    is the single-GPU step's (strong scaling); the step time is the max over
    ranks of each rank's CUDA-event time."""
    import torch
    import torch.distributed as dist
    from context_attention_long_b200 import api, exchange, inputs
    if world % 2:
        raise SystemExit("the unified (ring x Ulysses 2) part of the step needs an even number of GPUs")
    cfg, qb, kb, vb = inputs.config_inputs(WORKLOAD)
    B, S, H, D = qb.shape
    U = 2
    R = world // U
    lens, ring_lens, subs = multi_gpu_shards(S, world, U)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(int)
    a, b = off[rank], off[rank + 1]

    def shard(bits):
        return torch.from_numpy(np.ascontiguousarray(bits[:, a:b]).view(np.int16)).view(torch.bfloat16)

    hq, hk, hv = (shard(x).pin_memory() for x in (qb, kb, vb))
    q, k, v = (t.to(dev) for t in (hq, hk, hv))
    del qb, kb, vb
    ring_group, uly_group = exchange.unified_groups(R, U)
    stream = torch.cuda.current_stream()
    attn_flops = 4.0 * B * H * S * S * D
    step_flops = 2 * attn_flops
    launches_per_step = world + (1 + R + 1)     # ring steps; unified: pack, R ring steps, unpack

    def step(e=None):
        if e: e[0].record(stream)
        o_r, _ = exchange.ring_attention(q, k, v, None, lens, rotate_method="p2p")
        if e: e[1].record(stream)
        o_u, _ = exchange.unified_attention(q, k, v, ring_group, uly_group, ring_lens, subs)
        if e: e[2].record(stream)
        return o_r, o_u

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(dev)
    clocks.start()
    dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(args.steps):
        flush_l2(flush)       # between steps, outside the events
        step(ev[i])
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    dist.barrier()
    clocks.stop()
    per = np.array([[ev[i][j].elapsed_time(ev[i][j + 1]) for j in range(2)] for i in range(args.steps)])
    tot_ms, ring_tot_ms = max_over_ranks([per.sum(), per[:, 0].sum()], world, dist, dev)
    ms_per_step = tot_ms / args.steps
    ring_ms = ring_tot_ms / args.steps
    value = step_flops / (ms_per_step * 1e-3) / 1e12

    # end to end through the public API: this rank's shard uploaded from
    # pinned host memory and both outputs downloaded, every step
    ho_r, ho_u = torch.empty_like(hq).pin_memory(), torch.empty_like(hq).pin_memory()
    e2e_steps = max(3, min(args.steps, 10))
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        q.copy_(hq, non_blocking=True); k.copy_(hk, non_blocking=True); v.copy_(hv, non_blocking=True)
        o_r, o_u = step()
        ho_r.copy_(o_r, non_blocking=True); ho_u.copy_(o_u, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks([e0.elapsed_time(e1) / e2e_steps], world, dist, dev)[0]

    peaks, peaks_kind = load_peaks()
    peak_tf = float(peaks["bf16_tflops"])
    rank_ring_flops = attn_flops / world

    # The link as the exchanges use it: one ring hop of this rank's K and V
    # shard (send to the next rank, receive from the previous), timed on the
    # device, max over ranks; it feeds the exchange-selection model.
    hop_bytes = 2 * B * (b - a) * H * D * 2
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    kr, vr = torch.empty_like(k), torch.empty_like(v)

    def hop():
        ops = [dist.P2POp(dist.isend, k.view(torch.uint8).reshape(-1), nxt),
               dist.P2POp(dist.isend, v.view(torch.uint8).reshape(-1), nxt),
               dist.P2POp(dist.irecv, kr.view(torch.uint8).reshape(-1), prv),
               dist.P2POp(dist.irecv, vr.view(torch.uint8).reshape(-1), prv)]
        for w in dist.batch_isend_irecv(ops):
            w.wait()

    for _ in range(3):
        hop()
    dist.barrier()
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_hops = 10
    h0.record(stream)
    for _ in range(n_hops):
        hop()
    h1.record(stream)
    torch.cuda.synchronize()
    hop_ms = max_over_ranks([h0.elapsed_time(h1) / n_hops], world, dist, dev)[0]
    link_gbs = hop_bytes / (hop_ms * 1e-3) / 1e9
    rank_tflops = rank_ring_flops / (ring_ms * 1e-3) / 1e12
    exch_plan = {"inputs": {"link_gbs": round(link_gbs, 1), "link_kind": "measured: one ring hop of a K/V shard",
                            "attn_tflops": round(rank_tflops, 1), "hbm_gbs": float(peaks["hbm_gbs"])}}
    for causal in (False, True):
        pl = api.cpattn_plan_exchange(B, H, S, D, world, link_gbs, rank_tflops, float(peaks["hbm_gbs"]),
                                      causal=causal)
        exch_plan["causal" if causal else "non_causal"] = {
            "best": pl["best"], "us": {m: (None if pl[m]["seconds"] is None else round(pl[m]["seconds"] * 1e6, 1))
                                       for m in ("ring", "ulysses", "kv_gather")}}
    st, code = api.cpattn_device_status()
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1), RMS-normalised Q/K, bf16)",
        "config": config_block(cfg, world),
        "roofline": {"bound": "tensor", "kernel": "attn_fwd_kernel<128> ring steps incl. overlapped K/V rotation",
                     "achieved": rank_ring_flops / (ring_ms * 1e-3) / 1e12, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": rank_ring_flops / (ring_ms * 1e-3) / 1e12 / peak_tf,
                     "peak_kind": f"bf16_tflops burst, {peaks_kind}", "traffic": None},
        "gpu_launches": launches_per_step * args.steps, "clocks": clocks.summary(t0, t1),
        "e2e": {"value": step_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": 3 * B * S * H * D * 2, "d2h_bytes_per_step": 2 * B * S * H * D * 2,
                "note": "every rank uploads its Q/K/V shard and downloads both outputs; summed over ranks"},
        "device_status": code, "exchange_plan": exch_plan,
    }
    if rank == 0:
        print(json.dumps(line))
    del ring_group, uly_group
    dist.destroy_process_group()


def dit_extras(api, torch, dev, flush, peaks, inputs, link_gbs):
    """The image-DiT workload's other paths, timed each on its own: the step's
    kernels at that size, the causal variants, the backward, the fused
    projections, the exchange accounting and the exchange-selection model."""
    cfg, qb, kb, vb = inputs.config_inputs("dit")
    B, S, H, D = qb.shape
    P, U = cfg["ring_degree"], cfg["ulysses_degree"]
    q, k, v = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev) for x in (qb, kb, vb))
    stream = torch.cuda.current_stream()
    attn_flops = 4.0 * B * H * S * S * D
    peak_tf = float(peaks["bf16_tflops"])
    hbm = float(peaks["hbm_gbs"])
    tensor_bytes = B * S * H * D * 2
    qf, kf, vf = q.reshape(-1), k.reshape(-1), v.reshape(-1)
    yq, yk, yv, yo = (torch.empty_like(qf) for _ in range(4))
    out = torch.empty_like(qf)
    res = {}
    ms = median_event_ms(lambda: api.cpattn_ring_attention(q, k, v, P, stream=stream), flush, stream)
    res[f"ring_fused_p{P}"] = {"ms": ms, "TFLOP/s": attn_flops / (ms * 1e-3) / 1e12}
    ms = median_event_ms(lambda: api.cpattn_ulysses_permute_qkv(qf, kf, vf, B, S, H, D, U, yq=yq, yk=yk, yv=yv,
                                                                stream=stream), flush, stream)
    res[f"ulysses_permute_qkv_{U}"] = {"ms": ms, "GB/s": 6 * tensor_bytes / (ms * 1e-3) / 1e9}
    ms = median_event_ms(lambda: api.cpattn_head_sharded_attention(yq, yk, yv, B, S, H, D, U, yo=yo,
                                                                   stream=stream), flush, stream)
    res[f"head_sharded_attention_{U}"] = {"ms": ms, "TFLOP/s": attn_flops / (ms * 1e-3) / 1e12}
    ms = median_event_ms(lambda: api.cpattn_ulysses_unpermute(yo, B, S, H, D, U, x=out, stream=stream),
                         flush, stream)
    res[f"ulysses_unpermute_{U}_standalone"] = {"ms": ms, "GB/s": 2 * tensor_bytes / (ms * 1e-3) / 1e9}
    wsu = torch.empty(api.cpattn_ulysses_workspace_bytes(B, H, S, D), dtype=torch.uint8, device=dev)
    ms = median_event_ms(lambda: api.cpattn_ulysses_attention(qf, kf, vf, B, S, H, D, U, out=out, workspace=wsu,
                                                              stream=stream), flush, stream)
    res[f"ulysses_{U}_flow"] = {"ms": ms, "TFLOP/s": attn_flops / (ms * 1e-3) / 1e12,
                                "note": "Q/K/V permute + attention with the unpermute fused; 2 launches"}
    for key in res:
        if "GB/s" in res[key]:
            res[key]["frac_hbm"] = res[key]["GB/s"] / hbm
        else:
            res[key]["frac_bf16_peak"] = res[key]["TFLOP/s"] / peak_tf
    res.update(causal_paths(api, torch, flush, peaks, q, k, v, P, U))
    res.update(backward_paths(api, torch, flush, peaks, q, k, v, P))
    res.update(projection_paths(api, torch, flush, peaks, inputs, B, S, H, D, U))
    ring_tflops = res[f"ring_fused_p{P}"]["TFLOP/s"]

    # Accounting: what P GPUs would exchange per rank for this workload.
    exch = {}
    for mode, deg in (("ring", P), ("ulysses", U), ("kv_gather", P)):
        snd, rcv = api.cpattn_exchange_bytes(mode, B, H, S, D, deg)
        exch[f"{mode}_{deg}"] = {"send": snd[0], "recv": rcv[0]}
    exch["kv_gather_over_ulysses"] = exch[f"kv_gather_{P}"]["recv"] / max(1, exch[f"ulysses_{U}"]["recv"])
    # The exchange-selection model fed with this run's measured ring
    # throughput, the HBM bandwidth and the link bandwidth (--link-gbs;
    # default NVLink 5 nominal, an assumption, not a measurement).
    exch_plan = {"inputs": {"link_gbs": link_gbs,
                            "link_kind": "nominal assumption" if link_gbs == NOMINAL_LINK_GBS else "given",
                            "attn_tflops": round(ring_tflops, 1), "hbm_gbs": hbm}}
    for deg in (2, 4, 8):
        for causal in (False, True):
            pl = api.cpattn_plan_exchange(B, H, S, D, deg, link_gbs, ring_tflops, hbm, causal=causal)
            exch_plan[f"P{deg}" + ("_causal" if causal else "")] = {
                "best": pl["best"],
                "us": {m: (None if pl[m]["seconds"] is None else round(pl[m]["seconds"] * 1e6, 1))
                       for m in ("ring", "ulysses", "kv_gather")}}
    return {"workload": f"image-DiT B{B} H{H} S{S} D{D}", "kernels": res, "exchange_bytes_per_rank": exch,
            "exchange_plan": exch_plan}


def causal_flops(B, H, S, D):
    """4*D FLOPs per visible (query, key) pair; query i sees keys 0..i."""
    return 4.0 * B * H * D * S * (S + 1) / 2


def causal_paths(api, torch, flush, peaks, q, k, v, P, U):
    """The causal variants on the bench workload, outside the timed step: the
    fused causal ring and the causal Ulysses flow, each rep after an L2 flush."""
    B, S, H, D = q.shape
    stream = torch.cuda.current_stream()
    flops = causal_flops(B, H, S, D)
    peak_tf = float(peaks["bf16_tflops"])
    out = torch.empty_like(q)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    ws = torch.empty(api.cpattn_ulysses_workspace_bytes(B, H, S, D), dtype=torch.uint8, device=q.device)
    qf, kf, vf, of = q.reshape(-1), k.reshape(-1), v.reshape(-1), out.reshape(-1)

    res = {}
    for name, fn in (
        (f"causal_ring_fused_p{P}", lambda: api.cpattn_causal_ring_attention(q, k, v, P, out=out, lse=lse,
                                                                              stream=stream)),
        (f"causal_ulysses_{U}_flow", lambda: api.cpattn_causal_ulysses_attention(qf, kf, vf, B, S, H, D, U, out=of,
                                                                                 lse=lse, workspace=ws,
                                                                                 stream=stream)),
    ):
        ms = median_event_ms(fn, flush, stream)
        tf = flops / (ms * 1e-3) / 1e12
        res[name] = {"ms": ms, "TFLOP/s": tf, "frac_bf16_peak": tf / peak_tf,
                     "flops": "4*D per visible (query, key) pair: 2*B*H*D*S*(S+1)"}
    return res


def backward_flops(B, H, S, D, causal):
    """2.5x the forward's count (five S-sized matmuls against two), the usual
    accounting for an attention backward; causal: visible pairs only."""
    return 2.5 * (causal_flops(B, H, S, D) if causal else 4.0 * B * H * S * S * D)


def backward_paths(api, torch, flush, peaks, q, k, v, P):
    """The attention backward on the bench workload (dQ, dK, dV from the
    forward's output and LSE and a seeded upstream gradient), non-causal and
    causal, each rep after an L2 flush."""
    B, S, H, D = q.shape
    stream = torch.cuda.current_stream()
    gen = torch.Generator(device=q.device).manual_seed(7)
    do = torch.randn(q.shape, generator=gen, device=q.device).to(torch.bfloat16)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    # with the dS scratch the bindings allocate by default (all heads here)
    ws = torch.empty(api.backward_workspace_bytes(B, H, S), dtype=torch.uint8, device=q.device)
    peak_tf = float(peaks["bf16_tflops"])
    res = {}
    for causal in (False, True):
        fwd = api.cpattn_causal_ring_attention if causal else api.cpattn_ring_attention
        out, lse = fwd(q, k, v, P, stream=stream)

        def run():
            api.cpattn_attention_backward(q, k, v, out, lse, do, causal, dq, dk, dv, ws, stream=stream)

        ms = median_event_ms(run, flush, stream)
        tf = backward_flops(B, H, S, D, causal) / (ms * 1e-3) / 1e12
        res["attention_backward" + ("_causal" if causal else "")] = {
            "ms": ms, "TFLOP/s": tf, "frac_bf16_peak": tf / peak_tf,
            "flops": "2.5x the forward's (10*B*H*S^2*D; causal: visible pairs)", "launches": 3,
            "note": "row sums, dK/dV storing dS, dQ GEMM over the stored dS"}
    # the backward of the Ulysses flow (rank buffers; B = 1 here, so they are the full tensors)
    U = 4
    out, lse = api.cpattn_ulysses_attention(q.reshape(-1), k.reshape(-1), v.reshape(-1), B, S, H, D, U, stream=stream)
    wsu = torch.empty(api.backward_workspace_bytes(B, H, S, ulysses_D=D), dtype=torch.uint8, device=q.device)

    def run_u():
        api.cpattn_ulysses_attention_backward(q.reshape(-1), k.reshape(-1), v.reshape(-1), out, lse, do.reshape(-1),
                                              B, S, H, D, U, dq=dq.reshape(-1), dk=dk.reshape(-1), dv=dv.reshape(-1),
                                              workspace=wsu, stream=stream)

    ms = median_event_ms(run_u, flush, stream)
    tf = backward_flops(B, H, S, D, False) / (ms * 1e-3) / 1e12
    res[f"ulysses_{U}_backward_flow"] = {"ms": ms, "TFLOP/s": tf, "frac_bf16_peak": tf / peak_tf,
                                         "launches": 5, "note": "5 tensors permuted in (2 launches), the row sums of "
                                         "the 4 head ranks in one launch, dK/dV and the dQ GEMM over all of them, "
                                         "storing the gradients in the sequence-sharded layout"}
    return res


def projection_flops(B, S, H, D, Dm):
    """2*K FLOPs per output element (one multiply and one add per term):
    the Q/K/V projection (B*S x 3*H*D outputs, K = Dm) and the output
    projection (B*S x Dm outputs, K = H*D)."""
    return 2.0 * B * S * Dm * 3 * H * D, 2.0 * B * S * H * D * Dm


def projection_paths(api, torch, flush, peaks, inputs, B, S, H, D, U):
    """The Ulysses projections with the all-to-all fused in, on the bench
    workload's sizes (model width H*D), each rep after an L2 flush: the Q/K/V
    projection storing the head-sharded layout, and the output projection
    reading it in place.  For context, the unfused form with a library GEMM
    (torch.matmul, cuBLAS) and this library's permute kernels is timed beside
    them; it is not part of this library's path."""
    Dm = H * D                      # model width = heads x head dim (3072 on image-DiT)
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    xb, wb, wob = inputs.make_projection_inputs(B, S, H, D, Dm, 4321)
    x, w, wo = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev) for a in (xb, wb, wob))
    n = B * S * H * D
    yq, yk, yv, yo = (torch.empty(n, dtype=torch.bfloat16, device=dev) for _ in range(4))
    out = torch.empty(B * S * Dm, dtype=torch.bfloat16, device=dev)
    peak_tf = float(peaks["bf16_tflops"])
    f_qkv, f_out = projection_flops(B, S, H, D, Dm)
    res = {}

    def rec(name, fn, flops, note):
        ms = median_event_ms(fn, flush, stream)
        tf = flops / (ms * 1e-3) / 1e12
        res[name] = {"ms": ms, "TFLOP/s": tf, "frac_bf16_peak": tf / peak_tf, "note": note}

    rec(f"ulysses_{U}_qkv_projection_fused",
        lambda: api.cpattn_ulysses_qkv_projection(x, w, B, S, H, D, Dm, U, yq=yq, yk=yk, yv=yv, stream=stream),
        f_qkv, f"X W_qkv^T (Dm {Dm}) stored head-sharded, one launch; FLOPs 2*B*S*Dm*3*H*D")
    rec(f"ulysses_{U}_output_projection_fused",
        lambda: api.cpattn_ulysses_output_projection(yq, wo, B, S, H, D, Dm, U, out=out, stream=stream),
        f_out, "O W_o^T read from the head-sharded layout, one launch; FLOPs 2*B*S*H*D*Dm")
    x2 = x.view(B * S, Dm)
    w3 = w.view(3, H * D, Dm)
    q3, k3, v3 = (torch.empty(n, dtype=torch.bfloat16, device=dev) for _ in range(3))

    def unfused_qkv():
        for t, y in enumerate((q3, k3, v3)):
            torch.matmul(x2, w3[t].t(), out=y.view(B * S, H * D))
        api.cpattn_ulysses_permute_qkv(q3, k3, v3, B, S, H, D, U, yq=yq, yk=yk, yv=yv, stream=stream)

    def unfused_out():
        api.cpattn_ulysses_unpermute(yq, B, S, H, D, U, x=yo, stream=stream)
        torch.matmul(yo.view(B * S, H * D), wo.view(Dm, H * D).t(), out=out.view(B * S, Dm))

    rec("context_unfused_qkv_projection_cublas_plus_permute", unfused_qkv, f_qkv,
        "three library GEMMs (Q, K, V) and the Q/K/V permute kernel (context only)")
    rec("context_unfused_output_projection_unpermute_plus_cublas", unfused_out, f_out,
        "unpermute kernel and library GEMM (context only)")
    return res


def library_context_paths(torch, q, k, v, cflops):
    """Unsharded attention by torch's SDPA library backends on the same bf16
    (B, S, H, D) tensors (strided (B, H, S, D) views, no copy).  Context rows
    only: the pages run such a library kernel once per chunk; nothing of this
    library's path uses them."""
    from torch.nn.attention import SDPBackend, sdpa_kernel
    qt, kt, vt = (x.transpose(1, 2) for x in (q, k, v))

    def sdpa(backend, causal):
        def run():
            with sdpa_kernel([backend]):
                torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal)
        return run
    def sdpa_backward(backend, causal):
        # The graph is built once; each call runs only the library's backward.
        leaves = [x.detach().requires_grad_(True) for x in (q, k, v)]
        gen = torch.Generator(device=q.device).manual_seed(7)
        do = torch.randn(q.shape, generator=gen, device=q.device).to(q.dtype).transpose(1, 2)
        with sdpa_kernel([backend]):
            o = torch.nn.functional.scaled_dot_product_attention(*(x.transpose(1, 2) for x in leaves),
                                                                 is_causal=causal)

        def run():
            torch.autograd.grad(o, leaves, do, retain_graph=True)
        return run
    B, S, H, D = q.shape
    out = []
    for backend, tag in ((SDPBackend.CUDNN_ATTENTION, "cuDNN"), (SDPBackend.FLASH_ATTENTION, "FlashAttention-2")):
        out.append((f"library context: torch SDPA {tag}, unsharded", sdpa(backend, False)))
        out.append((f"library context: torch SDPA {tag}, unsharded, causal", sdpa(backend, True), cflops))
    for causal in (False, True):
        try:
            fn = sdpa_backward(SDPBackend.CUDNN_ATTENTION, causal)
        except RuntimeError as e:
            fn = e
        label = "library context: torch SDPA cuDNN backward" + (", causal" if causal else "")
        out.append((label, fn, backward_flops(B, H, S, D, causal)))
    return out


def run_sweep(args):
    """Every workload's paths, each timed on its own (median of `steps` reps,
    L2 flushed before each rep): attention TFLOP/s per path."""
    import torch
    from context_attention_long_b200 import api, build, inputs
    build.build()
    dev = torch.device("cuda", 0)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    peaks, kind = load_peaks()
    reps = max(3, args.steps)

    stream = torch.cuda.current_stream()

    def timeit(fn):
        return median_event_ms(fn, flush, stream, reps=reps, warmup=args.warmup)

    for name in ("tiny", "dit", "hires", "anything", "video"):
        cfg, qb, kb, vb = inputs.config_inputs(name)
        B, S, H, D = qb.shape
        q, k, v = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev) for x in (qb, kb, vb))
        del qb, kb, vb
        flops = 4.0 * B * H * S * S * D
        cflops = causal_flops(B, H, S, D)
        paths = []
        P = cfg["ring_degree"]
        lens = None
        if name == "anything":
            lens = inputs.ring_anything_lens(S, P, cfg["seed"])
        paths.append(("unsharded (the fused kernel with one shard: the single-GPU baseline)",
                      lambda: api.cpattn_ring_attention(q, k, v, 1, want_lse=True)))
        paths.append((f"ring fused P={P}" + (" (Ring Anything)" if lens else ""),
                      lambda: api.cpattn_ring_attention(q, k, v, P, lens, want_lse=True)))
        paths.append((f"causal ring fused P={P}" + (" (Ring Anything)" if lens else ""),
                      lambda: api.cpattn_causal_ring_attention(q, k, v, P, lens, want_lse=True), cflops))
        if name in ("tiny", "dit"):
            po = torch.empty((P, B, S, H, D), dtype=torch.float32, device=dev)
            pl = torch.empty((P, B, H, S), dtype=torch.float32, device=dev)
            ob = torch.empty_like(q)
            lo = torch.empty((B, H, S), dtype=torch.float32, device=dev)

            def unfused():
                for t in range(P):
                    api.cpattn_ring_step(q, k, v, P, t, lens, part_out=po[t], part_lse=pl[t])
                api.cpattn_lse_merge(po, pl, out_bf16=ob, lse_out=lo)
            paths.append((f"ring unfused P={P} (steps + LSE merge)", unfused))
        kvd = cfg.get("kv_gather_degree", P)
        if S % kvd == 0:
            paths.append((f"kv_gather {kvd}", lambda: api.cpattn_kv_gather_attention(q, k, v, kvd)))
        U = cfg["ulysses_degree"]
        if name == "video":
            ws = torch.empty(api.cpattn_unified_workspace_bytes(B, H, S, D), dtype=torch.uint8, device=dev)
            paths.append((f"unified ring {P} x Ulysses {U}",
                          lambda: api.cpattn_unified_attention(q, k, v, P, U, workspace=ws)))
            paths.append((f"causal unified ring {P} x Ulysses {U}",
                          lambda: api.cpattn_causal_unified_attention(q, k, v, P, U, workspace=ws), cflops))
        else:
            seq = inputs.front_loaded_splits(S, U) if name == "anything" else None
            heads = inputs.front_loaded_splits(H, U) if name == "anything" else None
            ws = torch.empty(api.cpattn_ulysses_workspace_bytes(B, H, S, D), dtype=torch.uint8, device=dev)
            qf, kf, vf = q.reshape(-1), k.reshape(-1), v.reshape(-1)
            paths.append((f"Ulysses {U}" + (" (Anything)" if seq else "") +
                          " flow: Q/K/V permute + attention (the unpermute fused in its epilogue)",
                          lambda: api.cpattn_ulysses_attention(qf, kf, vf, B, S, H, D, U, seq, heads, workspace=ws)))
            paths.append((f"causal Ulysses {U}" + (" (Anything)" if seq else "") + " flow",
                          lambda: api.cpattn_causal_ulysses_attention(qf, kf, vf, B, S, H, D, U, seq, heads,
                                                                      workspace=ws), cflops))
        if name in ("dit", "hires", "video"):
            gen = torch.Generator(device=dev).manual_seed(7)
            do = torch.randn(q.shape, generator=gen, device=dev).to(torch.bfloat16)
            bq, bk, bv = (torch.empty_like(q) for _ in range(3))
            bws = torch.empty(api.backward_workspace_bytes(B, H, S), dtype=torch.uint8, device=dev)
            o_f, l_f = api.cpattn_ring_attention(q, k, v, P, lens)
            o_c, l_c = api.cpattn_causal_ring_attention(q, k, v, P, lens)
            paths.append(("attention backward (dQ, dK, dV)",
                          lambda: api.cpattn_attention_backward(q, k, v, o_f, l_f, do, False, bq, bk, bv, bws),
                          backward_flops(B, H, S, D, False)))
            paths.append(("causal attention backward",
                          lambda: api.cpattn_attention_backward(q, k, v, o_c, l_c, do, True, bq, bk, bv, bws),
                          backward_flops(B, H, S, D, True)))
        if name in ("dit", "hires", "video"):
            paths += library_context_paths(torch, q, k, v, cflops)
        if name in ("dit", "video"):
            U_p = cfg["ulysses_degree"]
            for key, r in projection_paths(api, torch, flush, peaks, inputs, B, S, H, D, U_p).items():
                print(json.dumps({"workload": name, "shape": f"B{B} H{H} S{S} D{D} Dm{H * D}", "path": key,
                                  "ms": round(r["ms"], 4), "TFLOP/s": round(r["TFLOP/s"], 1),
                                  "frac_bf16_peak": round(r["frac_bf16_peak"], 4), "peak_kind": kind}), flush=True)
        for entry in paths:
            label, fn = entry[0], entry[1]
            try:
                if isinstance(fn, Exception):
                    raise fn
                ms = timeit(fn)
            except RuntimeError as e:    # a library backend that refuses this shape
                print(json.dumps({"workload": name, "path": label, "unavailable": str(e).splitlines()[0][:200]}),
                      flush=True)
                continue
            tf = (entry[2] if len(entry) > 2 else flops) / (ms * 1e-3) / 1e12
            print(json.dumps({"workload": name, "shape": f"B{B} H{H} S{S} D{D}", "path": label, "ms": round(ms, 4),
                              "TFLOP/s": round(tf, 1), "frac_bf16_peak": round(tf / float(peaks["bf16_tflops"]), 4),
                              "peak_kind": kind}), flush=True)
        st, code = api.cpattn_device_status()
        if st != 0:
            raise RuntimeError(f"device wait expired: {code:#x}")
        del q, k, v
        torch.cuda.empty_cache()


def run_single_kernel(args):
    """Profiling mode: `warmup + steps` launches of one kernel (or one flow) on
    the workload `--workload` (merge: P float32 partials of it), nothing else."""
    import torch
    from context_attention_long_b200 import api, build, inputs
    build.build()
    cfg, qb, kb, vb = inputs.config_inputs(args.workload)
    B, S, H, D = qb.shape
    P, U = cfg["ring_degree"], cfg["ulysses_degree"]
    dev = torch.device("cuda", 0)
    q, k, v = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev) for x in (qb, kb, vb))
    if args.kernel == "ring":
        fn = lambda: api.cpattn_ring_attention(q, k, v, P)
    elif args.kernel == "causal_ring":
        fn = lambda: api.cpattn_causal_ring_attention(q, k, v, P)
    elif args.kernel == "ring_step":
        fn = lambda: api.cpattn_ring_step(q, k, v, P, 1)
    elif args.kernel == "head_sharded":
        yq, yk, yv = (api.cpattn_ulysses_permute(t.reshape(-1), B, S, H, D, U) for t in (q, k, v))
        fn = lambda: api.cpattn_head_sharded_attention(yq, yk, yv, B, S, H, D, U)
    elif args.kernel == "backward":
        out, lse = api.cpattn_ring_attention(q, k, v, P)
        do = torch.randn(q.shape, device=dev).to(torch.bfloat16)
        fn = lambda: api.cpattn_attention_backward(q, k, v, out, lse, do)
    elif args.kernel == "permute_qkv":
        qf, kf, vf = q.reshape(-1), k.reshape(-1), v.reshape(-1)
        yq, yk, yv = torch.empty_like(qf), torch.empty_like(kf), torch.empty_like(vf)
        fn = lambda: api.cpattn_ulysses_permute_qkv(qf, kf, vf, B, S, H, D, U, yq=yq, yk=yk, yv=yv)
    elif args.kernel == "permute":
        fn = lambda: api.cpattn_ulysses_permute(q.reshape(-1), B, S, H, D, U)
    elif args.kernel == "unpermute":
        x = torch.empty_like(q.reshape(-1))
        fn = lambda: api.cpattn_ulysses_unpermute(q.reshape(-1), B, S, H, D, U, x=x)
    elif args.kernel == "unified":
        ws = torch.empty(api.cpattn_unified_workspace_bytes(B, H, S, D), dtype=torch.uint8, device=dev)
        fn = lambda: api.cpattn_unified_attention(q, k, v, P, U, workspace=ws)
    elif args.kernel in ("qkv_projection", "output_projection"):
        Dm = H * D
        xb, wb, wob = inputs.make_projection_inputs(B, S, H, D, Dm, 4321)
        x, w, wo = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev) for a in (xb, wb, wob))
        yq, yk, yv = api.cpattn_ulysses_qkv_projection(x, w, B, S, H, D, Dm, U)
        if args.kernel == "qkv_projection":
            fn = lambda: api.cpattn_ulysses_qkv_projection(x, w, B, S, H, D, Dm, U, yq=yq, yk=yk, yv=yv)
        else:
            fn = lambda: api.cpattn_ulysses_output_projection(yq, wo, B, S, H, D, Dm, U)
    else:
        po = torch.randn((P, B, S, H, D), device=dev)
        pl = torch.randn((P, B, H, S), device=dev)
        fn = lambda: api.cpattn_lse_merge(po, pl)
    t0 = time.perf_counter()
    for _ in range(args.warmup + args.steps):
        fn()
    torch.cuda.synchronize()
    st, code = api.cpattn_device_status()
    print(json.dumps({"kernel": args.kernel, "launches": args.warmup + args.steps, "status": st, "code": code,
                      "wall_s": time.perf_counter() - t0}))
    if st != 0:
        sys.exit(1)


if __name__ == "__main__":
    main()
