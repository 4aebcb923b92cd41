#!/usr/bin/env python
"""Benchmark of the fused pair-bias attention (features -> folded MLP ->
masked attention with the bias kept on chip) on the N=128 jets, P=128 slots,
H=8, D=16 workload.

One step = one call of pair_attention_forward over one batch of synthetic
jets (one kernel launch). Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): every rank processes its own batch (jets are
independent; no collective on the data path), so per-GPU work is fixed and
the scaling is weak. Timing: CUDA events on the launching stream, bracketed
by a barrier and a synchronize, max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from part_pair_bias_b200 import configs, shard, synth  # noqa: E402

L2_BYTES = 126 * 2 ** 20
MLP_FLOP_PER_PAIR = 2 * (4 * 64 + 64 * 64 + 64 * 64 + 64 * 8)          # 17,920 (algorithmic)
MMA_FLOP_PER_ROW = 2 * (16 * 64 + 64 * 64 + 64 * 64 + 64 * 16)         # 20,480 (issued per tile row)
# what the fused kernel computes in: MLP on tcgen05 with f16 operands, the
# hidden layers accumulated in f16 and the output layer in fp32; attention
# with bf16 operands and fp32 scores, softmax and accumulation
MLP_DTYPE = ("f16 MLP operands (hidden layers f16-accumulated, output layer fp32), "
             "bf16 Q/K/V/out with fp32 attention accumulate")
# backward MLP per unordered pair: recompute of layers 1-3, dL/dh3..dL/dh1
# (g W4, d3 W3, d2 W2) and the weight gradients dW4, dW3, dW2, dW1
BWD_FLOP_PER_PAIR = 2 * (4 * 64 + 2 * 64 * 64) + 2 * (8 * 64 + 2 * 64 * 64) + 2 * (8 * 64 + 2 * 64 * 64 + 64 * 4)
# issued per tile row by the MLP backward kernel: z1 and g W4 (K = 16), four
# 64 x 64 GEMMs, and the weight-gradient MMAs (dW4: 16 x 72, dW3, dW2: 64 x 72,
# dW1: 64 x 16 with the bias columns)
BWD_MMA_FLOP_PER_ROW = 2 * (2 * 16 * 64 + 4 * 64 * 64) + 2 * (16 * 72 + 2 * 64 * 72 + 64 * 16)
PROFILE = os.path.join(ROOT, "profiles", "k_fused_cluster_n128_p128.txt")
KERNEL_SOURCES = [os.path.join(ROOT, "part_pair_bias_b200", "csrc", f)
                  for f in ("pb_kernels.cuh", "pb_backward.cuh", "pb_device.cuh", "pairbias.cu")]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="n128_p128")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--sweep", action="store_true",
                    help="one JSON line per (workload, path) with times, rates and FLOP conventions")
    ap.add_argument("--sweep-workloads", default=None, help="comma list restricting --sweep's workloads")
    ap.add_argument("--sweep-paths", default=None, help="comma list restricting --sweep's paths")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def pair_counts(b):
    m = b.mult.astype(np.int64)
    unordered = m * (m + 1) // 2
    tiles = (unordered + 127) // 128
    return int(unordered.sum()), int(tiles.sum()), int((m * m).sum())


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d.get("bf16_tflops"), d.get("hbm_gbs"), "measured"
    return 1590.0, 6650.0, "fallback"


def kernel_sha():
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    if not os.path.exists(PROFILE):
        return None
    kv = {}
    for line in open(PROFILE):
        if ":" in line:
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    if kv.get("kernel_source_sha") != kernel_sha():
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi samples (SM clock, reasons) taken while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.rows, self.proc, self.window = [], None, None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        inside = [r for t, r in self.rows if t0 <= t <= t1]
        note = None
        if not inside:  # region shorter than the sampling period: nearest samples after its start
            inside = [r for t, r in self.rows if t >= t0][:3] or [self.rows[-1][1]]
            note = "timed region shorter than the 50 ms sampling period; nearest samples"
        sm = [float(r[1]) for r in inside if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in inside if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i in range(4) if len(r) > 5 + i and r[5 + i] == "Active"})
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
               "reasons": reasons, "samples": len(inside)}
        if note:
            out["note"] = note
        return out


def cpu_baseline(b, seconds, threads=None):
    """The fp64 oracle, as it stands, on the host cores (all of them, or
    `threads`): full batches until `seconds` have passed (at least one)."""
    import oracle
    oracle.build()
    prev = oracle.threads()
    if threads is not None:
        oracle.set_threads(threads)
    try:
        return _time_oracle(oracle, b, seconds)
    finally:
        oracle.set_threads(prev if threads is not None else 0)


def _time_oracle(oracle, b, seconds):
    t0 = time.perf_counter()
    passes = 0
    while True:
        oracle.forward(b)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            break
    return {"value": passes * b.N / dt, "unit": "jets/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{passes} pass(es) over the full {b.N}-jet batch, {dt:.1f} s"}


# --------------------------------------------------------------- our path

def run_ours(args, world, rank, local):
    from part_pair_bias_b200 import ops
    import torch.distributed as dist

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    wl = args.workload
    b = synth.make_jets(**configs.workload(wl, seed=shard.rank_seed(args.seed, rank)))
    unordered, tiles, ordered = pair_counts(b)
    mlp = ops.folded_mlp(b.params, dev)

    set_bytes = 4 * b.E.nbytes + (b.mask.nbytes if b.mask is not None else b.ptr.nbytes) + 4 * b.q.nbytes
    R = max(2, min(64, math.ceil(2 * L2_BYTES / set_bytes) + 1))
    sets = []
    for _ in range(R):
        jets = ops.jets_to_device(b, dev)
        q, k, v = (ops.bf16_to_device(x, dev) for x in (b.q, b.k, b.v))
        sets.append((jets, q, k, v, torch.empty_like(q)))

    def step(i):
        jets, q, k, v, out = sets[i % R]
        ops.pair_attention_forward(jets, mlp, None, q, k, v, out)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if ops.get_device_status():
        raise RuntimeError("device status set during warm-up")

    K = args.steps
    # The timed steps replay a CUDA graph of G consecutive steps (one launch
    # each, cycling over the R input sets), which removes the host's launch
    # gaps; steps beyond a whole number of replays are launched directly.
    # Fewer steps than one such graph are captured as one graph of exactly K
    # launches, replayed once.
    G = R * max(1, 170 // R)
    if K < G:
        G = K
    graph = None
    if K >= G:
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            for i in range(G):
                step(args.warmup + i)
        torch.cuda.current_stream().wait_stream(cap)
        graph.replay()  # warm-up of the captured launches
        torch.cuda.synchronize()
        if ops.get_device_status():
            raise RuntimeError("device status set during the graph warm-up")
    n_rep = K // G if graph is not None else 0
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    gpu_index = vis.split(",")[local] if vis else str(local)
    sampler = ClockSampler(gpu_index) if rank == 0 else None
    time.sleep(0.3 if sampler else 0)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    if graph is not None:
        # an untimed lead-in replay keeps the device busy while the host
        # submits the timed ones, so the start event is not followed by an
        # idle gap of graph submission
        graph.replay()
    start.record()
    for _ in range(n_rep):
        graph.replay()
    for i in range(n_rep * G, K):
        step(args.warmup + i)
    end.record()
    torch.cuda.synchronize()
    t1 = time.time()
    if world > 1:
        dist.barrier()
    clocks = sampler.summary(t0, t1) if sampler else None
    if sampler:
        sampler.stop()
    ms = start.elapsed_time(end)
    launch_ms = ms / K  # the timed region holds K launches of the one kernel and nothing else
    status = ops.get_device_status()

    # End to end through the public API from pinned host buffers: every step
    # copies its inputs in (one copy from a packed pinned buffer), runs the
    # call and copies its result out. Steps are double-buffered over three
    # streams (copy in, compute, copy out), so one step's copies overlap the
    # neighbouring steps' kernel and copies, as a serving loop would run them.
    parts = [("E", b.E), ("px", b.px), ("py", b.py), ("pz", b.pz),
             ("mask", b.mask) if b.mask is not None else ("ptr", b.ptr), ("q", b.q), ("k", b.k), ("v", b.v)]
    offs, total = {}, 0
    for name, arr in parts:
        offs[name] = (total, arr.nbytes)
        total += (arr.nbytes + 255) // 256 * 256  # every segment 256-byte aligned
    host_in = torch.empty(total, dtype=torch.uint8).pin_memory()
    for name, arr in parts:
        o, n = offs[name]
        host_in[o:o + n] = torch.from_numpy(np.ascontiguousarray(arr).view(np.uint8).reshape(-1))
    h2d = sum(arr.nbytes for _, arr in parts)

    def device_set():
        raw = torch.empty(total, dtype=torch.uint8, device=dev)

        def seg(name, dtype, shape):
            o, n = offs[name]
            return raw[o:o + n].view(dtype).view(shape)
        jets_e = ops.jets_to_device(b, dev)  # the descriptor's other fields (N, P, layout)
        for name in ("E", "px", "py", "pz"):
            setattr(jets_e, name, seg(name, torch.float32, (-1,)))
        if b.mask is not None:
            jets_e.mask = seg("mask", torch.uint8, (-1,))
        else:
            jets_e.ptr = seg("ptr", torch.int32, (-1,))
        qkv = [seg(name, torch.bfloat16, sets[0][1].shape) for name in ("q", "k", "v")]
        return raw, jets_e, qkv, torch.empty_like(sets[0][4])

    bufs = [device_set() for _ in range(2)]
    out_host = torch.empty(sets[0][4].shape, dtype=torch.bfloat16).pin_memory()
    d2h = out_host.numel() * out_host.element_size()
    Ke = max(1, min(K, 500))
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    loaded, ran, read = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [False, False]

    def e2e_step(i):
        j = i & 1
        raw, jets_e, (qd, kd, vd), outd = bufs[j]
        with torch.cuda.stream(s_in):
            if used[j]:
                s_in.wait_event(ran[j])  # the kernel two steps back has read these inputs
            raw.copy_(host_in, non_blocking=True)
            loaded[j].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(loaded[j])
            if used[j]:
                s_run.wait_event(read[j])  # the copy-out two steps back has read this output
            ops.pair_attention_forward(jets_e, mlp, None, qd, kd, vd, outd, stream=s_run)
            ran[j].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ran[j])
            out_host.copy_(outd, non_blocking=True)
            read[j].record(s_out)
        used[j] = True

    def join():
        cur = torch.cuda.current_stream()
        for st in (s_in, s_run, s_out):
            cur.wait_stream(st)

    torch.cuda.synchronize()
    for i in range(3):
        e2e_step(i)
    join()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    es.record()
    for st in (s_in, s_run, s_out):
        st.wait_stream(torch.cuda.current_stream())  # nothing starts before the start event
    for i in range(Ke):
        e2e_step(i)
    join()
    ee.record()
    torch.cuda.synchronize()
    e2e_ms = es.elapsed_time(ee)
    status |= ops.get_device_status()
    # the pipeline's last result against a plain call on the same inputs
    ref_out = torch.empty_like(sets[0][4])
    jets0, q0, k0, v0, _ = sets[0]
    ops.pair_attention_forward(jets0, mlp, None, q0, k0, v0, ref_out)
    torch.cuda.synchronize()
    if not torch.equal(out_host, ref_out.cpu()):
        raise RuntimeError("the pipelined end-to-end output differs from a plain call")

    ms, e2e_ms, launch_ms, status = shard.reduce_max([ms, e2e_ms, launch_ms, float(status)], device=dev)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    if status:
        raise RuntimeError(f"device status bits {int(status):#x} during the timed region")

    value = shard.job_rate(b.N * K, world, ms / 1e3)
    peak_tf, hbm_gbs, peak_src = measured_peaks()
    alg_flop = unordered * MLP_FLOP_PER_PAIR
    achieved_tf = alg_flop / (launch_ms / 1e3) / 1e12
    exec_tf = tiles * 128 * MMA_FLOP_PER_ROW / (launch_ms / 1e3) / 1e12
    dense_tf = b.N * b.P * b.P * MLP_FLOP_PER_PAIR / (launch_ms / 1e3) / 1e12
    traffic = profiled_traffic()
    line = {
        "metric": "jets/s for fused pair-bias attention (P=128,H=8,D=16); % bf16 tensor peak",
        "value": value,
        "unit": "jets/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": MLP_DTYPE,
        "data": "synthetic",
        "config": {"workload": wl, "jets_per_gpu": b.N, "P": b.P, "H": 8, "D": 16, "layout": b.layout,
                   "mean_multiplicity": float(b.mult.mean()), "path": "fused, 4-CTA clusters (bias in distributed shared memory)",
                   "l2": f"{R} rotating input sets of {set_bytes / 2**20:.1f} MiB (> 2x L2)",
                   "launch": (f"CUDA graph of {G} launches replayed {n_rep}x after an untimed lead-in replay"
                              if n_rep else "stream launches")
                   + (f" + {K - n_rep * G} stream launches" if n_rep and K > n_rep * G else ""),
                   "parallelism": f"data-parallel over jets x{world}, no collective"},
        "pairs_per_s": shard.job_rate(ordered * K, world, ms / 1e3),
        "gpu_launches": K,
        "roofline": {"bound": "tensor", "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": achieved_tf / peak_tf, "traffic": traffic,
                     "kernel": "k_fused_cluster", "launch_ms": launch_ms,
                     "flop_per_launch": alg_flop,
                     "flop_convention": "algorithmic: 17,920 per valid unordered pair (incl. diagonal)",
                     "exec_tflops": exec_tf, "dense_equiv_tflops": dense_tf,
                     "peak_source": f"{peak_src} bf16 dense burst (f16 runs at the same tensor rate)"},
        "clocks": clocks,
        "e2e": {"value": shard.job_rate(b.N * Ke, world, e2e_ms / 1e3), "unit": "jets/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": Ke,
                "pipeline": "double-buffered; copy in, kernel and copy out on three streams"},
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(b, args.cpu_seconds)
    print(json.dumps(line), flush=True)


# -------------------------------------------------------- reference arm

def run_reference(args, world, rank):
    """The fp64 oracle on the host cores, on the same workload and metric;
    each step is a bounded sample of 16 jets of the batch."""
    if rank != 0:
        return
    import oracle
    oracle.build()
    b = synth.make_jets(**configs.workload(args.workload, seed=args.seed))
    per = 16
    samples = [synth.slice_jets(b, lo, min(b.N, lo + per)) for lo in range(0, b.N, per)]
    for i in range(args.warmup):
        oracle.forward(samples[i % len(samples)])
    t0 = time.perf_counter()
    jets = 0
    for i in range(args.steps):
        s = samples[i % len(samples)]
        oracle.forward(s)
        jets += s.N
    dt = time.perf_counter() - t0
    value = jets / dt
    cores = oracle.threads()
    line = {
        "metric": "jets/s for fused pair-bias attention (P=128,H=8,D=16); % bf16 tensor peak",
        "value": value, "unit": "jets/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / max(1, args.steps), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": args.workload, "jets_per_step": per, "P": b.P, "H": 8, "D": 16},
        "cpu_baseline": {"value": value, "unit": "jets/s", "cores": cores, "kind": "oracle",
                         "sample": f"{per} jets of the {b.N}-jet batch per step, {args.steps} steps"},
        "e2e": {"value": value, "unit": "jets/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ sweep

def run_sweep(args):
    """One JSON line per (workload, path): device time (median of 20 launches
    after warm-up, L2 flushed before each), jets/s, valid ordered pairs/s,
    algorithmic GB/s, the MLP's TFLOP/s under the three conventions (alg:
    valid unordered pairs; exec: issued tile rows; dense: N P^2), and the
    host oracle's rate on a bounded sample of the workload (first jets)."""
    from part_pair_bias_b200 import ops
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
    peak_tf, hbm_gbs, peak_src = measured_peaks()

    def timed(fn, reps=20):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record()
            fn()
            s1.record()
            torch.cuda.synchronize()
            ts.append(s0.elapsed_time(s1))
        return statistics.median(ts)

    names = list(configs.ORDER) + ["n128_p128_full"]
    if args.sweep_workloads:
        names = [n for n in names if n in args.sweep_workloads.split(",")]
    only = set(args.sweep_paths.split(",")) if args.sweep_paths else None
    for name in names:
        if name == "n128_p128_full":
            b = synth.make_jets(**configs.workload("n128_p128", seed=args.seed, dist="full"))
        else:
            b = synth.make_jets(**configs.workload(name, seed=args.seed))
        unordered, tiles, ordered = pair_counts(b)
        valid = int(b.mult.sum())
        slots = b.N * b.P if b.layout == "padded" else valid
        jets = ops.jets_to_device(b, dev)
        mlp = ops.folded_mlp(b.params, dev)
        q, k, v = (ops.bf16_to_device(x, dev) for x in (b.q, b.k, b.v))
        out = torch.empty_like(q)
        feat = torch.empty((b.N, b.P, b.P, 4), device=dev)
        U = torch.empty((b.N, 8, b.P, b.P), device=dev, dtype=torch.bfloat16)
        ws = ops.workspace_for(jets, dev)
        bi = synth.make_block_inputs(b, args.seed)
        proj = ops.proj_to_device(bi, dev)
        x = ops.bf16_to_device(bi.x, dev)
        y = torch.empty_like(x)
        bws = torch.empty(ops.block_workspace_bytes(jets), dtype=torch.uint8, device=dev)
        inp = 17 * slots                      # momenta + mask (or ptr) per slot
        qkv = 3 * 256 * valid                 # Q, K, V rows of the valid particles
        paths = [
            ("features", lambda: ops.pairfeat_compute(jets, feat), inp + 16 * b.N * b.P * b.P, False),
            ("bias_bf16", lambda: ops.pairbias_mlp_forward(jets, mlp, U), inp + 2 * 8 * b.N * b.P * b.P, True),
            ("attention_reading_bias", lambda: ops.pair_attention_forward(jets, None, U, q, k, v, out),
             inp + qkv + 2 * 8 * ordered + 256 * slots, False),
            ("fused", lambda: ops.pair_attention_forward(jets, mlp, None, q, k, v, out), inp + qkv + 256 * slots, True),
        ]
        if ws is not None:
            paths.append(("fused_balanced", lambda: ops.pair_attention_forward(jets, mlp, None, q, k, v, out,
                                                                               workspace=ws),
                          inp + qkv + 256 * slots, True))
        paths.append(("block", lambda: ops.pair_block_forward(jets, mlp, proj, x, y, bws),
                      inp + 256 * slots + 256 * slots, True))
        mlp8 = ops.mlp_i8(b.params, dev)
        paths.append(("bias_bf16_int8", lambda: ops.pairbias_mlp_forward_i8(jets, mlp8, U),
                      inp + 2 * 8 * b.N * b.P * b.P, True))
        paths.append(("fused_int8", lambda: ops.pair_attention_forward_i8(jets, mlp8, q, k, v, out),
                      inp + qkv + 256 * slots, True))
        dout = ops.bf16_to_device(synth.make_upstream(b, args.seed), dev)
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
        grad = ops.MlpGrad(dev)
        gws = torch.empty(ops.backward_workspace_bytes(jets), dtype=torch.uint8, device=dev)
        # bytes: inputs twice (bias kernel, MLP backward), q/k/v/dout read, dq/dk/dv written,
        # the bf16 bias planes written, read and overwritten, dL/dU read per pair
        plane = 2 * 8 * b.N * b.P * b.P
        paths.append(("backward", lambda: ops.pair_attention_backward(jets, mlp, q, k, v, dout, dq, dk, dv, grad, gws),
                      2 * inp + 4 * 256 * valid + 3 * 256 * slots + 3 * plane + 2 * 8 * ordered, "bwd"))
        for path, fn, nbytes, has_mlp in paths:
            if only is not None and path not in only:
                continue
            ms = timed(fn)
            line = {"workload": name, "path": path, "seed": args.seed, "ms": ms, "jets_per_s": b.N / (ms / 1e3),
                    "pairs_per_s": ordered / (ms / 1e3), "alg_gbs": nbytes / (ms / 1e3) / 1e9,
                    "hbm_peak_gbs": hbm_gbs}
            if has_mlp == "bwd":
                line.update({"tflops_alg": unordered * (MLP_FLOP_PER_PAIR + BWD_FLOP_PER_PAIR) / (ms / 1e3) / 1e12,
                             "tflops_exec": tiles * 128 * (MMA_FLOP_PER_ROW + BWD_MMA_FLOP_PER_ROW) / (ms / 1e3) / 1e12,
                             "flop_convention": "alg: bias recompute 17,920 + backward 52,224 per valid unordered pair",
                             "peak_tflops": peak_tf, "peak_source": peak_src})
            elif has_mlp:
                line.update({"tflops_alg": unordered * MLP_FLOP_PER_PAIR / (ms / 1e3) / 1e12,
                             "tflops_exec": tiles * 128 * MMA_FLOP_PER_ROW / (ms / 1e3) / 1e12,
                             "tflops_dense": b.N * b.P * b.P * MLP_FLOP_PER_PAIR / (ms / 1e3) / 1e12,
                             "peak_tflops": peak_tf, "peak_source": peak_src})
            print(json.dumps(line), flush=True)
        if ops.get_device_status():
            raise RuntimeError(f"device status set on {name}")
        if args.no_cpu_baseline:
            continue
        sample = synth.slice_jets(b, 0, min(b.N, 16))
        for threads in (None, 1):
            cb = cpu_baseline(sample, args.cpu_seconds / 4, threads)
            print(json.dumps({"workload": name, "path": "oracle (host)" if threads is None else "oracle (1 thread)",
                              "seed": args.seed, "jets_per_s": cb["value"], "cores": cb["cores"],
                              "sample": cb["sample"]}), flush=True)


def main():
    args = parse()
    world, rank, local = dist_env()
    if args.sweep:
        run_sweep(args)
        return
    if args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
