#!/usr/bin/env python
"""Benchmark of the Q4_0 GEMV decode step on B200.

One step = one synthetic 27B-shaped decode step (M = 1): 64 layers x
(QKV 5120->7168, O 5120->5120, gate+up 5120->34816, down 17408->5120) Q4_0
GEMVs with the renorm chain, run through the C-ABI (q4gemv_run_stack) as one
persistent kernel launch (plus a 16-byte reset of its barrier words).
11.9 GB of weights per step, far larger than L2, so no flush is needed
between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--layers L runs an L-layer step instead (profiling captures only; the
reported workload then says so).

Under torchrun (N > 1) every rank runs an independent replica (same weights,
its own activation stream); there is no data-path collective, only a barrier
and a max-reduction of the timings.  Rank 0 prints one JSON line.

--shard runs the row-sharded step instead (q4gemv_run_stack_sharded): each
rank holds 1/N of every matrix's rows and every GEMV's output reaches every
rank before the next GEMV, so N GPUs share ONE decode step (strong scaling;
the reported bytes are the model's once per step).  --exchange peer (the
default) has each GEMV kernel store its rows into every rank's buffer over
CUDA IPC peer memory and stamp them; --exchange nccl all-gathers them with
NCCL after every GEMV instead.

--pipeline runs the pages' own multi-device split for comparison: contiguous
layer ranges, one per rank, the f16 hidden state sent from GPU to GPU (NCCL
send/recv) and from the last back to the first for the next token.  For one
autoregressive stream the ranges run one after another, so N GPUs hold 1/N
of the weights each but do not shorten the step.
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "achieved HBM GB/s (% of B200 peak) for Q4_0 GEMV; 27B-shaped decode steps/s"
L, HIDDEN, QKV_N, FFN = 64, 5120, 7168, 17408   # L: layers of the step (--layers)
DIMS = [(QKV_N, HIDDEN), (HIDDEN, HIDDEN), (2 * FFN, HIDDEN), (HIDDEN, FFN)]
SHAPE_NAMES = ["qkv_5120x7168", "o_5120x5120", "gate_up_5120x34816", "down_17408x5120"]
STEP_SEED = synth.workload_seed(4)
NOMINAL_HBM_GBS = 8000.0


def gemv_bytes(N: int, K: int) -> int:
    """Algorithmic bytes of one M=1 GEMV: Q4_0 weights (18 B per 32) + x + y."""
    return N * (K // 32) * 18 + 2 * K + 2 * N


STEP_GEMV_BYTES = L * sum(gemv_bytes(N, K) for N, K in DIMS)
STEP_WEIGHT_BYTES = L * sum(N * (K // 32) * 18 for N, K in DIMS)
WORKLOAD = ("27B-shaped decode step, M=1: 64 layers x (QKV 5120->7168, O 5120->5120, "
            "gate+up 5120->34816, down 17408->5120) Q4_0 GEMVs with unit-RMS renorm between "
            "matrices, one persistent kernel launch per step")
WORKLOAD_SHARD = ("27B-shaped decode step, M=1: 64 layers x (QKV 5120->7168, O 5120->5120, "
                  "gate+up 5120->34816, down 17408->5120) Q4_0 GEMVs with unit-RMS renorm between "
                  "matrices, every matrix row-sharded over the GPUs: per GEMV one kernel on each "
                  "GPU's rows, every GPU getting all rows before the next GEMV, replayed as one CUDA "
                  "graph")
WORKLOAD_GATED = ("27B-shaped decode step, M=1: 64 layers x (QKV 5120->7168, O 5120->5120, "
                  "gate+up 5120->34816, down 17408->5120) Q4_0 GEMVs with unit-RMS renorm between "
                  "matrices, each down GEMV fed SiLU(gate) * up of the gate+up output (computed in "
                  "its staging), one persistent kernel launch per step")
WORKLOAD_PIPE = ("27B-shaped decode step, M=1: 64 layers x (QKV 5120->7168, O 5120->5120, "
                 "gate+up 5120->34816, down 17408->5120) Q4_0 GEMVs with unit-RMS renorm between "
                 "matrices, split into contiguous layer ranges over the GPUs: one persistent kernel "
                 "per GPU and token, the f16 hidden state sent to the next GPU after each range and "
                 "back to the first for the next token (one autoregressive stream)")


KERNEL_SOURCES = ["stack.cuh", "gemv_dp2a.cuh", "partition.cuh", "device_common.cuh"]


def kernel_source_hash() -> str:
    """sha256 over the sources of the decode-step kernel (ties the ncu
    traffic figure in profiles/ to the code it was measured on)."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "q4_quantized_decode_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_tensor_peak():
    """Dense f16/bf16 tensor throughput (TFLOP/s, burst) and its source."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


# ------------------------------------------------------------------ multi-rank helpers

def max_over_ranks(dist, values, device=None):
    """Element-wise max of `values` over all ranks (device times are taken as
    the slowest rank's).  Works with gloo (CPU tensors) and nccl (CUDA)."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def step_throughput(world: int, steps: int, ms_max: float, bytes_per_step: int = None):
    """Whole-job GB/s and steps/s of `world` replicas that each ran `steps`
    steps, from the slowest rank's time in ms."""
    b = STEP_GEMV_BYTES if bytes_per_step is None else bytes_per_step
    secs = ms_max * 1e-3
    return world * b * steps / secs / 1e9, world * steps / secs


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "200"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = list(csv.reader(io.StringIO(self.tmp.read())))
        self.tmp.close()
        os.unlink(self.tmp.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for nm, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle timing

def oracle_sample(min_seconds: float, threads: int):
    """Times the fp64 oracle on whole layers of the workload (all four
    matrices) until at least `min_seconds` have elapsed; returns GB/s of
    Q4_0 bytes (+x,y) and a description of the sample."""
    import oracle
    x = synth.normal_f16(STEP_SEED, synth.act_id(0), max(HIDDEN, FFN))
    done_bytes, elapsed, layers = 0, 0.0, 0
    while elapsed < min_seconds and layers < L:
        for t, (N, K) in enumerate(DIMS):
            rows = synth.q4_0_matrix(STEP_SEED, synth.weight_id(4 * layers + t), N, K)
            t0 = time.perf_counter()
            oracle.q4_gemv(rows, K, x[None, :K], threads=threads)
            elapsed += time.perf_counter() - t0
            done_bytes += gemv_bytes(N, K)
        layers += 1
    return done_bytes / elapsed / 1e9, f"{layers} full layer(s) of the step ({done_bytes / 1e6:.0f} MB), fp64 oracle", elapsed


def oracle_layer_step(i: int, threads: int):
    """One reference step: all four GEMVs of layer i mod 64 of the workload,
    whole matrices, fp64 oracle.  Returns (bytes, seconds)."""
    import oracle
    l = i % L
    x = synth.normal_f16(STEP_SEED, synth.act_id(0), max(HIDDEN, FFN))
    done, dt = 0, 0.0
    for t, (N, K) in enumerate(DIMS):
        rows = synth.q4_0_matrix(STEP_SEED, synth.weight_id(4 * l + t), N, K)
        t0 = time.perf_counter()
        oracle.q4_gemv(rows, K, x[None, :K], threads=threads)
        dt += time.perf_counter() - t0
        done += gemv_bytes(N, K)
    return done, dt


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args, rank: int):
    """Reference arm: the fp64 CPU oracle as it stands, on the host cores."""
    if rank != 0:
        return 0
    threads = os.cpu_count() or 1
    # Warm-up steps are short (one GEMV each): they only load the oracle.
    for i in range(min(args.warmup, 1)):
        oracle_layer_step(i, threads)
    tot_b, tot_t = 0, 0.0
    for i in range(args.steps):
        b, dt = oracle_layer_step(i, threads)
        tot_b += b
        tot_t += dt
    gbs = tot_b / tot_t / 1e9
    sample = ("each step: one whole layer of the 27B-shaped step (QKV, O, gate+up and down of "
              "layer i mod 64, 186 MB of Q4_0), fp64 oracle; the step's GB/s")
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD, "parallelism": "replicas"},
        "decode_steps_per_s": gbs * 1e9 / STEP_GEMV_BYTES,
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm

def layer_range(world: int, rank: int, n_layers: int):
    """Contiguous layers [l0, l1) of `rank` in the layer-range pipeline: the
    pages' split of the model over devices, ranks in order, sizes within
    one layer of each other."""
    return rank * n_layers // world, (rank + 1) * n_layers // world


def build_weights(eng, torch, rank: int, l0: int = 0, l1: int = None):
    """Packed weights of layers [l0, l1) of the 64-layer step (all by
    default): generated on the host (seeded), copied to the device,
    repacked by the library's repack kernel."""
    layers = []
    host = {t: np.empty((N, (K // 32) * 18), dtype=np.uint8) for t, (N, K) in enumerate(DIMS)}
    staging = torch.empty(max(h.size for h in host.values()), dtype=torch.uint8, device="cuda")
    t_repack = 0.0
    for l in range(l0, L if l1 is None else l1):
        mats = []
        for t, (N, K) in enumerate(DIMS):
            synth.q4_0_matrix(STEP_SEED, synth.weight_id(4 * l + t), N, K, out=host[t])
            g = staging[: host[t].size]
            g.copy_(torch.from_numpy(host[t].reshape(-1)))
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            mats.append(eng.repack(g, N, K))
            torch.cuda.synchronize()
            t_repack += time.perf_counter() - t0
        layers.append(tuple(mats))
    del staging
    return layers, t_repack


def time_shapes(eng, torch, layers, reps: int = 5):
    """Per-shape M=1 GEMV timing: a CUDA graph of 64 launches, one per
    layer's matrix of that shape (64 distinct matrices, larger than L2)."""
    out = {}
    for t, (N, K) in enumerate(DIMS):
        x = torch.randn(K, device="cuda").half()
        y = torch.empty(N, device="cuda", dtype=torch.float16)
        s = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        eng.run(layers[0][t], x, N, K, out=y)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            for l in range(L):
                eng.run(layers[l][t], x, N, K, out=y)
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (reps * L)
        out[SHAPE_NAMES[t]] = {"us_per_launch": us, "GB/s": gemv_bytes(N, K) / us / 1e3,
                               "rows_per_s": N / us * 1e6}
        del g
    return out


def time_prefill(eng, torch, layers, M: int = 169, reps: int = 3):
    """The M > 16 tensor-core GEMM at a prompt length from the pages (169
    tokens) on the step's 64 distinct gate+up matrices (larger than L2): a
    CUDA graph of 64 launches.  Outside the timed step; context only."""
    N, K = DIMS[2]
    x = torch.from_numpy(synth.activations(STEP_SEED + 169, M, K).view(np.float16)).cuda()
    y = torch.empty(M, N, device="cuda", dtype=torch.float16)
    eng.run(layers[0][2], x, N, K, out=y)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for l in range(L):
            eng.run(layers[l][2], x, N, K, out=y)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    us = e0.elapsed_time(e1) * 1e3 / (reps * L)
    tp, kind = measured_tensor_peak()
    tflops = 2.0 * M * N * K / us / 1e6
    return {"shape": SHAPE_NAMES[2], "M": M, "us_per_launch": us, "tflops": tflops,
            "tensor_peak_tflops": tp, "tensor_peak_kind": kind, "tensor_frac": tflops / tp,
            "tensor_work_frac": 2 * tflops / tp,
            "note": "each weight enters the MMA as two exact binary16 parts: 2x the useful flops"}


def build_weights_sharded(eng, torch, q4, rank: int, world: int):
    """This rank's row slices of the 64-layer step's matrices (the rows
    q4gemv_shard_rows assigns it), repacked on the device; None for a slice
    of no rows."""
    layers = []
    t_repack = 0.0
    for l in range(L):
        mats = []
        for t, (N, K) in enumerate(DIMS):
            st, row0, rows, _ = q4.q4gemv_shard_rows(N, world, rank)
            if st != q4.Q4_OK:
                raise RuntimeError(f"shard_rows status {st}")
            if rows == 0:
                mats.append(None)
                continue
            full = synth.q4_0_matrix(STEP_SEED, synth.weight_id(4 * l + t), N, K)
            g = torch.from_numpy(np.ascontiguousarray(full[row0:row0 + rows]).reshape(-1)).cuda()
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            mats.append(eng.repack(g, rows, K))
            torch.cuda.synchronize()
            t_repack += time.perf_counter() - t0
        layers.append(tuple(mats))
    return layers, t_repack


def time_graph(torch, launch, n: int, reps: int = 5):
    """Mean time (us) of launch(j), j < n, captured as one CUDA graph and
    replayed `reps` times after a warm-up replay."""
    launch(0)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for j in range(n):
            launch(j)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e3 / (reps * n)


def extra_workloads(eng, torch, q4, layers):
    """The benchmark's other configurations, each timed over matrices that
    together exceed 4x L2 (the step's 64 distinct matrices of a shape, or
    rotating copies): the 1024x1024 GEMV (also single-launch latency), M = 4
    and 16 on both FFN shapes, Q8_0 at M = 1, 4, 16, the gated down GEMV, and the
    prefill GEMM at the pages' two prompt lengths."""
    peak, _ = measured_peaks()
    tpeak, tkind = measured_tensor_peak()
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    out = {}

    def hbm(us, nbytes, rows):
        return {"us_per_call": us, "GB/s": nbytes / us / 1e3, "frac_of_hbm_peak": nbytes / us / 1e3 / peak,
                "rows_per_s": rows / us * 1e6}

    # config 0: 1024 x 1024, M = 1
    N0 = K0 = 1024
    seed0 = synth.workload_seed(0)
    W0 = eng.repack(torch.from_numpy(synth.q4_0_matrix(seed0, synth.weight_id(0), N0, K0).reshape(-1)).cuda(), N0, K0)
    R0 = -(-4 * l2 // W0.numel())
    mats0 = [W0] + [W0.clone() for _ in range(R0 - 1)]
    x0 = torch.from_numpy(synth.activations(seed0, 1, K0).view(np.float16)).cuda()
    y0 = torch.empty(N0, dtype=torch.float16, device="cuda")
    us0 = time_graph(torch, lambda j: eng.run(mats0[j], x0, N0, K0, out=y0), R0, reps=3)
    lat = []
    for j in range(30):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        eng.run(mats0[j % R0], x0, N0, K0, out=y0)
        e1.record()
        torch.cuda.synchronize()
        lat.append(e0.elapsed_time(e1) * 1e3)
    out["gemv_1024x1024_m1"] = dict(hbm(us0, gemv_bytes(N0, K0), N0),
                                   single_launch_us_median=statistics.median(lat[5:]),
                                   rotating_copies=R0)
    del mats0

    # config 3: M = 4 and 16 on the FFN shapes (the step's 64 matrices of each)
    small = {}
    for M in (4, 16):
        for t in (2, 3):
            N, K = DIMS[t]
            x = torch.from_numpy(synth.activations(synth.workload_seed(3) + M, M, K).view(np.float16)).cuda()
            y = torch.empty(M, N, dtype=torch.float16, device="cuda")
            us = time_graph(torch, lambda j: eng.run(layers[j][t], x, N, K, out=y), L, reps=3)
            nbytes = N * (K // 32) * 18 + 2 * M * (K + N)
            small[f"M{M}_{SHAPE_NAMES[t]}"] = dict(hbm(us, nbytes, N), tflops=2.0 * M * N * K / us / 1e6)
    out["small_m"] = small

    # Q8_0 at M = 1, 4, 16 on the FFN shapes (rotating copies)
    q8 = {}
    for t in (2, 3):
        N, K = DIMS[t]
        Wq = eng.repack_q8_0(torch.from_numpy(synth.q8_0_matrix(synth.workload_seed(2), synth.weight_id(t), N, K)
                                              .reshape(-1)).cuda(), N, K)
        Rq = max(2, -(-4 * l2 // Wq.numel()))
        mats = [Wq] + [Wq.clone() for _ in range(Rq - 1)]
        for M in (1, 4, 16):
            x = torch.from_numpy(synth.activations(synth.workload_seed(2) + M, M, K).view(np.float16)).cuda()
            y = torch.empty(M, N, dtype=torch.float16, device="cuda")
            us = time_graph(torch, lambda j: eng.run_q8_0(mats[j], x, N, K, out=y), Rq, reps=3)
            q8[(f"M{M}_" if M > 1 else "") + SHAPE_NAMES[t]] = hbm(us, N * (K // 32) * 34 + 2 * M * (K + N), N)
        del mats, Wq
    out["q8_0"] = q8

    # the gated down GEMV: y = W_down (SiLU(gate) * up) from the 2*ffn gate+up output
    N, K = DIMS[3]
    gu = torch.from_numpy(synth.activations(synth.workload_seed(2) + 7, 1, 2 * K).view(np.float16)).cuda().reshape(-1)
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    us = time_graph(torch, lambda j: eng.run_swiglu(layers[j][3], gu, N, K, out=y), L, reps=3)
    out["gated_down_" + SHAPE_NAMES[3]] = hbm(us, N * (K // 32) * 18 + 4 * K + 2 * N, N)

    # prefill GEMM at the pages' prompt lengths (86, 169)
    for M in (86, 169):
        out[f"prefill_gemm_m{M}"] = time_prefill(eng, torch, layers, M=M)
    return out


def run_ours(args, rank: int, world: int, dist):
    import torch
    import q4_quantized_decode_b200 as q4
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    eng = q4.Q4Gemv(local)
    if args.shard and args.exchange == "nccl":
        # One communicator for the row-sharded step: rank 0's NCCL id, sent
        # to the others over the process group.
        uid = [q4.q4gemv_comm_unique_id()[1] if rank == 0 else None]
        if dist is not None and world > 1:
            dist.broadcast_object_list(uid, src=0)
        eng.init_comm(world, rank, uid[0])
    elif args.shard:
        # The peer exchange: every rank's buffer blob, gathered over the
        # process group, then every peer's buffer mapped.
        blob = eng.peer_export(world, rank, HIDDEN, QKV_N, FFN)
        blobs = [None] * world
        if dist is not None and world > 1:
            dist.all_gather_object(blobs, blob)
        else:
            blobs = [blob]
        eng.peer_open(blobs)
    if args.shard:
        layers, t_repack = build_weights_sharded(eng, torch, q4, rank, world)
    elif args.pipeline:
        layers, t_repack = build_weights(eng, torch, rank, *layer_range(world, rank, L))
    else:
        layers, t_repack = build_weights(eng, torch, rank)
    one_step = args.shard or args.pipeline   # the ranks share one step (and its input)
    act = 0 if one_step else rank
    x_host = torch.from_numpy(synth.normal_f16(STEP_SEED, synth.act_id(act), HIDDEN).view(np.float16)).pin_memory()
    out_host = torch.empty(HIDDEN, dtype=torch.float16).pin_memory()
    x_in = x_host.to(dev)
    x_out = torch.empty(HIDDEN, dtype=torch.float16, device=dev)
    stream = torch.cuda.current_stream()

    def pipeline_step(copy_in=None, copy_out=None):
        # One token of one decode stream through the layer-range pipeline:
        # rank r runs its layers on the hidden state from rank r - 1 and
        # sends its output on; the last rank's output is the next token's
        # input on rank 0 (autoregressive, so the stages cannot overlap).
        if world > 1 and rank > 0:
            dist.recv(x_in, src=rank - 1)
        elif copy_in is not None:
            x_in.copy_(copy_in, non_blocking=True)
        eng.run_stack(layers, x_in, HIDDEN, QKV_N, FFN, x_out=x_out)
        if world > 1:
            dist.send(x_out, dst=(rank + 1) % world)
            if rank == 0:
                dist.recv(x_in, src=world - 1)
        else:
            x_in.copy_(x_out)
        if copy_out is not None and rank == 0:
            copy_out.copy_(x_in, non_blocking=True)

    def step():
        if args.pipeline:
            pipeline_step()
        elif args.shard:
            eng.run_stack_sharded(layers, x_in, HIDDEN, QKV_N, FFN, x_out=x_out)
        elif args.gated:
            eng.run_stack_gated(layers, x_in, HIDDEN, QKV_N, FFN, x_out=x_out)
        else:
            eng.run_stack(layers, x_in, HIDDEN, QKV_N, FFN, x_out=x_out)

    def step_e2e():
        if args.pipeline:
            # the token's input from pinned host memory on rank 0, the next
            # input back to it
            pipeline_step(copy_in=x_host if rank == 0 else None, copy_out=out_host)
        elif args.shard:
            # the sharded call takes device vectors: the copies from and to
            # pinned host memory are made around it, every step
            x_in.copy_(x_host, non_blocking=True)
            eng.run_stack_sharded(layers, x_in, HIDDEN, QKV_N, FFN, x_out=x_out)
            out_host.copy_(x_out, non_blocking=True)
        elif args.gated:
            eng.run_stack_gated(layers, x_host, HIDDEN, QKV_N, FFN, x_out=out_host)
        else:
            eng.run_stack(layers, x_host, HIDDEN, QKV_N, FFN, x_out=out_host)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = eng.sync_status()
    if st != q4.Q4_OK:
        raise RuntimeError(f"device status {st}")

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(local).uuid)
        if uuid and not uuid.startswith("GPU-"):
            uuid = "GPU-" + uuid
    except Exception:
        uuid = None
    sampler = ClockSampler(uuid)

    def barrier():
        if dist is not None:
            dist.barrier()

    # ---- device-timed region: K steps, inputs resident in HBM
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier()
    ms = e0.elapsed_time(e1)

    # ---- end-to-end: the C-ABI call with HOST vectors (pinned), which copies
    # x to the device and the result back inside the call, every step
    step_e2e()   # descriptors (or the graph) for these pointers
    barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        step_e2e()
    f1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = f0.elapsed_time(f1)

    extras = rank == 0 and not args.no_per_shape and not one_step
    per_shape = time_shapes(eng, torch, layers) if extras else None
    others = extra_workloads(eng, torch, q4, layers) if extras else None
    if eng.sync_status() != q4.Q4_OK:
        raise RuntimeError("device status after timing")

    ms, ms_e2e = max_over_ranks(dist, [ms, ms_e2e], device=dev)
    # Every rank's steps are complete (synchronised before the reduction):
    # no rank stores into another's exchange buffer any more, and the step
    # graphs (which may hold NCCL calls) go before the process group.
    torch.cuda.synchronize()
    barrier()
    eng.close()
    if rank != 0:
        return 0

    ms_step = ms / args.steps
    # Replicas: every rank runs a whole step.  Sharded or pipelined: the ranks
    # share one.
    copies = 1 if one_step else world
    value, steps_per_s = step_throughput(copies, args.steps, ms)
    e2e_value, e2e_steps_per_s = step_throughput(copies, args.steps, ms_e2e)
    peak, peak_kind = measured_peaks()
    per_rank_gbs = STEP_GEMV_BYTES / (ms_step * 1e-3) / 1e9 / (world if one_step else 1)
    roofline = {
        "bound": "hbm", "achieved": per_rank_gbs, "peak": peak, "unit": "GB/s",
        "frac": per_rank_gbs / peak, "traffic": None,
        "kernel": ("q4::gemv_dp2a_kernel<1,16,3,6> (per rank: one launch per GEMV on its rows, "
                   "4L per step in one graph, plus the step-count update and the final renorm; "
                   "duration = step time; bytes = this rank's share of the step)"
                   if args.shard else
                   "q4::stack_kernel<16,3,6> (per rank: one persistent launch per token over its "
                   "layer range; duration = step time, all ranks in turn; bytes = this rank's share)"
                   if args.pipeline else
                   "q4::stack_kernel<16,3,6,true> (gated: one persistent launch per step)"
                   if args.gated else
                   "q4::stack_kernel<16,3,6> (one persistent launch per step, all 4L GEMVs and "
                   "the final renorm; duration = step time, which also holds the 16-byte "
                   "barrier-word reset before each launch)"),
        "peak_source": f"{peak_kind} hbm_gbs (copy) in MEASURED_PEAKS.json",
        "frac_of_nominal_8TBps": per_rank_gbs / NOMINAL_HBM_GBS,
    }
    traffic = os.path.join(ROOT, "profiles", "traffic_per_launch.json")
    if os.path.exists(traffic) and L == 64 and not one_step and not args.gated:
        with open(traffic) as f:
            tr = json.load(f)
        # Counters taken on another version of the kernel's source do not count.
        if tr.get("source_sha256") == kernel_source_hash():
            roofline["traffic"] = tr.get("bytes_per_launch")
            roofline["traffic_note"] = tr.get("note")
        else:
            roofline["traffic_note"] = "kernel source changed since the ncu capture: traffic unknown"
    cpu = None
    if not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        cgbs, sample, secs = oracle_sample(args.cpu_seconds, threads)
        c1, sample1, secs1 = oracle_sample(min(3.0, args.cpu_seconds), 1)
        cpu = {"value": cgbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"{sample}, {secs:.1f} s on {threads} host threads",
               "single_thread": {"value": c1, "unit": "GB/s", "sample": f"{sample1}, {secs1:.1f} s"},
               "cpu_model": cpu_model()}
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if one_step else "weak", "vs_baseline": None,
        "dtype": "q4_0 x f16 (s32 block sums, f32 accumulate)", "data": "synthetic",
        "config": {"workload": WORKLOAD_SHARD if args.shard else WORKLOAD_PIPE if args.pipeline else
                   WORKLOAD_GATED if args.gated else WORKLOAD,
                   "bytes_per_step": STEP_GEMV_BYTES,
                   "weight_bytes_per_step": STEP_WEIGHT_BYTES,
                   "l2": "inputs larger than L2 (11.9 GB of weights per step)",
                   "parallelism": ((f"row-sharded x{world} (NCCL all-gather after every GEMV)"
                                    if args.exchange == "nccl" else
                                    f"row-sharded x{world} (GEMV kernels store their rows into every "
                                    "rank's buffer over peer memory)")
                                   if args.shard else
                                   f"layer-range pipeline x{world} (hidden state sent between GPUs)"
                                   if args.pipeline else f"replicas x{world}"), "seed": STEP_SEED},
        "decode_steps_per_s": steps_per_s,
        "pct_of_8TBps_nominal": 100.0 * per_rank_gbs / NOMINAL_HBM_GBS,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": 2 * HIDDEN,
                "d2h_bytes_per_step": 2 * HIDDEN,
                "steps_per_s": e2e_steps_per_s},
        # one stack_kernel per step (and one 16-byte memset); sharded over NCCL: per
        # GEMV one kernel and one all-gather, and the final renorm; over peer memory:
        # per GEMV one kernel, the step-count update and the final unpack + renorm;
        # pipelined: one stack_kernel per GPU (this rank's count)
        "gpu_launches": args.steps * (((8 * L + 1) if args.exchange == "nccl" else (4 * L + 2))
                                      if args.shard else 1),
        "clocks": clocks,
        "repack_s_per_step_weights": t_repack,
        "per_shape_m1": per_shape,
        "other_configs": others,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_case(args):
    """Standalone GEMV timing on one shape (single-shape workloads and profiling): R
    copies of one packed matrix (R * size > 4 x L2 unless --rotate is given)
    launched in rotation inside a CUDA graph; prints one JSON line."""
    import torch
    import q4_quantized_decode_b200 as q4
    N, K = (int(v) for v in args.shape.lower().split("x"))
    M = args.M
    q8 = args.format == "q8_0"
    gated = args.act == "swiglu"
    if gated and (q8 or M != 1):
        raise SystemExit("--act swiglu: Q4_0 and M = 1 only")
    eng = q4.Q4Gemv(0)
    seed = synth.workload_seed(args.workload_seed)
    if q8:
        gguf = synth.q8_0_matrix(seed, synth.weight_id(0), N, K)
        W0 = eng.repack_q8_0(torch.from_numpy(gguf.reshape(-1)).cuda(), N, K)
        run = eng.run_q8_0
    else:
        gguf = synth.q4_0_matrix(seed, synth.weight_id(0), N, K)
        W0 = eng.repack(torch.from_numpy(gguf.reshape(-1)).cuda(), N, K)
        run = eng.run
        if gated:      # the down GEMV fed by a [gate | up] vector of 2K entries
            def run(W, x, N, K, out=None):
                return eng.run_swiglu(W, x.reshape(-1), N, K, out=out)
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    R = args.rotate or max(2, -(-4 * l2 // W0.numel()))
    mats = [W0] + [W0.clone() for _ in range(R - 1)]
    x = torch.from_numpy(synth.activations(seed, M, 2 * K if gated else K).view(np.float16)).cuda()
    y = torch.empty(M, N, dtype=torch.float16, device="cuda")
    run(mats[0], x, N, K, out=y)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for W in mats:
            run(W, x, N, K, out=y)
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    if eng.sync_status() != q4.Q4_OK:
        raise RuntimeError("device status")
    us = e0.elapsed_time(e1) * 1e3 / (args.steps * R)
    nbytes = N * (K // 32) * (34 if q8 else 18) + 2 * M * ((2 * K if gated else K) + N)
    peak, kind = measured_peaks()
    line = {"case": f"gemv {args.format}{' swiglu' if gated else ''} M={M} {N}x{K}", "N": N, "K": K, "M": M, "rotate": R,
            "us_per_launch": us, "GB/s": nbytes / us / 1e3,
            "frac_of_peak": nbytes / us / 1e3 / peak, "peak": peak, "peak_kind": kind,
            "rows_per_s": N / us * 1e6, "tflops": 2 * M * N * K / us / 1e6,
            "launches": args.steps * R}
    if M > q4.MAX_M_GEMV:
        # tensor-core GEMM: f16 products, bound by the tensor pipe (f16 = bf16 rate)
        tp, tkind = measured_tensor_peak()
        line.update({"tensor_peak_tflops": tp, "tensor_peak_kind": tkind,
                     "tensor_frac": line["tflops"] / tp})
    print(json.dumps(line), flush=True)
    eng.close()
    return 0


def set_layers(n: int):
    """Switch the step to n layers (profiling captures of a smaller case)."""
    global L, STEP_GEMV_BYTES, STEP_WEIGHT_BYTES, WORKLOAD
    L = n
    STEP_GEMV_BYTES = L * sum(gemv_bytes(N, K) for N, K in DIMS)
    STEP_WEIGHT_BYTES = L * sum(N * (K // 32) * 18 for N, K in DIMS)
    if n != 64:
        WORKLOAD = WORKLOAD.replace("64 layers", f"{n} layers (profiling case, not the benchmark)")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-shape", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--case", choices=["step", "gemv"], default="step",
                    help="step: the decode step (default); gemv: one shape, see --shape/--M")
    ap.add_argument("--shape", default="34816x5120", help="NxK for --case gemv")
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--rotate", type=int, default=0, help="matrix copies in rotation (0: > 4x L2)")
    ap.add_argument("--workload-seed", type=int, default=2)
    ap.add_argument("--format", choices=["q4_0", "q8_0"], default="q4_0", help="weights of --case gemv")
    ap.add_argument("--act", choices=["none", "swiglu"], default="none",
                    help="--case gemv: feed the GEMV SiLU(gate) * up of a 2K input (M = 1)")
    ap.add_argument("--layers", type=int, default=64, help="layers of the step (profiling only)")
    ap.add_argument("--shard", action="store_true",
                    help="row-shard every matrix over the ranks (one step shared by all GPUs)")
    ap.add_argument("--exchange", choices=["peer", "nccl"], default="peer",
                    help="--shard: how each GEMV's rows reach every rank")
    ap.add_argument("--gated", action="store_true",
                    help="the step with each down GEMV fed SiLU(gate) * up (q4gemv_run_stack_gated)")
    ap.add_argument("--pipeline", action="store_true",
                    help="split the layers into contiguous ranges over the ranks, the hidden state "
                         "passed from GPU to GPU (the pages' multi-device design; one stream)")
    args = ap.parse_args()
    if args.shard and args.pipeline:
        ap.error("--shard and --pipeline are two ways to split one step: pick one")
    if args.gated and (args.shard or args.pipeline):
        ap.error("--gated runs on one GPU per step (replicas)")
    if args.layers != 64:
        set_layers(args.layers)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    if args.case == "gemv":
        return run_case(args)
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist_mod
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = dist_mod
    try:
        return run_ours(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
