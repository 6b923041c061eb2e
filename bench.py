#!/usr/bin/env python
"""Benchmark of one ReLU linear-attention layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl la|reference]
                    [--workload NAME] [--op layer|reduce|apply|backward|causal|tconv|qkv]

A step is one pass of the layer's hot path over one batch of synthetic input:
the state reduce (S = sum phi(K)^T V, z = sum ReLU(K)) and the apply
(O = phi(Q) S / (ReLU(Q).z + eps)) of the default workload (the SANA-Video
480p layer, the largest single-layer call), or a whole block-causal video
(reset, 12 blocks x 5 calls) for the LongSANA workload. With --op reduce or
--op apply a step is one of the two halves alone (la_state_reduce, la_apply),
each its own kernel launch.
With --op backward a step is the layer's backward instead (dQ, dK, dV and the
state gradients from Q, K, V, the state and dO); with --op causal it is
token-causal attention over the workload's tokens (query n sees keys 0..n).
Both cover the non-causal workloads' shapes. With --op tconv a step is the
Mix-FFN's temporal depth-wise convolution over the video workload's latent
grid at the FFN width: a whole clip (sanavideo_480p), or one block reading and
updating the conv cache (longsana_block_causal).
Rank 0 prints one JSON line. Multi-GPU runs are weak-scaled: every rank runs
its own copy of the workload (heads and batches are independent), with no
collective on the data path; the time is the max over ranks.

--impl reference times the float64 CPU oracle (the only other program on the
path) on this host's cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "linear-attn tokens/s per layer at 1 B200; achieved HBM GB/s vs peak"
METRIC_BWD = "linear-attn backward tokens/s per layer at 1 B200; achieved HBM GB/s vs peak"
METRIC_CAUSAL = ("token-causal linear-attn tokens/s per layer at 1 B200; "
                 "achieved HBM GB/s vs peak")
METRIC_TCONV = "temporal-conv tokens/s per layer at 1 B200; achieved HBM GB/s vs peak"
METRIC_QKV = ("QKV projection + state reduce tokens/s per layer at 1 B200; "
              "achieved TFLOP/s vs bf16 peak")
METRIC_REDUCE = "linear-attn state-reduce tokens/s per layer at 1 B200; achieved HBM GB/s vs peak"
METRIC_APPLY = "linear-attn apply tokens/s per layer at 1 B200; achieved HBM GB/s vs peak"
METRICS = {"layer": METRIC, "backward": METRIC_BWD, "causal": METRIC_CAUSAL,
           "tconv": METRIC_TCONV, "qkv": METRIC_QKV, "reduce": METRIC_REDUCE,
           "apply": METRIC_APPLY}
# Channels of the temporal convolution: the FFN width of Sana-1.6B, which
# SANA-Video starts from (width 2240, FFN 5600).
FFN_WIDTH = 5600
OP_CONFIG = {"layer": {}, "backward": {"op": "backward (dQ, dK, dV, dS, dz)"},
             "reduce": {"op": "state reduce alone (S = sum phi(K)^T V, z = sum ReLU(K))"},
             "apply": {"op": "apply alone (O = phi(Q) S / (ReLU(Q).z + eps))"},
             "causal": {"op": "token-causal (query n sees keys 0..n), no carry"},
             "tconv": {"op": "temporal depth-wise conv 3x1x1 + shortcut", "channels": FFN_WIDTH},
             "qkv": {"op": "QKV projection (bf16 GEMM, bias) fused with the state reduce; "
                           "Q out, K and V never leave the chip"}}
DEFAULT_WORKLOAD = "sanavideo_480p"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
D = 32


# ---------------------------------------------------------------------------
# helpers


def env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def max_over_ranks(x: float, device=None) -> float:
    """The largest value of x over all ranks (x itself on a single process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaled_value(tokens_per_step: int, steps: int, world: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank processes its own copy of the workload,
    and the job takes as long as its slowest rank."""
    return world * tokens_per_step * steps / (ms_max / 1e3)


def rank_seed(rank: int) -> int:
    """Base input seed of a rank: each replica draws its own batch."""
    return 1000 * int(rank)


def layer_bytes(w, io_bytes=2):
    """Algorithmic HBM bytes of one layer: read Q, K, V, write O, write the state."""
    th = w.B * w.N * w.H
    state = w.B * w.H * (D * D + D) * 4
    # backward: read Q, K, V, dO and (S, z); write dQ, dK, dV and (dS, dz).
    # causal: the minimum, Q, K, V read once and O written once.
    # reduce: read K, V, write the state; apply: read Q and the state, write O.
    return {"attention_layer": 4 * th * D * io_bytes + state,
            "state_reduce": 2 * th * D * io_bytes + state,
            "apply": 2 * th * D * io_bytes + state,
            "attention_backward": 7 * th * D * io_bytes + 2 * state,
            "causal_attention": 4 * th * D * io_bytes}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, burst copy)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (no MEASURED_PEAKS.json)"


# Sources of each timed call's kernels: the kernel files and the device
# headers they include. A committed DRAM-traffic figure holds while these
# files are unchanged.
_DEVICE_HEADERS = ("la_common.cuh", "la_sm100.cuh", "la_tc_common.cuh")
KERNEL_SOURCES = {
    "attention_layer": ("la_tc.cu",) + _DEVICE_HEADERS,
    "la_block_causal_step": ("la_tc.cu",) + _DEVICE_HEADERS,
    "state_reduce": ("la_tc.cu",) + _DEVICE_HEADERS,
    "apply": ("la_tc.cu",) + _DEVICE_HEADERS,
    "attention_backward": ("la_backward_tc.cu",) + _DEVICE_HEADERS,
    "causal_attention": ("la_tc.cu", "la_causal_chunk.cu") + _DEVICE_HEADERS,
    "temporal_conv": ("la_conv.cu", "la_common.cuh", "la_sm100.cuh"),
    "qkv_state": ("la_qkv_tc.cu",) + _DEVICE_HEADERS,
}


def tensor_peaks():
    """Measured dense bf16 GEMM throughput (TFLOP/s): burst and sustained."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return ({"burst": float(m["bf16_tflops"]), "sustained": float(m["bf16_tflops_sustained"])},
                "measured (MEASURED_PEAKS.json bf16_tflops_sustained; the call is timed inside "
                "a seconds-long loop of back-to-back calls)")
    except Exception:
        return {"burst": 1590.0, "sustained": 1400.0}, "fallback 1.59 / 1.4 PFLOP/s"


def sources_sha(kernel):
    h = hashlib.sha256()
    for name in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(ROOT, "linear_attention_diffusion_b200", "csrc", name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload, kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None
    when there is none or the kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"traffic_{workload}.txt")
    if not os.path.exists(path):
        return None
    if kernel not in KERNEL_SOURCES:
        return None
    sha = sources_sha(kernel)
    for line in open(path):
        if line.startswith("#") or "=" not in line:
            continue
        kv = dict(tok.split("=", 1) for tok in line.split())
        if kv.get("kernel") == kernel and kv.get("sources_sha") == sha:
            return int(float(kv["dram_bytes_per_launch"]))
    return None


class ClockSampler:
    """nvidia-smi samples (every 100 ms) of the GPU this process uses."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = (uuid or "").lower()
        self.samples = []
        self.proc = None
        self.error = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception as e:  # no nvidia-smi
            self.error = str(e)

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            if self.uuid and self.uuid not in parts[0].lower():
                continue
            try:
                self.samples.append((time.time(), float(parts[1]), float(parts[2]),
                                     float(parts[3]) if parts[3] not in ("[N/A]", "") else None,
                                     parts[5:9]))
            except ValueError:
                pass

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "note": f"no nvidia-smi samples ({self.error or 'none parsed'})"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        note = "samples taken during the timed region"
        if not inside:
            mid = 0.5 * (t0 + t1)
            inside = sorted(self.samples, key=lambda s: abs(s[0] - mid))[:3]
            note = "timed region shorter than the 100 ms sampling period: nearest samples"
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in inside for i, v in enumerate(s[4])
                          if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(s[1] for s in inside),
                "sm_max_mhz": max(s[2] for s in inside), "reasons": reasons,
                "samples": len(inside), "note": note}


def cpu_cores_used():
    try:
        from threadpoolctl import threadpool_info
        n = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(w, seconds, max_reps=None, op="layer"):
    """Time the float64 oracle on a bounded sample of workload `w`.

    One call covers a subset of heads sized so that it takes at most about
    `seconds`/3; calls repeat until `seconds` have passed. Returns
    (tokens per second for the whole workload, description, cores)."""
    import numpy as np
    import oracle as orc

    dOa = wl.make_tensor((w.B, w.N, w.H, w.D), 3) if op == "backward" else None
    states = {}  # apply: the state of the sampled heads, reduced once, untimed

    def run(h_sub, Q, K, V, th):
        if op == "backward":
            orc.backward(Q, K, V, dOa[:, :, :h_sub], w.eps, th)
        elif op == "reduce":
            orc.state_reduce(K, V, th)
        elif op == "apply":
            orc.apply(Q, *states[h_sub], w.eps, th)
        elif op == "causal":
            orc.causal_attention(Q, K, V, w.eps, th)
        elif w.block_causal:
            Sc = np.zeros((w.B, h_sub, D, D))
            zc = np.zeros((w.B, h_sub, D))
            orc.block_causal_step(Q, K, V, Sc, zc, 1, w.eps, th)
        else:
            orc.attention(Q, K, V, w.eps, th)

    th = orc.rope_angles(w.T, w.Hh, w.W, 0, w.rope_base) if w.rope else None
    Qa, Ka, Va = wl.make_qkv(w, 0)
    h_sub = min(w.H, 2)
    if op == "apply":
        states[h_sub] = orc.state_reduce(Ka[:, :, :h_sub], Va[:, :, :h_sub], th)
    t = time.perf_counter()
    run(h_sub, Qa[:, :, :h_sub], Ka[:, :, :h_sub], Va[:, :, :h_sub], th)
    per_head = (time.perf_counter() - t) / h_sub
    h_sub = max(1, min(w.H, int((seconds / 3) / max(per_head, 1e-9))))
    Q, K, V = (x[:, :, :h_sub].contiguous() for x in (Qa, Ka, Va))
    if op == "apply":
        states[h_sub] = orc.state_reduce(K, V, th)
    reps, t0 = 0, time.perf_counter()
    while True:
        run(h_sub, Q, K, V, th)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds or (max_reps and reps >= max_reps):
            break
    per_call = el / reps
    full_call = per_call * w.H / h_sub
    if w.block_causal:
        calls = w.M * (w.steps + 1)
        tokens_per_s = w.M * w.N * w.B / (full_call * calls)
        desc = (f"oracle block_causal_step on {h_sub} of {w.H} heads of one {w.N}-token block, "
                f"{reps} calls in {el:.1f} s, scaled to {w.H} heads x {calls} calls per video")
    else:
        tokens_per_s = w.B * w.N / full_call
        what = {"backward": "backward", "causal": "causal_attention", "reduce": "state_reduce",
                "apply": "apply"}.get(op, "attention")
        desc = (f"oracle {what} on {h_sub} of {w.H} heads (B={w.B}, N={w.N}), {reps} calls "
                f"in {el:.1f} s, scaled to {w.H} heads")
    return tokens_per_s, desc, cpu_cores_used(), per_call, h_sub


# ---------------------------------------------------------------------------
# the CUDA path


def time_steps(args, step, stream, dev, world, n_sets, one_step_graphs, check_status):
    """Warm-up, then exactly args.steps steps timed on the device.

    ``step(i, evs)`` enqueues step i on ``stream`` (recording evs[0] and
    evs[1] around its launches when given). Steps are captured in CUDA graphs
    of ``chunk`` steps (one step per graph when ``one_step_graphs``) and
    replayed back to back between two events; a second graph with events
    around every step gives the per-step device durations. Returns
    (ms over all ranks' max, per-step us list, chunk, wall t0, wall t1).
    """
    import torch
    # warm-up, eager
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    torch.cuda.synchronize(dev)
    check_status()

    # chunk graph: C steps, with an event after every launch
    n_ev = 2
    chunk = n_sets * max(1, 100 // n_sets) if not one_step_graphs else 1
    chunk = min(chunk, args.steps) if args.steps > 0 else chunk
    chunk = max(1, chunk - chunk % n_sets) if chunk >= n_sets else chunk

    def capture(nsteps, with_events):
        evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(n_ev)]
               for _ in range(nsteps)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(nsteps):
                step(i, evs[i] if with_events else None)
        check_status()
        return g, evs

    g_chunk, _ = capture(chunk, with_events=False)
    full, rem = divmod(args.steps, chunk)
    g_rem = capture(rem, with_events=False)[0] if rem else None
    # a second graph with an event after every launch, for per-launch durations
    g_ev, ev_chunk = capture(chunk, with_events=True)

    # soak: the same graph, untimed, for about a second, so that clocks settle
    torch.cuda.synchronize(dev)
    t_soak = time.time()
    with torch.cuda.stream(stream):
        while time.time() - t_soak < args.soak:
            g_chunk.replay()
            torch.cuda.synchronize(dev)

    # timed region 1: exactly K steps, graph replays back to back (no events
    # between launches, so consecutive kernels overlap through programmatic
    # dependent launch exactly as they do for a user's stream)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(full):
            g_chunk.replay()
        if g_rem is not None:
            g_rem.replay()
        end.record(stream)
    torch.cuda.synchronize(dev)
    t1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    ms = start.elapsed_time(end)

    # timed region 2: the event graph, for the duration of each launch
    with torch.cuda.stream(stream):
        for _ in range(3):
            g_ev.replay()
    torch.cuda.synchronize(dev)
    seg = [[e[j].elapsed_time(e[j + 1]) for e in ev_chunk] for j in range(n_ev - 1)]
    seg_us = [1000.0 * statistics.mean(x) for x in seg]

    del g_chunk, g_rem, g_ev  # release the graphs before any collective teardown
    return max_over_ranks(ms, dev), seg_us, chunk, t0, t1


def run_la(args, w, rank, world, local_rank):
    import torch
    import linear_attention_diffusion_b200 as la

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    props = torch.cuda.get_device_properties(dev)
    uuid = str(getattr(props, "uuid", "") or "")
    sampler = ClockSampler(uuid)
    stream = torch.cuda.Stream(dev)
    lib = la._lib
    sp = stream.cuda_stream

    bwd = args.op == "backward"
    per_set = (4 if bwd else 3) * w.B * w.N * w.H * D * 2
    n_sets = max(1, min(8, math.ceil(2 * L2_BYTES / per_set)))
    if args.op in ("reduce", "apply"):
        # a step touches two of the set's tensors: rotate over at least two sets
        n_sets = max(2, min(8, math.ceil(2 * L2_BYTES / (per_set * 2 // 3))))
    if w.block_causal:
        n_sets = 5  # one set per call of a block; each set is far above L2
    sets = []
    for i in range(n_sets):
        if w.block_causal:
            q, k, v = wl.make_qkv(w, rank_seed(rank), block=0, step=i)
        else:
            q, k, v = wl.make_qkv(w, rank_seed(rank) + 10 * i)
        q, k, v = (x.to(dev) for x in (q, k, v))
        if bwd:
            # the set's dO and its forward state (computed once, untimed)
            g = wl.make_tensor(tuple(q.shape), rank_seed(rank) + 10 * i + 3).to(dev)
            _, Si, zi = la.attention(q, k, v, eps=w.eps,
                                     rope_grid=(w.T, w.Hh, w.W) if w.rope else None)
            sets.append((q, k, v, g, Si, zi))
        else:
            sets.append((q, k, v, torch.empty_like(q)))
    S = torch.zeros((w.B, w.H, D, D), device=dev)
    z = torch.zeros((w.B, w.H, D), device=dev)
    if bwd:
        grads = [torch.empty_like(sets[0][0]) for _ in range(3)] + [torch.empty_like(S),
                                                                    torch.empty_like(z)]
        grad_p = [t.data_ptr() for t in grads]

    def shape_at(t_offset=0):
        return la.make_shape(w.B, w.N, w.H, D, "bf16", w.rope, w.T, w.Hh, w.W, t_offset,
                             w.rope_base, w.eps)

    shape0 = shape_at(0)
    ws = la.workspace(shape0, dev, causal=args.op == "causal")
    ws_p, ws_n = ws.data_ptr(), ws.numel()
    S_p, z_p = S.data_ptr(), z.data_ptr()
    ptrs = [tuple(t.data_ptr() for t in s) for s in sets]
    keep = [shape_at(m * w.T) for m in range(max(1, w.M))]
    shapes = [ctypes.byref(s) for s in keep]
    status = []

    if args.op in ("reduce", "apply"):
        launches_per_step = 1
        if args.op == "apply":
            # the state the apply reads: the reduce of the first set (untimed)
            q0, k0, v0, _ = ptrs[0]
            status.append(lib.la_state_reduce(shapes[0], k0, v0, S_p, z_p, ws_p, ws_n, sp))
            torch.cuda.synchronize(dev)

        def step(i, evs=None):
            q, k, v, o = ptrs[i % n_sets]
            if evs is not None:
                evs[0].record(stream)
            if args.op == "reduce":
                status.append(lib.la_state_reduce(shapes[0], k, v, S_p, z_p, ws_p, ws_n, sp))
            else:
                status.append(lib.la_apply(shapes[0], q, S_p, z_p, o, sp))
            if evs is not None:
                evs[1].record(stream)
        kernel_names = ("state_reduce" if args.op == "reduce" else "apply",)
    elif args.op == "causal":
        # bf16: every chunk's state (+ the chunks' key sums with RoPE), their
        # prefix, then the chunks
        launches_per_step = 4 if w.rope else 3

        def step(i, evs=None):
            q, k, v, o = ptrs[i % n_sets]
            if evs is not None:
                evs[0].record(stream)
            status.append(lib.la_causal_attention(shapes[0], q, k, v, None, None, o, 0, ws_p,
                                                  ws_n, sp))
            if evs is not None:
                evs[1].record(stream)
        kernel_names = ("causal_attention",)
    elif bwd:
        launches_per_step = 2  # query side, then key side

        def step(i, evs=None):
            q, k, v, g, Si, zi = ptrs[i % n_sets]
            if evs is not None:
                evs[0].record(stream)
            status.append(lib.la_attention_backward(shapes[0], q, k, v, Si, zi, g, *grad_p,
                                                    ws_p, ws_n, sp))
            if evs is not None:
                evs[1].record(stream)
        kernel_names = ("attention_backward",)
    elif w.block_causal:
        calls_per_step = w.M * (w.steps + 1)
        # one or two kernels per call (see la_attention_launches); reset is memsets
        launches_per_step = la.la_attention_launches(keep[0]) * calls_per_step

        def step(i, evs=None):
            status.append(lib.la_state_reset(S_p, z_p, w.B, w.H, D, sp))
            c = 0
            for m in range(w.M):
                for s in range(w.steps + 1):
                    q, k, v, o = ptrs[s % n_sets]
                    upd = 1 if s == w.steps else 0
                    if evs is not None and upd == 0 and m == w.M - 1 and s == 0:
                        evs[0].record(stream)
                    status.append(lib.la_block_causal_step(shapes[m], q, k, v, S_p, z_p, o, upd,
                                                           ws_p, ws_n, sp))
                    if evs is not None and upd == 0 and m == w.M - 1 and s == 0:
                        evs[1].record(stream)
                    c += 1
        kernel_names = ("la_block_causal_step",)
    else:
        launches_per_step = la.la_attention_launches(keep[0])

        def step(i, evs=None):
            q, k, v, o = ptrs[i % n_sets]
            if evs is not None:
                evs[0].record(stream)
            status.append(lib.la_attention(shapes[0], q, k, v, S_p, z_p, o, ws_p, ws_n, sp))
            if evs is not None:
                evs[1].record(stream)
        kernel_names = ("attention_layer",)

    def check_status():
        bad = [s for s in status if s != 0]
        status.clear()
        if bad:
            raise RuntimeError(f"library call failed: {la.la_status_string(bad[0])} "
                               f"{la.la_last_error()}")

    ms_max, seg_us, chunk, t0, t1 = time_steps(args, step, stream, dev, world, n_sets,
                                               w.block_causal, check_status)

    # end-to-end through the public API with host buffers
    if args.e2e_steps <= 0:
        e2e = None
    elif bwd:
        e2e = run_e2e_backward(args, w, dev, stream, la, rank)
    elif args.op == "causal":
        e2e = run_e2e(args, w, dev, stream, la, rank, causal=True)
    elif args.op in ("reduce", "apply"):
        e2e = run_e2e_half(args, w, dev, stream, la, rank, args.op)
    else:
        e2e = run_e2e(args, w, dev, stream, la, rank)
    clocks = sampler.summary(t0, t1)
    sampler.stop()
    return {"ms": ms_max, "seg_us": seg_us, "kernel_names": kernel_names, "e2e": e2e,
            "clocks": clocks, "launches_per_step": launches_per_step, "n_sets": n_sets,
            "chunk": chunk, "per_set_bytes": per_set}


def run_tconv(args, w, rank, world, local_rank):
    """The temporal convolution over the video workload's latent grid."""
    import torch
    import linear_attention_diffusion_b200 as la

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(str(getattr(props, "uuid", "") or ""))
    stream = torch.cuda.Stream(dev)
    lib = la._lib
    sp = stream.cuda_stream
    C = FFN_WIDTH
    cshape = la.make_conv_shape(w.B, w.T, w.Hh, w.W, C)
    x = wl.make_tensor((w.B, w.T, w.Hh, w.W, C), rank_seed(rank) + 20).to(dev)
    y = torch.empty_like(x)
    wt = wl.make_tensor((C, 3), 21, torch.float32).to(dev)
    bias = wl.make_tensor((C,), 22, torch.float32).to(dev)
    # block-causal: the block reads the cache and leaves its last frame there
    cache = wl.make_tensor((w.B, w.Hh, w.W, C), 23).to(dev) if w.block_causal else None
    cache_p = None if cache is None else cache.data_ptr()
    per_set = x.numel() * x.element_size()
    status = []

    def step(i, evs=None):
        if evs is not None:
            evs[0].record(stream)
        status.append(lib.la_temporal_conv(ctypes.byref(cshape), x.data_ptr(), wt.data_ptr(),
                                           bias.data_ptr(), cache_p, cache_p, y.data_ptr(), sp))
        if evs is not None:
            evs[1].record(stream)

    def check_status():
        bad = [v for v in status if v != 0]
        status.clear()
        if bad:
            raise RuntimeError(f"library call failed: {la.la_status_string(bad[0])} "
                               f"{la.la_last_error()}")

    ms_max, seg_us, chunk, t0, t1 = time_steps(args, step, stream, dev, world, 1, False,
                                               check_status)
    e2e = None
    if args.e2e_steps > 0:
        steps = max(1, min(args.steps, args.e2e_steps))
        hx = x.cpu().pin_memory()
        hy = torch.empty_like(hx).pin_memory()

        def call(p, ins, outs, st):
            la.la_temporal_conv(cshape, ins[0], wt, bias, cache, cache, outs[0], st)

        ms = e2e_pipelined(dev, stream, [hx], [hy], call, 1, steps)
        e2e = {"ms_per_step": ms, "tokens_per_step": w.B * w.N, "steps": steps,
               "h2d_bytes_per_step": per_set, "d2h_bytes_per_step": per_set,
               "copies": "pipelined: copy-in, calls and copy-out on three streams, two buffer sets"}
    clocks = sampler.summary(t0, t1)
    sampler.stop()
    return {"ms": ms_max, "seg_us": seg_us, "kernel_names": ("temporal_conv",), "e2e": e2e,
            "clocks": clocks, "launches_per_step": 1, "n_sets": 1, "chunk": chunk,
            "per_set_bytes": per_set, "cache_bytes": 0 if cache is None else 2 * per_set // w.T}


def run_qkv(args, w, rank, world, local_rank):
    """The QKV projection fused with the state reduce, at the model's hidden
    width, with the unfused path (three cuBLAS projections through torch, then
    la_state_reduce) timed beside it for comparison."""
    import torch
    import torch.nn.functional as F
    import linear_attention_diffusion_b200 as la

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(str(getattr(props, "uuid", "") or ""))
    stream = torch.cuda.Stream(dev)
    lib = la._lib
    sp = stream.cuda_stream
    C = wl.hidden_width(w)
    HD = w.H * D
    X0, Wt, bias = wl.make_projection(w, C, seed=rank_seed(rank) + 30)
    per_set = X0.numel() * X0.element_size()
    n_sets = max(2, -(-2 * L2_BYTES // per_set))
    xs = [X0.to(dev)] + [wl.make_projection(w, C, seed=rank_seed(rank) + 30 + 10 * i)[0].to(dev)
                         for i in range(1, n_sets)]
    Wd, bd = Wt.to(dev), bias.to(dev)
    Q = torch.empty((w.B, w.N, w.H, D), dtype=torch.bfloat16, device=dev)
    S = torch.empty((w.B, w.H, D, D), device=dev)
    z = torch.empty((w.B, w.H, D), device=dev)
    shape = la.make_shape(w.B, w.N, w.H, D, "bf16", w.rope, w.T, w.Hh, w.W, 0, w.rope_base,
                          w.eps)
    ws_n = max(256, la.la_qkv_workspace_bytes(shape, C))
    ws = torch.empty(ws_n, dtype=torch.uint8, device=dev)
    status = []

    def step(i, evs=None):
        if evs is not None:
            evs[0].record(stream)
        status.append(lib.la_qkv_state(ctypes.byref(shape), C, xs[i % n_sets].data_ptr(),
                                       Wd.data_ptr(), bd.data_ptr(), Q.data_ptr(), S.data_ptr(),
                                       z.data_ptr(), ws.data_ptr(), ws_n, sp))
        if evs is not None:
            evs[1].record(stream)

    def check_status():
        bad = [v for v in status if v != 0]
        status.clear()
        if bad:
            raise RuntimeError(f"library call failed: {la.la_status_string(bad[0])} "
                               f"{la.la_last_error()}")

    ms_max, seg_us, chunk, t0, t1 = time_steps(args, step, stream, dev, world, n_sets, False,
                                               check_status)
    clocks = sampler.summary(t0, t1)

    # the unfused path on the same inputs: projections, then the state reduce
    Wq, Wk, Wv = (Wd[j * HD:(j + 1) * HD] for j in range(3))
    bq, bk, bv = (bd[j * HD:(j + 1) * HD] for j in range(3))
    Ku = torch.empty((w.B, w.N, HD), dtype=torch.bfloat16, device=dev)
    Vu = torch.empty_like(Ku)
    Qu = torch.empty_like(Ku)
    lws = la.workspace(shape, dev)

    def unfused(i, evs=None):
        x = xs[i % n_sets]
        if evs is not None:
            evs[0].record(stream)
        x2 = x.view(-1, C)
        torch.addmm(bq, x2, Wq.t(), out=Qu.view(-1, HD))
        torch.addmm(bk, x2, Wk.t(), out=Ku.view(-1, HD))
        torch.addmm(bv, x2, Wv.t(), out=Vu.view(-1, HD))
        la.la_state_reduce(shape, Ku, Vu, S, z, lws, sp)
        if evs is not None:
            evs[1].record(stream)

    ums, _, _, _, _ = time_steps(args, unfused, stream, dev, world, n_sets, False, lambda: None)
    e2e = None
    if args.e2e_steps > 0:
        steps = max(1, min(args.steps, args.e2e_steps))
        hx = X0.pin_memory()
        hq = torch.empty((w.B, w.N, w.H, D), dtype=torch.bfloat16).pin_memory()
        hs = torch.empty((w.B, w.H, D, D)).pin_memory()
        hz = torch.empty((w.B, w.H, D)).pin_memory()

        def call(p, ins, outs, st):
            la.la_qkv_state(shape, C, ins[0], Wd, bd, outs[0], outs[1], outs[2], ws, st)

        ms = e2e_pipelined(dev, stream, [hx], [hq, hs, hz], call, 1, steps)
        e2e = {"ms_per_step": ms, "tokens_per_step": w.B * w.N, "steps": steps,
               "h2d_bytes_per_step": per_set,
               "d2h_bytes_per_step": (hq.numel() * 2 + hs.numel() * 4 + hz.numel() * 4),
               "copies": "pipelined: copy-in, calls and copy-out on three streams, two buffer sets"}
    sampler.stop()
    flops = 2.0 * w.B * w.N * C * 3 * HD
    return {"ms": ms_max, "seg_us": seg_us, "kernel_names": ("qkv_state",), "e2e": e2e,
            "clocks": clocks, "launches_per_step": 2, "n_sets": n_sets, "chunk": chunk,
            "per_set_bytes": per_set, "flops": flops, "unfused_ms": ums / args.steps,
            "C": C}


def oracle_sample_qkv(w, seconds):
    """The float64 fused projection + state on a token subset, scaled to N."""
    import oracle as orc
    C = wl.hidden_width(w)
    X, Wt, b = wl.make_projection(w, C, seed=30)
    th_all = orc.rope_angles(w.T, w.Hh, w.W, 0, w.rope_base) if w.rope else None
    n_sub = min(w.N, 256)
    Xs = X[:1, :n_sub]
    th = None if th_all is None else th_all[:n_sub]
    reps, t0 = 0, time.perf_counter()
    while True:
        orc.qkv_state(Xs, Wt, b, w.H, th)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    per_call = el / reps * (w.B * w.N) / n_sub
    desc = (f"oracle qkv_state on {n_sub} of {w.B * w.N} tokens (C = {C}), {reps} calls in "
            f"{el:.1f} s, scaled to {w.B * w.N} tokens")
    return w.B * w.N / per_call, desc, cpu_cores_used(), per_call


def oracle_sample_tconv(w, seconds):
    """The float64 temporal convolution on a channel subset, scaled to FFN_WIDTH."""
    import oracle as orc
    c_sub = 8
    x = wl.make_tensor((w.B, w.T, w.Hh, w.W, c_sub), 20)
    wt = wl.make_tensor((c_sub, 3), 21, __import__("torch").float32)
    f = wl.make_tensor((w.B, w.Hh, w.W, c_sub), 23) if w.block_causal else None
    reps, t0 = 0, time.perf_counter()
    while True:
        orc.temporal_conv(x, wt, None, f)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    per_call = el / reps * FFN_WIDTH / c_sub
    desc = (f"oracle temporal_conv on {c_sub} of {FFN_WIDTH} channels ({w.T}x{w.Hh}x{w.W}), "
            f"{reps} calls in {el:.1f} s, scaled to {FFN_WIDTH} channels")
    return w.B * w.N / per_call, desc, cpu_cores_used(), per_call


def e2e_pipelined(dev, compute, host_in, host_out, call, passes_per_step, steps):
    """Time ``steps`` steps of ``passes_per_step`` library calls each, every
    call with its inputs copied in from pinned host memory and its outputs
    copied back to pinned host memory.

    Copies in run on one stream, the calls on ``compute`` and copies out on a
    third stream, with two device buffer sets, so the copies of neighbouring
    calls overlap a call (both copy directions at once). ``call(p, ins, outs,
    stream)`` enqueues call p. Returns ms per step (CUDA events)."""
    import torch
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    bin_ = [[torch.empty_like(h, device=dev) for h in host_in] for _ in range(2)]
    bout = [[torch.empty_like(h, device=dev) for h in host_out] for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def one(p):
        s = p % 2
        if p >= 2:
            h2d.wait_event(ev_done[s])      # call p - 2 has read this input set
        with torch.cuda.stream(h2d):
            for d_, h_ in zip(bin_[s], host_in):
                d_.copy_(h_, non_blocking=True)
        ev_in[s].record(h2d)
        compute.wait_event(ev_in[s])
        if p >= 2:
            compute.wait_event(ev_out[s])   # copy-out of call p - 2 is done with this set
        call(p, bin_[s], bout[s], compute)
        ev_done[s].record(compute)
        d2h.wait_event(ev_done[s])
        with torch.cuda.stream(d2h):
            for h_, d_ in zip(host_out, bout[s]):
                h_.copy_(d_, non_blocking=True)
        ev_out[s].record(d2h)

    for p in range(passes_per_step):  # warm-up step
        one(p)
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(h2d)
    for p in range(steps * passes_per_step):
        one(p)
    d2h.wait_stream(compute)
    d2h.wait_stream(h2d)
    end.record(d2h)
    torch.cuda.synchronize(dev)
    return start.elapsed_time(end) / steps


def run_e2e_half(args, w, dev, stream, la, rank, op):
    """The reduce or the apply alone through la_state_reduce / la_apply: the
    reduce copies K, V in and S, z out; the apply copies Q, S, z in and O out
    (pipelined over three streams, e2e_pipelined)."""
    import torch
    steps = max(1, min(args.steps, args.e2e_steps))
    q, k, v = wl.make_qkv(w, 1000 * rank + 7)
    shape = la.make_shape(w.B, w.N, w.H, D, "bf16", w.rope, w.T, w.Hh, w.W, 0, w.rope_base,
                          w.eps)
    ws = la.workspace(shape, dev)
    S = torch.zeros((w.B, w.H, D, D), device=dev)
    z = torch.zeros((w.B, w.H, D), device=dev)
    la.la_state_reduce(shape, k.to(dev), v.to(dev), S, z, ws, stream)
    torch.cuda.synchronize(dev)
    hS, hz = S.cpu().pin_memory(), z.cpu().pin_memory()
    if op == "reduce":
        hin = [x.pin_memory() for x in (k, v)]
        hout = [torch.empty_like(hS).pin_memory(), torch.empty_like(hz).pin_memory()]

        def call(p, ins, outs, st):
            la.la_state_reduce(shape, ins[0], ins[1], outs[0], outs[1], ws, st)
    else:
        hin = [q.pin_memory(), hS, hz]
        hout = [torch.empty_like(hin[0]).pin_memory()]

        def call(p, ins, outs, st):
            la.la_apply(shape, ins[0], ins[1], ins[2], outs[0], st)

    ms = e2e_pipelined(dev, stream, hin, hout, call, 1, steps)
    nb = lambda ts: sum(t.numel() * t.element_size() for t in ts)
    return {"ms_per_step": ms, "tokens_per_step": w.B * w.N, "steps": steps,
            "h2d_bytes_per_step": nb(hin), "d2h_bytes_per_step": nb(hout),
            "copies": "pipelined: copy-in, calls and copy-out on three streams, two buffer sets"}


def run_e2e(args, w, dev, stream, la, rank, causal=False):
    """Same metric through la_attention / la_block_causal_step /
    la_causal_attention, every call copying its Q, K, V in from pinned host
    memory and its O out (pipelined over three streams, e2e_pipelined)."""
    import torch
    steps = max(1, min(args.steps, args.e2e_steps))
    if w.block_causal:
        q, k, v = wl.make_qkv(w, 1000 * rank, block=0, step=0)
    else:
        q, k, v = wl.make_qkv(w, 1000 * rank + 7)
    hin = [x.pin_memory() for x in (q, k, v)]
    hout = [torch.empty_like(hin[0]).pin_memory()]
    S = torch.zeros((w.B, w.H, D, D), device=dev)
    z = torch.zeros((w.B, w.H, D), device=dev)
    shapes = [la.make_shape(w.B, w.N, w.H, D, "bf16", w.rope, w.T, w.Hh, w.W, m * w.T,
                            w.rope_base, w.eps) for m in range(max(1, w.M))]
    ws = la.workspace(shapes[0], dev, causal=causal)
    per = w.steps + 1

    def call(p, ins, outs, st):
        if causal:
            la.la_causal_attention(shapes[0], *ins, None, None, outs[0], 0, ws, st)
        elif w.block_causal:
            i = p % (w.M * per)
            if i == 0:
                la.la_state_reset(S, z, w.B, w.H, D, st)
            la.la_block_causal_step(shapes[i // per], *ins, S, z, outs[0],
                                    1 if i % per == w.steps else 0, ws, st)
        else:
            la.la_attention(shapes[0], *ins, S, z, outs[0], ws, st)

    passes = w.M * per if w.block_causal and not causal else 1
    ms = e2e_pipelined(dev, stream, hin, hout, call, passes, steps)
    tokens = (w.M if (w.block_causal and not causal) else 1) * w.B * w.N
    nb = hin[0].numel() * hin[0].element_size()
    return {"ms_per_step": ms, "tokens_per_step": tokens, "steps": steps,
            "h2d_bytes_per_step": 3 * nb * passes, "d2h_bytes_per_step": nb * passes,
            "copies": "pipelined: copy-in, calls and copy-out on three streams, two buffer sets"}


def run_e2e_backward(args, w, dev, stream, la, rank):
    """The backward through la_attention_backward, every call copying Q, K, V,
    dO in and dQ, dK, dV out (pipelined); the state is reduced again inside
    the call (S = z = NULL), as a caller holding only host tensors would do."""
    import torch
    steps = max(1, min(args.steps, args.e2e_steps))
    q, k, v = wl.make_qkv(w, 1000 * rank + 7)
    g = wl.make_tensor(tuple(q.shape), 1000 * rank + 10)
    hin = [x.pin_memory() for x in (q, k, v, g)]
    hout = [torch.empty_like(hin[0]).pin_memory() for _ in range(3)]
    dS = torch.empty((w.B, w.H, D, D), device=dev)
    dz = torch.empty((w.B, w.H, D), device=dev)
    shape = la.make_shape(w.B, w.N, w.H, D, "bf16", w.rope, w.T, w.Hh, w.W, 0, w.rope_base,
                          w.eps)
    ws = la.workspace(shape, dev)

    def call(p, ins, outs, st):
        la.la_attention_backward(shape, ins[0], ins[1], ins[2], None, None, ins[3], *outs, dS,
                                 dz, ws, st)

    ms = e2e_pipelined(dev, stream, hin, hout, call, 1, steps)
    nb = hin[0].numel() * hin[0].element_size()
    return {"ms_per_step": ms, "tokens_per_step": w.B * w.N, "steps": steps,
            "h2d_bytes_per_step": 4 * nb, "d2h_bytes_per_step": 3 * nb,
            "copies": "pipelined: copy-in, calls and copy-out on three streams, two buffer sets"}


# ---------------------------------------------------------------------------


def config_of(w, world, n_sets=None, per_set=None):
    c = {"workload": w.name, "model": "Sana-1.6B" if w.H == 70 else "Sana-0.6B",
         "global_batch": w.B * world, "seq_len": w.N, "heads": w.H, "head_dim": D,
         "rope": "3d 8/12/12 base 1e4" if w.rope else "none", "eps": w.eps,
         "parallelism": f"dp{world} (independent replicas)", "io": "bf16",
         "accumulate": "f32"}
    if w.outlier_frac:
        c["k_outliers"] = f"{w.outlier_frac:.0%} of K entries x{w.outlier_scale:g}"
    if w.block_causal:
        c.update({"blocks": w.M, "block_tokens": w.N, "passes_per_block": w.steps + 1,
                  "video_tokens": w.M * w.N})
    if n_sets is not None:
        c["l2"] = (f"inputs larger than L2: {n_sets} rotating input sets of "
                   f"{per_set / 1e6:.0f} MB ({n_sets * per_set / 1e6:.0f} MB > 126 MB L2)")
    return c


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["la", "reference"], default="la")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(wl.WORKLOADS))
    # --e2e-steps 0 and --cpu-seconds 0 leave out the end-to-end and CPU
    # legs (for profiler runs; the timed region is the same either way).
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--soak", type=float, default=1.0)
    ap.add_argument("--ref-budget", type=float, default=150.0,
                    help="seconds of oracle work for --impl reference (warm-up and steps)")
    ap.add_argument("--op", choices=["layer", "reduce", "apply", "backward", "causal", "tconv",
                                     "qkv"],
                    default="layer")
    args = ap.parse_args()
    w = wl.WORKLOADS[args.workload]
    if args.op in ("backward", "causal", "qkv", "reduce", "apply") and w.block_causal:
        ap.error(f"--op {args.op} covers the non-causal workloads")
    if args.op == "tconv" and not w.rope:
        ap.error("--op tconv needs a video workload (sanavideo_480p, longsana_block_causal)")
    if args.steps is None:
        per_step_us = {"sana0.6b_512px": 10, "sana1.6b_1024px": 30, "sana1.6b_4k": 120,
                       "sanavideo_480p": 250, "longsana_block_causal": 12000}[w.name]
        if args.op in ("backward", "causal"):
            per_step_us *= 10
        elif args.op == "tconv":
            per_step_us = 200
        elif args.op == "qkv":
            per_step_us *= 8
        args.steps = max(10, int(0.5e6 / per_step_us))
    args.warmup = max(args.warmup, 3)

    world = env_int("WORLD_SIZE", 1)
    rank = env_int("RANK", 0)
    local_rank = env_int("LOCAL_RANK", 0)

    if args.impl == "reference":
        return main_reference(args, w, rank, world)

    import torch
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    r = {"tconv": run_tconv, "qkv": run_qkv}.get(args.op, run_la)(args, w, rank, world,
                                                                  local_rank)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    ms_step = r["ms"] / args.steps
    tokens_step = (w.M * w.N * w.B) if (w.block_causal and args.op == "layer") else w.B * w.N
    value = weak_scaled_value(tokens_step, args.steps, world, r["ms"])
    peak, peak_src = peaks()
    lb = layer_bytes(w)
    lb["temporal_conv"] = 2 * r["per_set_bytes"] + r.get("cache_bytes", 0)
    # The unit timed is one library call: its average duration is the timed
    # region (back-to-back graph replays, no events between launches) divided
    # by the calls in it. The event graph's per-call figure, which also holds
    # the events' own cost and loses the overlap of consecutive calls, is
    # reported beside it.
    if w.block_causal and args.op == "layer":
        name = "la_block_causal_step"
        calls = w.M * (w.steps + 1)
        alg = 4 * w.B * w.N * w.H * D * 2 + 2 * w.B * w.H * (D * D + D) * 4
        dur_us = ms_step * 1e3 / calls
        kernels = {name: {"avg_us": dur_us, "algorithmic_bytes": alg,
                          "gbs": alg / (dur_us * 1e-6) / 1e9,
                          "launches": r["launches_per_step"] // calls,
                          "event_graph_us": r["seg_us"][0],
                          "note": "update=0 call, event graph; avg over all 60 calls"}}
        dom = name
        traffic = profiled_traffic(w.name, name)
    elif args.op == "qkv":
        kernels, dom, traffic = {}, None, None
    else:
        kernels = {}
        for nm, us in zip(r["kernel_names"], r["seg_us"]):
            dur_us = ms_step * 1e3  # one call per step
            kernels[nm] = {"avg_us": dur_us, "algorithmic_bytes": lb[nm],
                           "gbs": lb[nm] / (dur_us * 1e-6) / 1e9,
                           "launches": r["launches_per_step"], "event_graph_us": us}
        dom = max(kernels, key=lambda k: kernels[k]["avg_us"])
        traffic = profiled_traffic(w.name, dom)
    kd = kernels.get(dom)
    if args.op == "qkv":
        # a dense contraction: tensor-bound against the measured bf16 GEMM peak
        tf_peak, tf_src = tensor_peaks()
        dur_us = ms_step * 1e3
        tflops = r["flops"] / (dur_us * 1e-6) / 1e12
        roofline = {"bound": "tensor", "kernel": "qkv_state", "achieved": round(tflops, 1),
                    "peak": tf_peak["sustained"], "unit": "TFLOP/s",
                    "frac": round(tflops / tf_peak["sustained"], 4),
                    "frac_of_burst": round(tflops / tf_peak["burst"], 4),
                    "traffic": profiled_traffic(w.name, "qkv_state"),
                    "algorithmic_flops": r["flops"], "avg_launch_us": round(dur_us, 3),
                    "event_graph_us": round(r["seg_us"][0], 3), "launches_per_call": 2,
                    "peak_source": tf_src,
                    "unfused_us": round(r["unfused_ms"] * 1e3, 3),
                    "unfused_note": ("the same result through three cuBLAS projections "
                                     "(torch.addmm with bias) writing Q, K, V, then "
                                     "la_state_reduce reading K and V back")}
    else:
      roofline = {"bound": "hbm", "kernel": dom, "achieved": round(kd["gbs"], 1),
                "peak": peak, "unit": "GB/s", "frac": round(kd["gbs"] / peak, 4),
                "traffic": traffic, "algorithmic_bytes": kd["algorithmic_bytes"],
                "avg_launch_us": round(kd["avg_us"], 3), "peak_source": peak_src,
                "per_kernel": {k: {"avg_us": round(v["avg_us"], 3), "gbs": round(v["gbs"], 1),
                                   "frac": round(v["gbs"] / peak, 4),
                                   "event_graph_us": round(v["event_graph_us"], 3),
                                   "launches_per_call": v["launches"]}
                               for k, v in kernels.items()},
                "avg_launch_note": ("call duration = timed region / calls (back-to-back "
                                    "graph replays); event_graph_us = the same call with "
                                    "events around it in a second graph")}
    e = r["e2e"]
    e2e = None if e is None else {
        "value": world * e["tokens_per_step"] / (e["ms_per_step"] / 1e3), "unit": "tokens/s",
        "h2d_bytes_per_step": e["h2d_bytes_per_step"],
        "d2h_bytes_per_step": e["d2h_bytes_per_step"], "steps": e["steps"],
        "ms_per_step": round(e["ms_per_step"], 4), "copies": e.get("copies"),
        "api": ("la_attention_backward" if args.op == "backward" else
                "la_state_reduce" if args.op == "reduce" else
                "la_apply" if args.op == "apply" else
                "la_causal_attention" if args.op == "causal" else
                "la_temporal_conv" if args.op == "tconv" else
                "la_qkv_state" if args.op == "qkv" else
                "la_block_causal_step" if w.block_causal else "la_attention")}
    out = {"metric": METRICS[args.op], "value": value, "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
           "latency_us": ms_step * 1e3, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1), bf16)",
           "config": dict(config_of(w, world, r["n_sets"], r["per_set_bytes"]),
                          **OP_CONFIG[args.op]),
           "roofline": roofline, "e2e": e2e,
           "gpu_launches": r["launches_per_step"] * args.steps,
           "clocks": r["clocks"], "graph_chunk_steps": r["chunk"], "soak_s": args.soak}
    if world == 1 and args.cpu_seconds > 0 and args.op in ("tconv", "qkv"):
        sampler_fn = oracle_sample_tconv if args.op == "tconv" else oracle_sample_qkv
        tps, desc, cores, _ = sampler_fn(w, args.cpu_seconds)
        out["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": cores,
                               "kind": "oracle", "sample": desc}
    elif world == 1 and args.cpu_seconds > 0:
        tps, desc, cores, _, _ = oracle_sample(w, args.cpu_seconds, op=args.op)
        out["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": cores,
                               "kind": "oracle", "sample": desc}
    print(json.dumps(out), flush=True)


def main_reference(args, w, rank, world):
    """The float64 oracle, timed as it stands on the host's cores."""
    if rank != 0:
        return
    budget = float(getattr(args, "ref_budget", 150.0))  # seconds: warm-up + timed steps
    per = budget / (args.steps + args.warmup)
    if args.op in ("tconv", "qkv"):
        sampler_fn = oracle_sample_tconv if args.op == "tconv" else oracle_sample_qkv
        tps, desc, cores, per_call = sampler_fn(w, min(per * args.steps, 60.0))
        out = {"impl": "reference", "metric": METRICS[args.op], "value": tps, "unit": "tokens/s",
               "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
               "ms_per_step": per_call * 1e3, "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "f64",
               "data": "synthetic (seeded N(0,1), bf16 inputs read exactly)",
               "config": dict(config_of(w, world), **OP_CONFIG[args.op]),
               "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle", "sample": desc},
               "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                       "d2h_bytes_per_step": 0}}
        print(json.dumps(out), flush=True)
        return
    _, _, cores, per_call, h_sub = oracle_sample(w, min(per, 3.0), max_reps=1, op=args.op)
    # each step: one oracle call on h_sub heads (at most `per` seconds)
    import oracle as orc
    import numpy as np
    th = orc.rope_angles(w.T, w.Hh, w.W, 0, w.rope_base) if w.rope else None
    Q, K, V = (x[:, :, :h_sub].contiguous() for x in wl.make_qkv(w, 0))
    bwd = args.op == "backward"
    dO = wl.make_tensor((w.B, w.N, w.H, w.D), 3)[:, :, :h_sub].contiguous() if bwd else None
    S0, z0 = orc.state_reduce(K, V, th) if args.op == "apply" else (None, None)

    def call():
        if bwd:
            orc.backward(Q, K, V, dO, w.eps, th)
        elif args.op == "reduce":
            orc.state_reduce(K, V, th)
        elif args.op == "apply":
            orc.apply(Q, S0, z0, w.eps, th)
        elif args.op == "causal":
            orc.causal_attention(Q, K, V, w.eps, th)
        elif w.block_causal:
            orc.block_causal_step(Q, K, V, np.zeros((w.B, h_sub, D, D)),
                                  np.zeros((w.B, h_sub, D)), 1, w.eps, th)
        else:
            orc.attention(Q, K, V, w.eps, th)

    for _ in range(args.warmup):
        call()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        call()
    el = time.perf_counter() - t0
    per_call = el / args.steps
    full_call = per_call * w.H / h_sub
    if w.block_causal:
        calls = w.M * (w.steps + 1)
        value = w.M * w.N * w.B / (full_call * calls)
        ms_step = full_call * calls * 1e3
        sample = (f"each step: oracle block_causal_step on {h_sub} of {w.H} heads of one block; "
                  f"scaled to {w.H} heads x {calls} calls per video")
    else:
        value = w.B * w.N / full_call
        ms_step = full_call * 1e3
        what = {"backward": "backward", "causal": "causal_attention", "reduce": "state_reduce",
                "apply": "apply"}.get(args.op, "attention")
        sample = f"each step: oracle {what} on {h_sub} of {w.H} heads; scaled to {w.H} heads"
    out = {"impl": "reference", "metric": METRICS[args.op], "value": value, "unit": "tokens/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded N(0,1), bf16 inputs read exactly)",
           "config": dict(config_of(w, world), **OP_CONFIG[args.op]),
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
