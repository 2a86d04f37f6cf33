#!/usr/bin/env python
"""Benchmark of the sparse FFN layer forward (tokens/s per layer, % of roofline).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl sfn|reference]

One step is one call of ``sfn_sparse_ffn_forward_ws`` (the whole path:
predictor, bank top-k, sparse gate/up, sparse down) on one batch of T tokens
of the workload.  Steps rotate over several distinct layers whose total size
is far above the 126 MB L2, so no step finds its weights in L2.  Steps are
replayed from a CUDA graph (no host launch gaps) and timed with CUDA events
on the launching stream, synchronised on both sides, max over ranks.

With N > 1 (torchrun), every rank runs its own copy of the workload on its own
GPU (tokens are independent: weak scaling, no collective on the data path);
``value`` is the tokens of all ranks divided by the slowest rank's time.

``--impl reference`` times the fp64 CPU oracle instead (the only reference
there is), on the host cores, same workload and metric; on N > 1 only rank 0
runs it.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse-FFN layer tokens/s at T=1..32K; % of HBM or bf16 tensor roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TIMED_STAGES = 16


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "batched_decode", "prefill", "long_prefill"])
    ap.add_argument("--impl", default="sfn", choices=["sfn", "reference"])
    ap.add_argument("--k", type=int, default=None, help="override top-k (e.g. 64: dense mask)")
    ap.add_argument("--method", default="sfn", choices=["sfn", "dense4x", "backward"],
                    help="sfn: the predictor-gated sparse FFN; dense4x: the pages' post-hoc "
                         "comparison (dense gate/up, amplitude top-k, sparse down); backward: "
                         "the layer's backward with the surrogate top-k gradient")
    ap.add_argument("--shard", default="tokens", choices=["tokens", "banks"],
                    help="tokens: every rank runs the whole layer on its own tokens (weak "
                         "scaling); banks: the ranks split one layer's banks and sum their "
                         "float32 partial outputs with an all-reduce (strong scaling)")
    ap.add_argument("--temperature", type=float, default=1.0,
                    help="surrogate temperature of --method backward")
    ap.add_argument("--path", default="auto",
                    choices=["auto", "cuda_core", "tensor"],
                    help="kernels to use (the library picks by token count when auto)")
    ap.add_argument("--workloads", default="all", choices=["all", "one"],
                    help="all (default): with the default decode workload, also measure the "
                         "batched-decode, prefill and long-prefill workloads and report them "
                         "under 'workloads'; one: only --workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--settle", type=float, default=1.0,
                    help="seconds of untimed load before timing (clock settling)")
    return ap.parse_args(argv)


# --------------------------------------------------------------------------- helpers

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, source="fallback")


def default_steps(name, extra=False):
    # about a second of timed GPU work at the current kernel speeds; the
    # workloads measured beside the headline line take about a quarter second
    if extra:
        return {"decode": 10000, "batched_decode": 2000, "prefill": 100, "long_prefill": 20}[name]
    return {"decode": 40000, "batched_decode": 4000, "prefill": 200, "long_prefill": 30}[name]


def rotation_layers(name):
    # decode working sets are < L2 per step: rotate 8 distinct layers (2.95 GB)
    return {"decode": 8, "batched_decode": 4, "prefill": 1, "long_prefill": 1}[name]


def aggregate_max(value, world, device=None):
    """Max of a float over ranks (the slowest rank's time)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background (read only)."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.out = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [r for r in csv.reader(io.StringIO(self.out.read())) if len(r) >= 10]
        os.unlink(self.out.name)
        mine = [r for r in rows if self.uuid and self.uuid in r[1]] or rows
        loaded = [r for r in mine if _num(r[5]) and _num(r[5]) >= 50] or mine
        sm = [_num(r[2]) for r in loaded if _num(r[2])]
        smax = [_num(r[3]) for r in loaded if _num(r[3])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i in range(4)
                          if r[6 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples_under_load": len(loaded)}


def _num(s):
    try:
        return float(s.strip())
    except (ValueError, AttributeError):
        return None


# stage name -> the source files that define its kernel
KERNEL_SOURCES = {
    "pred_h": ["predict_topk.cu"], "logits_topk": ["predict_topk.cu"],
    "ffn": ["gather_ffn.cu"], "reduce": ["gather_ffn.cu"],
    "tc_h": ["tc_path.cu", "tc_util.cuh"], "tc_logits_topk": ["tc_path.cu", "tc_util.cuh"],
    "tc_gateup": ["tc_path.cu", "tc_util.cuh"], "tc_down": ["tc_path.cu", "tc_util.cuh"],
}
COMMON_SOURCES = ["sfn_internal.cuh", "async_util.cuh"]


def _code_only(text):
    """C/C++ source without comments and blank space, so that a digest
    changes with the code and not with its comments."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_digest(kernel):
    """Digest of the code (comments left out) a stage's kernel is compiled
    from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "predictor_gated_channel_b200", "csrc")
    for name in sorted(KERNEL_SOURCES.get(kernel, []) + COMMON_SOURCES):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:12]


def traffic_from_profiles(kernel, workload):
    """DRAM bytes per launch (read + write) from the committed ncu summary
    profiles/dram_traffic.txt, if its source digest still matches the
    kernel's sources; None otherwise."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel \
                and parts[1] == workload:
            if parts[3] != source_digest(kernel):
                return None
            return float(parts[2])
    return None


# ------------------------------------------------------------------ algorithmic work

def stage_work(wl, T, union_channels):
    """Algorithmic bytes and useful FLOPs of each stage for one call on T tokens.

    union_channels: number of distinct kept channels over the T tokens (the
    rows of Wg, Wu, Wd that must be read at least once).  Tensor-core stages
    count the same useful work; their dense tiles do more arithmetic."""
    e = 2 if wl.dtype == "bf16" else 4
    d, d_i, r, d_s, nb = wl.d, wl.d_i, wl.r, wl.d_s, wl.n_banks
    pred_h = {"bytes": r * d * e + T * d * e + T * r * 4, "flops": 2 * T * d * r}
    logits = {"bytes": d_i * r * e + T * r * 4 + T * nb * 8 + T * d_s * 8,
              "flops": 2 * T * r * d_i}
    ffn = {"bytes": 3 * union_channels * d * e + T * d * e + T * d_s * 8,
           "flops": 6 * T * d_s * d}
    return {
        "pred_h": pred_h, "logits_topk": logits, "ffn": ffn,
        "reduce": {"bytes": T * d * e, "flops": 0},
        "tc_h": pred_h, "tc_logits_topk": logits,
        "tc_gateup": {"bytes": 2 * union_channels * d * e + T * d * e + T * d_i * e,
                      "flops": 4 * T * d_s * d},
        "tc_down": {"bytes": union_channels * d * e + T * d_i * e + T * d * e,
                    "flops": 2 * T * d_s * d},
        # Dense-4x: gate and up are dense (the mask depends on them)
        "dense4x_gateup": {"bytes": 2 * d_i * d * e + T * d * e + T * d_i * e + T * nb * 8,
                           "flops": 4 * T * d_i * d},
        # backward: g, u, da; dWd, dWg, dWu; dx (two d_i contractions) are 8
        # T d d_i GEMMs, plus dh, dB (T d_i r each) and dA, dx (T r d each)
        "bwd_gemm": {"bytes": 5 * d_i * d * e + 3 * d_i * d * 4 + 2 * d_i * r * e
                              + T * d_i * (3 * 4 + 4 * e) + 2 * T * d * e + T * d * 4,
                     "flops": 2 * T * (8 * d * d_i + 2 * d_i * r + 2 * r * d)},
        "bwd_elem": {"bytes": T * d_i * (4 * 4 + 4 * e) + T * nb * 12, "flops": 0},
        "bwd_tau": {"bytes": T * d_i * 4 + T * nb * 12, "flops": 0},
    }


def useful_flops_per_token(wl, method="sfn"):
    """Predictor (2dr + 2r d_i) + kept gate and up (4 d d_s) + kept down (2 d d_s);
    Dense-4x: dense gate and up (4 d d_i) + kept down (2 d d_s)."""
    if method == "dense4x":
        return 2 * (2 * wl.d * wl.d_i + wl.d * wl.d_s)
    if method == "backward":  # predictor recompute + the backward's contractions
        return 2 * (wl.d * wl.r + wl.r * wl.d_i + 8 * wl.d * wl.d_i + 2 * wl.d_i * wl.r
                    + 2 * wl.r * wl.d)
    return 2 * (wl.d * wl.r + wl.r * wl.d_i + 3 * wl.d * wl.d_s)


# ---------------------------------------------------------------------- the GPU arm

def run_sfn(args, rank, world, local):
    import torch

    from predictor_gated_channel_b200 import _capi
    from predictor_gated_channel_b200 import build as sfn_build

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (there is no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    sfn_build.build()
    L = _capi.lib()

    K = args.steps if args.steps is not None else default_steps(args.workload)
    W = max(3, args.warmup if args.warmup is not None else 20)
    line = measure(args, args.workload, K, W, rank, world, dev, L, main=True)
    if extra_workloads_wanted(args, world):
        line_w = {}
        for name in EXTRA_WORKLOADS:
            torch.cuda.empty_cache()
            sub = measure(args, name, default_steps(name, extra=True), W, rank, world, dev, L,
                          main=False)
            if sub is not None:
                line_w[name] = summarize(sub)
        if line is not None:
            line["workloads"] = line_w
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return line


# the other workloads of the metric, measured in the default run beside the
# headline decode line (each with its own steps, timing, roofline and clocks)
EXTRA_WORKLOADS = ("batched_decode", "prefill", "long_prefill")


def extra_workloads_wanted(args, world):
    return (args.workloads == "all" and world == 1 and args.workload == "decode"
            and args.method == "sfn" and args.k is None and args.shard == "tokens"
            and args.path == "auto")


def summarize(line):
    """The per-workload entry of the headline line."""
    keys = ("value", "unit", "steps", "warmup", "ms_per_step", "roofline", "step_roofline",
            "mask_union_channels", "clocks", "gpu_launches", "step_time_spread", "e2e",
            "cpu_baseline")
    out = {k: line.get(k) for k in keys}
    out["workload"] = line["config"]["workload"]
    out["dtype"] = line["dtype"]
    out["stages"] = {n: {"us_per_step": v["us_per_step"], "share": v["share"]}
                     for n, v in line["stages"].items()}
    return out


def measure(args, workload, K, W, rank, world, dev, L, main):
    """Time K steps of one workload (after W warm-up steps); rank 0 returns
    its JSON line, the other ranks None."""
    import numpy as np
    import torch

    import predictor_gated_channel_b200 as sfn
    from predictor_gated_channel_b200 import _capi
    from predictor_gated_channel_b200.inputs import (WORKLOADS, make_layer_device,
                                                     make_tokens_device)
    if world > 1:
        import torch.distributed as dist

    wl = WORKLOADS[workload]
    if args.k is not None:
        wl = wl.with_(k=args.k)
    T = wl.T
    S = rotation_layers(workload)
    peaks = load_peaks()

    shard = args.shard == "banks"
    if shard and (args.method != "sfn" or wl.dtype != "bf16"):
        raise SystemExit("bench.py: --shard banks runs the bf16 forward")
    # bank shards: every rank holds the same layer and tokens and keeps its banks
    seed = 0 if shard else rank
    layers = [make_layer_device(wl, dev, seed=seed, layer=i) for i in range(S)]
    xs = [make_tokens_device(wl, dev, seed=seed, layer=i) for i in range(S)]
    wl_full = wl
    if shard:
        b0, b1 = sfn.bank_shard(wl.n_banks, rank, world)
        rows = slice(b0 * wl.bank, b1 * wl.bank)
        for lay in layers:
            for n in ("B", "Wg", "Wu", "Wd"):
                lay[n] = lay[n][rows]
        wl = wl.with_(d_i=(b1 - b0) * wl.bank)
    ys = [torch.empty((T, wl.d), dtype=torch.float32 if shard else wl.torch_dtype, device=dev)
          for _ in range(S)]
    ms = [torch.empty((T, wl.n_banks), dtype=torch.int64, device=dev) for _ in range(S)]
    dense4x = args.method == "dense4x"
    backward = args.method == "backward"
    if (dense4x or backward) and wl.dtype != "bf16":
        raise SystemExit(f"bench.py: --method {args.method} runs on bf16 workloads")
    if dense4x:
        ws_bytes = L.sfn_dense4x_workspace_bytes(T, wl.d, wl.d_i, wl.bank, wl.k)
    elif backward:
        ws_bytes = L.sfn_backward_workspace_bytes(T, wl.d, wl.d_i, wl.r, wl.bank, wl.k)
        # dy per rotation layer; one set of float32 gradients, overwritten every step
        gen = torch.Generator(device=dev).manual_seed(1000 + rank)
        dys = [torch.randn((T, wl.d), device=dev, generator=gen).to(torch.bfloat16)
               for _ in range(S)]
        gshape = {"dx": (T, wl.d), "dA": (wl.r, wl.d), "dB": (wl.d_i, wl.r),
                  "dWg": (wl.d_i, wl.d), "dWu": (wl.d_i, wl.d), "dWd": (wl.d_i, wl.d)}
        grads = {n: torch.empty(sh, dtype=torch.float32, device=dev) for n, sh in gshape.items()}
    else:
        ws_bytes = sfn.workspace_bytes(T, wl.d, wl.d_i, wl.r, wl.bank, wl.k, wl.torch_dtype)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    path_id = {"auto": 0, "cuda_core": 1, "tensor": 2}[args.path]
    stream = torch.cuda.Stream(device=dev)

    def call(i, st_ptr):
        lay = layers[i]
        ptrs = [xs[i].data_ptr(), lay["A"].data_ptr(), lay["B"].data_ptr(),
                lay["Wg"].data_ptr(), lay["Wu"].data_ptr(), lay["Wd"].data_ptr(),
                ys[i].data_ptr(), ms[i].data_ptr(), T, wl.d, wl.d_i, wl.r, wl.bank, wl.k]
        if backward:
            gp = [grads[n].data_ptr() for n in ("dx", "dA", "dB", "dWg", "dWu", "dWd")]
            rc = L.sfn_sparse_ffn_backward(*ptrs[:6], dys[i].data_ptr(), args.temperature, *gp,
                                           ptrs[7], T, wl.d, wl.d_i, wl.r, wl.bank, wl.k,
                                           ws.data_ptr(), ws_bytes, st_ptr)
        elif dense4x:
            rc = L.sfn_dense4x_forward(ptrs[0], ptrs[3], ptrs[4], ptrs[5], ptrs[6], ptrs[7], T,
                                       wl.d, wl.d_i, wl.bank, wl.k, ws.data_ptr(), ws_bytes,
                                       st_ptr)
        elif shard:
            rc = L.sfn_sparse_ffn_forward_partial(*ptrs, path_id, ws.data_ptr(), ws_bytes,
                                                  st_ptr)
            if world > 1:
                _capi.check(rc, "sfn_sparse_ffn_forward_partial")
                import torch.distributed as dist
                dist.all_reduce(ys[i])  # sum of the ranks' partial outputs
        elif wl.dtype == "bf16":
            rc = L.sfn_sparse_ffn_forward_path(*ptrs, path_id, ws.data_ptr(), ws_bytes, st_ptr)
        else:
            rc = L.sfn_sparse_ffn_forward_f32_ws(*ptrs, ws.data_ptr(), ws_bytes, st_ptr)
        _capi.check(rc, "sfn_sparse_ffn_forward")

    # eager warm-up (also compiles kernel attributes outside capture)
    with torch.cuda.stream(stream):
        for i in range(S):
            call(i, stream.cuda_stream)
    stream.synchronize()

    # graphs: one of S steps, and one of (K mod S) steps
    def capture(n):
        if n == 0:
            return None, 0
        g = torch.cuda.CUDAGraph()
        c0 = L.sfn_kernel_launch_count()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
            for i in range(n):
                call(i % S, stream.cuda_stream)
        return g, L.sfn_kernel_launch_count() - c0

    eager = shard and world > 1  # steps with a collective run eagerly
    if eager:
        g_full = g_rem = None
        c0 = L.sfn_kernel_launch_count()
        with torch.cuda.stream(stream):
            call(0, stream.cuda_stream)
        stream.synchronize()
        launches_per_step = L.sfn_kernel_launch_count() - c0
    else:
        g_full, launches_full = capture(S)
        g_rem, launches_rem = capture(K % S)
        launches_per_step = launches_full / S

    def replay(nsteps):
        if eager:
            for j in range(nsteps):
                call(j % S, stream.cuda_stream)
            return
        for _ in range(nsteps // S):
            g_full.replay()
        if nsteps % S:
            assert nsteps % S == K % S
            g_rem.replay()

    sampler = None
    if rank == 0:
        uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", "") or "")
        sampler = ClockSampler(uuid).start()

    # warm-up: W untimed steps, then keep the GPU loaded ~1 s so clocks settle
    with torch.cuda.stream(stream):
        if eager:
            # a fixed number of steps: every rank must make the same collective calls
            replay(W + int(args.settle * 1000))
        else:
            for _ in range(W // S):
                g_full.replay()
            for i in range(W % S):
                call(i, stream.cuda_stream)
            t_settle = time.time()
            while time.time() - t_settle < args.settle:
                g_full.replay()
        stream.synchronize()

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        replay(K)
        ev1.record(stream)
    stream.synchronize()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    elapsed_ms = ev0.elapsed_time(ev1)
    clocks = sampler.stop() if sampler else None
    elapsed_ms_max = aggregate_max(elapsed_ms, world, dev)

    # mask statistics of the last step on each layer: union of kept channels
    unions = []
    for i in range(S):
        m = ms[i].cpu().numpy().view(np.uint64)
        bits = np.unpackbits(m.view(np.uint8), bitorder="little").reshape(T, -1)
        unions.append(int(bits.any(axis=0).sum()))
    union = int(round(sum(unions) / len(unions)))

    # spread of the step time: R event-bracketed replays of the S-step graph
    dist_line = None
    if not eager:
        R = 50 if T <= 4096 else 10
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(R)]
        with torch.cuda.stream(stream):
            for a, b in evs:
                a.record(stream)
                g_full.replay()
                b.record(stream)
        stream.synchronize()
        per_step = sorted(a.elapsed_time(b) / S for a, b in evs)

        def pct(q):
            return per_step[min(R - 1, int(round(q * (R - 1))))]
        dist_line = {"reps": R, "steps_per_rep": S, "p10_ms": pct(0.1), "p50_ms": pct(0.5),
                     "p90_ms": pct(0.9)}

    # per-stage kernel times (a separate pass of eager steps, events on the stream)
    n_stage_steps = min(K, max(S, 2000 if T <= 64 else 8 * S))
    with torch.cuda.stream(stream):
        for i in range(S):
            call(i, stream.cuda_stream)
        stream.synchronize()
        _capi.check(L.sfn_timing_begin(), "sfn_timing_begin")
        for j in range(n_stage_steps):
            call(j % S, stream.cuda_stream)
        import ctypes
        ms_arr = (ctypes.c_double * TIMED_STAGES)()
        n_arr = (ctypes.c_uint64 * TIMED_STAGES)()
        _capi.check(L.sfn_timing_end(ms_arr, n_arr, TIMED_STAGES), "sfn_timing_end")
    stages = {}
    for s_id in range(TIMED_STAGES):
        if n_arr[s_id]:
            name = L.sfn_stage_name(s_id).decode()
            stages[name] = {"launches": int(n_arr[s_id]), "ms_total": ms_arr[s_id],
                            "us_per_launch": 1e3 * ms_arr[s_id] / n_arr[s_id],
                            # a stage may run more than once per step (split-K sums,
                            # the backward's groups of GEMMs): work is per step
                            "us_per_step": 1e3 * ms_arr[s_id] / n_stage_steps}
    tot = sum(v["ms_total"] for v in stages.values()) or 1.0
    for v in stages.values():
        v["share"] = v["ms_total"] / tot
    work = stage_work(wl, T, union)
    if "tc_gateup" in stages and "tc_logits_topk" not in stages:
        # one token tile: the logits GEMM and its top-k run inside the gate/up kernel
        work["tc_gateup"] = {k: work["tc_gateup"][k] + work["tc_logits_topk"][k]
                             for k in ("bytes", "flops")}
    bound = "hbm" if T <= 256 else "tensor"
    if "tc_down" in stages and "reduce" in stages:  # split-K partial sums
        work["reduce"] = {"bytes": T * wl.d * 4, "flops": 0}
    dom = max(stages, key=lambda n: stages[n]["ms_total"])
    dom_s = stages[dom]["us_per_step"] * 1e-6
    if bound == "hbm":
        achieved = work[dom]["bytes"] / dom_s / 1e9
        peak, unit = peaks["hbm_gbs"], "GB/s"
    else:
        # the tensor-bound steps keep the GPU loaded for seconds (settling and
        # timing), under the power cap: the sustained GEMM peak applies
        achieved = work[dom]["flops"] / dom_s / 1e12
        peak, unit = peaks["bf16_tflops_sustained"], "TFLOP/s"
    traffic = traffic_from_profiles(dom, workload)
    for n, v in stages.items():
        v["alg_bytes_per_launch"] = work[n]["bytes"]
        v["alg_gbs"] = work[n]["bytes"] / (v["us_per_step"] * 1e-6) / 1e9

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e and not backward and not shard:
        n_e2e = min(K, 300 if T <= 64 else (10 if main else 3))
        x_host = [xs[i].cpu().pin_memory() for i in range(S)]
        y_host = torch.empty((T, wl.d), dtype=wl.torch_dtype).pin_memory()
        m_host = torch.empty((T, wl.n_banks), dtype=torch.int64).pin_memory()
        x_dev = torch.empty_like(xs[0])
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for j in range(n_e2e):
                i = j % S
                # host input in, the C ABI call, host output back: what a caller does
                x_dev.copy_(x_host[i], non_blocking=True)
                lay = layers[i]
                if dense4x:
                    rc = L.sfn_dense4x_forward(x_dev.data_ptr(), lay["Wg"].data_ptr(),
                                               lay["Wu"].data_ptr(), lay["Wd"].data_ptr(),
                                               ys[i].data_ptr(), ms[i].data_ptr(), T, wl.d,
                                               wl.d_i, wl.bank, wl.k, ws.data_ptr(), ws_bytes,
                                               stream.cuda_stream)
                elif wl.dtype == "bf16":
                    rc = L.sfn_sparse_ffn_forward_path(
                        x_dev.data_ptr(), lay["A"].data_ptr(), lay["B"].data_ptr(),
                        lay["Wg"].data_ptr(), lay["Wu"].data_ptr(), lay["Wd"].data_ptr(),
                        ys[i].data_ptr(), ms[i].data_ptr(), T, wl.d, wl.d_i, wl.r, wl.bank,
                        wl.k, path_id, ws.data_ptr(), ws_bytes, stream.cuda_stream)
                else:
                    rc = L.sfn_sparse_ffn_forward_f32_ws(
                        x_dev.data_ptr(), lay["A"].data_ptr(), lay["B"].data_ptr(),
                        lay["Wg"].data_ptr(), lay["Wu"].data_ptr(), lay["Wd"].data_ptr(),
                        ys[i].data_ptr(), ms[i].data_ptr(), T, wl.d, wl.d_i, wl.r, wl.bank,
                        wl.k, ws.data_ptr(), ws_bytes, stream.cuda_stream)
                _capi.check(rc, "e2e forward")
                y_host.copy_(ys[i], non_blocking=True)
                m_host.copy_(ms[i], non_blocking=True)
                stream.synchronize()  # the caller reads the step's result
            e1.record(stream)
        stream.synchronize()
        e2e_ms = aggregate_max(e0.elapsed_time(e1), world, dev)
        e2e = {"value": world * T * n_e2e / (e2e_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": int(xs[0].numel() * xs[0].element_size()),
               "d2h_bytes_per_step": int(ys[0].numel() * ys[0].element_size()
                                          + ms[0].numel() * ms[0].element_size()),
               "steps": n_e2e}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the workloads beside the headline line take a shorter sample
        cpu = cpu_baseline(wl, {k: v.cpu() for k, v in layers[0].items()}, xs[0].cpu(),
                           budget_s=15.0 if main else 5.0, method=args.method)

    if world > 1:
        dist.barrier()
    del g_full, g_rem
    if rank != 0:
        return None

    # token replicas: every rank processes its own T tokens; bank shards: the
    # ranks share one batch of T tokens
    value = (1 if shard else world) * T * K / (elapsed_ms_max * 1e-3)
    # the path's algorithmic minimum: predictor weights, kept rows, x and y
    if dense4x:
        step_bytes = sum(work[n]["bytes"] for n in ("dense4x_gateup", "tc_down"))
    elif backward:
        step_bytes = sum(work[n]["bytes"] for n in ("pred_h", "logits_topk", "bwd_gemm",
                                                    "bwd_elem", "bwd_tau"))
    else:
        step_bytes = sum(work[n]["bytes"] for n in ("pred_h", "logits_topk", "ffn", "reduce"))
    step_flops = T * useful_flops_per_token(wl, args.method)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": elapsed_ms_max / K, "higher_is_better": True,
        "scaling": "strong" if shard else "weak", "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic",
        "config": {
            "workload": f"{wl_full.name}: T={T} d={wl_full.d} d_i={wl_full.d_i} r={wl_full.r} "
                        f"bank={wl_full.bank} k={wl_full.k} {wl_full.dtype}",
            "T": T, "d": wl_full.d, "d_i": wl_full.d_i, "r": wl_full.r, "bank": wl_full.bank,
            "k": wl_full.k, "method": args.method,
            "l2": (f"inputs larger than L2: steps rotate over {S} distinct layers "
                   f"({S * sum(v.numel() * v.element_size() for v in layers[0].values()) / 1e9:.2f}"
                   " GB of weights)"),
            "parallelism": (f"bank shards x{world} (all-reduce of float32 partial y)" if shard
                            else f"replica x{world} (token batches independent)"),
            "path": args.path,
            "timing": ("eager steps (each ends in an all-reduce)" if eager else
                       "CUDA graph replay of the steps") + ", CUDA events on the launching stream",
            **({"shard": f"rank 0 holds banks {b0}..{b1 - 1}; roofline figures are per rank"}
               if shard else {}),
        },
        "roofline": {"bound": bound, "kernel": dom, "achieved": achieved, "peak": peak,
                     "unit": unit, "frac": achieved / peak, "traffic": traffic,
                     "peak_source": peaks["source"],
                     "peak_kind": "copy bandwidth" if bound == "hbm" else "sustained bf16 GEMM",
                     "alg_per_launch": work[dom]["bytes"] if bound == "hbm" else work[dom]["flops"]},
        "step_roofline": {
            "bytes_per_step": step_bytes, "flops_per_step_useful": step_flops,
            "achieved_gbs": step_bytes / (elapsed_ms_max / K * 1e-3) / 1e9,
            "frac_hbm": step_bytes / (elapsed_ms_max / K * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "achieved_tflops_useful": step_flops / (elapsed_ms_max / K * 1e-3) / 1e12,
            "frac_tensor": step_flops / (elapsed_ms_max / K * 1e-3) / 1e12
                           / peaks["bf16_tflops_sustained"],
        },
        "step_time_spread": dist_line,
        "stages": stages,
        "mask_union_channels": union,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(round(launches_per_step * K * world)),
        "clocks": clocks,
    }
    return line


def cpu_baseline(wl, layer_host, x_host, budget_s=15.0, method="sfn"):
    """The oracle, as it stands, on a bounded sample of the same workload."""
    import numpy as np

    import oracle
    oracle.build()
    cores = oracle.num_threads()

    def run(xb):
        if method == "dense4x":
            oracle.dense4x(xb, layer_host["Wg"], layer_host["Wu"], layer_host["Wd"], wl.bank,
                           wl.k)
        elif method == "backward":
            dy = np.random.default_rng(1000).standard_normal(xb.shape)
            oracle.backward(xb, layer_host["A"], layer_host["B"], layer_host["Wg"],
                            layer_host["Wu"], layer_host["Wd"], dy, wl.bank, wl.k, 1.0)
        else:
            oracle.forward(xb, layer_host["A"], layer_host["B"], layer_host["Wg"],
                           layer_host["Wu"], layer_host["Wd"], wl.bank, wl.k)

    t0 = time.perf_counter()
    run(x_host[:1])
    t1 = time.perf_counter() - t0
    # about budget_s of work: one token on one core took t1, tokens run on `cores`
    # threads (assumed ~70 % parallel efficiency)
    n = max(1, min(16384, int(0.7 * budget_s * max(cores, 1) / max(t1, 1e-3))))
    import torch
    reps = math.ceil(n / x_host.shape[0])
    xb = torch.cat([x_host] * reps)[:n]
    t0 = time.perf_counter()
    run(xb)
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": UNIT, "cores": min(cores, n), "kind": "oracle",
            "sample": f"{n} tokens of the {wl.name} workload (T={wl.T} per step) through the "
                      f"fp64 oracle ({method}), OpenMP over tokens, {dt:.1f} s"}


# ---------------------------------------------------------------- the reference arm

def run_reference(args, rank, world):
    if rank != 0:
        return None
    import numpy as np
    import torch

    import oracle
    from predictor_gated_channel_b200.inputs import WORKLOADS, make_layer, make_tokens
    wl = WORKLOADS[args.workload]
    if args.k is not None:
        wl = wl.with_(k=args.k)
    oracle.build()
    cores = oracle.num_threads()
    K = args.steps if args.steps is not None else default_steps(args.workload)
    W = max(3, args.warmup if args.warmup is not None else 20)
    layer = make_layer(wl)
    # one step = one forward on a bounded sample of the workload's T tokens
    T_step = min(wl.T, max(1, cores))
    x = make_tokens(wl, T=T_step * 4)

    def step(j):
        s = (j % 4) * T_step
        if args.method == "dense4x":
            oracle.dense4x(x[s:s + T_step], layer["Wg"], layer["Wu"], layer["Wd"], wl.bank, wl.k)
        elif args.method == "backward":
            dy = np.random.default_rng(1000 + j).standard_normal((T_step, wl.d))
            oracle.backward(x[s:s + T_step], layer["A"], layer["B"], layer["Wg"], layer["Wu"],
                            layer["Wd"], dy, wl.bank, wl.k, args.temperature)
        else:
            oracle.forward(x[s:s + T_step], layer["A"], layer["B"], layer["Wg"], layer["Wu"],
                           layer["Wd"], wl.bank, wl.k)

    t0 = time.perf_counter()
    step(0)
    t_one = time.perf_counter() - t0
    budget = 150.0
    W_eff = min(W, max(1, int(20.0 / max(t_one, 1e-3))))
    K_eff = min(K, max(1, int(budget / max(t_one, 1e-3))))
    for j in range(W_eff):
        step(j)
    t0 = time.perf_counter()
    for j in range(K_eff):
        step(j)
    dt = time.perf_counter() - t0
    value = T_step * K_eff / dt
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": K_eff, "warmup": W_eff, "ms_per_step": 1e3 * dt / K_eff,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"{wl.name}: T={wl.T} d={wl.d} d_i={wl.d_i} r={wl.r} "
                               f"bank={wl.bank} k={wl.k} {wl.dtype}",
                   "T": wl.T, "d": wl.d, "d_i": wl.d_i, "r": wl.r, "bank": wl.bank, "k": wl.k,
                   "method": args.method},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(cores, T_step),
                         "kind": "oracle",
                         "sample": f"{T_step} tokens per step (of T={wl.T}), {K_eff} steps"
                                   + (f" (of {K} requested; capped to ~{budget:.0f} s)"
                                      if K_eff < K else "")},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_env()
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        line = run_sfn(args, rank, world, local)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
