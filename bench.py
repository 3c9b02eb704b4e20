#!/usr/bin/env python
"""Benchmark of the gated delta-rule forward on B200.

One step = one chunked forward (pdn_chunk_fwd) of the Preconditioned GDN
layer workload: B=4 sequences x T=4096 tokens x H=16 heads, d_k = d_v = 128,
bf16 q/k/v/o, fp32 state, scalar decay, diagonal preconditioner. Inputs are
resident in HBM before the timed region; L2 is flushed (256 MiB write) between
timed steps. The JSON line also carries:
  e2e         the same metric end to end through pdn_chunk_fwd_host from
              pinned HOST buffers (host->device inputs and device->host
              output, final state and accumulator per step, overlapped with
              the compute over batch slices);
  roofline    one pdn_chunk_fwd call (its kernels timed as one launch by the
              CUDA events around it) against the measured bf16 tensor peak;
  decode      the recurrent decode workload (256 sequences x 16 heads,
              fp32 state, 1024 steps), tokens/s and HBM roofline;
  workloads   the other forward workloads (Preconditioned KDA B8 T8192;
              FG2-GDN and Gated DeltaNet-2 B2 T32768; preconditioned linear
              attention and FG2-GDN+ at the headline shape): tokens/s, tensor and
              HBM fractions, and per-kernel CUDA-event times (also given for
              the headline layer under roofline.kernel_ms);
  backward    the gradient of the headline layer (pdn_chunk_bwd, every
              input's gradient from dO and dS_T): tokens/s and its fraction
              of the fp32 CUDA-core peak (an ALU-bound pass);
  backward_prologue  the same from the layer's raw projections (gradients
              through the fused prologue's activations);
  train_step  one forward + backward of the headline layer in training mode
              (the forward saves delta and the chunk-start states, the
              backward skips its forward sweep), against the plain pair;
  cpu_baseline the fp64 oracle on the host cores on a bounded sample.
Multi-GPU (torchrun): every rank runs its own independent batch (weak
scaling, no collective on the data path); the time is the max over ranks.

`--impl reference` times the fp64 CPU oracle (the only reference this path
has) on the same workload, on a bounded sample per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# Algorithmic tensor-core work of the chunk form per (token, head) at chunk C:
# 2C(3 d_k + 2 d_v) for the C^2 products (M, P, Y, U, P.Delta) and
# 6 d_k d_v for the state products (Y S^T, Q S^T, Delta^T W).
def chunk_flops_per_token_head(C, dk, dv):
    return 2 * C * (3 * dk + 2 * dv) + 6 * dk * dv


def fwd_bytes_per_token_head(w):
    """Inputs read once + output written once (bf16 q, k, v, o; fp32 scalar
    gates; per-channel gates at the element size)."""
    es = 2 if w.dtype == "bf16" else 4
    b = es * (2 * w.dk + 2 * w.dv)
    if w.variant in ("FG2_GDN",):
        b += es * w.dk
    elif w.variant == "FG2_GDN_PLUS":
        b += es * (w.dk + w.dv)
    elif w.variant != "GDN2":
        b += 4
    if w.variant == "GDN2":
        b += es * (w.dk + w.dv)
    if w.decay == "scalar":
        b += 4
    elif w.decay == "channel":
        b += es * w.dk
    return b


def decode_bytes_per_token_head(w):
    """State read + write (fp32), accumulator read + write, token inputs and output."""
    es = 2 if w.dtype == "bf16" else 4
    b = 8 * w.dk * w.dv + es * (2 * w.dk + 2 * w.dv) + 4 + 4
    if w.variant in ("PDN", "PGDN", "PKDA"):
        b += 8 * w.dk
    return b


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def traffic_for(kernel_key, files):
    """DRAM traffic per launch from the committed ncu summary, or None when
    the kernel sources changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel_key)
    if not d or d.get("source_hash") != kernel_source_hash(files):
        return None
    return d.get("bytes_per_launch")


# Sources of the kernels one pdn_chunk_fwd call launches on the d = 128 bf16
# workloads (the three-kernel tensor-core path that automatic selection picks).
CHUNK_SOURCES = ["linear_recurrence_sequence_chunked_b200/csrc/chunk_split.cu",
                 "linear_recurrence_sequence_chunked_b200/csrc/tiles.cuh",
                 "linear_recurrence_sequence_chunked_b200/csrc/common.cuh",
                 "linear_recurrence_sequence_chunked_b200/csrc/ptx.cuh"]
DECODE_SOURCES = ["linear_recurrence_sequence_chunked_b200/csrc/decode.cu",
                  "linear_recurrence_sequence_chunked_b200/csrc/common.cuh"]


# ------------------------------------------------------------------ multi-rank host logic
def rank_seed(seed, rank):
    """Each rank draws its own independent batch (weak scaling: per-GPU work
    is fixed, nothing is exchanged on the data path)."""
    return seed + 1000 * rank


def max_over_ranks(x, world, device=None):
    """The slowest rank's device time; one all-reduce of a scalar (any
    torch.distributed backend), outside the data path."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(units_per_rank, world, ms_max):
    """Whole-job units per second: every rank's units over the max time."""
    return world * units_per_rank / (ms_max / 1e3)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle timing
def oracle_sample_rate(w, target_s=12.0, nthreads=None):
    """Times the fp64 oracle on a bounded sample of workload w (whole chains of
    T tokens). Returns (tokens/s, threads used, sample description)."""
    import oracle
    from linear_recurrence_sequence_chunked_b200.workloads import make_inputs
    nthreads = nthreads or os.cpu_count() or 1
    oracle.build()
    # probe: one chain per thread over a short prefix to size the sample
    Tp = min(w.T, 256)
    x = make_inputs(w.replace(seed=w.seed + 17), B=max(1, -(-nthreads // w.H)), T=Tp)
    t0 = time.perf_counter()
    oracle.forward(w.variant, x["q"], x["k"], x["v"], log_alpha=x["log_alpha"], beta=x["beta"],
                   erase=x["erase"], write=x["write"], x=w.precond_x, eps=w.precond_eps,
                   nthreads=nthreads)
    dt = max(time.perf_counter() - t0, 1e-6)
    chains_probe = x["k"].shape[0] * w.H
    rate = chains_probe * Tp / dt  # token-heads per second
    # whole chains of T tokens, batches of H heads, about target_s of work
    chains = max(1, int(rate * target_s / w.T))
    Bs = max(1, min(w.B * 4, -(-chains // w.H)))
    x = make_inputs(w, B=Bs)
    t0 = time.perf_counter()
    oracle.forward(w.variant, x["q"], x["k"], x["v"], log_alpha=x["log_alpha"], beta=x["beta"],
                   erase=x["erase"], write=x["write"], x=w.precond_x, eps=w.precond_eps,
                   nthreads=nthreads)
    dt = time.perf_counter() - t0
    tok = Bs * w.T  # tokens (all H heads) processed
    desc = "%d sequences x %d tokens x %d heads (%s, d=%d), fp64 token loop, %d threads" % (
        Bs, w.T, w.H, w.variant, w.dk, nthreads)
    return tok / dt, nthreads, desc, dt


# ------------------------------------------------------------------ GPU arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    from linear_recurrence_sequence_chunked_b200 import build as pdn_build
    from linear_recurrence_sequence_chunked_b200 import pdn
    from linear_recurrence_sequence_chunked_b200.workloads import WORKLOADS, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    if rank == 0:
        pdn_build.build()
    if world > 1:
        dist.barrier()
    pdn.load()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def mor(x):
        return max_over_ranks(x, world, dev)

    w = WORKLOADS[args.workload]
    peaks, peaks_kind = load_peaks()
    # each rank: its own independent batch (different seed)
    wr = w.replace(seed=rank_seed(w.seed, rank))
    x = make_inputs(wr, device=dev, generator_device=dev)
    g = {n: x[n] for n in ("log_alpha", "beta", "erase", "write")}
    impl = args.kernel
    o = torch.empty(w.B, w.T, w.H, w.dv, dtype=x["v"].dtype, device=dev)
    prob = pdn.make_problem(w.variant, w.B, w.T, w.H, w.dk, w.dv, x["k"].dtype, w.decay, w.chunk,
                            impl, w.q_scale, w.precond_x, w.precond_eps)
    ws_bytes = pdn.pdn_chunk_fwd_workspace(prob)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    ST = torch.empty(w.B, w.H, w.dv, w.dk, dtype=torch.float32, device=dev)
    AT = torch.empty(w.B, w.H, w.dk, dtype=torch.float32, device=dev) \
        if w.variant in pdn.PRECOND_VARIANTS else None
    tens = pdn.make_tensors(x["q"], x["k"], x["v"], o, **g, ST=ST, AT=AT)
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def step():
        rc = pdn.pdn_chunk_fwd(prob, tens, ws.data_ptr(), ws.numel(), sptr)
        if rc != pdn.PDN_OK:
            raise pdn.PdnError(rc, "pdn_chunk_fwd")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if pdn.device_error() != pdn.PDN_OK:
        raise SystemExit("device error during warm-up")

    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    with ClockSampler(gpu_index) as clk:
        barrier()
        for i in range(args.steps):
            flush.fill_(float(i))  # > L2: no reuse of the previous step's lines
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        barrier()
    clocks = clk.summary()
    ms_local = sum(a.elapsed_time(b) for a, b in ev)
    ms = mor(ms_local)
    tokens = world * w.B * w.T * args.steps
    value = throughput(w.B * w.T * args.steps, world, ms)
    ms_launch = ms_local / args.steps
    flops = chunk_flops_per_token_head(w.chunk, w.dk, w.dv) * w.B * w.T * w.H
    ach_tflops = flops / (ms_launch / 1e3) / 1e12
    peak = peaks["bf16_tflops"]
    if pdn.device_error() != pdn.PDN_OK:
        raise SystemExit("device error during the timed region")
    impl_id = pdn.pdn_chunk_fwd_impl(prob)
    tc = impl_id == pdn.IMPLS["tc"]
    kernel_name = {1: "simt", 2: "tcgen05 split (K0 key energy + prefix, K1 intra-chunk, K2 state)"
                   }.get(impl_id, "?")
    launches_per_step = 1
    if impl_id == pdn.IMPLS["tc"]:
        launches_per_step = 4 if w.variant in pdn.PRECOND_VARIANTS else 2

    result = {
        "metric": "fwd tokens/s per layer (H16,d128,T4K) + % roofline; decode tokens/s",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if tc else "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "variant": w.variant, "B": w.B, "T": w.T, "H": w.H,
                   "d_k": w.dk, "d_v": w.dv, "chunk": w.chunk, "inputs": w.dtype,
                   "state": "f32", "kernel": kernel_name,
                   "per_gpu_batch": w.B, "global_batch": w.B * world,
                   "l2": "flushed between timed steps (256 MiB write)",
                   "parallelism": "dp%d" % world},
        "roofline": {"bound": "tensor", "achieved": ach_tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": ach_tflops / peak, "peak_kind": peaks_kind + " bf16 burst",
                     "launch": "one pdn_chunk_fwd call (%d kernels), CUDA events on its stream"
                               % launches_per_step,
                     "flops_per_launch": flops,
                     "traffic": traffic_for("chunk_fwd:" + w.name, CHUNK_SOURCES)},
        "clocks": clocks,
        "gpu_launches": args.steps * launches_per_step,
    }

    result["roofline"]["kernel_ms"] = profiled_kernel_ms(pdn, prob, tens, ws, sptr)

    # ---------------- e2e: pinned host buffers, copies inside the timed region
    if not args.no_e2e:
        hx = {n: (t.cpu().pin_memory() if t is not None else None) for n, t in x.items()}
        ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        # the final state (and accumulator) come back too: what a caller
        # continuing the sequence needs
        hST = torch.empty(ST.shape, dtype=ST.dtype).pin_memory()
        hAT = torch.empty(AT.shape, dtype=AT.dtype).pin_memory() if AT is not None else None
        dx = {n: (torch.empty_like(t, device=dev) if t is not None else None) for n, t in hx.items()}
        dtens = pdn.make_tensors(dx["q"], dx["k"], dx["v"], o, dx["log_alpha"], dx["beta"],
                                 dx["erase"], dx["write"], ST=ST, AT=AT)
        h2d = sum(t.numel() * t.element_size() for t in hx.values() if t is not None)
        d2h = sum(t.numel() * t.element_size() for t in (ho, hST, hAT) if t is not None)

        htens = pdn.make_host_tensors(hx["q"], hx["k"], hx["v"], ho, hx["log_alpha"],
                                      hx["beta"], hx["erase"], hx["write"], ST=hST, AT=hAT)
        slices = w.B  # one batch element per part: copy in / compute / copy out overlap

        def e2e_step():
            rc = pdn.pdn_chunk_fwd_host(prob, htens, dtens, ws.data_ptr(), ws.numel(), slices,
                                        sptr)
            if rc != pdn.PDN_OK:
                raise pdn.PdnError(rc, "pdn_chunk_fwd_host")

        for _ in range(max(1, args.warmup)):
            e2e_step()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        barrier()
        ems = mor(e0.elapsed_time(e1))
        result["e2e"] = {"value": tokens / (ems / 1e3), "unit": "tokens/s",
                         "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                         "ms_per_step": ems / args.steps,
                         "path": "pdn_chunk_fwd_host, %d batch slices" % slices}
        result["gpu_launches"] += args.steps * launches_per_step * slices
        del hx, ho, hST, hAT, dx

    # ---------------- the other forward workloads
    if not args.no_extra:
        del ws
        torch.cuda.empty_cache()
        result["workloads"] = {}
        for name in EXTRA_WORKLOADS:
            fused = name.endswith("+prologue")
            r = bench_workload(args, WORKLOADS[name.split("+")[0]], dev, stream, peaks, peaks_kind,
                               rank, mor, barrier, fused_prologue=fused)
            result["workloads"][name] = r
            result["gpu_launches"] += r["gpu_launches"]
            torch.cuda.empty_cache()

    # ---------------- backward of the headline layer
    if not args.no_backward:
        torch.cuda.empty_cache()
        result["backward"] = bench_backward(args, w, dev, stream, rank, mor, barrier)
        result["backward_prologue"] = bench_backward(args, w, dev, stream, rank, mor, barrier,
                                                     raw=True)
        result["gpu_launches"] += (result["backward"]["gpu_launches"]
                                   + result["backward_prologue"]["gpu_launches"])
        torch.cuda.empty_cache()
        if tc:
            result["train_step"] = bench_train(args, w, dev, stream, rank, mor, barrier,
                                               result["ms_per_step"]
                                               + result["backward"]["ms_per_step"])
            result["gpu_launches"] += result["train_step"]["gpu_launches"]
            torch.cuda.empty_cache()

    # ---------------- decode workload
    if not args.no_decode:
        result["decode"] = bench_decode(args, dev, stream, peaks, peaks_kind, world, rank,
                                        mor, barrier)
        result["gpu_launches"] += result["decode"]["gpu_launches"]

    # ---------------- CPU baseline (rank 0, N=1 only)
    if world == 1 and not args.no_cpu_baseline:
        rate, cores, desc, secs = oracle_sample_rate(w, target_s=args.cpu_seconds)
        result["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores,
                                  "kind": "oracle", "sample": desc, "seconds": secs}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# "+prologue": the same layer from raw projections, with L2 normalisation,
# sigmoid gains and the softplus decay fused into the kernels
EXTRA_WORKLOADS = ("pkda_bf16_8k", "fg2_bf16_32k", "gdn2_bf16_32k", "pla_bf16_4k", "fg2p_bf16_4k",
                   "pgdn_bf16_4k+prologue")


def profiled_kernel_ms(pdn, prob, tens, ws, sptr, reps=3):
    """Mean per-stage milliseconds of pdn_chunk_fwd (CUDA events between its
    kernels, outside the timed region): key-energy prefix, intra-chunk
    kernel, state kernel."""
    acc = None
    for _ in range(reps):
        rc, ms = pdn.pdn_chunk_fwd_profiled(prob, tens, ws.data_ptr(), ws.numel(), sptr)
        if rc != pdn.PDN_OK:
            raise pdn.PdnError(rc, "pdn_chunk_fwd_profiled")
        acc = ms if acc is None else [a + b for a, b in zip(acc, ms)]
    names = ["k0_key_energy", "k1_intra", "k2_state"] if len(acc) == 3 else ["chunk_simt"]
    return {n: v / reps for n, v in zip(names, acc)}


def bench_workload(args, w, dev, stream, peaks, peaks_kind, rank, mor, barrier,
                   fused_prologue=False):
    """Times `args.steps` forward calls of workload w (inputs resident in HBM
    and larger than L2, so no flush), after warm-up."""
    import torch

    from linear_recurrence_sequence_chunked_b200 import pdn
    from linear_recurrence_sequence_chunked_b200.workloads import (make_inputs, make_raw_inputs,
                                                                   raw_prologue)

    wr = w.replace(seed=rank_seed(w.seed, rank))
    bits, dscale = raw_prologue(w) if fused_prologue else (0, 1.0)
    x = (make_raw_inputs if fused_prologue else make_inputs)(wr, device=dev, generator_device=dev)
    g = {n: x[n] for n in ("log_alpha", "beta", "erase", "write")}
    o = torch.empty(w.B, w.T, w.H, w.dv, dtype=x["v"].dtype, device=dev)
    prob = pdn.make_problem(w.variant, w.B, w.T, w.H, w.dk, w.dv, x["k"].dtype, w.decay, w.chunk,
                            "auto", w.q_scale, w.precond_x, w.precond_eps, bits, dscale)
    ws_bytes = pdn.pdn_chunk_fwd_workspace(prob)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    ST = torch.empty(w.B, w.H, w.dv, w.dk, dtype=torch.float32, device=dev)
    AT = torch.empty(w.B, w.H, w.dk, dtype=torch.float32, device=dev) \
        if w.variant in pdn.PRECOND_VARIANTS else None
    tens = pdn.make_tensors(x["q"], x["k"], x["v"], o, **g, ST=ST, AT=AT)
    sptr = stream.cuda_stream

    def step():
        rc = pdn.pdn_chunk_fwd(prob, tens, ws.data_ptr(), ws.numel(), sptr)
        if rc != pdn.PDN_OK:
            raise pdn.PdnError(rc, "pdn_chunk_fwd")

    for _ in range(args.warmup):
        step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    barrier()
    ms_local = e0.elapsed_time(e1)
    ms = mor(ms_local)
    if pdn.device_error() != pdn.PDN_OK:
        raise SystemExit("device error during the %s timed region" % w.name)
    per = ms_local / args.steps
    flops = chunk_flops_per_token_head(w.chunk, w.dk, w.dv) * w.B * w.T * w.H
    nbytes = fwd_bytes_per_token_head(w) * w.B * w.T * w.H + 4 * w.B * w.H * w.dv * w.dk
    launches = 4 if w.variant in pdn.PRECOND_VARIANTS else 2
    res = {"variant": w.variant, "B": w.B, "T": w.T, "H": w.H, "d": w.dk, "inputs": w.dtype,
           "prologue": "fused (raw projections)" if fused_prologue else "none",
           "value": w.B * w.T * args.steps / (ms / 1e3), "unit": "tokens/s",
           "ms_per_step": ms / args.steps,
           "tensor": {"achieved": flops / (per / 1e3) / 1e12, "peak": peaks["bf16_tflops"],
                      "unit": "TFLOP/s", "frac": flops / (per / 1e3) / 1e12 / peaks["bf16_tflops"],
                      "flops_per_launch": flops},
           "hbm": {"achieved": nbytes / (per / 1e3) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                   "frac": nbytes / (per / 1e3) / 1e9 / peaks["hbm_gbs"],
                   "bytes_per_launch": nbytes},
           "peak_kind": peaks_kind,
           "kernel_ms": profiled_kernel_ms(pdn, prob, tens, ws, sptr),
           "l2": "inputs larger than L2 (no flush)",
           "gpu_launches": args.steps * launches}
    del x, g, o, ws, ST, AT, tens
    return res


# fp32 CUDA-core peak from the unit counts and the maximum SM clock: 148 SMs x
# 128 fp32 lanes x 2 flops (FMA) x 1965 MHz
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def bwd_flops_per_token_head(dk, dv):
    """Elementwise state work of the four backward sweeps per (token, head),
    an FMA counted as 2: forward delta sweep 5, reverse cotangent sweep 7,
    forward dq'/dr sweep 7, reverse dw sweep 7 flops per state element."""
    return 26 * dk * dv


def bench_backward(args, w, dev, stream, rank, mor, barrier, raw=False):
    """Times `args.steps` pdn_chunk_bwd calls of the headline layer (inputs and
    cotangents resident in HBM, larger than L2), after warm-up; with `raw`,
    from the raw projections through the fused prologue."""
    import torch

    from linear_recurrence_sequence_chunked_b200 import pdn
    from linear_recurrence_sequence_chunked_b200.workloads import (make_inputs, make_raw_inputs,
                                                                   raw_prologue)

    wr = w.replace(seed=rank_seed(w.seed, rank))
    if raw:
        x = make_raw_inputs(wr, device=dev, generator_device=dev)
        bits, dscale = raw_prologue(w)
    else:
        x = make_inputs(wr, device=dev, generator_device=dev)
        bits, dscale = 0, 1.0
    gen = torch.Generator(device=dev).manual_seed(rank_seed(7, rank))
    dO = torch.randn(w.B, w.T, w.H, w.dv, generator=gen, device=dev).to(x["v"].dtype)
    dST = torch.randn(w.B, w.H, w.dv, w.dk, generator=gen, device=dev)
    prob = pdn.make_problem(w.variant, w.B, w.T, w.H, w.dk, w.dv, x["k"].dtype, w.decay, w.chunk,
                            "auto", w.q_scale, w.precond_x, w.precond_eps, bits, dscale)
    f32 = dict(dtype=torch.float32, device=dev)
    g = {n: torch.empty_like(x[n], **f32) for n in ("q", "k", "v")}
    g["log_alpha"] = torch.empty_like(x["log_alpha"], **f32)
    g["beta"] = torch.empty_like(x["beta"], **f32)
    g["S0"] = torch.empty(w.B, w.H, w.dv, w.dk, **f32)
    g["A0"] = torch.empty(w.B, w.H, w.dk, **f32)
    tens = pdn.make_tensors(x["q"], x["k"], x["v"], None, x["log_alpha"], x["beta"])
    grads = pdn.make_grads(dO, dST, g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], None, None,
                           g["S0"], g["A0"])
    ws = torch.empty(pdn.pdn_chunk_bwd_workspace(prob), dtype=torch.uint8, device=dev)
    sptr = stream.cuda_stream

    def step():
        rc = pdn.pdn_chunk_bwd(prob, tens, grads, ws.data_ptr(), ws.numel(), sptr)
        if rc != pdn.PDN_OK:
            raise pdn.PdnError(rc, "pdn_chunk_bwd")

    for _ in range(args.warmup):
        step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    barrier()
    ms_local = e0.elapsed_time(e1)
    ms = mor(ms_local)
    if pdn.device_error() != pdn.PDN_OK:
        raise SystemExit("device error during the backward timed region")
    per = ms_local / args.steps
    flops = bwd_flops_per_token_head(w.dk, w.dv) * w.B * w.T * w.H
    # preconditioner prefix (block totals of k.k, carries), generic vectors,
    # the row sweeps (one launch), F2, R2, the chain rules; the decay's
    # final-state term and suffix sum (3 scan passes; the decay map's
    # derivative under the prologue); the preconditioner's suffix (block
    # totals, carries, dk update)
    launches = 2 + 1 + 1 + 2 + 1 + (1 + 3 + (1 if bits else 0)) + 3
    res = {"workload": w.name, "variant": w.variant, "value": w.B * w.T * args.steps / (ms / 1e3),
           "unit": "tokens/s", "ms_per_step": ms / args.steps,
           "roofline": {"bound": "alu", "achieved": flops / (per / 1e3) / 1e12,
                        "peak": FP32_ALU_TFLOPS, "unit": "TFLOP/s",
                        "frac": flops / (per / 1e3) / 1e12 / FP32_ALU_TFLOPS,
                        "flops_per_launch": flops,
                        "peak_kind": "fp32 CUDA-core peak from unit counts x 1965 MHz"},
           "gradients": ("q, k, v, log_alpha, beta, S0, A0 (fp32) from dO and dS_T"
                         + (", with respect to the raw projections (fused prologue)" if raw else "")),
           "l2": "inputs larger than L2 (no flush)",
           "gpu_launches": args.steps * launches}
    del x, dO, dST, g, ws, grads, tens
    return res


def bench_train(args, w, dev, stream, rank, mor, barrier, plain_ms):
    """Times `args.steps` training steps of the headline layer in training
    mode: pdn_chunk_fwd_save (the forward, also leaving every token's delta and
    the chunk-start states) then pdn_chunk_bwd_saved (the backward without its
    forward sweep). Each half is also timed alone; `plain_ms` is the forward
    plus backward measured above, for comparison."""
    import torch

    from linear_recurrence_sequence_chunked_b200 import pdn
    from linear_recurrence_sequence_chunked_b200.workloads import make_inputs

    wr = w.replace(seed=rank_seed(w.seed, rank))
    x = make_inputs(wr, device=dev, generator_device=dev)
    gen = torch.Generator(device=dev).manual_seed(rank_seed(7, rank))
    dO = torch.randn(w.B, w.T, w.H, w.dv, generator=gen, device=dev).to(x["v"].dtype)
    dST = torch.randn(w.B, w.H, w.dv, w.dk, generator=gen, device=dev)
    prob = pdn.make_problem(w.variant, w.B, w.T, w.H, w.dk, w.dv, x["k"].dtype, w.decay, w.chunk,
                            "auto", w.q_scale, w.precond_x, w.precond_eps)
    f32 = dict(dtype=torch.float32, device=dev)
    o = torch.empty(w.B, w.T, w.H, w.dv, dtype=x["v"].dtype, device=dev)
    ST = torch.empty(w.B, w.H, w.dv, w.dk, **f32)
    AT = torch.empty(w.B, w.H, w.dk, **f32) if w.variant in pdn.PRECOND_VARIANTS else None
    delta = torch.empty(w.B, w.H, w.T, w.dv, **f32)
    ckpt = torch.empty(w.B, w.H, (w.T + 63) // 64, w.dk, w.dv, **f32)
    g = {n: torch.empty_like(x[n], **f32) for n in ("q", "k", "v")}
    g["log_alpha"] = torch.empty_like(x["log_alpha"], **f32)
    g["beta"] = torch.empty_like(x["beta"], **f32)
    g["S0"] = torch.empty(w.B, w.H, w.dv, w.dk, **f32)
    g["A0"] = torch.empty(w.B, w.H, w.dk, **f32)
    tens = pdn.make_tensors(x["q"], x["k"], x["v"], o, x["log_alpha"], x["beta"], ST=ST, AT=AT)
    grads = pdn.make_grads(dO, dST, g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], None, None,
                           g["S0"], g["A0"])
    fws = torch.empty(max(1, pdn.pdn_chunk_fwd_workspace(prob)), dtype=torch.uint8, device=dev)
    bws = torch.empty(pdn.pdn_chunk_bwd_workspace(prob), dtype=torch.uint8, device=dev)
    sptr = stream.cuda_stream

    def fwd():
        rc = pdn.pdn_chunk_fwd_save(prob, tens, delta.data_ptr(), ckpt.data_ptr(), fws.data_ptr(),
                                    fws.numel(), sptr)
        if rc != pdn.PDN_OK:
            raise pdn.PdnError(rc, "pdn_chunk_fwd_save")

    def bwd():
        rc = pdn.pdn_chunk_bwd_saved(prob, tens, grads, delta.data_ptr(), ckpt.data_ptr(),
                                     bws.data_ptr(), bws.numel(), sptr)
        if rc != pdn.PDN_OK:
            raise pdn.PdnError(rc, "pdn_chunk_bwd_saved")

    def timed(body):
        for _ in range(args.warmup):
            body()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            body()
        e1.record(stream)
        barrier()
        return mor(e0.elapsed_time(e1)) / args.steps

    ms = timed(lambda: (fwd(), bwd()))
    ms_fwd = timed(fwd)
    ms_bwd = timed(bwd)
    if pdn.device_error() != pdn.PDN_OK:
        raise SystemExit("device error during the training-step timed region")
    fwd_launches = 4 if w.variant in pdn.PRECOND_VARIANTS else 2
    launches = fwd_launches + 2 + 1 + 1 + 2 + 1 + 4 + 3
    res = {"workload": w.name, "variant": w.variant,
           "value": w.B * w.T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
           "forward_save_ms": ms_fwd, "backward_saved_ms": ms_bwd,
           "plain_step_ms": plain_ms, "speedup_vs_plain": plain_ms / ms if plain_ms else None,
           "what": ("pdn_chunk_fwd_save + pdn_chunk_bwd_saved: the forward leaves delta and the "
                    "chunk-start states (fp32), the backward skips its forward row sweep; "
                    "gradients at bf16 accuracy"),
           "l2": "inputs larger than L2 (no flush)",
           # the step loop, then the forward and the backward loops alone
           "gpu_launches": 2 * args.steps * launches}
    del x, dO, dST, g, fws, bws, grads, tens, delta, ckpt
    return res


def bench_decode(args, dev, stream, peaks, peaks_kind, world, rank, mor, barrier):
    import torch

    from linear_recurrence_sequence_chunked_b200 import pdn
    from linear_recurrence_sequence_chunked_b200.workloads import WORKLOADS, make_inputs

    w = WORKLOADS["pgdn_decode_256"]
    steps = args.decode_steps
    wr = w.replace(seed=rank_seed(w.seed, rank))
    x = make_inputs(wr, device=dev, generator_device=dev, T=steps)
    # step-major copies so that each step's token slice is contiguous
    xs = {n: (t.transpose(0, 1).contiguous() if t is not None else None) for n, t in x.items()}
    del x
    S = torch.zeros(w.B, w.H, w.dv, w.dk, dtype=torch.float32, device=dev)
    A = torch.zeros(w.B, w.H, w.dk, dtype=torch.float32, device=dev)
    o = torch.empty(steps, w.B, 1, w.H, w.dv, dtype=torch.bfloat16, device=dev)
    prob = pdn.make_problem(w.variant, w.B, 1, w.H, w.dk, w.dv, torch.bfloat16, w.decay, 64,
                            "auto", w.q_scale, w.precond_x, w.precond_eps)
    tens = []
    for s in range(steps):
        sl = {n: (t[s] if t is not None else None) for n, t in xs.items()}
        tens.append(pdn.make_tensors(sl["q"], sl["k"], sl["v"], o[s], sl["log_alpha"],
                                     sl["beta"], None, None, S, S, A, A))
    sptr = stream.cuda_stream
    lib = pdn.load()

    def run(s):
        rc = pdn.pdn_decode_step(prob, tens[s], sptr)
        if rc != pdn.PDN_OK:
            raise pdn.PdnError(rc, "pdn_decode_step")

    for s in range(min(args.warmup, steps)):
        run(s)
    S.zero_()
    A.zero_()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(steps):
        run(s)
    e1.record(stream)
    barrier()
    if pdn.device_error() != pdn.PDN_OK:
        raise SystemExit("device error in decode")
    ms_local = e0.elapsed_time(e1)
    ms = mor(ms_local)
    per_step = ms_local / steps
    byts = decode_bytes_per_token_head(w) * w.B * w.H
    gbs = byts / (per_step / 1e3) / 1e9
    return {"workload": w.name, "value": throughput(w.B * steps, world, ms), "unit": "tokens/s",
            "steps": steps, "ms_per_step": ms / steps, "gpu_launches": steps,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                         "peak_kind": peaks_kind + " copy", "frac_of_8tbs_spec": gbs / 8000.0,
                         "bytes_per_launch": byts,
                         "traffic": traffic_for("decode:" + w.name, DECODE_SOURCES)},
            "l2": "state (268 MB) larger than L2"}


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    from linear_recurrence_sequence_chunked_b200.workloads import WORKLOADS
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    secs = max(0.5, min(20.0, 150.0 / max(1, args.steps + args.warmup), args.cpu_seconds))
    rates = []
    desc = cores = None
    for i in range(args.warmup + args.steps):
        rate, cores, desc, _ = oracle_sample_rate(w, target_s=secs)
        if i >= args.warmup:
            rates.append(rate)
    value = statistics.mean(rates)
    tok_per_step = w.B * w.T
    out = {"impl": "reference",
           "metric": "fwd tokens/s per layer (H16,d128,T4K) + % roofline; decode tokens/s",
           "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": tok_per_step / value * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic",
           "config": {"workload": w.name, "variant": w.variant, "B": w.B, "T": w.T, "H": w.H,
                      "d_k": w.dk, "d_v": w.dv, "chunk": w.chunk, "inputs": w.dtype,
                      "reference": "fp64 CPU oracle (token loop), bounded sample per step"},
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                            "sample": desc},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0},
           "gpu_launches": 0}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="pgdn_bf16_4k")
    ap.add_argument("--kernel", choices=["auto", "simt", "tc"], default="auto")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the Preconditioned KDA 8k and FG2 / GDN-2 32k workloads")
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
