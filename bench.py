"""Benchmark of the SSD chunked-scan forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one ssd_forward over the whole workload (every step of the path: the
cumulative decay, the diagonal blocks, the chunk states, the state passing and
the outputs), inputs resident in HBM.  Each rank runs the full per-GPU workload
(weak scaling; ranks share nothing, the work has no data-path collective).
L2 is flushed (a 512 MiB write) before every timed step, outside the timed
events.  Times are CUDA events on the launching stream, the median of the K
steps, max over ranks.  ``--impl reference`` times the float64 oracle on the
host cores on a bounded sample of the same workload (rank 0 only).
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

METRIC = "SSD chunked-scan fwd Mtokens/s and % of roofline (HBM or tensor pipe)"
DEFAULT_WORKLOAD = "long_L65536_H64_P128_N256_G8"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ----------------------------------------------------------------------------- helpers
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def algorithmic(w, ndocs):
    """Compulsory bytes and causal flops of one forward over workload ``w``."""
    T, H, P, N, G, Q = w.tokens, w.nheads, w.headdim, w.dstate, w.ngroups, w.chunk_size
    ein = 2 if w.dtype == "bf16" else 4
    states = ndocs * H * N * P * 4
    byts = T * H * P * ein * 2 + T * H * ein + 2 * T * G * N * ein + states + 12 * H
    if w.init != "zero":
        byts += states
    flops_tok_head = Q * P + 4 * N * P + Q * N * G / H + 2 * N * P / Q
    return byts, T * H * flops_tok_head


# the sources each measured kernel is built from (its recorded DRAM traffic stays
# valid while these are unchanged)
KERNEL_SOURCES = {
    "tc": ("ssd_tc.cu", "ssd_tc2.cu", "tc_common.cuh", "ssd_internal.h"),
    "tc128": ("ssd_tc_wide.cu", "tc_common.cuh", "ssd_internal.h"),
    "simt": ("ssd_simt.cu", "ssd_internal.h"),
    "step": ("ssd_step.cu", "ssd_internal.h"),
}


def kernel_source_hash(path_name="tc"):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "structured_state_space_chunked_b200", "csrc")
    for fn in KERNEL_SOURCES[path_name]:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, path_name):
    """dram bytes per launch from a committed ncu summary, if the kernels are unchanged."""
    fn = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(fn) as f:
            rec = json.load(f)
        e = rec[workload][path_name]
        if e.get("source_hash") == kernel_source_hash(path_name):
            return float(e["dram_bytes_per_launch"]), e.get("kernel")
    except Exception:
        pass
    return None, None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []
        self.mark = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def region(self, t0, t1):
        self.mark = (t0, t1)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        t0, t1 = self.mark or (0, float("inf"))
        rows = [l for (t, l) in self.lines if t0 - 0.06 <= t <= t1 + 0.06] or [l for _, l in self.lines]
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            parts = [p.strip() for p in r.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- ranks
def dist_setup(n):
    """One process per GPU; the process group only coordinates (barrier, max time)."""
    import torch
    from structured_state_space_chunked_b200 import dist as sdist
    rank, world, local = sdist.env_ranks()
    if world != n:
        raise SystemExit(f"--gpus {n} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    pg = sdist.init("nccl", timeout_s=120, device=torch.device("cuda", local))
    return rank, world, local, pg


def barrier(pg):
    from structured_state_space_chunked_b200 import dist as sdist
    sdist.barrier(pg)


def max_over_ranks(pg, v):
    import torch
    from structured_state_space_chunked_b200 import dist as sdist
    return sdist.max_over_ranks(v, pg, device=torch.device("cuda", torch.cuda.current_device()))


# ----------------------------------------------------------------------------- oracle arm
def oracle_sample_throughput(w, inp, budget_s):
    """Time the oracle on a subset of heads over every sequence of the workload.

    Returns (Mtokens/s in whole-token units, number of heads, seconds): the
    oracle computed `k` of the H heads for all tokens, i.e. T * k / H whole tokens.
    """
    import oracle
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].cpu().numpy()
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}

    def run(k):
        t0 = time.perf_counter()
        oracle.oracle_forward(cpu["x"], cpu["dt"], cpu["A"], cpu["B"], cpu["C"], cpu["D"],
                              cpu["dt_bias"], cpu["initial_states"], cu_seqlens=cu,
                              heads=list(range(k)))
        return time.perf_counter() - t0

    # the oracle runs its (sequence, head) items in parallel over its threads: size the
    # head sample so that every thread is busy for about the budget
    threads = oracle.oracle_threads()
    seqs = int(inp["x"].shape[0]) if inp["cu_seqlens"] is None else int(inp["cu_seqlens"].numel() - 1)
    k = 1
    t = run(k)
    if t < 0.5 * budget_s and k < w.nheads:
        waves = max(1, int(budget_s / max(t, 1e-6)))
        k = int(min(w.nheads, max(1, (waves * threads) // max(seqs, 1))))
        t = run(k)
    reps = 1
    if t < 0.25 * budget_s:  # the whole workload is quick: repeat it
        reps = int(min(50, max(1, 0.5 * budget_s / max(t, 1e-6))))
        t = sum(run(k) for _ in range(reps)) / reps
    return (w.tokens * k / w.nheads) / t / 1e6, k, t, min(threads, seqs * k)


# ----------------------------------------------------------------------------- main
def run_step(args, w, rank, world, local, pg, hbm_peak, peak_kind):
    """--op step: ``ssd_step`` over a decode batch with the workload's head shape.

    A step reads and writes every sequence's fp32 state (8 N P bytes per head) plus
    the token's x, dt, B, C and y; that is its compulsory traffic and the kernel is
    HBM-bound.  The state is updated in place, step after step; L2 is flushed before
    every timed step.
    """
    import math
    import numpy as np
    import torch

    from structured_state_space_chunked_b200 import ssd

    dev = torch.device("cuda", local)
    bsz, H, P, N, G = args.decode_batch, w.nheads, w.headdim, w.dstate, w.ngroups
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    g = torch.Generator(device="cpu").manual_seed(1234 + rank)
    x = torch.randn(bsz, H, P, generator=g).to(dev, td)
    dt = torch.randn(bsz, H, generator=g).to(dev, td)
    A = (-torch.exp(torch.rand(H, generator=g) * math.log(16))).to(dev)
    B = (torch.randn(bsz, G, N, generator=g) / math.sqrt(N)).to(dev, td)
    C = (torch.randn(bsz, G, N, generator=g) / math.sqrt(N)).to(dev, td)
    D = torch.randn(H, generator=g).to(dev)
    u = torch.exp(torch.rand(H, generator=g) * (math.log(1e-1) - math.log(1e-3)) + math.log(1e-3))
    bias = torch.log(torch.expm1(u)).to(dev)
    state = (0.1 * torch.randn(bsz, H, N, P, generator=g)).to(dev)
    y = torch.empty(bsz, H, P, dtype=td, device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ssd.ssd_step(x, dt, A, B, C, state, D, bias, y=y)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.2)
    barrier(pg)
    t_wall0 = time.time()
    for i in range(args.steps):
        flush.fill_(float(i))
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    barrier(pg)
    t_wall1 = time.time()
    clk.region(t_wall0, t_wall1)
    time.sleep(0.1)
    clocks = clk.stop()
    ms = statistics.median(a.elapsed_time(b) for a, b in zip(starts, ends))
    ms = max_over_ranks(pg, ms)
    ein = 2 if w.dtype == "bf16" else 4
    byts = bsz * H * (8 * N * P + 2 * P * ein + ein) + 2 * bsz * G * N * ein + 12 * H
    achieved = byts / (ms * 1e-3) / 1e9
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        nb = min(bsz, 32)
        args_cpu = [t[:nb].cpu() for t in (state, x, dt)] + [A.cpu()] + [t[:nb].cpu() for t in (B, C)]
        t0 = time.perf_counter()
        reps = 0
        while time.perf_counter() - t0 < 2.0:
            oracle.oracle_step(*args_cpu, D.cpu(), bias.cpu())
            reps += 1
        dtc = (time.perf_counter() - t0) / reps
        cpu = {"value": nb / dtc / 1e6, "unit": "Mtokens/s", "cores": 1, "kind": "oracle",
               "sample": f"float64 numpy step oracle, {nb} of {bsz} sequences, {reps} repetitions"}
    if rank == 0:
        line = {
            "metric": "SSD decode step (ssd_step) Mtokens/s and % of HBM roofline",
            "value": bsz * world / (ms * 1e-3) / 1e6, "unit": "Mtokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": f"decode step, {w.name} head shape", "decode_batch": bsz,
                       "nheads": H, "headdim": P, "dstate": N, "ngroups": G,
                       "parallelism": f"dp{world} (independent replicas)",
                       "l2": "flushed before every timed step (512 MiB write, outside the events)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak,
                         "traffic": recorded_traffic(f"decode_b{bsz}_{w.name}", "step")[0],
                         "peak_source": f"{peak_kind} (MEASURED_PEAKS.json burst)" if peak_kind == "measured"
                         else "fallback", "algorithmic_bytes_per_launch": byts,
                         "kernel": "ssd_step_kernel"},
            "cpu_baseline": cpu, "e2e": None, "gpu_launches": args.steps, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def run_bwd(args, w, rank, world, local, pg, hbm_peak, tc_peak, peak_kind):
    """--op backward: ``ssd_backward`` over the workload (all gradients, fp32).

    Algorithmic flops per token and head, for chunks of Q tokens: 2 Q (2 P + 3 N)
    (the in-chunk products W, V, dC, dB, gB) + 8 N P (the state-sized products of
    dC, dB, gB and the per-chunk cotangent sum) + 2 N P (the forward's chunk states,
    recomputed).  bf16 inputs with P a multiple of 64 (up to 256) and N = 64 or 128
    take the tensor-core path (Q = 128, one block per 64-column slice of P): its
    roofline is the measured bf16 tensor rate.  Every other shape runs
    on the CUDA cores (Q = 64) against the fp32 FMA rate, 148 SMs x 128 lanes x 2 x
    1965 MHz = 74.4 TFLOP/s.  L2 is flushed before every timed step.
    """
    import torch

    from structured_state_space_chunked_b200 import inputs as I
    from structured_state_space_chunked_b200 import ssd

    dev = torch.device("cuda", local)
    inp = I.make_inputs(w, device=dev)
    ndocs = w.batch if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1
    dy, dfin = I.make_cotangents(w, ndocs, device=dev)
    bsz, L = inp["x"].shape[:2]
    H, P, N, G = w.nheads, w.headdim, w.dstate, w.ngroups
    h = ssd.SSD(bsz, L, H, P, N, G, w.torch_dtype,
                max_docs=0 if inp["cu_seqlens"] is None else ndocs, device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        return h.backward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], dy, inp["D"],
                          inp["dt_bias"], inp["initial_states"], dfin, inp["cu_seqlens"])

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    if h.status() != 0:
        raise SystemExit("device status set during warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.2)
    barrier(pg)
    t_wall0 = time.time()
    for i in range(args.steps):
        flush.fill_(float(i))
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    barrier(pg)
    t_wall1 = time.time()
    clk.region(t_wall0, t_wall1)
    time.sleep(0.1)
    clocks = clk.stop()
    ms = statistics.median(a.elapsed_time(b) for a, b in zip(starts, ends))
    ms = max_over_ranks(pg, ms)
    T = bsz * L
    on_tc = w.dtype == "bf16" and P % 64 == 0 and P <= 256 and N in (64, 128)
    Q = 128 if on_tc else 64
    flops = float(T) * H * (2 * Q * (2 * P + 3 * N) + 10 * N * P)
    if on_tc:
        bound, peak = "tensor", tc_peak
        peak_source = (f"{peak_kind} bf16 tensor rate (MEASURED_PEAKS.json burst)" if peak_kind == "measured"
                       else "fallback bf16 tensor rate")
    else:
        bound, peak = "alu", 148 * 128 * 2 * 1965e6 / 1e12
        peak_source = "derived: 148 SMs x 128 fp32 lanes x 2 x 1965 MHz"
    achieved = flops / (ms * 1e-3) / 1e12
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        heads = [0]
        cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].cpu().numpy()
        cpu_in = [inp[k].cpu() for k in ("x", "dt", "A", "B", "C")]
        t0 = time.perf_counter()
        oracle.oracle_backward(*cpu_in, dy.cpu(), inp["D"].cpu(), inp["dt_bias"].cpu(),
                               None if inp["initial_states"] is None else inp["initial_states"].cpu(),
                               dfin.cpu(), cu_seqlens=cu, heads=heads)
        dtc = time.perf_counter() - t0
        cpu = {"value": T * len(heads) / H / dtc / 1e6, "unit": "Mtokens/s",
               "cores": min(oracle.oracle_threads(), ndocs), "kind": "oracle",
               "sample": f"float64 backward oracle, head 0 of {H} over all {ndocs} documents, "
                         "scaled to the whole layer"}
    if rank == 0:
        line = {
            "metric": "SSD chunked-scan backward (ssd_backward) Mtokens/s and % of roofline (tensor or fp32 FMA)",
            "value": T * world / (ms * 1e-3) / 1e6, "unit": "Mtokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "nheads": H,
                       "headdim": P, "dstate": N, "ngroups": G, "input_dtype": w.dtype,
                       "parallelism": f"dp{world} (independent replicas)",
                       "l2": "flushed before every timed step (512 MiB write, outside the events)"},
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": None, "peak_source": peak_source,
                         "algorithmic_flops_per_launch": flops, "chunk": Q,
                         "kernel": ("kb_chunk_tc + kb_states_tc x2 + kb_state_pass + k_cumsum + k_state_pass"
                                    if on_tc and N == 128 else
                                    "kb_chunk_tc + kb_chunk_dstate + kb_state_pass + the forward's state kernels"
                                    if on_tc else
                                    "kb_chunk + kb_chunk_dstate + kb_state_pass + the forward's state kernels")},
            "cpu_baseline": cpu, "e2e": None, "gpu_launches": 11 * args.steps, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def run_ext(args, w, rank, world, local, pg, hbm_peak, peak_kind):
    """--op ext: ``ssd_forward_ext`` over the workload with the ReLU feature map on B
    and C and the denominator normalisation (the scan of a ones column).

    Compulsory bytes: B and C read and their mapped copies written; the numerator
    scan's x, dt, mapped B and C read, y written, final states written; the
    denominator scan's dt, mapped B and C read and its output written;
    the division's y read and written, x and the denominator read.  L2 is flushed
    before every timed step.
    """
    import torch

    from structured_state_space_chunked_b200 import inputs as I
    from structured_state_space_chunked_b200 import ssd

    if w.varlen_tokens:
        raise SystemExit("--op ext takes a batch-mode workload")
    dev = torch.device("cuda", local)
    inp = I.make_inputs(w, device=dev)
    bsz, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    fmap = ssd.SSD_FMAP_RELU
    N2 = ssd.feature_map_dim(fmap, N)
    h = ssd.SSD(bsz, L, H, P, N, G, w.torch_dtype, device=dev)
    y = torch.empty(bsz, L, H, P, dtype=w.torch_dtype, device=dev)
    fin = torch.empty(bsz, H, N2, P, dtype=torch.float32, device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        h.forward_ext(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["dt_bias"],
                      w.chunk_size, feature_map=fmap, normalize=True, y=y, final_states=fin)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    if h.status() != 0:
        raise SystemExit("device status set during warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.2)
    barrier(pg)
    t_wall0 = time.time()
    for i in range(args.steps):
        flush.fill_(float(i))
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    barrier(pg)
    t_wall1 = time.time()
    clk.region(t_wall0, t_wall1)
    time.sleep(0.1)
    clocks = clk.stop()
    ms = statistics.median(a.elapsed_time(b) for a, b in zip(starts, ends))
    ms = max_over_ranks(pg, ms)
    es = 2 if w.dtype == "bf16" else 4
    T = bsz * L
    # the operation's compulsory bytes, as for the plain forward: x, dt, B, C read once, y and
    # the final (mapped) states written once, A, D, dt_bias; the mapped copies, the
    # denominator and any second pass over y are the implementation's own traffic
    byts = T * H * P * 2 * es + T * H * es + 2 * T * G * N * es + bsz * H * N2 * P * 4 + 12 * H
    achieved = byts / (ms * 1e-3) / 1e9
    # the library's choice: the denominator beside the numerator on a second stream and a
    # division pass when the numerator's units leave a quarter of the SMs idle, else the
    # denominator first and the division folded into the numerator kernel
    units = bsz * H * (P // 64)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    if 4 * units > 3 * sms:
        ext_kernels = ("fmap_ew_kernel (B and C) + den_chunk_gram_kernel x2 + den_pass_kernel + "
                       "ssd_tc_fused<1, true> (division in its epilogue)")
        ext_launches = 5
    else:
        ext_kernels = ("fmap_ew_kernel (B and C) + ssd_tc_fused, beside it on a second stream "
                       "den_chunk_gram_kernel x2 + den_pass_kernel; then normalize_kernel")
        ext_launches = 6
    if rank == 0:
        line = {
            "metric": "SSD forward with ReLU feature map and denominator normalisation (ssd_forward_ext) "
                      "Mtokens/s and % of HBM roofline",
            "value": T * world / (ms * 1e-3) / 1e6, "unit": "Mtokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "feature_map": "relu", "normalize": True, "batch": bsz,
                       "seqlen": L, "nheads": H, "headdim": P, "dstate": N, "ngroups": G,
                       "parallelism": f"dp{world} (independent replicas)",
                       "l2": "flushed before every timed step (512 MiB write, outside the events)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "traffic": None,
                         "peak_source": f"{peak_kind} (MEASURED_PEAKS.json burst)" if peak_kind == "measured"
                         else "fallback", "algorithmic_bytes_per_launch": byts,
                         "kernel": ext_kernels},
            "cpu_baseline": None, "e2e": None, "gpu_launches": ext_launches * args.steps, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def run_cp(args, w, rank, world, local, pg, hbm_peak, peak_kind):
    """--op cp: the device steps one context-parallel rank adds to its own forward.

    The workload is the rank's slice (batch mode); the rank is the last of
    --cp-ranks, which has the longest combine.  Timed per step: ssd_cp_logdecay,
    ssd_cp_combine, ssd_cp_correct (the all-gather between them is a collective
    and is not part of this one-GPU measurement).  Compulsory bytes: dt read, cs
    written and read, C read, y read and written, every rank's final state and log
    decay read, h_in and the final state written.
    """
    import torch

    from structured_state_space_chunked_b200 import inputs as I
    from structured_state_space_chunked_b200 import ssd

    if w.varlen_tokens:
        raise SystemExit("--op cp takes a batch-mode workload")
    dev = torch.device("cuda", local)
    inp = I.make_inputs(w, device=dev)
    R = args.cp_ranks
    bsz, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    y = torch.randn(bsz, L, H, P, device=dev).to(w.torch_dtype)
    S_all = 0.1 * torch.randn(R, bsz, H, N, P, device=dev)
    ld_all = -torch.rand(R, bsz, H, device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    corr_ev = []

    def step(i=None):
        cs, ld = ssd.cp_logdecay(inp["dt"], inp["A"], inp["dt_bias"], headdim=P, dstate=N, ngroups=G)
        h_in, fin = ssd.cp_combine(R - 1, S_all, ld_all, inp["initial_states"], dt_dtype=w.torch_dtype)
        if i is not None:
            corr_ev[i][0].record(stream)
        ssd.cp_correct(inp["C"], cs, h_in, y)
        if i is not None:
            corr_ev[i][1].record(stream)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    corr_ev.extend((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps))
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.2)
    barrier(pg)
    t_wall0 = time.time()
    for i in range(args.steps):
        flush.fill_(float(i))
        starts[i].record(stream)
        step(i)
        ends[i].record(stream)
    barrier(pg)
    t_wall1 = time.time()
    clk.region(t_wall0, t_wall1)
    time.sleep(0.1)
    clocks = clk.stop()
    ms = statistics.median(a.elapsed_time(b) for a, b in zip(starts, ends))
    ms = max_over_ranks(pg, ms)
    corr_ms = statistics.median(a.elapsed_time(b) for a, b in corr_ev)
    on_tc = w.dtype == "bf16" and P % 64 == 0 and P <= 256 and N % 64 == 0 and N <= 256
    ein = 2 if w.dtype == "bf16" else 4
    T = bsz * L
    byts = (T * H * ein + 2 * T * H * 4 + T * G * N * ein + 2 * T * H * P * ein
            + R * bsz * H * (N * P + 1) * 4 + 2 * bsz * H * N * P * 4)
    flops = 2.0 * T * H * N * P
    achieved = byts / (ms * 1e-3) / 1e9
    if rank == 0:
        line = {
            "metric": "SSD context-parallel rank steps (log decay, combine, correction) Mtokens/s",
            "value": T * world / (ms * 1e-3) / 1e6, "unit": "Mtokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": f"context-parallel rank {R - 1} of {R}, slice = {w.name}",
                       "batch": bsz, "seqlen": L, "nheads": H, "headdim": P, "dstate": N,
                       "ngroups": G, "parallelism": f"dp{world} (independent replicas)",
                       "l2": "flushed before every timed step (512 MiB write, outside the events)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "traffic": None,
                         "peak_source": f"{peak_kind} (MEASURED_PEAKS.json burst)" if peak_kind == "measured"
                         else "fallback", "algorithmic_bytes_per_launch": byts,
                         "correction_us": corr_ms * 1e3,
                         "correction_tflops_achieved": flops / (corr_ms * 1e-3) / 1e12,
                         "kernel": "cp_logdecay_kernel + cp_combine_kernel + "
                                   + ("cp_correct_tc_kernel" if on_tc else "cp_correct_kernel")},
            "cpu_baseline": None, "e2e": None, "gpu_launches": 3 * args.steps, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--unit-columns", type=int, default=64, choices=[64, 128],
                    help="column width of the tensor-core kernel's work units")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--op", default="forward",
                    choices=["forward", "step", "cp", "backward", "ext"],
                    help="forward: the chunked scan (default); step: one decode token per "
                         "sequence (ssd_step) with the workload's head shape; cp: the device "
                         "steps a context-parallel rank adds to its forward (log decay, "
                         "combine over --cp-ranks ranks, output correction), the workload "
                         "being the rank's slice; backward: ssd_backward over the workload; "
                         "ext: ssd_forward_ext with the ReLU feature map and normalisation")
    ap.add_argument("--cp-ranks", type=int, default=4, help="ranks for --op cp")
    ap.add_argument("--decode-batch", type=int, default=256,
                    help="sequences per ssd_step call (--op step)")
    args = ap.parse_args()
    # at least 10 untimed warm-up steps (the reported "warmup" is the count run)
    args.warmup = max(args.warmup, 10)

    import torch
    from structured_state_space_chunked_b200 import inputs as I
    from structured_state_space_chunked_b200 import ssd

    w = I.workload(args.workload)
    rank, world, local, pg = dist_setup(args.gpus)
    hbm_peak, tc_peak, peak_kind = peaks()
    if args.op == "step":
        run_step(args, w, rank, world, local, pg, hbm_peak, peak_kind)
        return
    if args.op == "cp":
        run_cp(args, w, rank, world, local, pg, hbm_peak, peak_kind)
        return
    if args.op == "backward":
        run_bwd(args, w, rank, world, local, pg, hbm_peak, tc_peak, peak_kind)
        return
    if args.op == "ext":
        run_ext(args, w, rank, world, local, pg, hbm_peak, peak_kind)
        return

    if args.impl == "reference":
        if rank != 0:
            return
        import oracle
        inp = I.make_inputs(w, device="cpu")
        budget = max(0.05, min(10.0, 150.0 / (args.steps + args.warmup)))
        _v, kh, _t, ref_cores = oracle_sample_throughput(w, inp, budget)
        import oracle as _o
        cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].numpy()

        def ref_step():
            _o.oracle_forward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                              inp["dt_bias"], inp["initial_states"], cu_seqlens=cu,
                              heads=list(range(kh)))

        for _ in range(args.warmup):
            ref_step()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            ref_step()
        wall = time.perf_counter() - t0
        value = (w.tokens * kh / w.nheads) * args.steps / wall / 1e6
        sample = (f"float64 oracle, heads 0..{kh - 1} of {w.nheads} over all {w.tokens} tokens "
                  f"per step; whole-token throughput = tokens * {kh} / {w.nheads} / time")
        line = {
            "impl": "reference", "metric": METRIC, "value": value, "unit": "Mtokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * wall / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name},
            "cpu_baseline": {"value": value, "unit": "Mtokens/s", "cores": ref_cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "Mtokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return

    dev = torch.device("cuda", local)
    inp = I.make_inputs(w, device=dev)
    ndocs = inp["cu_seqlens"].numel() - 1 if inp["cu_seqlens"] is not None else w.batch
    bsz, L = inp["x"].shape[:2]
    h = ssd.SSD(bsz, L, w.nheads, w.headdim, w.dstate, w.ngroups, w.torch_dtype,
                max_docs=ndocs if inp["cu_seqlens"] is not None else 0, device=dev)
    path = {"auto": ssd.SSD_PATH_AUTO, "simt": ssd.SSD_PATH_SIMT, "tc": ssd.SSD_PATH_TC}[args.path]
    if path != ssd.SSD_PATH_AUTO:
        h.force_path(path)
    if args.unit_columns != 64:
        h.tc_unit_columns(args.unit_columns)
    plan = h.plan(w.chunk_size, ndocs if inp["cu_seqlens"] is not None else 0)
    path_name = {0: "simt", 1: "tc"}[plan.path if path == ssd.SSD_PATH_AUTO else path]
    if path_name == "tc" and args.unit_columns == 128:
        path_name = "tc128"
    y = torch.empty_like(inp["x"])
    fin = torch.empty(ndocs, w.nheads, w.dstate, w.headdim, dtype=torch.float32, device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        h.forward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["dt_bias"],
                  w.chunk_size, inp["initial_states"], inp["cu_seqlens"], y=y, final_states=fin)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    if h.status() != 0:
        raise SystemExit("device status error during warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.2)
    barrier(pg)
    t_wall0 = time.time()
    for i in range(args.steps):
        flush.fill_(float(i))
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    barrier(pg)
    t_wall1 = time.time()
    clk.region(t_wall0, t_wall1)
    time.sleep(0.1)
    clocks = clk.stop()
    st = h.status()
    if st != 0:
        raise SystemExit(f"device status {st} in the timed region")
    # the median step (CUDA events), then the max over ranks
    ms = statistics.median(s.elapsed_time(e) for s, e in zip(starts, ends))
    ms = max_over_ranks(pg, ms)
    tokens_all = w.tokens * world
    value = tokens_all / (ms * 1e-3) / 1e6

    byts, flops = algorithmic(w, ndocs)
    achieved_gbs = byts / (ms * 1e-3) / 1e9
    achieved_tf = flops / (ms * 1e-3) / 1e12
    traffic, traffic_kernel = recorded_traffic(w.name, path_name)
    t_hbm = byts / (hbm_peak * 1e9)
    t_tc = flops / (tc_peak * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved_gbs / hbm_peak, "traffic": traffic}
    else:
        roof = {"bound": "tensor", "achieved": achieved_tf, "peak": tc_peak, "unit": "TFLOP/s",
                "frac": achieved_tf / tc_peak, "traffic": traffic}
    roof.update({"peak_source": f"{peak_kind} (MEASURED_PEAKS.json burst)" if peak_kind == "measured"
                 else "fallback", "algorithmic_bytes_per_launch": byts,
                 "causal_flops_per_launch": flops, "tensor_tflops_achieved": achieved_tf,
                 "roofline_us": 1e6 * max(t_hbm, t_tc), "frac_of_roofline": 1e3 * max(t_hbm, t_tc) / ms,
                 "kernel": traffic_kernel or {"tc": "ssd_tc_fused<1>" if w.dstate <= 128
                                              else "ssd_tc_fused2<2>",
                                              "tc128": "ssd_tc_wide"}.get(path_name, "simt (4-5 kernels)")})

    # end to end through the host-buffer entry point (pinned host memory)
    host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in inp.items()}
    yh = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    fh = torch.empty(fin.shape, dtype=torch.float32).pin_memory()
    h2d = sum(v.numel() * v.element_size() for k, v in host.items() if v is not None)
    d2h = yh.numel() * yh.element_size() + fh.numel() * fh.element_size()

    def e2e_step():
        h.forward_host(host["x"], host["dt"], host["A"], host["B"], host["C"], host["D"],
                       host["dt_bias"], w.chunk_size, host["initial_states"], host["cu_seqlens"],
                       y=yh, final_states=fh)

    e2e = None
    if args.e2e_steps > 0:
        for _ in range(3):
            e2e_step()
        barrier(pg)
        t0 = time.perf_counter()
        for _ in range(args.e2e_steps):
            e2e_step()
        barrier(pg)
        e2e_s = max_over_ranks(pg, (time.perf_counter() - t0) / args.e2e_steps)
        e2e = {"value": tokens_all / e2e_s / 1e6, "unit": "Mtokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": 1e3 * e2e_s}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        v, kh, t, used = oracle_sample_throughput(w, inp, 12.0)
        cpu = {"value": v, "unit": "Mtokens/s", "cores": used, "kind": "oracle",
               "sample": f"float64 oracle, heads 0..{kh - 1} of {w.nheads} over all {w.tokens} "
                         f"tokens in {t:.2f} s; whole-token throughput = tokens * {kh} / "
                         f"{w.nheads} / time"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "Mtokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen,
                       "nheads": w.nheads, "headdim": w.headdim, "dstate": w.dstate,
                       "ngroups": w.ngroups, "chunk_size": w.chunk_size,
                       "tokens_per_gpu": w.tokens, "path": path_name,
                       "parallelism": f"dp{world} (independent replicas)",
                       "l2": "flushed before every timed step (512 MiB write, outside the events)"},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": int(plan.kernels) * args.steps, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    h.close()
    if pg is not None:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
