#!/usr/bin/env python
"""Benchmark of the Multi-Scale Retention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference]

One JSON line on stdout (rank 0).  A step is one chunkwise forward of the
6.7B-shaped workload (B=2 sequences of 8192 tokens, 16 heads, d_k=256,
d_v=512, chunk 512, per-head GroupNorm + swish gate fused, final f32 state
emitted) through the C ABI, inputs resident in HBM.  Every step reads about
0.8 GB of inputs, far more than the 126 MB L2, so no flush is needed between
steps.  The same run also times
  * the two kernels of the step separately (CUDA events between the state and
    output calls, on the launching stream) for the roofline of the dominant
    one,
  * the recurrent decode workload (128 sequences x 16 heads, d_k=256,
    d_v=512, f32 state initialised by a chunkwise prefill of 8192 tokens,
    1024 single-token steps),
  * the end-to-end call with pinned host buffers (host->device copies of the
    inputs and device->host copy of the output inside the timed region),
  * the fp64 CPU oracle on a bounded sample of the same workload (rank 0, N=1).

--impl reference times the oracle alone (the CPU reference arm).

Multi-GPU: each rank runs its own batch of independent sequences (weak
scaling, no collective on the data path); the step time is the maximum over
ranks, and the value counts the tokens of all ranks.
"""

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from linear_recurrent_sequence_retention_b200 import workloads as W  # noqa: E402

METRIC = "retention fwd tokens/s & % bf16 tensor peak; decode steps/s & HBM GB/s % peak"
HEADLINE = "msr_6p7b_b2_h16_t8192_dk256_dv512_c512"
HEADLINE_6P7B = HEADLINE                # fixed: --workload may change HEADLINE
DECODE = "decode_6p7b_n128_h16_dk256_dv512"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TC_SOURCE = os.path.join(ROOT, "linear_recurrent_sequence_retention_b200", "csrc", "chunkwise_tc.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "chunkwise_output_kernel_6p7b_t8192_traffic.json")


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# algorithmic counts (per token and head), stated with the roofline
# ---------------------------------------------------------------------------

def alg_counts(wl, chunk):
    """Per token-head: flops of the output kernel (intra-chunk causal product
    and the decayed read of the state), of the state kernel (state update),
    and the bytes every step must move (q, k, v, g read; y written)."""
    C, dk, dv = chunk, wl.dk, wl.dv
    flops_out = (C + 1) * (dk + dv) + 2 * dk * dv
    flops_state = 2 * dk * dv
    bytes_in = 2 * (2 * dk + dv) + (2 * dv if wl.norm_gate else 0)
    bytes_out = 2 * dv
    return flops_out, flops_state, bytes_in, bytes_out


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)),
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, world):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle, as it stands, on a bounded sample
# ---------------------------------------------------------------------------

def sample_len(wl, i):
    """Token count of the i-th sampled (sequence, head) pair of a workload."""
    if wl.varlen:
        nseq, lo, hi = wl.varlen
        return int(W.varlen_lengths(nseq, lo, hi, seed=0)[i % nseq])
    return wl.T


def n_pairs(wl):
    return (wl.varlen[0] if wl.varlen else wl.B) * wl.H


def oracle_sample_step(wl, seed, chunk):
    """One (sequence, head) of the workload through the oracle: the chunkwise
    form over all its tokens, then GroupNorm + gate when the workload has it."""
    import oracle
    q, k, v, g = W.make_qkvg(1, sample_len(wl, seed), 1, wl.dk, wl.dv, "bf16", seed=seed,
                             gate=wl.norm_gate)
    f = W.to_f64
    gam = W.head_gammas(wl.H)[seed % wl.H]
    t0 = time.perf_counter()
    o, _ = oracle.retention_chunkwise(f(q)[0, :, 0], f(k)[0, :, 0], f(v)[0, :, 0], gam, chunk)
    if wl.norm_gate:
        oracle.norm_gate(o[:, None, :], f(g)[0][:, None, :])
    return time.perf_counter() - t0


def blas_threads():
    try:
        import threadpoolctl
        n = [i["num_threads"] for i in threadpoolctl.threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return len(os.sched_getaffinity(0))


def cpu_baseline(wl, budget_s=15.0):
    """Oracle throughput in tokens/s (one token = all H heads), timed on a
    sample of whole (sequence, head) pairs for about ``budget_s`` seconds."""
    done, elapsed, token_heads = 0, 0.0, 0
    while elapsed < budget_s or done == 0:
        elapsed += oracle_sample_step(wl, done, wl.chunk)
        token_heads += sample_len(wl, done)
        done += 1
        if done >= n_pairs(wl):
            break
    what = "chunkwise form + GroupNorm/gate" if wl.norm_gate else "chunkwise form"
    return {"value": token_heads / wl.H / elapsed, "unit": "tokens/s",
            "cores": blas_threads(), "kind": "oracle",
            "sample": f"{done} of {n_pairs(wl)} (sequence, head) pairs of {wl.name}, "
                      f"{token_heads} token-heads, {what} in numpy float64; "
                      f"tokens/s counts a token once all {wl.H} heads are done"}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def traffic_from_profile(workload):
    """DRAM bytes per launch of the output kernel at the workload's full size,
    from the committed ncu figures (a small JSON file), only if they were taken
    on this workload and on the current kernel source."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
        sha = hashlib.sha256(open(TC_SOURCE, "rb").read()).hexdigest()
        if d.get("source_sha256") != sha or d.get("workload") != workload:
            return None
        return float(d["dram_bytes_per_launch_full_size"])
    except (OSError, ValueError, KeyError, TypeError):
        return None


def config_of(wl, world):
    Bx, Tx, nst, cu = shape_of(wl)
    in_mb = Bx * Tx * wl.H * (2 * wl.dk + wl.dv + (wl.dv if wl.norm_gate else 0)) * 2 / 1e6
    cfg = {"workload": wl.name, "B_per_gpu": Bx, "T": Tx, "H": wl.H, "d_k": wl.dk, "d_v": wl.dv,
           "chunk": wl.chunk,
           "epilogue": ("per-head GroupNorm (eps 1e-5) + swish gate, y bf16" if wl.norm_gate
                        else "none, o bf16"),
           "state_out": "f32 final state" if wl.state_out else "none",
           "parallelism": f"dp{world}",
           "l2": (f"inputs ({in_mb:.0f} MB per step) larger than L2; no flush" if in_mb >= 264
                  else f"inputs ({in_mb:.0f} MB per step) near or below L2 size: L2 flushed "
                       "(256 MB write) between timed steps, outside the per-step events")}
    if cu is not None:
        cfg["packed"] = f"{nst} sequences, {Tx} tokens, cu_seqlens"
    return cfg


def shape_of(wl):
    """(B, T, number of sequences, cu_seqlens or None) of a chunkwise workload; a
    packed variable-length batch is one row of all its tokens."""
    if wl.varlen:
        nseq, lo, hi = wl.varlen
        cu = W.cu_seqlens_of(W.varlen_lengths(nseq, lo, hi, seed=0))
        return 1, int(cu[-1]), nseq, cu
    return wl.B, wl.T, wl.B, None


def run_headline(args, world, rank, pk, pk_kind):
    from linear_recurrent_sequence_retention_b200 import ops
    wl = W.WORKLOADS[HEADLINE]
    dev = torch.device("cuda")
    Bx, Tx, nst, cu = shape_of(wl)
    q, k, v, g = W.make_qkvg(Bx, Tx, wl.H, wl.dk, wl.dv, "bf16", seed=rank, gate=wl.norm_gate,
                             device=dev)
    cu = None if cu is None else torch.from_numpy(cu).to(dev)
    gam = W.head_gammas(wl.H)
    y = torch.empty(Bx, Tx, wl.H, wl.dv, device=dev, dtype=torch.bfloat16)
    S = torch.empty(nst, wl.H, wl.dk, wl.dv, device=dev, dtype=torch.float32) if wl.state_out else None
    ws = ops.alloc_workspace(ops.chunkwise_workspace_size(torch.bfloat16, wl.chunk, Bx, Tx, wl.H,
                                                          wl.dk, wl.dv, nst if cu is not None else 0),
                             dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record()
        ops.chunkwise_states(k, v, gam, wl.chunk, cu_seqlens=cu, state_out=S, workspace=ws)
        if ev is not None:
            ev[1].record()
        ops.chunkwise_outputs(q, k, v, gam, wl.chunk, ws, cu_seqlens=cu, g=g, out=y)
        if ev is not None:
            ev[2].record()

    # inputs that fit in L2 are flushed between timed steps (a 256 MB write,
    # outside the per-step events), so every step reads them from HBM
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v, g) if t is not None)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if in_bytes < (252 << 20) else None
    for _ in range(args.warmup):
        step()
    ops.check_device_error()
    K = args.steps
    # the timed region: K whole steps, nothing recorded between the two kernels
    # of a step (an event there adds a launch gap); with an L2 flush between
    # steps, each step is bracketed by its own pair of events instead
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    start.record()
    for i in range(K):
        if flush is not None:
            flush.fill_(i & 0xff)
            sev[i][0].record()
        step()
        if flush is not None:
            sev[i][1].record()
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    ops.check_device_error()
    ms_total = start.elapsed_time(end)
    if flush is not None:     # the step time is the sum of the steps' own events
        ms_total = float(np.sum([e[0].elapsed_time(e[1]) for e in sev]))
    # per-kernel durations (state pass, output pass) for the roofline: the same
    # steps on the same stream right after the timed region, with events
    # between the kernels
    Kk = max(3, min(K, 20))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(Kk)]
    for i in range(Kk):
        if flush is not None:
            flush.fill_(i & 0xff)
        step(evs[i])
    torch.cuda.synchronize()
    ops.check_device_error()
    ms_state = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    ms_out = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    ms_step = max_over_ranks(ms_total / K, world)
    tokens = sum_over_ranks(Bx * Tx, world)
    value = tokens / (ms_step / 1e3)

    # roofline of the dominant (output) kernel.  The chunkwise path is a dense
    # contraction judged on the tensor pipe: algorithmic flops at the
    # workload's own chunk length over the kernel's event time against the
    # bf16 peak; its HBM fraction is reported beside it.  The kernels may
    # evaluate short chunks as longer ones (same result, more intra-chunk
    # work), so the flops at the executed chunk are given too.
    f_out, f_state, b_in, b_out = alg_counts(wl, wl.chunk)
    c_exec = ops.chunkwise_executed_chunk(torch.bfloat16, wl.chunk, wl.dk, wl.dv)
    f_out_x, f_state_x, _, _ = alg_counts(wl, c_exec)
    units = Bx * Tx * wl.H                          # token-heads per launch
    flops_launch = f_out * units
    bytes_launch = (b_in + b_out) * units
    t_out = ms_out / 1e3
    peak_bw = pk["hbm_gbs"]
    peak_tf = pk["bf16_tflops"]
    traffic = traffic_from_profile(wl.name)
    ach = flops_launch / t_out / 1e12
    roof = {"bound": "tensor", "achieved": ach, "peak": peak_tf, "unit": "TFLOP/s",
            "frac": ach / peak_tf, "traffic": traffic,
            "kernel": "output_kernel (tcgen05)", "peak_source": f"{pk_kind} bf16 (burst)",
            "algorithmic_flops_per_launch": flops_launch, "launch_ms": ms_out,
            "executed_chunk": c_exec,
            "flops_per_launch_at_executed_chunk": f_out_x * units,
            "hbm": {"achieved_gbs": bytes_launch / t_out / 1e9, "peak_gbs": peak_bw,
                    "frac": bytes_launch / t_out / 1e9 / peak_bw,
                    "algorithmic_bytes_per_launch": bytes_launch}}
    step_flops = (f_out + f_state) * units
    tensor = {"achieved_tflops": step_flops / (ms_step / 1e3) / 1e12,
              "peak_tflops": peak_tf, "frac": step_flops / (ms_step / 1e3) / 1e12 / peak_tf,
              "peak_source": f"{pk_kind} bf16 (burst)",
              "spec_peak_tflops": 2250.0,
              "frac_of_spec": step_flops / (ms_step / 1e3) / 1e12 / 2250.0,
              "algorithmic_flops_per_step": step_flops,
              "executed_chunk": c_exec,
              "flops_per_step_at_executed_chunk": (f_out_x + f_state_x) * units,
              "counting": f"per token-head (C+1)(dk+dv) + 4 dk dv, C={wl.chunk}"}
    step_bytes = (b_in + b_out) * units + (nst * wl.H * wl.dk * wl.dv * 4 if wl.state_out else 0)
    hbm = {"achieved_gbs": step_bytes / (ms_step / 1e3) / 1e9, "peak_gbs": peak_bw,
           "frac": step_bytes / (ms_step / 1e3) / 1e9 / peak_bw,
           "algorithmic_bytes_per_step": step_bytes}
    kernels = {"state_kernel_ms": ms_state, "output_kernel_ms": ms_out, "step_ms": ms_total / K,
               "note": f"kernel durations from {Kk} event-instrumented steps run right after "
                       "the timed region (events between the two kernels add a launch gap, "
                       "so the timed steps carry none)"}

    # end to end through the public API with pinned host buffers.  Every step
    # copies its inputs host->device, runs the call and copies its outputs
    # device->host.  Timed two ways: serial (one stream), and streamed (a
    # copy-in stream, the compute stream and a copy-out stream with two
    # buffer sets, so step i+1's inputs and step i-1's outputs cross PCIe --
    # full duplex -- while step i computes); the streamed figure is the value.
    e2e = None
    if not args.no_e2e:
        ins = [t for t in (q, k, v, g) if t is not None]
        nb = 2
        hins = [[t.to("cpu").pin_memory() for t in ins] for _ in range(nb)]
        dins = [[torch.empty_like(t) for t in ins] for _ in range(nb)]
        ys = [y] + [torch.empty_like(y) for _ in range(nb - 1)]
        Ss = [S] + [None if S is None else torch.empty_like(S) for _ in range(nb - 1)]
        hys = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(nb)]
        hSs = [None if S is None else torch.empty(S.shape, dtype=S.dtype).pin_memory()
               for _ in range(nb)]
        s_cmp = torch.cuda.current_stream()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(nb)]
        ev_done = [torch.cuda.Event() for _ in range(nb)]
        ev_out = [torch.cuda.Event() for _ in range(nb)]

        def call(b, stream):
            di = dins[b]
            ops.chunkwise_fwd(di[0], di[1], di[2], gam, wl.chunk, cu_seqlens=cu,
                              g=di[3] if g is not None else None, out=ys[b], state_out=Ss[b],
                              workspace=ws, stream=stream)

        def serial_step():
            for d, hsrc in zip(dins[0], hins[0]):
                d.copy_(hsrc, non_blocking=True)
            call(0, s_cmp)
            hys[0].copy_(ys[0], non_blocking=True)
            if hSs[0] is not None:
                hSs[0].copy_(Ss[0], non_blocking=True)

        def streamed_step(i):
            b = i % nb
            if i >= nb:
                s_in.wait_event(ev_done[b])        # step i-nb finished reading buffer set b
            with torch.cuda.stream(s_in):
                for d, hsrc in zip(dins[b], hins[b]):
                    d.copy_(hsrc, non_blocking=True)
                ev_in[b].record(s_in)
            s_cmp.wait_event(ev_in[b])
            if i >= nb:
                s_cmp.wait_event(ev_out[b])        # step i-nb's outputs have left buffer set b
            call(b, s_cmp)
            ev_done[b].record(s_cmp)
            s_out.wait_event(ev_done[b])
            with torch.cuda.stream(s_out):
                hys[b].copy_(ys[b], non_blocking=True)
                if hSs[b] is not None:
                    hSs[b].copy_(Ss[b], non_blocking=True)
                ev_out[b].record(s_out)

        Ke = max(3, min(K, 10))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(2):
            serial_step()
        barrier(world)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(Ke):
            serial_step()
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
        ms_serial = max_over_ranks(e0.elapsed_time(e1) / Ke, world)
        for i in range(2 * nb):
            streamed_step(i)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        e0.record(s_cmp)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(Ke):
            streamed_step(i)
        s_cmp.wait_event(ev_out[(Ke - 1) % nb])    # the last outputs are on the host
        e1.record(s_cmp)
        torch.cuda.synchronize()
        barrier(world)
        ms_e2e = max_over_ranks(e0.elapsed_time(e1) / Ke, world)
        ops.check_device_error()
        h2d = sum(t.numel() * t.element_size() for t in hins[0])
        d2h = hys[0].numel() * hys[0].element_size() + (
            0 if hSs[0] is None else hSs[0].numel() * hSs[0].element_size())
        e2e = {"value": tokens / (ms_e2e / 1e3), "unit": "tokens/s", "ms_per_step": ms_e2e,
               "steps": Ke, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "api": "ops.chunkwise_fwd (C ABI retention_chunkwise_fwd) from pinned host memory; "
                      "copy-in, compute and copy-out on three streams with two buffer sets",
               "serial": {"value": tokens / (ms_serial / 1e3), "ms_per_step": ms_serial,
                          "api": "the same call with both copies on the compute stream"}}
        del hins, dins, ys, Ss, hys, hSs
    del q, k, v, g, y, ws
    torch.cuda.empty_cache()
    return {"value": value, "ms_per_step": ms_step, "roofline": roof, "tensor": tensor,
            "hbm": hbm, "kernels": kernels, "e2e": e2e, "clocks": clocks,
            "gpu_launches": (3 if cu is not None else 2) * K, "wl": wl}  # timed region only


def run_decode(args, world, rank, pk, pk_kind):
    from linear_recurrent_sequence_retention_b200 import ops
    wl = W.WORKLOADS[DECODE]
    dev = torch.device("cuda")
    N, H, dk, dv = wl.B, wl.H, wl.dk, wl.dv
    gam = W.head_gammas(H)
    S = torch.empty(N, H, dk, dv, device=dev, dtype=torch.float32)
    # prefill: state-only chunkwise pass over 8192 tokens, in groups of sequences
    grp = min(16, N)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000 + rank)
    sc = 1.0 / math.sqrt(dk)
    ws = None
    for n0 in range(0, N, grp):
        kk = (torch.randn(grp, wl.T, H, dk, generator=gen, device=dev) * sc).to(torch.bfloat16)
        vv = (torch.randn(grp, wl.T, H, dv, generator=gen, device=dev) * sc).to(torch.bfloat16)
        if ws is None:
            ws = ops.alloc_workspace(ops.chunkwise_workspace_size(torch.bfloat16, wl.chunk, grp,
                                                                  wl.T, H, dk, dv), dev)
        ops.chunkwise_states(kk, vv, gam, wl.chunk, state_out=S[n0:n0 + grp], workspace=ws)
        del kk, vv
    torch.cuda.synchronize()
    del ws
    steps = wl.decode_steps
    qs = (torch.randn(steps, N, H, dk, generator=gen, device=dev) * sc).to(torch.bfloat16)
    ks = (torch.randn(steps, N, H, dk, generator=gen, device=dev) * sc).to(torch.bfloat16)
    vs = (torch.randn(steps, N, H, dv, generator=gen, device=dev) * sc).to(torch.bfloat16)
    o = torch.empty(N, H, dv, device=dev, dtype=torch.float32)
    for i in range(max(3, args.warmup)):
        ops.recurrent_step(qs[i], ks[i], vs[i], gam, S, out=o)
    ops.check_device_error()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        ops.recurrent_step(qs[i], ks[i], vs[i], gam, S, out=o)
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    ops.check_device_error()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    state_bytes = N * H * dk * dv * 4
    step_bytes = 2 * state_bytes + N * H * (2 * dk + dv) * 2 + N * H * dv * 4
    ach = step_bytes / (ms / 1e3) / 1e9
    ranks_tokens = sum_over_ranks(N, world)

    # the same tokens, Tn = 16 per call: one pass over the state per 16 tokens
    Tn = 16
    calls = steps // Tn
    qm, km, vm = (x.view(calls, Tn, N, H, -1).transpose(1, 2).contiguous() for x in (qs, ks, vs))
    om = torch.empty(N, Tn, H, dv, device=dev, dtype=torch.float32)
    for i in range(max(3, args.warmup)):
        ops.recurrent_steps(qm[i % calls], km[i % calls], vm[i % calls], gam, S, out=om)
    ops.check_device_error()
    barrier(world)
    torch.cuda.synchronize()
    e0.record()
    for i in range(calls):
        ops.recurrent_steps(qm[i], km[i], vm[i], gam, S, out=om)
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    ops.check_device_error()
    ms_m = max_over_ranks(e0.elapsed_time(e1) / calls, world)
    call_bytes = 2 * state_bytes + N * Tn * H * (2 * dk + dv) * 2 + N * Tn * H * dv * 4
    ach_m = call_bytes / (ms_m / 1e3) / 1e9
    multi = {"tokens_per_call": Tn, "calls": calls, "ms_per_call": ms_m,
             "tokens_per_s": ranks_tokens * Tn / (ms_m / 1e3),
             "speedup_vs_single_step": (ms * Tn) / ms_m,
             "roofline": {"bound": "hbm", "achieved": ach_m, "peak": pk["hbm_gbs"], "unit": "GB/s",
                          "frac": ach_m / pk["hbm_gbs"], "peak_source": pk_kind,
                          "algorithmic_bytes_per_launch": call_bytes,
                          "kernel": "decode_multi_tc_kernel"}}
    del qs, ks, vs, qm, km, vm, S, o, om
    torch.cuda.empty_cache()
    return {"workload": wl.name, "steps": steps, "ms_per_step": ms,
            "steps_per_s": 1e3 / ms, "tokens_per_s": ranks_tokens / (ms / 1e3),
            "roofline": {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / pk["hbm_gbs"], "peak_source": pk_kind,
                         "frac_of_8tbs": ach / 8000.0,
                         "algorithmic_bytes_per_launch": step_bytes,
                         "kernel": "decode_step_kernel"},
            "multi_token": multi,
            "gpu_launches": steps + calls}


BACKWARD = "msr_b4_h8_t2048_dk128_dv256_c128"


def fp32_fma_peak_tflops(pk):
    """float32 FMA roofline of the CUDA cores: SMs x 128 lanes x 2 flops x the
    maximum SM clock (MEASURED_PEAKS' sm_max_mhz, else the part's 1965 MHz)."""
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    mhz = float(pk.get("sm_max_mhz", 1965.0))
    return sms * 128 * 2 * mhz * 1e6 / 1e12


def run_backward(args, world, rank, pk, pk_kind):
    """The chunkwise backward (dQ, dK, dV and the initial-state gradient from
    dO) on the B=4, T=2048, H=8, d_k=128, d_v=256, chunk-128 workload.  bf16
    inputs run on the tensor-core forward kernels (three retentions, bf16 MMAs,
    roofline: the bf16 tensor peak), timed without and with a final-state
    gradient; the same values as float32 inputs (`cuda_core` below) run on CUDA
    cores in float32 (roofline: the float32 FMA peak)."""
    from linear_recurrent_sequence_retention_b200 import ops
    wl = W.WORKLOADS[BACKWARD]
    dev = torch.device("cuda")
    B, T, H, dk, dv, C = wl.B, wl.T, wl.H, wl.dk, wl.dv, wl.chunk
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=rank, gate=False, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(2000 + rank)
    do = torch.randn(B, T, H, dv, generator=gen, device=dev).to(torch.bfloat16)
    dS = torch.randn(B, H, dk, dv, generator=gen, device=dev)
    gam = W.head_gammas(H)
    ws = ops.alloc_workspace(max(ops.chunkwise_bwd_workspace_size(dt, C, B, T, H, dk, dv)
                                 for dt in (torch.bfloat16, torch.float32)), dev)
    # per token-head: three intra-chunk causal products (C+1)(dk+dv) each, three
    # state reads 2 dk dv each, two state recurrences 2 dk dv each
    flops = (3 * (C + 1) * (dk + dv) + 10 * dk * dv) * B * T * H
    tokens = sum_over_ranks(B * T, world)

    def timed(dstate, reps, x=(q, k, v, do)):
        for _ in range(max(3, args.warmup)):
            ops.chunkwise_bwd(*x, gam, C, d_state_out=dstate, return_d_state=True, workspace=ws)
        ops.check_device_error()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            ops.chunkwise_bwd(*x, gam, C, d_state_out=dstate, return_d_state=True, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
        ops.check_device_error()
        return max_over_ranks(e0.elapsed_time(e1) / reps, world)

    reps_tc, reps_cc = 20, 5
    ms_tc = timed(None, reps_tc)
    ms_tc_ds = timed(dS, reps_tc)
    x32 = tuple(t.float() for t in (q, k, v, do))
    ms_cc = timed(dS, reps_cc, x32)
    del x32
    ach_tc = flops / (ms_tc / 1e3) / 1e12
    ach_cc = flops / (ms_cc / 1e3) / 1e12
    peak_tc = pk["bf16_tflops"]
    peak_cc = fp32_fma_peak_tflops(pk)
    del q, k, v, do, dS, ws
    torch.cuda.empty_cache()
    big = backward_6p7b(args, world, rank, pk, pk_kind)
    return {"workload": wl.name, "input_dtype": "bf16", "ms_per_call": ms_tc,
            "tokens_per_s": tokens / (ms_tc / 1e3),
            "ms_per_call_with_d_state_out": ms_tc_ds,
            "path": "tensor cores: three forward retentions (dQ; dV and dK on the sequences "
                    "read backwards) plus token-reversal copies",
            "roofline": {"bound": "tensor", "achieved": ach_tc, "peak": peak_tc,
                         "unit": "TFLOP/s", "frac": ach_tc / peak_tc,
                         "peak_source": f"{pk_kind} bf16 (burst)",
                         "algorithmic_flops_per_call": flops,
                         "counting": f"per token-head 3 (C+1)(dk+dv) + 10 dk dv, C={C}",
                         "kernel": "state_kernel + output_kernel (x3), flip_tokens_kernel"},
            "cuda_core": {"with": "float32 inputs (the same values) and a final-state gradient",
                          "ms_per_call": ms_cc,
                          "tokens_per_s": tokens / (ms_cc / 1e3),
                          "roofline": {"bound": "alu", "achieved": ach_cc, "peak": peak_cc,
                                       "unit": "TFLOP/s", "frac": ach_cc / peak_cc,
                                       "peak_source": "derived: SMs x 128 FP32 lanes x 2 flops "
                                                      "x max SM clock",
                                       "kernel": "chunk_grad_simt_kernel + chunk_state_simt_kernel"}},
            "6p7b": big,
            "gpu_launches": 13 * reps_tc + 15 * reps_tc + 5 * reps_cc + big["gpu_launches"]}


def backward_6p7b(args, world, rank, pk, pk_kind):
    """The backward at the 6.7B-shaped workload (B=2, T=8192, H=16, d_k=256,
    d_v=512, chunk 512, bf16, with a final-state gradient): tensor cores, the
    dQ and dK retentions in two d_v halves each."""
    from linear_recurrent_sequence_retention_b200 import ops
    wl = W.WORKLOADS[HEADLINE_6P7B]
    dev = torch.device("cuda")
    B, T, H, dk, dv, C = wl.B, wl.T, wl.H, wl.dk, wl.dv, wl.chunk
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=rank, gate=False, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(3000 + rank)
    do = torch.randn(B, T, H, dv, generator=gen, device=dev).to(torch.bfloat16)
    dS = torch.randn(B, H, dk, dv, generator=gen, device=dev)
    gam = W.head_gammas(H)
    ws = ops.alloc_workspace(ops.chunkwise_bwd_workspace_size(torch.bfloat16, C, B, T, H, dk, dv), dev)
    flops = (3 * (C + 1) * (dk + dv) + 10 * dk * dv) * B * T * H
    reps = 5
    for _ in range(max(3, args.warmup)):
        ops.chunkwise_bwd(q, k, v, do, gam, C, d_state_out=dS, return_d_state=True, workspace=ws)
    ops.check_device_error()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        ops.chunkwise_bwd(q, k, v, do, gam, C, d_state_out=dS, return_d_state=True, workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    ops.check_device_error()
    ms = max_over_ranks(e0.elapsed_time(e1) / reps, world)
    ach = flops / (ms / 1e3) / 1e12
    del q, k, v, do, dS, ws
    torch.cuda.empty_cache()
    return {"workload": wl.name, "ms_per_call_with_d_state_out": ms,
            "tokens_per_s": sum_over_ranks(B * T, world) / (ms / 1e3),
            "roofline": {"bound": "tensor", "achieved": ach, "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": ach / pk["bf16_tflops"],
                         "peak_source": f"{pk_kind} bf16 (burst)",
                         "algorithmic_flops_per_call": flops,
                         "counting": f"per token-head 3 (C+1)(dk+dv) + 10 dk dv, C={C}",
                         "kernel": "state_kernel + output_kernel (x5: dQ and dK in two d_v "
                                   "halves), flip_tokens_kernel, split_heads_kernel"},
            "gpu_launches": reps * 22}


def run_rope(args, world, rank, pk, pk_kind):
    """Rotary position encoding of q and k of the 6.7B-shaped workload (B=2,
    T=8192, H=16, d_k=256, bf16): one streaming pass, HBM-bound (reads q and
    k, writes the rotated copies)."""
    from linear_recurrent_sequence_retention_b200 import ops
    wl = W.WORKLOADS["msr_6p7b_b2_h16_t8192_dk256_dv512_c512"]
    dev = torch.device("cuda")
    q, k, _, _ = W.make_qkvg(wl.B, wl.T, wl.H, wl.dk, 8, "bf16", seed=rank, gate=False, device=dev)
    qo, ko = torch.empty_like(q), torch.empty_like(k)
    for _ in range(max(3, args.warmup)):
        ops.rope(q, k, q_out=qo, k_out=ko)
    reps = 20
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        ops.rope(q, k, q_out=qo, k_out=ko)
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    ops.check_device_error()
    ms = max_over_ranks(e0.elapsed_time(e1) / reps, world)
    nbytes = 4 * q.numel() * q.element_size()             # q, k read; rotated q, k written
    ach = nbytes / (ms / 1e3) / 1e9
    del q, k, qo, ko
    torch.cuda.empty_cache()
    ab = rope_forward_ab(args, world, rank)
    return {"workload": f"{wl.name} q,k", "ms_per_call": ms,
            "tokens_per_s": sum_over_ranks(wl.B * wl.T, world) / (ms / 1e3),
            "roofline": {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / pk["hbm_gbs"], "peak_source": pk_kind,
                         "algorithmic_bytes_per_launch": nbytes, "kernel": "rope_kernel"},
            "forward_with_rope": ab,
            "gpu_launches": reps + ab["gpu_launches"]}


def rope_forward_ab(args, world, rank):
    """The 6.7B-shaped forward (GroupNorm + gate, y bf16, final state) on
    rotated q and k through the one-call entry (retention_chunkwise_fwd_rope:
    the rotary pass over q and k, then the two chunkwise passes), and the
    share of the rotary pass in it."""
    from linear_recurrent_sequence_retention_b200 import ops
    wl = W.WORKLOADS[HEADLINE_6P7B]          # whatever --workload times
    dev = torch.device("cuda")
    B, T, H, dk, dv, C = wl.B, wl.T, wl.H, wl.dk, wl.dv, wl.chunk
    q, k, v, g = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=rank, gate=True, device=dev)
    gam = W.head_gammas(H)
    y = torch.empty(B, T, H, dv, device=dev, dtype=torch.bfloat16)
    S = torch.empty(B, H, dk, dv, device=dev, dtype=torch.float32)
    ws = ops.alloc_workspace(ops.chunkwise_fwd_rope_workspace_size(C, B, T, H, dk, dv), dev)

    def call():
        ops.chunkwise_fwd(q, k, v, gam, C, g=g, out=y, state_out=S, workspace=ws,
                          rope_base=10000.0)

    reps = 20
    for _ in range(max(3, args.warmup)):
        call()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        call()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    ops.check_device_error()
    ms = max_over_ranks(e0.elapsed_time(e1) / reps, world)
    del q, k, v, g, y, S, ws
    torch.cuda.empty_cache()
    return {"workload": wl.name, "entry": "retention_chunkwise_fwd_rope", "ms_per_call": ms,
            "tokens_per_s": sum_over_ranks(B * T, world) / (ms / 1e3),
            "kernels": "rope_kernel (q, k) + state + output",
            "gpu_launches": reps * 3}


def run_rla(args, world, rank, pk, pk_kind):
    """Residual linear attention, window 512 (the RAttention page's setting), on
    the B=4, T=2048, H=8, d_k=128, d_v=256 shape with bf16 inputs: one pass
    mapping and shifting the inputs, then the chunkwise retention at gamma = 1
    on the tensor-core kernels (256-token chunks)."""
    from linear_recurrent_sequence_retention_b200 import ops
    wl = W.WORKLOADS[BACKWARD]
    dev = torch.device("cuda")
    B, T, H, dk, dv, w, C = wl.B, wl.T, wl.H, wl.dk, wl.dv, 512, 256
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=rank, gate=False, device=dev)
    out = torch.empty(B, T, H, dv, device=dev, dtype=torch.bfloat16)
    ws = ops.alloc_workspace(ops.lib().retention_rla_workspace_size(ops.RET_BF16, B, T, H, dk, dv, 0), dev)
    for _ in range(max(3, args.warmup)):
        ops.rla_fwd(q, k, v, w, out=out, workspace=ws)
    reps = 20
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        ops.rla_fwd(q, k, v, w, out=out, workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    ops.check_device_error()
    ms = max_over_ranks(e0.elapsed_time(e1) / reps, world)
    flops = ((C + 1) * (dk + dv) + 4 * dk * dv) * B * T * H
    ach = flops / (ms / 1e3) / 1e12
    del q, k, v, out, ws
    torch.cuda.empty_cache()
    return {"workload": f"{wl.name} rla window {w}", "ms_per_call": ms,
            "tokens_per_s": sum_over_ranks(B * T, world) / (ms / 1e3),
            "roofline": {"bound": "tensor", "achieved": ach, "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": ach / pk["bf16_tflops"],
                         "peak_source": f"{pk_kind} bf16 (burst)",
                         "algorithmic_flops_per_call": flops,
                         "counting": f"per token-head (C+1)(dk+dv) + 4 dk dv, C={C} (the retention "
                                     "inside; the feature pass is HBM traffic)",
                         "kernel": "rla_inputs_kernel + state_kernel + output_kernel"},
            "gpu_launches": 3 * reps}


def run_parallel(args, world, rank, pk, pk_kind):
    """The parallel form (Q K^T * D) V on the tensor cores, bf16 inputs, f32
    accumulation, bf16 output, at the head shapes of the two chunkwise
    workloads: each call is the fp16 copy of v and one output-kernel launch
    over every causal 128 x 128 (query, key) block pair."""
    from linear_recurrent_sequence_retention_b200 import ops
    dev = torch.device("cuda")
    res = {}
    launches = 0
    for name in (HEADLINE_6P7B, BACKWARD):
        wl = W.WORKLOADS[name]
        B, T, H, dk, dv = wl.B, wl.T, wl.H, wl.dk, wl.dv
        q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=rank, gate=False, device=dev)
        gam = W.head_gammas(H)
        o = torch.empty(B, T, H, dv, device=dev, dtype=torch.bfloat16)
        ws = ops.alloc_workspace(ops.parallel_workspace_size(torch.bfloat16, B, T, H, dk, dv), dev)
        for _ in range(max(3, args.warmup)):
            ops.parallel_fwd(q, k, v, gam, out=o, workspace=ws)
        reps = 10
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            ops.parallel_fwd(q, k, v, gam, out=o, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
        ops.check_device_error()
        ms = max_over_ranks(e0.elapsed_time(e1) / reps, world)
        # causal pairs (n, m <= n): (q_n . k_m) and its weight times v_m
        flops = B * H * T * (T + 1) * (dk + dv)
        ach = flops / (ms / 1e3) / 1e12
        rb = -(-T // 128)
        executed = B * H * rb * (rb + 1) // 2 * 128 * 128 * 2 * (dk * (2 if dv > 256 else 1) + dv)
        res[name] = {"ms_per_call": ms, "tokens_per_s": sum_over_ranks(B * T, world) / (ms / 1e3),
                     "roofline": {"bound": "tensor", "achieved": ach, "peak": pk["bf16_tflops"],
                                  "unit": "TFLOP/s", "frac": ach / pk["bf16_tflops"],
                                  "peak_source": f"{pk_kind} bf16 (burst)",
                                  "algorithmic_flops_per_call": flops,
                                  "executed_flops_per_call": executed,
                                  "counting": "B H T (T+1) (dk + dv): the causal half of Q K^T "
                                              "and of P V; executed adds the masked half of "
                                              "the diagonal blocks and, for dv = 512, the "
                                              "Q K^T repeated by the second dv half",
                                  "kernel": "v16_kernel + output_kernel"}}
        launches += 2 * reps
        del q, k, v, o, ws
        torch.cuda.empty_cache()
    return {"workloads": res, "gpu_launches": launches}


def main():
    global HEADLINE
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mine", "reference"], default="mine")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--backward-only", action="store_true", help="backward only (profiling)")
    ap.add_argument("--parallel-only", action="store_true", help="parallel form only (profiling)")
    ap.add_argument("--no-rope", action="store_true")
    ap.add_argument("--no-rla", action="store_true")
    ap.add_argument("--no-parallel", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--workload", default=HEADLINE,
                    choices=[n for n, w in W.WORKLOADS.items() if w.dtype == "bf16" and not w.decode_steps],
                    help="chunkwise workload to time (default: the 6.7B-shaped headline)")
    ap.add_argument("--B", type=int, default=None, help="override the headline batch (profiling)")
    ap.add_argument("--T", type=int, default=None, help="override the headline length (profiling)")
    ap.add_argument("--no-headline", action="store_true", help="decode only (profiling)")
    ap.add_argument("--decode-N", type=int, default=None, help="override the decode batch (profiling)")
    ap.add_argument("--decode-steps", type=int, default=None, help="override the decode steps")
    args = ap.parse_args()
    if args.warmup < 3:
        log("warm-up below 3 steps is not allowed; using 3")
        args.warmup = 3
    world, rank, local = dist_setup()
    pk, pk_kind = peaks()
    if args.decode_N or args.decode_steps:
        import dataclasses
        base = W.WORKLOADS[DECODE]
        N, st = args.decode_N or base.B, args.decode_steps or base.decode_steps
        W.WORKLOADS[DECODE] = dataclasses.replace(base, B=N, decode_steps=st,
                                                  name=f"{base.name}@N{N}_steps{st}")
    HEADLINE = args.workload
    if args.B or args.T:
        import dataclasses
        base = W.WORKLOADS[HEADLINE]
        B, T = args.B or base.B, args.T or base.T
        W.WORKLOADS[HEADLINE] = dataclasses.replace(base, B=B, T=T,
                                                    name=f"{base.name}@B{B}_T{T}")
    wl = W.WORKLOADS[HEADLINE]

    if args.impl == "reference":
        # The CPU reference arm: the fp64 oracle, rank 0 only, bounded samples.
        if rank == 0:
            for i in range(args.warmup):
                oracle_sample_step(wl, i, wl.chunk)
            times = [oracle_sample_step(wl, i, wl.chunk) for i in range(args.steps)]
            ms = 1e3 * float(np.sum(times)) / args.steps
            toks = float(np.mean([sample_len(wl, i) for i in range(args.steps)]))
            val = toks / wl.H / (ms / 1e3)
            line = {"metric": METRIC, "value": val, "unit": "tokens/s", "impl": "reference",
                    "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                    "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                    "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                    "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "H": wl.H,
                               "d_k": wl.dk, "d_v": wl.dv, "chunk": wl.chunk,
                               "step": "one (sequence, head) pair of the workload"},
                    "cpu_baseline": {"value": val, "unit": "tokens/s", "kind": "oracle",
                                     "cores": blas_threads(),
                                     "sample": f"each step: one of the {n_pairs(wl)} (sequence, "
                                               f"head) pairs ({toks:.0f} tokens on average), "
                                               "numpy float64"},
                    "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                            "d2h_bytes_per_step": 0}}
            print(json.dumps(line), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    assert torch.cuda.is_available(), "bench.py needs a CUDA device (use --impl reference for the CPU arm)"
    if args.backward_only:
        bwd = run_backward(args, world, rank, pk, pk_kind)
        if rank == 0:
            print(json.dumps({"metric": METRIC, "backward": bwd, "n_gpus": world}), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    if args.parallel_only:
        par = run_parallel(args, world, rank, pk, pk_kind)
        if rank == 0:
            print(json.dumps({"metric": METRIC, "parallel": par, "n_gpus": world}), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    if args.no_headline:
        dec = run_decode(args, world, rank, pk, pk_kind)
        if rank == 0:
            print(json.dumps({"metric": METRIC, "decode": dec, "n_gpus": world}), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    head = run_headline(args, world, rank, pk, pk_kind)
    dec = None if args.no_decode else run_decode(args, world, rank, pk, pk_kind)
    bwd = None if args.no_backward else run_backward(args, world, rank, pk, pk_kind)
    rope = None if args.no_rope else run_rope(args, world, rank, pk, pk_kind)
    rla = None if args.no_rla else run_rla(args, world, rank, pk, pk_kind)
    par = None if args.no_parallel else run_parallel(args, world, rank, pk, pk_kind)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(wl, args.cpu_seconds)
    if rank == 0:
        line = {
            "metric": METRIC,
            "value": head["value"],
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": head["ms_per_step"],
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": config_of(wl, world),
            "roofline": head["roofline"],
            "tensor": head["tensor"],
            "hbm": head["hbm"],
            "kernels": head["kernels"],
            "backward": bwd,
            "rope": rope,
            "rla": rla,
            "parallel": par,
            "e2e": head["e2e"],
            "cpu_baseline": cpu,
            "clocks": head["clocks"],
            "gpu_launches": (head["gpu_launches"] + (dec["gpu_launches"] if dec else 0)
                             + (bwd["gpu_launches"] if bwd else 0)
                             + (rope["gpu_launches"] if rope else 0)
                             + (rla["gpu_launches"] if rla else 0)
                             + (par["gpu_launches"] if par else 0)),
            "arithmetic": "tensor-core MMAs (tcgen05) with f32 accumulation: q, k as bf16; "
                          "v, the decayed scores, the decayed query rows, zeta*K and the "
                          "carried state as fp16",
            # last, so that a reader keeping only the line's tail still has it
            "decode": dec,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
