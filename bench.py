#!/usr/bin/env python
"""Benchmark of the multi-scale retention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one chunkwise-recurrent retention forward (fused GroupNorm) over
the 6.7B-class layer at 8k context: batch 8, 16 heads, 8192 tokens, d_k 256,
d_v 512, chunk 512, bf16 inputs, decays gamma_h = 1 - 2^(-5-h).  The headline
`value` is tokens/s of that step (batch x sequence tokens, all heads), timed
with CUDA events on the launching stream with the inputs resident in HBM.
The inputs (3.2 GB per step) are far larger than the 126 MB L2, so no flush
is needed between steps.  The same line carries:
  roofline      the chunk-output kernel (the larger of the two the chunkwise
                call launches), timed live between events, against the
                measured bf16 tensor peak; the state-scan kernel and the
                whole call are reported beside it
  e2e           the same metric through the public API with pinned host
                buffers: host->device copy of q, k, v and device->host copy
                of o inside the timed region
  decode        the recurrent step (batch 8, 16 heads, 256 x 512 state) after
                an 8192-token chunkwise prefill, 1024 steps over 4 rotating
                states so the 256 MB working set exceeds L2; % of measured HBM
  parallel      the parallel form on the 1.3B-class layer (8 x 8 heads x 2048)
  long_64k      chunkwise over 65536 tokens (1 x 16 heads)
  gated         the headline step with the output gate swish(G) (.) GN(o)
  backward      the chunkwise backward on the 1.3B-class layer
  rotate        the xPos rotation of q and k of the 6.7B-class 8k layer, in
                place; % of measured HBM
  cpu_baseline  the float64 CPU oracle on a bounded sample of the same
                workload (rank 0, N = 1 only)
With --gpus N > 1 the script re-runs itself under torchrun (one process per
GPU; the driver may also launch it under torchrun directly).  Every rank runs
the same per-GPU step on its own GPU (weak scaling, no collective on the data
path); the time is the max over ranks and `value` counts the tokens of all
ranks.  --plumbing-check runs that launch and aggregation on CPU over gloo.

--impl reference times the CPU oracle (the only reference this build has)
on a bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "retention fwd tokens/s (chunkwise, % bf16 TC peak); decode steps/s (% HBM BW)"
WORKLOAD = "l6p7b_8k_bf16"

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# algorithmic work (causal pairs only; no split, padding or recompute counted)
# ---------------------------------------------------------------------------

def chunk_lengths(N, C):
    return [min(C, N - s) for s in range(0, N, C)]


def chunkwise_flops(B, H, N, dk, dv, C, state_in=False, state_out=False):
    Ls = chunk_lengths(N, C)
    intra = sum(L * (L + 1) for L in Ls) * (dk + dv)
    inter = sum(2 * dk * dv * L for i, L in enumerate(Ls) if i > 0 or state_in)
    state = sum(2 * dk * dv * L for i, L in enumerate(Ls) if i < len(Ls) - 1 or state_out)
    return B * H * (intra + inter + state)


def chunkwise_phase_flops(B, H, N, dk, dv, C, state_in=False, state_out=False):
    """(states phase, output phase) shares of chunkwise_flops: the chunk
    states K^T (V (.) zeta), and the intra-chunk plus cross-chunk outputs."""
    Ls = chunk_lengths(N, C)
    state = sum(2 * dk * dv * L for i, L in enumerate(Ls) if i < len(Ls) - 1 or state_out)
    return B * H * state, chunkwise_flops(B, H, N, dk, dv, C, state_in, state_out) - B * H * state


def chunkwise_bytes(B, H, N, dk, dv, elem=2, state_in=False, state_out=False):
    io = B * H * N * (2 * dk + 2 * dv) * elem
    st = 4 * B * H * dk * dv * (int(state_in) + int(state_out))
    return io + st


def parallel_flops(B, H, N, dk, dv):
    return B * H * N * (N + 1) * (dk + dv)


def step_bytes(B, H, dk, dv, elem=2):
    return B * H * (8 * dk * dv + elem * (2 * dk + dv) + elem * dv)


def step_flops(B, H, dk, dv):
    return B * H * 4 * dk * dv


# ---------------------------------------------------------------------------
# distributed plumbing (weak scaling: no collective on the data path)
# ---------------------------------------------------------------------------

def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def init_dist(backend):
    import datetime

    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def max_over_ranks(x: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def global_throughput(units_per_rank_per_step: float, steps: int, world: int, t_max_s: float):
    return units_per_rank_per_step * steps * world / t_max_s


# ---------------------------------------------------------------------------
# measurement helpers
# ---------------------------------------------------------------------------

# Sources that decide what the chunk-output kernel does (its code, the
# headers it includes and the tensor maps it is launched with).
OUT_KERNEL_SOURCES = ("tc_out.cu", "sm100.cuh", "common.cuh", "tmap.cu", "tmap.h")


def kernel_source_hash(names=OUT_KERNEL_SOURCES):
    """Hash of the CUDA sources of the chunk-output kernel: stored profiler
    counters are only valid for it."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_recurrent_sequence_scale_b200", "csrc")
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def stored_traffic(workload):
    """DRAM bytes per launch of the chunk-output kernel from the committed ncu
    summary, or None when that kernel changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("source_hash") != kernel_source_hash():
        return None
    return d.get("per_launch_bytes", {}).get(workload)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def smi_index(local: int) -> int:
    """nvidia-smi index of this process's CUDA device."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [x.strip() for x in vis.split(",") if x.strip()]
    if local < len(ids) and ids[local].isdigit():
        return int(ids[local])
    return local


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
             "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.6)

    def stop(self):
        if self.proc is None:
            return
        time.sleep(0.3)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        rows = []
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 11:
                continue
            try:
                rows.append({"sm": float(f[2]), "max": float(f[3]), "util": float(f[5]),
                             "reasons": f[6], "hw": f[7], "hwt": f[8], "swt": f[9], "pc": f[10]})
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        loaded = [r for r in rows if r["util"] >= 50] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pc", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["max"] for r in rows), "reasons": sorted(reasons),
                "samples": len(loaded)}


def timed(fn, steps, warmup, stream, device, phases=None):
    """Run fn warmup times, then time exactly `steps` calls with CUDA events on
    `stream`, bracketed by a barrier and a device synchronize on both sides.
    Returns (seconds of this rank, max seconds over ranks).  With `phases` (a
    list of callables that together make one call of fn) each step runs the
    phases with an event between them, and a third value lists the seconds
    each phase took over all steps."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    nb = steps * (len(phases) if phases else 1) + 1
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(nb)]
    j = 0
    ev[0].record(stream)
    for _ in range(steps):
        for f in (phases or [fn]):
            f()
            j += 1
            ev[j].record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    t = ev[0].elapsed_time(ev[-1]) / 1e3
    if not phases:
        return t, max_over_ranks(t, device)
    P = len(phases)
    per = [sum(ev[s * P + i].elapsed_time(ev[s * P + i + 1]) for s in range(steps)) / 1e3
           for i in range(P)]
    return t, max_over_ranks(t, device), per


def make_qkv(torch, B, H, N, dk, dv, device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    s = 1.0 / math.sqrt(dk)
    q = (torch.randn((B, H, N, dk), device=device, generator=g) * s).to(torch.bfloat16)
    k = (torch.randn((B, H, N, dk), device=device, generator=g) * s).to(torch.bfloat16)
    v = (torch.randn((B, H, N, dv), device=device, generator=g) * s).to(torch.bfloat16)
    gam = torch.tensor([1.0 - 2.0 ** (-5 - h) for h in range(H)], dtype=torch.float32,
                       device=device)
    return q, k, v, gam


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample of the same workload)
# ---------------------------------------------------------------------------

def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = [x.get("num_threads", 0) for x in info if x.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample(heads_max: int, budget_s: float):
    """Run the CPU oracle's chunkwise form (+GroupNorm) head by head on the
    workload's own per-head inputs until the budget is spent.  Returns
    (tokens/s counted like the GPU metric, heads done, seconds)."""
    import oracle
    from linear_recurrent_sequence_scale_b200 import workloads as wl
    w = wl.WORKLOADS[WORKLOAD]
    gam = wl.msr_gammas(w.H)
    done, spent = 0, 0.0
    while done < heads_max and (done == 0 or spent < budget_s):
        b, h = divmod(done, w.H)
        q, k, v = wl.make_head_inputs(w, b % w.B, h)
        t0 = time.perf_counter()
        o, _ = oracle.chunkwise(q.exact[None, None], k.exact[None, None], v.exact[None, None],
                                [float(gam[h])], w.chunk)
        oracle.group_norm(o, w.gn_eps)
        spent += time.perf_counter() - t0
        done += 1
    # a token of the metric carries all H heads
    return done * w.N / w.H / spent, done, spent


def run_reference(args):
    rank, world = dist_env()[:2]
    if rank != 0:
        return 0
    from linear_recurrent_sequence_scale_b200 import workloads as wl
    w = wl.WORKLOADS[WORKLOAD]
    # size each step so that warmup + steps end within about two minutes of
    # wall time (drawing a head's inputs costs about what the oracle does);
    # the timed figure counts the oracle's own time only, since the GPU arm's
    # inputs are resident before its timed region starts
    oracle_sample(1, 0.0)  # first call: imports and allocator warm-up
    t_wall = time.perf_counter()
    oracle_sample(1, 0.0)
    per_head = time.perf_counter() - t_wall
    heads = max(1, min(w.B * w.H,
                       int(120.0 / max(per_head, 1e-3) / max(1, args.steps + args.warmup))))
    for _ in range(args.warmup):
        oracle_sample(heads, 1e9)
    dt = 0.0
    for _ in range(args.steps):
        dt += oracle_sample(heads, 1e9)[2]
    value = heads * w.N / w.H * args.steps / dt
    cores = blas_threads()
    sample = (f"{heads} of {w.B * w.H} (batch, head) pairs of the {WORKLOAD} workload per step, "
              f"full 8192 tokens, chunk {w.chunk}, GroupNorm; float64 numpy oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": w.B, "seq_len": w.N, "heads": w.H,
                   "dk": w.dk, "dv": w.dv, "chunk": w.chunk, "parallelism": "cpu"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args):
    import torch

    import linear_recurrent_sequence_scale_b200 as ret
    from linear_recurrent_sequence_scale_b200 import workloads as wl

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist("nccl")
    ret.load_library()
    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    stream = torch.cuda.current_stream(device)
    launches = 0

    def want(name):
        return args.only in ("all", name)

    # defaults when the headline is not run (--only <sub-benchmark>)
    w = wl.WORKLOADS[WORKLOAD]
    B, H, N, dk, dv, C, eps = w.B, w.H, w.N, w.dk, w.dv, w.chunk, w.gn_eps
    value = t_max = roofline = e2e = None
    headline_launches = 0
    clocks = ClockSampler(smi_index(local))
    if want("headline"):
        # ---------------- headline: chunkwise on the 6.7B-class layer at 8k ----------------
        w = wl.WORKLOADS[WORKLOAD]
        B, H, N, dk, dv, C, eps = w.B, w.H, w.N, w.dk, w.dv, w.chunk, w.gn_eps
        if args.batch:
            B = args.batch  # smaller copy of the workload, for profiler captures only
        q, k, v, gam = make_qkv(torch, B, H, N, dk, dv, device, seed=1000 + rank)
        o = torch.empty((B, H, N, dv), dtype=torch.bfloat16, device=device)
        ws = torch.empty(ret.chunkwise_workspace_bytes(B, H, N, dk, dv, C, torch.bfloat16),
                         dtype=torch.uint8, device=device)
        step = lambda: ret.chunkwise(q, k, v, gam, C, gn_eps=eps, out=o, workspace=ws)
        # the same call in its two phases, so that each kernel's time is measured
        # live: ret_chunkwise does these two calls on one stream
        phases = [lambda: ret.chunkwise_states(k, v, gam, C, ws),
                  lambda: ret.chunkwise_output(q, k, v, gam, C, ws, gn_eps=eps, out=o)]
        clocks = ClockSampler(smi_index(local))
        clocks.start()
        # the step as a user calls it (one ret_chunkwise per step): `value`
        t_local, t_max = timed(step, args.steps, args.warmup, stream, device)
        # the same steps split into the two phases with an event between them:
        # each kernel's duration for the roofline line (the one-call form also
        # lets the output kernel start while the state scan drains, which the
        # split run cannot show)
        _, _, t_phase = timed(step, args.steps, 1, stream, device, phases)
        clocks.stop()
        launches += 2 * args.steps  # state scan + chunk output per call
        headline_launches = launches  # the headline timed region
        launches += 2 * args.steps    # the phase-split run
        tokens = B * N
        value = global_throughput(tokens, args.steps, world, t_max)
        F = chunkwise_flops(B, H, N, dk, dv, C)
        F_states, F_out = chunkwise_phase_flops(B, H, N, dk, dv, C)
        Bytes = chunkwise_bytes(B, H, N, dk, dv)
        call_s = t_local / args.steps
        out_s = t_phase[1] / args.steps
        states_s = t_phase[0] / args.steps
        achieved = F_out / out_s / 1e12
        traffic = stored_traffic(WORKLOAD)
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": traffic,
                    "kernel": "k3::chunk_out_tc (ret_chunkwise_output), the dominant kernel",
                    "peak_source": f"{peak_src} bf16 burst; sustained "
                                   f"{peaks.get('bf16_tflops_sustained')}",
                    "algorithmic_flop_per_launch": F_out,
                    "kernel_ms": out_s * 1e3,
                    "share_of_step": out_s / (out_s + states_s),
                    "other_kernel": {"name": "k2::state_scan_tc (ret_chunkwise_states)",
                                     "ms": states_s * 1e3, "algorithmic_flop": F_states,
                                     "tflops": F_states / states_s / 1e12,
                                     "frac": F_states / states_s / 1e12 / peak},
                    "whole_call": {"algorithmic_flop": F, "tflops": F / call_s / 1e12,
                                   "frac": F / call_s / 1e12 / peak,
                                   "algorithmic_bytes": Bytes,
                                   "hbm_gbs": Bytes / call_s / 1e9,
                                   "hbm_frac": Bytes / call_s / 1e9 / peaks.get("hbm_gbs", 6650.0)}}
        del ws

        # ---------------- e2e through the public API with host buffers ----------------
        # Every step copies q, k, v from pinned host memory and o back, one
        # cudaMemcpyAsync per tensor slice.  The batch is cut into slices (one
        # batch row each) so that the copies of one slice overlap the kernels
        # of another: host->device on one stream, the retention call on the
        # compute stream, device->host on a third, ordered by events.
        e2e = None
        if not args.skip_e2e:
            hq = q.to("cpu").pin_memory()
            hk = k.to("cpu").pin_memory()
            hv = v.to("cpu").pin_memory()
            ho = torch.empty((B, H, N, dv), dtype=torch.bfloat16).pin_memory()
            dq_, dk_, dv_ = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            do_ = torch.empty_like(o)
            ws1 = torch.empty(ret.chunkwise_workspace_bytes(1, H, N, dk, dv, C, torch.bfloat16),
                              dtype=torch.uint8, device=device)
            ws_slices = [ws1, torch.empty_like(ws1)]
            h2d = torch.cuda.Stream(device)
            d2h = torch.cuda.Stream(device)

            def e2e_step():
                h2d.wait_stream(stream)  # after the previous step (and the start event)
                for b in range(B):
                    ev_in = torch.cuda.Event()
                    with torch.cuda.stream(h2d):
                        dq_[b].copy_(hq[b], non_blocking=True)
                        dk_[b].copy_(hk[b], non_blocking=True)
                        dv_[b].copy_(hv[b], non_blocking=True)
                        ev_in.record(h2d)
                    stream.wait_event(ev_in)
                    ret.chunkwise(dq_[b:b + 1], dk_[b:b + 1], dv_[b:b + 1], gam, C, gn_eps=eps,
                                  out=do_[b:b + 1], workspace=ws_slices[b & 1])
                    ev_o = torch.cuda.Event()
                    ev_o.record(stream)
                    with torch.cuda.stream(d2h):
                        d2h.wait_event(ev_o)
                        ho[b].copy_(do_[b], non_blocking=True)
                # the step ends when its last output has reached the host
                stream.wait_stream(d2h)

            e_steps = max(3, min(args.steps, 20))
            te_local, te_max = timed(e2e_step, e_steps, 1, stream, device)
            launches += 2 * B * e_steps
            e2e = {"value": global_throughput(tokens, e_steps, world, te_max), "unit": "tokens/s",
                   "h2d_bytes_per_step": hq.nbytes + hk.nbytes + hv.nbytes,
                   "d2h_bytes_per_step": ho.nbytes, "steps": e_steps,
                   "pipeline": f"{B} batch-row slices, copies overlapped with compute"}
            del hq, hk, hv, ho, dq_, dk_, dv_, do_, ws_slices, ws1
        del q, k, v, o
        torch.cuda.empty_cache()

    extra = {}
    sub_steps = max(3, min(args.steps, 20))
    if not args.skip_sub:
        # ---------------- decode ----------------
        if want("decode"):
            wd = wl.WORKLOADS["decode_6p7b"]
            qd, kd, vd, gd = make_qkv(torch, wd.B, wd.H, wd.N, wd.dk, wd.dv, device, seed=2000 + rank)
            s0 = torch.empty((wd.B, wd.H, wd.dk, wd.dv), dtype=torch.float32, device=device)
            ret.chunkwise(qd, kd, vd, gd, wd.chunk, state_out=s0)  # prefill (untimed)
            launches += 0
            del qd, kd, vd
            states = [s0.clone() for _ in range(4)]
            T = wl.DECODE_STEPS
            g = torch.Generator(device=device)
            g.manual_seed(3000 + rank)
            sc = 1.0 / math.sqrt(wd.dk)
            tq = (torch.randn((T, wd.B, wd.H, wd.dk), device=device, generator=g) * sc).bfloat16()
            tk = (torch.randn((T, wd.B, wd.H, wd.dk), device=device, generator=g) * sc).bfloat16()
            tv = (torch.randn((T, wd.B, wd.H, wd.dv), device=device, generator=g) * sc).bfloat16()
            od = torch.empty((wd.B, wd.H, wd.dv), dtype=torch.bfloat16, device=device)

            def decode_run():
                for t in range(T):
                    ret.step(tq[t], tk[t], tv[t], gd, states[t & 3], out=od)

            # the 1024-step loop timed REPS times; the median per step is reported
            REPS = 7
            plain = [timed(decode_run, 1, 1 if r == 0 else 0, stream, device)[0] / T
                     for r in range(REPS)]
            launches += T * REPS
            per_step = statistics.median(plain)
            sb = step_bytes(wd.B, wd.H, wd.dk, wd.dv)
            # the same 1024 steps replayed from a CUDA graph (launch cost hidden)
            graph_step = None
            try:
                gs = torch.cuda.Stream(device)
                gs.wait_stream(stream)
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.stream(gs):
                    decode_run()  # warm (also sets kernel attributes outside capture)
                    with torch.cuda.graph(graph, stream=gs):
                        decode_run()
                stream.wait_stream(gs)
                replays = [timed(graph.replay, 1, 1 if r == 0 else 0, stream, device)[0] / T
                           for r in range(REPS)]
                launches += T * REPS
                graph_step = statistics.median(replays)
                del graph
            except Exception as ex:  # capture is an optimisation, not a requirement
                graph_step = None
                extra["decode_graph_error"] = str(ex)[:200]
            best = min(x for x in (per_step, graph_step) if x is not None)
            extra["decode"] = {
                "workload": "decode_6p7b", "steps_per_s": world / max_over_ranks(best, device),
                "us_per_step": best * 1e6, "us_per_step_launches": per_step * 1e6,
                "us_per_step_graph": None if graph_step is None else graph_step * 1e6,
                "repetitions": REPS, "statistic": "median of the 1024-step loop timed 7 times",
                "us_per_step_graph_all": None if graph_step is None else [x * 1e6 for x in replays],
                "us_per_step_launches_all": [x * 1e6 for x in plain],
                "tokens_per_s": wd.B * world / max_over_ranks(best, device),
                "roofline": {"bound": "hbm", "achieved": sb / best / 1e9,
                             "peak": peaks.get("hbm_gbs", 6650.0), "unit": "GB/s",
                             "frac": sb / best / 1e9 / peaks.get("hbm_gbs", 6650.0),
                             "algorithmic_bytes_per_step": sb},
                "note": "1024 steps over 4 rotating 64 MiB states (working set 256 MiB > L2)"}
            # the same loop with the xPos rotation of q and k fused into the step
            # (ret_step_rotated, token positions 8192 + t), plain launches
            thd = torch.from_numpy(wl.rotation_angles(wd.dk, seed=1)).to(device)

            def decode_run_rot():
                for t in range(T):
                    ret.step(tq[t], tk[t], tv[t], gd, states[t & 3], out=od, theta=thd,
                             pos=wd.N + t)

            rot = [timed(decode_run_rot, 1, 1 if r == 0 else 0, stream, device)[0] / T
                   for r in range(3)]
            launches += 3 * T
            extra["decode"]["rotated_us_per_step_launches"] = statistics.median(rot) * 1e6
            del states, tq, tk, tv, s0
            torch.cuda.empty_cache()

        # ---------------- parallel form, 1.3B-class layer ----------------
        if want("l1p3b"):
            wp = wl.WORKLOADS["l1p3b_bf16"]
            qp, kp, vp, gp = make_qkv(torch, wp.B, wp.H, wp.N, wp.dk, wp.dv, device, seed=4000 + rank)
            op = torch.empty_like(vp)
            tpar, _ = timed(lambda: ret.parallel(qp, kp, vp, gp, out=op), sub_steps, 3, stream, device)
            launches += sub_steps
            Fp = parallel_flops(wp.B, wp.H, wp.N, wp.dk, wp.dv)
            cs_ = tpar / sub_steps
            wsp = torch.empty(ret.chunkwise_workspace_bytes(wp.B, wp.H, wp.N, wp.dk, wp.dv, wp.chunk,
                                                            torch.bfloat16),
                              dtype=torch.uint8, device=device)
            tch, _ = timed(lambda: ret.chunkwise(qp, kp, vp, gp, wp.chunk, out=op, workspace=wsp),
                           sub_steps, 3, stream, device)
            launches += 2 * sub_steps
            # the same call split into its two kernels, each timed live
            _, _, tph = timed(None, sub_steps, 0, stream, device,
                              [lambda: ret.chunkwise_states(kp, vp, gp, wp.chunk, wsp),
                               lambda: ret.chunkwise_output(qp, kp, vp, gp, wp.chunk, wsp,
                                                            out=op)])
            launches += 2 * sub_steps
            Fc = chunkwise_flops(wp.B, wp.H, wp.N, wp.dk, wp.dv, wp.chunk)
            Bc = chunkwise_bytes(wp.B, wp.H, wp.N, wp.dk, wp.dv)
            Fcs, Fco = chunkwise_phase_flops(wp.B, wp.H, wp.N, wp.dk, wp.dv, wp.chunk)
            extra["l1p3b"] = {
                "workload": "l1p3b_bf16",
                "parallel": {"tokens_per_s": wp.B * wp.N / cs_, "ms": cs_ * 1e3,
                             "tflops": Fp / cs_ / 1e12, "frac_tc": Fp / cs_ / 1e12 / peak},
                "chunkwise": {"tokens_per_s": wp.B * wp.N / (tch / sub_steps),
                              "ms": tch / sub_steps * 1e3,
                              "tflops": Fc / (tch / sub_steps) / 1e12,
                              "frac_tc": Fc / (tch / sub_steps) / 1e12 / peak,
                              "hbm_frac": Bc / (tch / sub_steps) / 1e9 / peaks.get("hbm_gbs", 6650.0),
                              "states_ms": tph[0] / sub_steps * 1e3,
                              "output_ms": tph[1] / sub_steps * 1e3,
                              "states_tflops": Fcs / (tph[0] / sub_steps) / 1e12,
                              "output_tflops": Fco / (tph[1] / sub_steps) / 1e12}}
            del qp, kp, vp, op, wsp
            torch.cuda.empty_cache()

        # ---------------- long context 64k ----------------
        if want("long_64k"):
            wlg = wl.WORKLOADS["long_64k_bf16"]
            ql, kl, vl, gl = make_qkv(torch, wlg.B, wlg.H, wlg.N, wlg.dk, wlg.dv, device,
                                      seed=5000 + rank)
            ol = torch.empty_like(vl)
            sl = torch.empty((wlg.B, wlg.H, wlg.dk, wlg.dv), dtype=torch.float32, device=device)
            wsl = torch.empty(ret.chunkwise_workspace_bytes(wlg.B, wlg.H, wlg.N, wlg.dk, wlg.dv,
                                                            wlg.chunk, torch.bfloat16),
                              dtype=torch.uint8, device=device)
            tl, _ = timed(lambda: ret.chunkwise(ql, kl, vl, gl, wlg.chunk, out=ol, state_out=sl,
                                                workspace=wsl), sub_steps, 3, stream, device)
            launches += 2 * sub_steps
            Fl = chunkwise_flops(wlg.B, wlg.H, wlg.N, wlg.dk, wlg.dv, wlg.chunk, state_out=True)
            cl = tl / sub_steps
            extra["long_64k"] = {"workload": "long_64k_bf16", "tokens_per_s": wlg.N / cl,
                                 "ms": cl * 1e3, "tflops": Fl / cl / 1e12,
                                 "frac_tc": Fl / cl / 1e12 / peak}
            del ql, kl, vl, ol, sl, wsl
            torch.cuda.empty_cache()

        # ---------------- backward on the 1.3B-class layer ----------------
        if want("backward"):
            wb = wl.WORKLOADS["l1p3b_bf16"]
            qb, kb, vb, gb = make_qkv(torch, wb.B, wb.H, wb.N, wb.dk, wb.dv, device, seed=7000 + rank)
            dob = (torch.randn(vb.shape, device=device) * 0.1).bfloat16()
            wsb = torch.empty(ret.load_library().ret_chunkwise_backward_workspace(
                wb.B, wb.H, wb.N, wb.dk, wb.dv, wb.chunk, ret.RET_BF16), dtype=torch.uint8,
                device=device)
            tb, _ = timed(lambda: ret.chunkwise_backward(qb, kb, vb, gb, wb.chunk, dob, workspace=wsb),
                          3, 1, stream, device)
            # bf16: six row reversals, three forward calls of two kernels each and
            # the d state_in scaling
            launches += 3 * 13
            Fb = 2 * chunkwise_flops(wb.B, wb.H, wb.N, wb.dk, wb.dv, wb.chunk)
            cb = tb / 3
            extra["backward"] = {"workload": "l1p3b_bf16 chunkwise backward (dq, dk, dv)",
                                 "ms": cb * 1e3, "tokens_per_s": wb.B * wb.N / cb,
                                 "tflops": Fb / cb / 1e12,
                                 "note": "bf16: three forward chunkwise calls of permuted and "
                                         "row-reversed inputs on the tensor cores; flops counted "
                                         "as twice the forward's"}
            del qb, kb, vb, dob, wsb
            torch.cuda.empty_cache()

        # ---------------- xPos rotation of q and k, 6.7B-class 8k layer ----------------
        if want("rotate"):
            wr = wl.WORKLOADS["l6p7b_8k_bf16"]
            qr, kr, vr, _ = make_qkv(torch, wr.B, wr.H, wr.N, wr.dk, wr.dv, device, seed=8000 + rank)
            del vr
            thr = torch.from_numpy(wl.rotation_angles(wr.dk, seed=1)).to(device)
            tr, _ = timed(lambda: (ret.rotate(qr, thr, 0, out=qr), ret.rotate(kr, thr, 0, out=kr)),
                          sub_steps, 3, stream, device)
            launches += 2 * sub_steps
            Br = 2 * 2 * qr.numel() * qr.element_size()   # q and k, each read and written once
            cr = tr / sub_steps
            extra["rotate"] = {"workload": "l6p7b_8k_bf16 xPos rotation of q and k, in place",
                               "ms": cr * 1e3, "hbm_gbs": Br / cr / 1e9,
                               "hbm_frac": Br / cr / 1e9 / peaks.get("hbm_gbs", 6650.0)}
            del qr, kr
            torch.cuda.empty_cache()

        # ---------------- gated output on the headline workload ----------------
        if want("gated"):
            qg, kg, vg, gg = make_qkv(torch, w.B, w.H, w.N, w.dk, w.dv, device, seed=6000 + rank)
            gate = torch.randn(vg.shape, device=device).bfloat16()
            og = torch.empty_like(vg)
            wsg = torch.empty(ret.chunkwise_workspace_bytes(w.B, w.H, w.N, w.dk, w.dv, w.chunk,
                                                            torch.bfloat16),
                              dtype=torch.uint8, device=device)
            tg, _ = timed(lambda: ret.chunkwise(qg, kg, vg, gg, w.chunk, gn_eps=w.gn_eps, out=og,
                                                workspace=wsg, gate=gate),
                          sub_steps, 3, stream, device)
            tu, _ = timed(lambda: ret.chunkwise(qg, kg, vg, gg, w.chunk, gn_eps=w.gn_eps, out=og,
                                                workspace=wsg),
                          sub_steps, 3, stream, device)
            launches += 4 * sub_steps
            cg_ = tg / sub_steps
            Fg = chunkwise_flops(w.B, w.H, w.N, w.dk, w.dv, w.chunk)
            extra["gated"] = {"workload": WORKLOAD + " with swish(gate) * GroupNorm(o)",
                              "tokens_per_s": w.B * w.N / cg_, "ms": cg_ * 1e3,
                              "ungated_ms": tu / sub_steps * 1e3,
                              "tflops": Fg / cg_ / 1e12, "frac_tc": Fg / cg_ / 1e12 / peak,
                              "gate_bytes": gate.numel() * gate.element_size()}
            del qg, kg, vg, og, wsg, gate
            torch.cuda.empty_cache()

    # ---------------- CPU oracle baseline ----------------
    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        val, heads, spent = oracle_sample(w.B * w.H, args.cpu_budget)
        cpu = {"value": val, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{heads} of {w.B * w.H} (batch, head) pairs of {WORKLOAD}, full "
                         f"{w.N} tokens, chunk {w.chunk}, GroupNorm; {spent:.1f} s of CPU work"}

    dev_err = ret.device_error()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": None if t_max is None else t_max / args.steps * 1e3,
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD if not args.batch else f"{WORKLOAD} (batch {B})",
                       "global_batch": B * world, "seq_len": N, "heads": H,
                       "dk": dk, "dv": dv, "chunk": C, "group_norm_eps": eps,
                       "parallelism": f"dp{world} (independent (batch, head) problems per GPU)",
                       "l2": "inputs 3.2 GB per step > 126 MB L2; no flush"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": headline_launches, "gpu_launches_all_timed": launches,
            "clocks": clocks.summary(), "device_error": dev_err,
        }
        line.update(extra)
        print(json.dumps(line), flush=True)
    return 0


def free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_launch_command(gpus: int, argv, port: int):
    """The torchrun command that runs this script once per GPU (one process
    per GPU, rendezvous on 127.0.0.1)."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={gpus}", "--master-addr=127.0.0.1", f"--master-port={port}",
            os.path.abspath(__file__), *argv]


def launch_ranks(gpus: int, argv) -> int:
    """Re-run this script under torchrun with `gpus` ranks; rank 0 prints the
    line.  Used when --gpus N > 1 is given outside torchrun."""
    return subprocess.call(rank_launch_command(gpus, argv, free_port()))


def run_plumbing_check(args):
    """The multi-rank plumbing without a GPU: every rank joins a gloo group,
    reports a fixed per-rank time (rank r takes 0.5 + r seconds for `steps`
    steps of the headline's tokens) and rank 0 prints n_gpus, the max time
    and the whole-job throughput, exactly as the GPU run aggregates them."""
    rank, world = init_dist("gloo")
    from linear_recurrent_sequence_scale_b200 import workloads as wl
    w = wl.WORKLOADS[WORKLOAD]
    t_local = 0.5 + rank
    barrier()
    t_max = max_over_ranks(t_local)
    value = global_throughput(w.B * w.N, args.steps, world, t_max)
    if rank == 0:
        print(json.dumps({"plumbing_check": True, "n_gpus": world, "gpus_requested": args.gpus,
                          "t_max_s": t_max, "value": value, "unit": "tokens/s"}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1,
                    help="GPUs (ranks); outside torchrun, N > 1 re-runs this script under it")
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of CPU oracle work for cpu_baseline")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-sub", action="store_true", help="headline only")
    ap.add_argument("--only", default="all",
                    choices=["all", "headline", "decode", "l1p3b", "long_64k", "backward", "rotate",
                             "gated"],
                    help="run one part (profiler captures); the line then lacks the others")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the headline batch (smaller profiler captures only)")
    ap.add_argument("--plumbing-check", action="store_true",
                    help="CPU only: run the rank launch and the cross-rank aggregation over gloo, "
                         "no kernels")
    raw = list(sys.argv[1:] if argv is None else argv)
    args = ap.parse_args(raw)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return launch_ranks(args.gpus, raw)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but {world} ranks were launched")
    if args.plumbing_check:
        try:
            return run_plumbing_check(args)
        finally:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()
    if args.impl == "reference":
        return run_reference(args)
    try:
        return run_ours(args)
    finally:
        try:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()
        except Exception:
            pass


if __name__ == "__main__":
    sys.exit(main())
