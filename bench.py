#!/usr/bin/env python
"""Throughput benchmark of the B200 KDA library (kda_chunk_fwd / kda_recurrent_step).

One step = one kda_chunk_fwd over the long-context bf16 prefill workload
(B=1, H=32, T=1,048,576, d=128, chunk 64, random initial state; the
largest single-GPU workload): in-chunk gate cumsum and decay factors, the
C x C score matrices, the triangular (UT/WY) solve, the W/U products, the
sequential state pass (with the chunk-parallel scan for few long chains)
and the outputs.  The training-shape prefill (B=8, H=32, T=8192) and the
small prefill (B=1, H=16, T=4096) are timed under the same rules and
reported under "prefill_other_workloads"; the single-token decode kernel is
measured on its own workload (256 sequences x 32 heads, d=128, 1000
consecutive steps) under "decode"; the backward pass under "backward".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one rank per GPU) every rank runs the same workload on
its own seeded sequences: the units are independent, so there is no
collective on the data path ("scaling": "weak"); timing is the device time
of each rank, max over ranks.  `--impl reference` times the fp64 CPU oracle
(the only reference this operator has) on a bounded prefix of the same
workload and prints its line from rank 0.
"""
from __future__ import annotations

import argparse
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

METRIC = "KDA prefill tokens/s & TFLOP/s (% bf16 peak); decode GB/s (% HBM peak), 1×B200"
DATA = ("synthetic, seeded: q,k ~N(0,1) L2-normalised per token; v ~N(0,1); beta=sigmoid(N(0,1)); "
        "g=logsigmoid(N(3,1)) per channel; S0 ~N(0,0.1^2)")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------- accounting
def prefill_flops_per_token_head(d: int, C: int = 64) -> float:
    """Algorithmic FLOPs of the chunked method per token and head (triangle-aware):
    A_kk, A_qk, the triangular inverse, W, U, A_qk V' and the three state-pass
    products, divided by the chunk length."""
    akk = 2 * C * (C - 1) / 2 * d
    aqk = 2 * C * (C + 1) / 2 * d
    tri = 3 * 2 * C * (C + 1) / 2 * d
    inv = C * (C - 1) * (C - 2) / 3  # forward substitution of the unit triangle, 83,328 at C=64
    state = 3 * 2 * C * d * d
    return (akk + aqk + tri + inv + state) / C


def prefill_bytes(B, T, H, dk, dv, elem=2, state_in=True, state_out=True) -> float:
    """Algorithmic HBM bytes of one call: q,k,g,v,beta read, o written, the fp32 state read/written once."""
    per_tok = (3 * dk + dv + 1 + dv) * elem
    st = B * H * dk * dv * 4
    return B * T * H * per_tok + st * (int(state_in) + int(state_out))


def prep_input_bytes(B, T, H, dk, dv, elem=2) -> float:
    """Algorithmic bytes of the prep kernel alone: its inputs q, k, the
    per-channel g, v and beta (the record it writes is an intermediate)."""
    return B * T * H * (3 * dk + dv + 1) * elem


def backward_bytes(B, T, H, dk, dv, elem=2) -> float:
    """Algorithmic HBM bytes of one backward call: q, k, g, v, beta, dL/do read;
    dq, dk, dg, dv, dbeta written; S0 and dL/dS_T read, dL/dS0 written (fp32)."""
    per_tok = ((3 * dk + 2 * dv + 1) + (3 * dk + dv + 1)) * elem
    return B * T * H * per_tok + 3 * B * H * dk * dv * 4


def backward_macs(B, T, H, dk, dv, chunk=64) -> float:
    """Tensor-core multiply-adds the chunkwise backward issues (full tiles):
    the chunk operands (P, Aqk, W, U), the forward replay (V', S), the reverse
    sweep (dV', dS), the d_v contractions (dAqk, dT, T^T dU, dO S0^T, dW,
    dKbar) and the rest (dT, T^T dW, dA, dQ+, dK-, dK+), per chunk and head."""
    c = chunk
    per = (2 * c * c * dk + c * c * (dk + dv)) + 2 * c * dk * dv + (c * dv * (c + dk) + 2 * dk * dv * c) \
        + (2 * c * c * dv + c * dv * c + 3 * c * dk * dv) + (2 * c * c * dk + 2 * c ** 3 + 4 * c * c * dk)
    return B * H * -(-T // c) * per


def decode_bytes(N, H, dk, dv, elem=2) -> float:
    return N * H * (2 * dk * dv * 4 + (3 * dk + 2 * dv + 1) * elem)


# Dense tf32 / bf16 tensor throughput of the B200 (nominal 1.1 / 2.25 PFLOP/s),
# applied to the measured bf16 peak to get a tf32 peak.
TF32_PER_BF16 = 1.1 / 2.25


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def weak_scaling_value(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return units_per_rank * world / max_seconds


def reduce_max(x: float, device=None) -> float:
    """Max of a float over all ranks (no-op without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled in the background."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, interval_ms: int = 20):
        self.path = tempfile.mktemp(prefix="kda_clocks_", suffix=".csv")
        self.proc = None
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", f"-lms", str(interval_ms)],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i in range(4) if r[i].lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------- oracle leg
def oracle_throughput(cfg, tokens: int, nthreads: int = 0):
    """Times the fp64 oracle on all heads of the workload's first `tokens`
    tokens; returns (tokens/s of the workload, seconds, threads)."""
    import oracle
    from gated_delta_rule_67_b200.workloads import make_config_inputs
    x = make_config_inputs(cfg, device="cpu", T=tokens)
    args = [x[n] for n in ("q", "k", "v", "g", "beta")]
    import numpy as np
    f64 = [np.ascontiguousarray(a.double().numpy()) for a in args]
    s0 = None if x["initial_state"] is None else x["initial_state"].double().numpy()
    t0 = time.perf_counter()
    oracle.kda_forward(*f64, cfg.scale, s0, nthreads=nthreads)
    dt = time.perf_counter() - t0
    return cfg.B * tokens / dt, dt, oracle.max_threads() if nthreads <= 0 else nthreads


PREFILL_SOURCES = ["gated_delta_rule_67_b200/csrc/kda_prefill_bf16.cu", "gated_delta_rule_67_b200/csrc/sm100.cuh"]


def bench_config(cfg, world):
    """The `config` object of both arms' JSON lines (same keys on both)."""
    return {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "T": cfg.T, "dk": cfg.dk, "dv": cfg.dv,
            "chunk": cfg.chunk, "l2": "inputs larger than L2, and L2 flushed (256 MiB write) between timed steps",
            "parallelism": f"dp{world}: independent sequences per GPU, no collective"}


def run_reference(args, cfg):
    """The reference arm: the fp64 oracle on the host cores, same workload/metric."""
    import oracle
    oracle.build()
    # Size each step's sample so the whole --steps/--warmup run takes about a minute.
    probe_tok = 64
    _, dt_probe, cores = oracle_throughput(cfg, probe_tok)
    budget = 60.0 / max(1, args.steps + args.warmup)
    tokens = int(max(16, min(cfg.T, probe_tok * budget / max(dt_probe, 1e-6))))
    for _ in range(args.warmup):
        oracle_throughput(cfg, tokens)
    times = []
    for _ in range(args.steps):
        _, dt, cores = oracle_throughput(cfg, tokens)
        times.append(dt)
    total = sum(times)
    value = cfg.B * tokens * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": DATA,
        "config": bench_config(cfg, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"all {cfg.H} heads x first {tokens} of {cfg.T} tokens per step "
                                   f"(fp64 token-by-token recurrence, OpenMP over heads x 16-column blocks)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- our arm
def traffic_from_profile(kernel_sources):
    """DRAM bytes per call from the committed ncu summary, if it was taken on
    the kernel sources as they are now (else None)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None, None
    with open(p) as f:
        d = json.load(f)
    h = hashlib.sha256()
    for s in kernel_sources:
        with open(os.path.join(ROOT, s), "rb") as fh:
            h.update(fh.read())
    if d.get("source_sha256") != h.hexdigest():
        return None, d
    return d, d


NOMINAL_HBM_GBS = 8000.0  # B200 datasheet HBM3e bandwidth, for context beside the measured copy peak


def hbm_fracs(achieved_gbs, peaks):
    """Fraction of the measured copy peak (the roofline denominator) and of the
    nominal datasheet figure; flags a kernel that reads above the measured copy."""
    d = {"frac": achieved_gbs / peaks["hbm_gbs"], "frac_nominal": achieved_gbs / NOMINAL_HBM_GBS}
    if achieved_gbs > peaks["hbm_gbs"]:
        d["above_measured_peak"] = True
    return d


class PrefillCase:
    """One prefill workload resident on the device: seeded inputs, outputs, workspace."""

    def __init__(self, cfg, rank, dev):
        import torch
        from gated_delta_rule_67_b200 import kda_chunk_fwd_workspace_size
        from gated_delta_rule_67_b200.workloads import make_prefill_inputs
        self.cfg = cfg
        x = make_prefill_inputs(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, cfg.torch_dtype, cfg.s0_std,
                                seed=cfg.seed + 1000 * rank, device=dev)
        self.ins = [x[n] for n in ("q", "k", "v", "g", "beta")]
        self.s0 = x["initial_state"]
        self.o = torch.empty_like(x["v"])
        self.sT = torch.empty((cfg.B, cfg.H, cfg.dk, cfg.dv), dtype=torch.float32, device=dev)
        nws = kda_chunk_fwd_workspace_size(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, cfg.chunk, cfg.torch_dtype)
        self.ws = torch.empty(max(1, nws), dtype=torch.uint8, device=dev)

    def call(self, evs=None, ins=None):
        from gated_delta_rule_67_b200 import kda_chunk_fwd
        kda_chunk_fwd(*(ins or self.ins), self.cfg.scale, self.s0, chunk=self.cfg.chunk, o=self.o,
                      final_state=self.sT, workspace=self.ws, events=evs)

    def nbytes(self):
        c = self.cfg
        return prefill_bytes(c.B, c.T, c.H, c.dk, c.dv, 4 if c.dtype == "f32" else 2, self.s0 is not None, True)


def time_calls(case, steps, warmup, flush, stream, sampler_gpu=None, world=1, dev=None):
    """W untimed calls, then K calls each bracketed by CUDA events on the launching
    stream, L2 flushed (a 256 MiB write) before every call outside the events.
    Returns (per-call ms list, clocks summary or None)."""
    import torch
    import torch.distributed as dist
    for _ in range(warmup):
        flush.zero_()
        case.call()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    for pair in evs:  # materialise the event handles
        for e in pair:
            e.record(stream)
    torch.cuda.synchronize()
    sampler = ClockSampler(sampler_gpu) if sampler_gpu else None
    if sampler:
        time.sleep(0.1)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        evs[i][0].record(stream)
        case.call()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = None
    if sampler:
        sampler.stop()
        clocks = sampler.summary()
    return [a.elapsed_time(b) for a, b in evs], clocks


def run_ours(args, cfg):
    import torch
    import torch.distributed as dist
    from gated_delta_rule_67_b200 import kda_chunk_fwd, kda_chunk_fwd_launch_count, kda_recurrent_step
    from gated_delta_rule_67_b200.workloads import DECODE_BF16, PREFILL_CONFIGS, make_decode_inputs

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)
    peaks, peaks_kind = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > 126 MB of L2
    stream = torch.cuda.current_stream(dev)
    gpu_id = str(torch.cuda.get_device_properties(dev).uuid)
    gpu_id = gpu_id if gpu_id.startswith("GPU-") else "GPU-" + gpu_id

    # ---- the headline workload (inputs resident in HBM, independent sequences per rank)
    case = PrefillCase(cfg, rank, dev)
    step_ms, clocks = time_calls(case, args.steps, args.warmup, flush, stream, gpu_id, world, dev)
    # The timed calls record events only around each call (an event recorded
    # between two kernels would hold the second one back until the first has
    # drained); the prep / state-pass split comes from separate profiled calls.
    split_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(min(args.steps, 10))]
    for trip in split_evs:  # materialise the event handles before the library records them
        for e in trip:
            e.record(stream)
    torch.cuda.synchronize()
    for trip in split_evs:
        flush.zero_()
        case.call(trip)
    torch.cuda.synchronize()
    prep_ms = [a.elapsed_time(b) for a, b, _ in split_evs]
    state_ms = [b.elapsed_time(c) for _, b, c in split_evs]
    total_s = reduce_max(sum(step_ms) / 1e3, dev)
    tokens = cfg.B * cfg.T
    value = weak_scaling_value(tokens * args.steps, world, total_s)
    ms_per_step = 1e3 * total_s / args.steps
    flops = prefill_flops_per_token_head(cfg.dk) * tokens * cfg.H
    nbytes = case.nbytes()
    mean_prep, mean_state = statistics.mean(prep_ms), statistics.mean(state_ms)
    launches_per_step = kda_chunk_fwd_launch_count(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, cfg.chunk, cfg.torch_dtype)
    dom = "kda_state_pass+scan" if mean_state >= mean_prep else "kda_chunk_prep"

    # ---- roofline of the operator call (its kernels together)
    call_s = ms_per_step / 1e3
    achieved = nbytes / call_s / 1e9
    prof, _ = traffic_from_profile(PREFILL_SOURCES)
    traffic = None if prof is None else prof.get("bytes_per_call", {}).get(cfg.name)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                **hbm_fracs(achieved, peaks), "traffic": traffic,
                "scope": f"whole kda_chunk_fwd call ({launches_per_step} launches); algorithmic bytes "
                         f"{nbytes / 1e6:.2f} MB per call (1282 B per token-head + 2 x 64 KiB state per chain); "
                         f"peak = {peaks_kind} hbm_gbs; traffic = ncu DRAM bytes per call"
                         + ("" if prof is None else f" ({prof.get('traffic_note', '')})"),
                "kernels": {"kda_chunk_prep": {"ms": mean_prep, "share": mean_prep / (mean_prep + mean_state)},
                            "kda_state_pass+scan": {"ms": mean_state,
                                                    "share": mean_state / (mean_prep + mean_state)}},
                "dominant": dom}
    # the prep kernel on its own: its algorithmic bytes are its inputs (q, k, v,
    # the per-channel g and beta); the record it writes is an intermediate
    prep_bytes = prep_input_bytes(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv)
    prep_gbs = prep_bytes / (mean_prep / 1e3) / 1e9
    roofline["dominant_kernel"] = {
        "name": "kda_chunk_prep", "ms": mean_prep, "algorithmic_bytes": prep_bytes, "achieved": prep_gbs,
        **hbm_fracs(prep_gbs, peaks),
        "traffic": None if prof is None else prof.get("prep_bytes_per_launch", {}).get(cfg.name),
        "scope": "one prep launch: q, k, v, g, beta read (1026 B per token-head at d = 128); CUDA events "
                 "around it in separate calls; traffic = ncu DRAM bytes of the launch (reads its inputs, "
                 "writes the 74 KB record per 64-token tile)"}
    tflops = flops / call_s / 1e12

    # ---- end to end through the public API: every step copies its inputs from
    # pinned host memory into the device buffers and reads o and the final state back
    h_ins = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t) for t in case.ins]
    h_s0 = None if case.s0 is None else torch.empty(case.s0.shape, dtype=torch.float32, pin_memory=True).copy_(case.s0)
    h_o = torch.empty(case.o.shape, dtype=case.o.dtype, pin_memory=True)
    h_sT = torch.empty(case.sT.shape, dtype=torch.float32, pin_memory=True)
    e2e_steps = max(3, min(args.steps, args.e2e_steps))

    def e2e_step():
        for d, hsrc in zip(case.ins, h_ins):
            d.copy_(hsrc, non_blocking=True)
        if case.s0 is not None:
            case.s0.copy_(h_s0, non_blocking=True)
        case.call()
        h_o.copy_(case.o, non_blocking=True)
        h_sT.copy_(case.sT, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record()
    for _ in range(e2e_steps):
        e2e_step()
    eb.record()
    torch.cuda.synchronize()
    e2e_s = reduce_max(ea.elapsed_time(eb) / 1e3, dev)
    h2d = sum(t.numel() * t.element_size() for t in h_ins) + (0 if h_s0 is None else h_s0.numel() * 4)
    d2h = h_o.numel() * h_o.element_size() + h_sT.numel() * 4
    e2e = {"value": weak_scaling_value(tokens * e2e_steps, world, e2e_s), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps}
    del h_ins, h_s0, h_o, h_sT, case
    torch.cuda.empty_cache()

    # ---- the other prefill workloads, same timing rules (extra keys; the headline is above)
    others = {}
    for name in args.also:
        c = PREFILL_CONFIGS[name]
        oc = PrefillCase(c, rank, dev)
        ms, _ = time_calls(oc, args.steps, args.warmup, flush, stream, None, world, dev)
        s = reduce_max(sum(ms) / 1e3, dev) / args.steps
        gb = oc.nbytes() / s / 1e9
        tr = None if prof is None else prof.get("bytes_per_call", {}).get(c.name)
        others[c.name] = {"us_per_call": s * 1e6, "tokens_per_s": weak_scaling_value(c.B * c.T, world, s),
                          "calls": args.steps, "algorithmic_bytes": oc.nbytes(), "achieved_gbs": gb,
                          **hbm_fracs(gb, peaks), "traffic": tr,
                          "tflops": prefill_flops_per_token_head(c.dk) * c.B * c.T * c.H / s / 1e12,
                          "launches": kda_chunk_fwd_launch_count(c.B, c.T, c.H, c.dk, c.dv, c.chunk, c.torch_dtype)}
        del oc
        torch.cuda.empty_cache()

    # ---- the scalar-gate forms and the fused input preparation on the bench-sized prefill
    variants = None
    if not args.no_variants:
        import torch.nn.functional as F
        from gated_delta_rule_67_b200.binding import KDA_PREP_ALL
        from gated_delta_rule_67_b200.workloads import PREFILL_BF16, make_head_gates, make_raw_prefill_inputs
        vc = PREFILL_BF16
        base = PrefillCase(vc, rank, dev)
        ins, s0, o, sT, ws = base.ins, base.s0, base.o, base.sT, base.ws
        gh = make_head_gates((vc.B, vc.T, vc.H), 1, vc.torch_dtype, seed=vc.seed + 7 + 1000 * rank, device=dev)
        raw = make_raw_prefill_inputs(vc.B, vc.T, vc.H, vc.dk, vc.dv, vc.torch_dtype, vc.s0_std,
                                      vc.seed + 11 + 1000 * rank, dev)
        rq, rk, rv, rg, rb = (raw[n] for n in ("q", "k", "v", "g", "beta"))
        nvar = max(3, min(args.steps, 100))

        def timed(fn):
            for _ in range(3):
                fn()
            ts = []
            for _ in range(nvar):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b))
            us = 1e3 * reduce_max(statistics.median(ts), dev)
            return {"us_per_call": us, "tokens_per_s": weak_scaling_value(vc.B * vc.T, world, us / 1e6),
                    "calls": nvar}

        def unfused():  # the same preparation as separate PyTorch ops ahead of the call (comparison only)
            qn = (rq.float() * torch.rsqrt((rq.float() ** 2).sum(-1, keepdim=True) + 1e-6)).to(rq.dtype)
            kn = (rk.float() * torch.rsqrt((rk.float() ** 2).sum(-1, keepdim=True) + 1e-6)).to(rk.dtype)
            kda_chunk_fwd(qn, kn, rv, F.logsigmoid(rg.float()).to(rg.dtype), torch.sigmoid(rb.float()).to(rb.dtype),
                          vc.scale, s0, chunk=vc.chunk, o=o, final_state=sT, workspace=ws)

        variants = {
            "workload": vc.name,
            "kda_channel_gate": timed(lambda: base.call()),
            "gated_deltanet_head_gate": timed(lambda: kda_chunk_fwd(ins[0], ins[1], ins[2], gh, ins[4], vc.scale, s0,
                                                                    chunk=vc.chunk, o=o, final_state=sT,
                                                                    workspace=ws)),
            "deltanet_no_gate": timed(lambda: kda_chunk_fwd(ins[0], ins[1], ins[2], None, ins[4], vc.scale, s0,
                                                            chunk=vc.chunk, o=o, final_state=sT, workspace=ws)),
            "fused_input_prep": timed(lambda: kda_chunk_fwd(rq, rk, rv, rg, rb, vc.scale, s0, chunk=vc.chunk, o=o,
                                                            final_state=sT, workspace=ws, prep=KDA_PREP_ALL)),
            "unfused_prep_torch_then_call": timed(unfused),
            "note": "median per call, L2 flushed between calls; raw inputs ~ N(0,1) (q, k, v, beta), "
                    "N(3,1) (g) before preparation; the unfused line runs the preparation as PyTorch ops "
                    "before the call, for comparison only",
        }
        del raw, gh, base, ins, s0, o, sT, ws
        torch.cuda.empty_cache()

    # ---- backward pass on the bench-sized prefill and on the training shape
    backward = None
    if not args.no_backward:
        backward = {}
        for name in args.backward_workloads:
            backward[name] = time_backward(PREFILL_CONFIGS[name], args.backward_calls, rank, world, dev, flush,
                                           stream, peaks)
            torch.cuda.empty_cache()

    # ---- decode kernel on its own workload (the last device timing: a timing
    # taken right after its 1000 HBM-bound steps came out up to 8 % slower)
    decode = None
    if not args.no_decode:
        dc = DECODE_BF16
        nsteps = args.decode_steps
        y = make_decode_inputs(nsteps, dc.N, dc.H, dc.dk, dc.dv, dc.torch_dtype, dc.s0_std, dc.seed + rank, dev)
        st = y["state"]
        od = torch.empty((dc.N, dc.H, dc.dv), dtype=dc.torch_dtype, device=dev)
        for t in range(min(5, nsteps)):
            kda_recurrent_step(y["q"][t], y["k"][t], y["v"][t], y["g"][t], y["beta"][t], st, dc.scale, o=od)
        torch.cuda.synchronize()
        da, db = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        da.record()
        for t in range(nsteps):
            kda_recurrent_step(y["q"][t], y["k"][t], y["v"][t], y["g"][t], y["beta"][t], st, dc.scale, o=od)
        db.record()
        torch.cuda.synchronize()
        d_s = reduce_max(da.elapsed_time(db) / 1e3, dev) / nsteps
        gbs = decode_bytes(dc.N, dc.H, dc.dk, dc.dv) / d_s / 1e9
        decode = {"workload": dc.name, "us_per_step": d_s * 1e6, "steps": nsteps,
                  "value": gbs * world, "unit": "GB/s", **hbm_fracs(gbs, peaks),
                  "tokens_per_s": dc.N * world / d_s, "kernel": "decode_step_kernel (1 launch/step)",
                  "bytes_per_step": decode_bytes(dc.N, dc.H, dc.dk, dc.dv)}
        del y

    # ---- CPU baseline: the oracle on the host cores (rank 0, N = 1 only), on a
    # labelled prefix of the headline workload (the oracle's cost is linear in T,
    # so its tokens/s on the prefix is its rate on the whole sequence)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ctoks = min(cfg.T, args.cpu_tokens)
        v, dt, cores = oracle_throughput(cfg, ctoks)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"all {cfg.H} heads x first {ctoks} of {cfg.T} tokens, one pass ({dt:.2f} s), "
                         f"fp64 token-by-token recurrence; rate extrapolated linearly to the whole sequence"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": cfg.dtype, "data": DATA, "config": bench_config(cfg, world),
            "tflops": tflops, "tflops_frac_bf16": tflops / peaks["bf16_tflops"],
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks, "prefill_other_workloads": others, "decode": decode, "variants": variants,
            "backward": backward,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def time_backward(cfg, calls, rank, world, dev, flush, stream, peaks):
    """Median device time of kda_backward over `calls` calls (L2 flushed between)."""
    import torch
    from gated_delta_rule_67_b200 import kda_backward
    from gated_delta_rule_67_b200.binding import load as load_lib
    from gated_delta_rule_67_b200.workloads import make_cotangents, make_prefill_inputs
    x = make_prefill_inputs(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, cfg.torch_dtype, cfg.s0_std,
                            seed=cfg.seed + 1000 * rank, device=dev)
    d_o, d_s = make_cotangents(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, cfg.torch_dtype, seed=cfg.seed + 13 + 1000 * rank,
                               device=dev)
    bws = torch.empty(max(1, int(load_lib().kda_backward_workspace_size(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv,
                                                                         1 if cfg.dtype == "bf16" else 0))),
                      dtype=torch.uint8, device=dev)
    bargs = (x["q"], x["k"], x["v"], x["g"], x["beta"], d_o, cfg.scale, x["initial_state"], d_s)
    for _ in range(2):
        kda_backward(*bargs, workspace=bws)
    torch.cuda.synchronize()
    ts = []
    for _ in range(calls):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        kda_backward(*bargs, workspace=bws)
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    bs = reduce_max(statistics.median(ts) / 1e3, dev)
    tokens = cfg.B * cfg.T
    bbytes = backward_bytes(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, 2 if cfg.dtype == "bf16" else 4)
    bflops = 2 * backward_macs(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv)
    bf16_in = cfg.dtype == "bf16"
    # the tensor-core products run on bf16 operands for bf16 inputs, on tf32 (three-term split) for fp32
    mma_peak = peaks["bf16_tflops"] * (1.0 if bf16_in else TF32_PER_BF16)
    gbs = bbytes / bs / 1e9
    return {"us_per_call": bs * 1e6, "tokens_per_s": weak_scaling_value(tokens, world, bs),
            "calls": calls, "algorithmic_bytes": bbytes, "achieved_gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
            "issued_tflops": bflops / bs / 1e12, "mma_dtype": "bf16" if bf16_in else "tf32x3",
            "mma_peak_tflops": mma_peak, "frac_mma_peak": bflops / bs / 1e12 / mma_peak,
            "workspace_bytes": bws.numel(), "launches": 4,
            "kernel": "chunkwise: bwd_prep, bwd_pass (forward replay + reverse dS sweep), bwd_local_a, "
                      "bwd_local_b"}


def main(argv=None):
    from gated_delta_rule_67_b200.workloads import LONG_BF16, PREFILL_BF16, PREFILL_CONFIGS, TINY_F32, TRAIN_BF16
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=LONG_BF16.name, choices=sorted(PREFILL_CONFIGS),
                    help="headline prefill workload (default: the largest single-GPU one, T = 1,048,576)")
    ap.add_argument("--also", nargs="*", default=[TRAIN_BF16.name, PREFILL_BF16.name, TINY_F32.name],
                    help="further prefill workloads timed under the same rules (extra keys)")
    ap.add_argument("--backward-workloads", nargs="*", default=[PREFILL_BF16.name, TRAIN_BF16.name])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-variants", action="store_true", help="skip the gate-variant / fused-prep timings")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward-pass timing")
    ap.add_argument("--backward-calls", type=int, default=20)
    ap.add_argument("--cpu-tokens", type=int, default=32768)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    cfg = PREFILL_CONFIGS[args.workload]
    if args.impl == "reference":
        if int(os.environ.get("RANK", 0)) != 0:
            return 0
        run_reference(args, cfg)
        return 0
    run_ours(args, cfg)
    return 0


if __name__ == "__main__":
    sys.exit(main())
