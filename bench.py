#!/usr/bin/env python3
"""Benchmark of the KDA forward pass on B200: chunked-prefill tokens/s with its HBM roofline fraction,
plus the fused decode step's state GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload {1,2,3,4,5}] [--impl {ours,reference}]

One step = one pass of the forward pass over one batch of the workload with inputs resident in
HBM: one ``kda_chunk_fwd`` call for the prefill workloads (1-4), one ``kda_recurrent_step`` call for
the decode workload (5).  The headline line is workload 4 (B1 T65536 H8->HV32, the largest
single-GPU configuration); the other prefill workloads (2, 3) and the decode workload (5) are
measured in the same run and reported as extra keys, each with its own roofline.

Rank 0 prints ONE JSON line.  ``--gpus N`` with N > 1 relaunches this script under
torch.distributed.run (one process per GPU, rendezvous on 127.0.0.1) unless it already runs under
it.  Every rank runs the same workload on its own GPU over its own independent (b, hv) shard -- the
forward pass has no exchange step, so there is no collective on the data path (weak scaling); a
barrier and a MAX all-reduce of the device times are the only communication.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from kimi_delta_attention_33_b200.inputs import (GATE_STANDARD, MLA_DECODE, WORKLOADS, make_inputs,  # noqa: E402
                                                 make_mla_inputs)

METRIC = "KDA fwd tokens/s (chunked prefill) & decode-step state GB/s, % of roofline, 1 B200"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
# source file of the kernels each kda_chunk_fwd schedule runs (keys: kda.SCHEDULE_* values)
PREFILL_KERNEL_FILES = {0: "kimi_delta_attention_33_b200/csrc/kda_chunk_simt.cu",
                        1: "kimi_delta_attention_33_b200/csrc/kda_chunk_tc.cu",
                        2: "kimi_delta_attention_33_b200/csrc/kda_chunk_split.cu",
                        3: "kimi_delta_attention_33_b200/csrc/kda_chunk_split.cu"}
DECODE_KERNEL_FILE = "kimi_delta_attention_33_b200/csrc/kda_decode.cu"
MLA_KERNEL_FILE = "kimi_delta_attention_33_b200/csrc/kda_mla.cu"


# ------------------------------------------------------------------------ algorithmic counts ---

def elt_bytes(w):
    return 2 if w.dtype == torch.bfloat16 else 4


def prefill_bytes(w) -> int:
    """Bytes the forward pass must move: q, k once per H head, v, g_raw, beta, A_log, dt_bias and S0
    (when given) read; o and S_T written.  Per-chunk states and intermediates are not counted."""
    e = elt_bytes(w)
    B, T, H, HV, K, V = w.B, w.T, w.H, w.HV, w.K, w.V
    rd = 2 * B * T * H * K * e + B * T * HV * V * e + B * T * HV * K * e + B * T * HV * e + HV * 4 + HV * K * 4
    if w.S0_std is not None:
        rd += B * HV * K * V * 4
    wr = B * T * HV * V * e + B * HV * K * V * 4
    return rd + wr


def prefill_flops(w) -> float:
    """2 flops per multiply-add, triangles counted half: A, R, W, U (C*K/2 or C*V/2 each), the solve
    (C^2/6), the three K x V state products and A.E (C*V/2), per token and value head."""
    C, K, V = w.chunk, w.K, w.V
    per = 2 * (4 * (C * K / 2) + C * C / 6 + 3 * K * V + C * V / 2)
    return per * w.B * w.T * w.HV


def decode_bytes(w) -> int:
    """Per decode step: S read and written (fp32), q, k per H head, v, g_raw, beta, A_log, dt_bias, o."""
    e = elt_bytes(w)
    B, H, HV, K, V = w.B, w.H, w.HV, w.K, w.V
    return (2 * B * HV * K * V * 4 + 2 * B * H * K * e + B * HV * V * e + B * HV * K * e + B * HV * e + HV * 4
            + HV * K * 4 + B * HV * V * e)


def mla_bytes(B, T, H, d_q, d_v, r) -> int:
    """Absorbed MLA decode: the latent cache, both up-projections, q read once; o written (bf16)."""
    return 2 * (B * T * r + H * d_q * r + H * d_v * r + B * H * d_q + B * H * d_v)


def mla_flops(B, T, H, d_q, d_v, r) -> float:
    """q W_UK, the scores, the weighted latent sum and the W_UV projection, 2 flops per multiply-add."""
    return 2.0 * B * H * (d_q * r + 2 * T * r + d_v * r)


# -------------------------------------------------------------------------------- peaks etc ----

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 1632.8)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, 1590.0, "fallback"


def _sha(path):
    with open(os.path.join(ROOT, path), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def ncu_traffic(kernel_file: str, wid: int):
    """DRAM bytes per launch from the committed ncu summary, or None when absent or stale."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            table = json.load(f)
    except Exception:
        return None
    ent = table.get(f"{kernel_file}#{wid}")
    if not ent or ent.get("source_sha256") != _sha(kernel_file):
        return None
    return ent.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------------- clocks -----

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only) while running."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons = [], set()
        self.period, self.stop_evt, self.thread, self.max_mhz = period_s, threading.Event(), None, None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        except Exception:
            self.nv = None

    def _run(self):
        while not self.stop_evt.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.get_reasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join()

    def summary(self):
        if self.nv is None:
            return None
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------------------ distributed ---

def dist_setup(backend: str = "nccl"):
    """One process per GPU from the torch.distributed.run environment.  The bench uses NCCL; the
    CPU tests of this plumbing pass backend="gloo" (no device is touched then)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend == "nccl":
        torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    """MAX of a per-rank scalar over all ranks (every rank gets the result)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(w, rank: int) -> int:
    """Seed of a rank's input shard: rank 0 draws the workload's own inputs (seed 1000 + id, as the
    parity tests do), every other rank an independent shard of the same shape."""
    return 1000 + w.wid + 7919 * rank


def aggregate(units_per_step: int, steps: int, local_total_ms: float, ws: int):
    """Whole-job throughput under weak scaling: every rank processed units_per_step per step on its
    own shard; the job took as long as its slowest rank.  Returns (value per second, ms per step)."""
    total_ms = max_over_ranks(local_total_ms, ws)
    return ws * units_per_step * steps / (total_ms / 1e3), total_ms / steps


# ----------------------------------------------------------------------------- our arm -------

def _step_inputs_decode(x, w, dev):
    """Per-step contiguous slices [steps, B, ...] of the decode token stream."""
    return {n: x[n].to(dev).transpose(0, 1).contiguous() for n in ("q", "k", "v", "g", "beta")}


def l2_note(w) -> str:
    """How the timed steps keep the L2 cache from serving the inputs: a flush between steps for a
    workload whose bytes fit in L2 twice over, else nothing (its inputs alone exceed L2)."""
    small = (not w.is_decode) and prefill_bytes(w) < 2 * (126 << 20)
    return "flushed between timed steps (256 MiB write)" if small else "inputs larger than L2"


def workload_config(w, ws):
    """The `config` object of a line; identical for both arms of the same workload."""
    return {"workload": f"workload {w.wid}: {w.name}", "B": w.B, "T": w.T, "H": w.H, "HV": w.HV, "K": w.K,
            "V": w.V, "chunk": w.chunk, "gate": "standard" if w.gate_mode == GATE_STANDARD else "safe",
            "inputs": "bf16" if w.dtype == torch.bfloat16 else "fp32", "state": "fp32",
            "S0": w.S0_std is not None, "l2": l2_note(w),
            "parallelism": f"dp{ws} (independent (b, hv) shards per GPU, no collective)"}


def _time_steps(step, steps, stream, dev, flush, ws, clk=None):
    """Device time (ms) of each of `steps` calls of step(i), CUDA events on `stream`, bracketed by a
    barrier and a synchronize on both sides; `flush` (or None) is zeroed before every step."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(ws)
    torch.cuda.synchronize(dev)
    if clk is not None:
        clk.__enter__()
    try:
        for i in range(steps):
            if flush is not None:
                flush.zero_()
            evs[i][0].record(stream)
            step(i)
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
    finally:
        if clk is not None:
            clk.__exit__()
    barrier(ws)
    return [a.elapsed_time(b) for a, b in evs]


def _roofline(bytes_per_launch, flops, sec_per_launch, hbm_peak, peak_kind, kernel_file, wid):
    achieved = bytes_per_launch / sec_per_launch / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "peak_kind": peak_kind,
            "unit": "GB/s", "frac": round(achieved / hbm_peak, 4), "traffic": ncu_traffic(kernel_file, wid),
            "kernel_file": kernel_file, "algorithmic_bytes_per_launch": bytes_per_launch}
    if flops:
        roof["algorithmic_flops_per_launch"] = flops
        roof["achieved_tflops"] = round(flops / sec_per_launch / 1e12, 2)
    return roof


class Prefill:
    """One prefill workload resident on the device: inputs, outputs and the workspace that selects
    the fastest schedule, and one ``kda_chunk_fwd`` call per step."""

    def __init__(self, w, seed, dev, kda):
        self.w, self.kda, self.dev = w, kda, dev
        self.x = make_inputs(w, seed=seed, device=str(dev))
        self.ws_bytes = kda.workspace_size(w.B, w.T, w.H, w.HV, w.K, w.V, w.chunk)
        self.workspace = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.o = torch.empty(w.B, w.T, w.HV, w.V, dtype=w.dtype, device=dev)
        self.S_T = torch.empty(w.B, w.HV, w.K, w.V, dtype=torch.float32, device=dev)
        self.sched = kda.schedule(w.B, w.T, w.H, w.HV, w.K, w.V, w.chunk, w.dtype, self.ws_bytes)
        self.kernel_file = PREFILL_KERNEL_FILES[self.sched]
        self.launches = kda.schedule_launches(w.B, w.T, w.H, w.HV, w.K, w.V, w.chunk, w.dtype, self.ws_bytes)

    def step(self, i=0):
        x, w = self.x, self.w
        self.kda.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["S0"],
                           chunk=w.chunk, gate_mode=w.gate_mode, lower_bound=w.lower_bound, o=self.o, S_T=self.S_T,
                           workspace=self.workspace)

    def measure(self, steps, warmup, ws, flush, hbm_peak, peak_kind, clk=None):
        w = self.w
        for i in range(warmup):
            self.step(i)
        torch.cuda.synchronize(self.dev)
        self.kda.read_status(self.workspace)
        stream = torch.cuda.current_stream(self.dev)
        ms = _time_steps(self.step, steps, stream, self.dev, flush if l2_note(w).startswith("flushed") else None,
                         ws, clk)
        self.kda.read_status(self.workspace)
        value, ms_per_step = aggregate(w.B * w.T, steps, sum(ms), ws)
        # one library call per step: its kernels are timed together, since the algorithmic bytes
        # belong to the pass as a whole
        roof = _roofline(prefill_bytes(w), prefill_flops(w), (sum(ms) / steps) / 1e3, hbm_peak, peak_kind,
                         self.kernel_file, w.wid)
        roof["schedule"] = self.kda.SCHEDULE_NAMES[self.sched]
        roof["kernels_per_call"] = self.launches
        return value, ms_per_step, roof


def measure_decode(w, seed, dev, kda, hbm_peak, peak_kind, ws=1, steps=None, warmup=3, clk=None):
    """`steps` consecutive kda_recurrent_step calls (default: the workload's 128) on the workload's token
    stream, the state updated in place; returns (tokens/s, ms per step, roofline)."""
    x = make_inputs(w, seed=seed, device=str(dev))
    steps_in = _step_inputs_decode(x, w, dev)
    S = x["S0"].clone()
    o = torch.empty(w.B, w.HV, w.V, dtype=w.dtype, device=dev)
    nsteps = steps_in["q"].shape[0]
    steps = steps or w.decode_steps

    def step(i):
        t = i % nsteps
        kda.recurrent_step(steps_in["q"][t], steps_in["k"][t], steps_in["v"][t], steps_in["g"][t],
                           steps_in["beta"][t], S, x["A_log"], x["dt_bias"], gate_mode=w.gate_mode,
                           lower_bound=w.lower_bound, o=o)
    for i in range(warmup):
        step(i)
    # 512 MiB of state per step: far more than L2, no flush needed
    ms = _time_steps(lambda i: step(warmup + i), steps, torch.cuda.current_stream(dev), dev, None, ws, clk)
    value, ms_per_step = aggregate(w.B, steps, sum(ms), ws)
    roof = _roofline(decode_bytes(w), 0, (sum(ms) / steps) / 1e3, hbm_peak, peak_kind, DECODE_KERNEL_FILE, w.wid)
    return value, ms_per_step, roof


def measure_mla(dev, kda, hbm_peak, peak_kind, bf16_peak, steps=50, warmup=3):
    """The absorbed MLA decode step on its decode workload (B64 T4096 H96 d_q = d_v = 128 r = 512)."""
    cfg = MLA_DECODE
    x = {k: (v.to(dev) if v is not None else None) for k, v in make_mla_inputs(**cfg, device=str(dev)).items()}
    ws = torch.empty(kda.mla_decode_workspace_size(cfg["B"], cfg["T"], cfg["H"], cfg["d_q"], cfg["d_v"], cfg["r"]),
                     dtype=torch.uint8, device=dev)
    o = torch.empty(cfg["B"], cfg["H"], cfg["d_v"], dtype=torch.bfloat16, device=dev)

    def step(i):
        kda.mla_decode(x["q"], x["W_UK"], x["W_UV"], x["c"], x["lengths"], o=o, workspace=ws)
    for i in range(warmup):
        step(i)
    # the 268 MB latent cache is larger than L2: no flush needed
    ms = _time_steps(step, steps, torch.cuda.current_stream(dev), dev, None, 1)
    sec = (sum(ms) / steps) / 1e3
    nb, nf = mla_bytes(**cfg), mla_flops(**cfg)
    roof = _roofline(nb, nf, sec, hbm_peak, peak_kind, MLA_KERNEL_FILE, 6)
    roof["flop_bound_frac"] = round(nf / sec / 1e12 / bf16_peak, 4)
    return {"workload": "absorbed MLA decode B64 T4096 H96 d_q=d_v=128 r=512 (bf16)", "steps": steps,
            "us_per_step": round(sec * 1e6, 2), "tokens_per_s": round(cfg["B"] / sec, 1), "roofline": roof,
            "kernels_per_call": 3}


def backward_bytes(w) -> int:
    """Reverse mode: the forward inputs and dO read (dtype), S0 if any; dq, dk, dv, dg, dbeta, dS0 written (fp32)."""
    e = elt_bytes(w)
    B, T, H, HV, K, V = w.B, w.T, w.H, w.HV, w.K, w.V
    rd = 2 * B * T * H * K * e + 2 * B * T * HV * V * e + B * T * HV * K * e + B * T * HV * e + HV * 4 + HV * K * 4
    if w.S0_std is not None:
        rd += B * HV * K * V * 4
    wr = 4 * (2 * B * T * H * K + B * T * HV * V + B * T * HV * K + B * T * HV + B * HV * K * V + HV + HV * K)
    return rd + wr


def measure_backward(dev, kda, hbm_peak, peak_kind, wid=2, steps=10, warmup=3):
    """kda_backward on a prefill workload's shape (gradients of every input, gate included)."""
    w = WORKLOADS[wid]
    x = make_inputs(w, seed=rank_seed(w, 0), device=str(dev))
    gen = torch.Generator(device=str(dev)).manual_seed(5)
    dO = torch.randn(w.B, w.T, w.HV, w.V, generator=gen, device=dev).to(w.dtype)
    out = {}
    ws = torch.empty(kda.backward_workspace_size(w.B, w.T, w.H, w.HV, w.K, w.V), dtype=torch.uint8, device=dev)

    def step(i):
        kda.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], dO, x["A_log"], x["dt_bias"], x["S0"], None,
                     gate_mode=w.gate_mode, lower_bound=w.lower_bound, workspace=ws, out=out)
    step(0)  # fills `out`; later calls reuse its buffers
    for i in range(warmup):
        step(i)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ms = _time_steps(step, steps, torch.cuda.current_stream(dev), dev, flush, 1)
    sec = (sum(ms) / steps) / 1e3
    roof = _roofline(backward_bytes(w), 0, sec, hbm_peak, peak_kind, "kimi_delta_attention_33_b200/csrc/kda_backward.cu",
                     wid)
    return {"workload": f"reverse mode on workload {wid}: {w.name}", "steps": steps, "ms_per_step": round(sec * 1e3, 4),
            "tokens_per_s": round(w.B * w.T / sec, 1), "roofline": roof, "bound_note": "CUDA cores, latency of the "
            "per-token reductions; the HBM roofline is given for reference"}


EXTRA_STEPS = {1: 200, 2: 200, 3: 40, 4: 20}


def run_mla_only(args, ws, rank, local):
    """`--workload 6`: the absorbed MLA decode alone (profiler captures and quick looks; not the headline)."""
    from kimi_delta_attention_33_b200 import kda
    dev = torch.device("cuda", local)
    hbm_peak, bf16_peak, peak_kind = measured_peaks()
    r = measure_mla(dev, kda, hbm_peak, peak_kind, bf16_peak, steps=args.steps, warmup=args.warmup)
    if rank == 0:
        print(json.dumps({"metric": METRIC, "value": r["tokens_per_s"], "unit": "tokens/s", "n_gpus": ws,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["us_per_step"] / 1e3,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                          "data": "synthetic", "config": {"workload": r["workload"]}, "roofline": r["roofline"],
                          "gpu_launches": args.steps * 3}), flush=True)


def measure_fallbacks(dev, kda, hbm_peak, peak_kind, steps=20):
    """The paths outside the two tensor-core schedules, timed on workload 2's sizes: the CUDA-core kernel
    (value/key width 64, and chunk 16, both bf16) and the two-pass schedule with every chunk on the exact
    decay path (dt_bias far positive: every gate value near the lower bound, so the in-chunk decay span
    exceeds the factorised operands' limit)."""
    w2 = WORKLOADS[2]
    cases = {"cuda_core_K64_V64": w2.scaled(K=64, V=64), "cuda_core_chunk16": w2.scaled(chunk=16),
             "two_pass_exact_decay_path": w2.scaled(dt_bias_mean=6.0, dt_bias_std=0.0)}
    out = {}
    for name, w in cases.items():
        pf = Prefill(w, rank_seed(w, 0), dev, kda)
        v, mps, r = pf.measure(steps, 3, 1, None, hbm_peak, peak_kind)
        out[name] = {"sizes": f"B{w.B} T{w.T} H{w.H} HV{w.HV} K{w.K} V{w.V} C{w.chunk}", "schedule": r["schedule"],
                     "ms_per_step": round(mps, 5), "tokens_per_s": round(v, 1), "roofline_frac": r["frac"],
                     "kernel_file": r["kernel_file"]}
        del pf
        torch.cuda.empty_cache()
    return out


def run_ours(args, ws, rank, local):
    from kimi_delta_attention_33_b200 import kda
    if args.workload == 6:
        return run_mla_only(args, ws, rank, local)
    dev = torch.device("cuda", local)
    w = WORKLOADS[args.workload]
    if args.B is not None:
        w = w.scaled(B=args.B)
    if args.T is not None:
        w = w.scaled(T=args.T)
    torch.manual_seed(0)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    hbm_peak, _, peak_kind = measured_peaks()
    clk = ClockSampler(local, period_s=0.002)

    if w.is_decode:
        value, ms_per_step, roof = measure_decode(w, rank_seed(w, rank), dev, kda, hbm_peak, peak_kind, ws,
                                                  steps=args.steps, warmup=args.warmup, clk=clk)
        launches_per_step, x = 1, None
    else:
        pf = Prefill(w, rank_seed(w, rank), dev, kda)
        value, ms_per_step, roof = pf.measure(args.steps, args.warmup, ws, flush, hbm_peak, peak_kind, clk)
        launches_per_step, x = pf.launches, pf.x
        sched = pf.sched
        del pf

    line = None
    if rank == 0:
        e2e = None if args.no_e2e else run_e2e(args, w, x if x is not None else make_inputs(w, device=str(dev)),
                                               dev, kda)
        line = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None,
                "dtype": "f32" if w.is_decode or sched == kda.SCHEDULE_CUDA_CORE else "tf32",
                "data": "synthetic", "config": workload_config(w, ws), "roofline": roof, "e2e": e2e,
                "gpu_launches": args.steps * launches_per_step, "clocks": clk.summary()}
    x = None
    torch.cuda.empty_cache()

    # the other workloads, measured in the same run on rank 0 (extra keys, each with its roofline)
    if rank == 0 and not args.no_extras:
        extras = {}
        want = set(args.extras.split(",")) if args.extras else None

        def wanted(key):
            return want is None or key in want
        for wid in (2, 3, 4):
            if wid == w.wid or not wanted(f"workload{wid}"):
                continue
            pf = Prefill(WORKLOADS[wid], rank_seed(WORKLOADS[wid], 0), dev, kda)
            v, mps, r = pf.measure(EXTRA_STEPS[wid], 3, 1, flush, hbm_peak, peak_kind)
            extras[f"workload{wid}"] = {"workload": workload_config(WORKLOADS[wid], 1)["workload"],
                                        "steps": EXTRA_STEPS[wid], "ms_per_step": round(mps, 5),
                                        "tokens_per_s": round(v, 1), "roofline": r}
            del pf
            torch.cuda.empty_cache()
        if not w.is_decode and wanted("decode"):
            w5 = WORKLOADS[5]
            v, mps, r = measure_decode(w5, rank_seed(w5, 0), dev, kda, hbm_peak, peak_kind)
            extras["decode"] = {"workload": workload_config(w5, 1)["workload"], "steps": w5.decode_steps,
                                "us_per_step": round(mps * 1e3, 2), "tokens_per_s": round(v, 1),
                                "state_GBps": r["achieved"], "frac": r["frac"], "roofline": r}
        torch.cuda.empty_cache()
        if wanted("mla_decode"):
            extras["mla_decode"] = measure_mla(dev, kda, hbm_peak, peak_kind, measured_peaks()[1])
            torch.cuda.empty_cache()
        if wanted("backward"):
            extras["backward"] = measure_backward(dev, kda, hbm_peak, peak_kind)
            torch.cuda.empty_cache()
        if wanted("fallbacks"):
            extras["fallbacks"] = measure_fallbacks(dev, kda, hbm_peak, peak_kind)
        line.update(extras)
    if rank == 0:
        line["cpu_baseline"] = cpu_baseline(w) if (ws == 1 and not args.no_cpu_baseline) else None
        print(json.dumps(line), flush=True)


def run_e2e(args, w, x, dev, kda):
    """Same metric through the public API with host buffers: every step copies its inputs from pinned
    host memory to the device, makes the call, and copies its result back, all inside the timed
    region.  Two buffer sets and three streams overlap step i's call with step i+1's input copies and
    step i-1's result copies, as a serving loop would."""
    names = ("q", "k", "v", "g", "beta")
    h2d_s, comp_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    nbuf = 2
    if w.is_decode:
        inputs = names
        host = [{n: x[n][:, 0].contiguous().cpu().pin_memory() for n in inputs} for _ in range(nbuf)]
        S = x["S0"].clone()
        outs = [torch.empty(w.B, w.HV, w.V, dtype=w.dtype, device=dev) for _ in range(nbuf)]
        out_host = [torch.empty(w.B, w.HV, w.V, dtype=w.dtype).pin_memory() for _ in range(nbuf)]
        units = w.B

        def launch(devb, j):
            kda.recurrent_step(devb["q"], devb["k"], devb["v"], devb["g"], devb["beta"], S, x["A_log"], x["dt_bias"],
                               gate_mode=w.gate_mode, lower_bound=w.lower_bound, o=outs[j])
            return (outs[j],)
        results_host = [(out_host[j],) for j in range(nbuf)]
    else:
        inputs = names + (("S0",) if x["S0"] is not None else ())
        host = [{n: x[n].cpu().pin_memory() for n in inputs} for _ in range(nbuf)]
        ws_bytes = kda.workspace_size(w.B, w.T, w.H, w.HV, w.K, w.V, w.chunk)
        workspace = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)  # calls are ordered on comp_s
        o_dev = [torch.empty(w.B, w.T, w.HV, w.V, dtype=w.dtype, device=dev) for _ in range(nbuf)]
        S_dev = [torch.empty(w.B, w.HV, w.K, w.V, dtype=torch.float32, device=dev) for _ in range(nbuf)]
        results_host = [(torch.empty(o_dev[0].shape, dtype=w.dtype).pin_memory(),
                         torch.empty(S_dev[0].shape, dtype=torch.float32).pin_memory()) for _ in range(nbuf)]
        units = w.B * w.T

        def launch(devb, j):
            kda.chunk_fwd(devb["q"], devb["k"], devb["v"], devb["g"], devb["beta"], x["A_log"], x["dt_bias"],
                          devb.get("S0"), chunk=w.chunk, gate_mode=w.gate_mode, lower_bound=w.lower_bound, o=o_dev[j],
                          S_T=S_dev[j], workspace=workspace)
            return (o_dev[j], S_dev[j])
    devbufs = [{n: torch.empty_like(host[j][n], device=dev) for n in inputs} for j in range(nbuf)]
    ev_in = [torch.cuda.Event() for _ in range(nbuf)]
    ev_done = [torch.cuda.Event() for _ in range(nbuf)]
    ev_out = [torch.cuda.Event() for _ in range(nbuf)]

    def step(i):
        j = i % nbuf
        with torch.cuda.stream(h2d_s):  # inputs of step i, once step i - nbuf's call released the buffer
            if i >= nbuf:
                h2d_s.wait_event(ev_done[j])
            for n in inputs:
                devbufs[j][n].copy_(host[j][n], non_blocking=True)
            ev_in[j].record(h2d_s)
        with torch.cuda.stream(comp_s):  # the call, once its inputs landed and its outputs were read back
            comp_s.wait_event(ev_in[j])
            if i >= nbuf:
                comp_s.wait_event(ev_out[j])
            res = launch(devbufs[j], j)
            ev_done[j].record(comp_s)
        with torch.cuda.stream(d2h_s):  # the step's result back to the host
            d2h_s.wait_event(ev_done[j])
            for dst, src in zip(results_host[j], res):
                dst.copy_(src, non_blocking=True)
            ev_out[j].record(d2h_s)

    for i in range(max(args.warmup, 1)):
        step(i)
    torch.cuda.synchronize(dev)
    n = max(3, min(args.steps, 50))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(h2d_s)
    for i in range(n):
        step(i)
    d2h_s.wait_stream(h2d_s)
    d2h_s.wait_stream(comp_s)
    b.record(d2h_s)
    torch.cuda.synchronize(dev)
    sec = a.elapsed_time(b) / 1e3 / n
    h2d = sum(host[0][k].numel() * host[0][k].element_size() for k in inputs)
    d2h = sum(t.numel() * t.element_size() for t in results_host[0])
    return {"value": round(units / sec, 1), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": n, "overlap": "inputs of step i+1 and results of step i-1 "
            "copy while step i runs (two buffer sets, three streams)",
            # the host link's rates over the timed steps: at a PCIe link's rate the call is copy-bound
            "h2d_GBps": round(h2d / sec / 1e9, 1), "d2h_GBps": round(d2h / sec / 1e9, 1)}


# ------------------------------------------------------------------------ CPU oracle legs -----

def _oracle_sample(w, budget_s: float):
    """A bounded sample of the workload for the float64 oracle: a subset of (b, hv) pairs over a prefix
    of the tokens, sized to roughly `budget_s` seconds on this host.  Returns the callable and a
    description; the callable returns the number of workload tokens it stands for (token-heads / HV)."""
    import oracle
    threads = max(1, oracle.num_threads())
    per_token_head = 7.0 * w.K * w.V          # double flops of one recurrence step
    rate = 0.8e9 * threads                    # rough oracle speed, only used to size the sample
    T = w.T
    max_th = budget_s * rate / per_token_head
    pairs = max(1, min(w.pairs, int(max_th // T)))
    if pairs == 1 and T > max_th:
        T = max(16, int(max_th))
    pairs = min(pairs, w.pairs)
    sub = w.scaled(T=T)
    x = make_inputs(sub)
    G = w.HV // w.H
    sel = [(b, hv) for b in range(w.B) for hv in range(w.HV)][:pairs]

    def run():
        for b, hv in sel:
            h = hv // G
            s0 = None if x["S0"] is None else x["S0"][b:b + 1, hv:hv + 1]
            oracle.forward(x["q"][b:b + 1, :, h:h + 1], x["k"][b:b + 1, :, h:h + 1], x["v"][b:b + 1, :, hv:hv + 1],
                           x["g"][b:b + 1, :, hv:hv + 1], x["beta"][b:b + 1, :, hv:hv + 1], x["A_log"][hv:hv + 1],
                           x["dt_bias"][hv:hv + 1], s0, gate_mode=w.gate_mode, lower_bound=w.lower_bound)
        return pairs * T / w.HV

    desc = (f"{pairs} of {w.pairs} (b, hv) pairs x {T} of {w.T} tokens"
            f" ({pairs * T} token-heads = {pairs * T / w.HV:.1f} workload tokens), one pair per oracle call")
    return run, desc, threads


def cpu_baseline(w):
    run, desc, threads = _oracle_sample(w, budget_s=4.0)
    t0 = time.perf_counter()
    tokens, reps = 0.0, 0
    while True:
        tokens += run()
        reps += 1
        el = time.perf_counter() - t0
        if el >= 10.0 or reps >= 50:
            break
    return {"value": round(tokens / el, 2), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{desc}; repeated {reps}x in {el:.1f} s on {os.cpu_count()} host cores",
            "host_cpu_count": os.cpu_count()}


def run_reference(args):
    """The oracle as it stands, timed on the host cores, on this arm's workload, metric and unit."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if args.workload == 6:
        return run_reference_mla(args, ws)
    w = WORKLOADS[args.workload]
    run, desc, threads = _oracle_sample(w, budget_s=2.0)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    tokens = sum(run() for _ in range(args.steps))
    el = time.perf_counter() - t0
    v = round(tokens / el, 2)
    print(json.dumps({"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
                      "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
                      "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
                      "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                      "config": workload_config(w, ws),
                      "note": "the float64 oracle on the host cores; the config's L2 note describes the GPU arm",
                      "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                       "sample": desc + " per step"},
                      "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
          flush=True)


def run_reference_mla(args, ws):
    """The MLA decode oracle on the host, one sequence of the decode workload per step."""
    from oracle import mla
    x = make_mla_inputs(**MLA_DECODE)
    for _ in range(args.warmup):
        mla.absorbed(x["q"][:1], x["W_UK"], x["W_UV"], x["c"][:1])
    t0 = time.perf_counter()
    for i in range(args.steps):
        b = i % MLA_DECODE["B"]
        mla.absorbed(x["q"][b:b + 1], x["W_UK"], x["W_UV"], x["c"][b:b + 1])
    el = time.perf_counter() - t0
    v = round(args.steps / el, 2)
    print(json.dumps({"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": ws,
                      "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
                      "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                      "data": "synthetic",
                      "config": {"workload": "absorbed MLA decode B64 T4096 H96 d_q=d_v=128 r=512 (bf16)"},
                      "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
                                       "sample": "one sequence per step"},
                      "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
          flush=True)


def run_dry_plumbing(args):
    """The multi-rank plumbing alone, on CPU (gloo): set-up, barrier, MAX over ranks and the weak-
    scaling aggregate of a synthetic per-rank time, and rank 0's one line.  Touches no device; for
    testing ``--gpus N`` without GPUs."""
    ws, rank, local = dist_setup(backend="gloo")
    try:
        barrier(ws)
        value, ms_per_step = aggregate(1000, args.steps, 10.0 * (rank + 1) * args.steps, ws)
        if rank == 0:
            print(json.dumps({"dry_plumbing": True, "n_gpus": ws, "steps": args.steps, "value": value,
                              "ms_per_step": ms_per_step, "scaling": "weak"}), flush=True)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


def relaunch_under_torchrun(n: int) -> int:
    """Run this script again as n ranks under torch.distributed.run (rendezvous on 127.0.0.1), with
    the same arguments; returns the launcher's exit status."""
    import socket
    import subprocess
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.run(cmd).returncode


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=4, choices=[1, 2, 3, 4, 5, 6],
                    help="1-5: the KDA workloads (4, the largest single-GPU prefill, is the headline); "
                         "6: the absorbed MLA decode alone")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the other workloads' extra keys")
    ap.add_argument("--extras", default=None,
                    help="comma-separated subset of the extra keys to measure (workload2, workload3, workload4, "
                         "decode, mla_decode, backward, fallbacks); all by default")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--dry-plumbing", action="store_true",
                    help="multi-rank plumbing only, on CPU over gloo (no device is touched)")
    ap.add_argument("--B", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiler captures; not a bench line)")
    ap.add_argument("--T", type=int, default=None,
                    help="override the workload's length (smaller cases for profiler captures; not a bench line)")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch_under_torchrun(args.gpus))
    if args.steps is None:
        args.steps = {1: 200, 2: 200, 3: 40, 4: 20, 5: 128, 6: 50}[args.workload] if args.impl == "ours" else 10
    if args.dry_plumbing:
        run_dry_plumbing(args)
        return
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup
    if args.impl == "reference":
        run_reference(args)
        return
    ws, rank, local = dist_setup()
    try:
        run_ours(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
