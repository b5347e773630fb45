#!/usr/bin/env python
"""Throughput of exact tiled attention (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one pass of the whole hot path over one batch of the workload:
the fused forward (O and LSE), then the backward's three stages (D / LSE
preprocess, the dK/dV/dQ kernel, the dQ conversion). The default workload is
the Llama-7B-shaped causal case (B=4, H=32, N=4096, d=128, bf16), the one the
forward >= 60% / backward >= 45% of dense-BF16 peak targets are stated on.
Inputs are seeded synthetic N(0,1) values rounded to bf16; each of Q, K, V, dO
(134 MB) is larger than the 126 MB L2, so no flush is needed between steps.

Prints one JSON line (rank 0). Under torchrun every rank runs its own copy of
the workload (independent batches, no collective on the data path: weak
scaling); the timed region is bracketed by a barrier and a device
synchronisation on both sides and its duration is the maximum over ranks.

``--impl reference`` times the fp64 CPU oracle instead (the only other
implementation of this computation here), on the same workload, metric and
unit, one bounded sample (one batch-head, forward + backward) per step.

``--workload fp32_n512_d32`` (one head, N = 512, d = 32, fp32, the lesson's
NumPy example shape) has no backward: a step is one fp32 forward on the CUDA
cores, L2 is flushed before each timed launch and only the launches are timed.
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
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_io_aware_45_b200 import inputs  # noqa: E402

METRIC = "attention fwd+bwd TFLOPS at 1 B200 and % of dense-BF16 tensor peak"
UNIT = "TFLOP/s"
FALLBACK_PEAK_TFLOPS = 1590.0
REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama7b_causal",
                    choices=list(inputs.WORKLOADS) + [VARLEN_NAME])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--window", type=int, default=-1,
                    help="sliding window: each query sees at most this many earlier keys "
                         "(fa_fwd_window / fa_bwd_window with left = W, on the causal workload)")
    ap.add_argument("--deterministic", action="store_true",
                    help="backward through fa_bwd_deterministic (run-to-run identical dQ)")
    return ap.parse_args()


def workload_config(w: inputs.Workload, world: int, deterministic: bool = False,
                    window: int = -1) -> dict:
    return {"workload": f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.N} d={w.d} "
                        f"{'causal' if w.causal else 'non-causal'}"
                        f"{' block-sparse' if w.sparse else ''} bf16 fwd+bwd",
            "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "causal": w.causal,
            "block_sparse": w.sparse, "grad_dtype": "f32", "deterministic_dq": deterministic,
            "window_left": window,
            "parallelism": f"dp{world}: rank r owns global batch rows [rB, rB+B), all KV heads",
            "l2": "no flush: each of Q, K, V, dO is larger than L2 (126 MB)"
                  if w.B * w.Hq * w.N * w.d * 2 > 126e6 else "working set may fit L2"}


def forward_only_config(w: inputs.Workload, world: int) -> dict:
    return {"workload": f"{w.name}: B={w.B} H={w.Hq} N={w.N} d={w.d} "
                        f"{'causal' if w.causal else 'non-causal'} {w.dtype} forward",
            "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "causal": w.causal,
            "block_sparse": w.sparse, "parallelism": f"dp{world}: rank r owns global batch rows [rB, rB+B), all KV heads",
            "l2": "flushed before every timed launch (a 256 MB write; inputs are 64 KB each)"}


def step_flops(w: inputs.Workload, mask) -> tuple[float, float]:
    fwd = inputs.flops(w, mask=mask, backward=False)
    bwd = inputs.flops(w, mask=mask, backward=True)
    return fwd, bwd


# ---------------------------------------------------------------- CPU oracle timing

def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(w: inputs.Workload, x: dict, b: int, h: int):
    """Runs the oracle forward + backward (forward only for a workload
    without a backward) of one (batch, query head) and returns (seconds,
    algorithmic FLOPs of that sample)."""
    from oracle import attention as orc
    hk = h // w.group
    q = x["q"][b:b + 1, h:h + 1]
    k = x["k"][b:b + 1, hk:hk + 1]
    v = x["v"][b:b + 1, hk:hk + 1]
    t0 = time.perf_counter()
    O, _ = orc.forward(q, k, v, w.scale, w.causal, x["mask"])
    if w.backward:
        do = x["do"][b:b + 1, h:h + 1]
        orc.backward(q, k, v, do, w.scale, w.causal, x["mask"], O=O)
    dt = time.perf_counter() - t0
    per = (14.0 if w.backward else 4.0) * w.d * inputs.allowed_count(w.N, w.causal, x["mask"])
    return dt, per


def cpu_baseline(w, x, budget_s=20.0) -> dict:
    secs, fl, n = 0.0, 0.0, 0
    # at least one unit; several while they are short (a forward-only unit of
    # the fp32 workload takes milliseconds, so it is repeated)
    cap = 4 if w.backward else 1000
    while n == 0 or (secs < budget_s * 0.5 and n < cap):
        dt, f = oracle_sample(w, x, n % w.B, (n * 7) % w.Hq)
        secs += dt
        fl += f
        n += 1
    what = "forward+backward" if w.backward else "forward"
    return {"value": fl / secs / 1e12, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{n} (batch, head) units of {w.B * w.Hq}, {what} in fp64 "
                      f"NumPy ({secs:.1f} s)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = inputs.WORKLOADS[args.workload]
    x = inputs.make_inputs(w)
    world = int(os.environ.get("WORLD_SIZE", args.gpus))
    times, fl = [], 0.0
    for i in range(args.warmup + args.steps):
        dt, f = oracle_sample(w, x, i % w.B, (i * 7) % w.Hq)
        if i >= args.warmup:
            times.append(dt)
            fl += f
    total = sum(times)
    val = fl / total / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, world) if w.backward else forward_only_config(w, world),
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": oracle_threads(),
                             "kind": "oracle",
                             "sample": "one (batch, head) unit per step, "
                                       f"{'forward+backward' if w.backward else 'forward'} "
                                       "in fp64 NumPy"},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        sm, smax, reasons = [], [], set()
        for line in open(self.path):
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                mask = int(f[4], 16)
            except ValueError:
                continue
            for bit, name in REASON_BITS.items():
                if mask & bit and name != "gpu_idle":
                    reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- multi-rank helpers

def max_over_ranks(ms: float, device=None) -> float:
    """The slowest rank's time (the whole job ends when it ends); ms itself
    when not running under an initialised process group of more than one."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_units(world: int, rank: int, B: int, Hkv: int) -> list:
    """The (global batch row, KV head) units rank ``rank`` owns. The units of
    attention are independent (no exchange step on the pages' path), so the
    job is partitioned, not replicated: the global problem holds ``world``
    times the per-rank batch, and rank r owns batch rows r*B .. r*B + B - 1
    with every KV head (each unit brings its group of query heads). Per-GPU
    work stays fixed as ranks are added (weak scaling) and no collective
    touches the data; rank r's rows are drawn with seed r."""
    if not (0 <= rank < world):
        raise ValueError("rank outside the job")
    return [(rank * B + b, hk) for b in range(B) for hk in range(Hkv)]


def job_tflops(flops_per_rank_step: float, steps: int, world: int, ms: float) -> float:
    """Whole-job throughput under weak scaling: every rank runs the same
    per-rank workload (its own seeded batch), so the job does world times
    the per-rank work in the slowest rank's time."""
    return flops_per_rank_step * steps * world / (ms / 1e3) / 1e12


# ---------------------------------------------------------------- our arm

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            return json.load(open(p)), "measured"
        except Exception:
            pass
    return None, "fallback"


# A timed region at least this long runs under the 1 kW power cap on B200:
# the kernels' cycle counts stay the same while the SM clock falls (measured:
# 2-20 steps of the llama7b-shaped step at 1,965 MHz, 200 steps at ~1,770 MHz
# with sw_power_cap active; per-kernel times x clock agree within 1 %).
LONG_REGION_MS = 250.0


def select_bf16_peak(peaks, kind: str, timed_ms: float, clocks: dict):
    """The dense bf16 peak a kernel's time is compared with: the measured
    sustained figure (a seconds-long GEMM loop under the power cap) when the
    timed region ran long enough to reach the cap, or its clock record shows
    the cap holding the SM clock below its maximum; else the burst figure.
    Returns (peak, peak_kind, burst, sustained)."""
    burst = (peaks or {}).get("bf16_tflops", FALLBACK_PEAK_TFLOPS)
    sustained = (peaks or {}).get("bf16_tflops_sustained")
    sm, smax = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    capped = ("sw_power_cap" in (clocks.get("reasons") or []) and sm is not None
              and smax is not None and sm < 0.98 * smax)
    if sustained and (capped or timed_ms >= LONG_REGION_MS):
        why = f"timed region {timed_ms:.0f} ms" + (", SM clock held below max by the power cap"
                                                    if capped else "")
        return sustained, f"{kind} sustained bf16 ({why})", burst, sustained
    return burst, f"{kind} burst bf16 (timed region {timed_ms:.0f} ms)", burst, sustained


def tensor_roofline(kernel: str, ach: float, peak_sel, traffic):
    peak, kind, burst, sustained = peak_sel
    return {"bound": "tensor", "kernel": kernel, "achieved": ach, "peak": peak,
            "unit": "TFLOP/s", "frac": ach / peak, "peak_kind": kind,
            "frac_of_burst": ach / burst,
            "frac_of_sustained": (ach / sustained) if sustained else None, "traffic": traffic}


def traffic_record(kernel_file: str, workload: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, or None if the kernel's source changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    src = os.path.join(ROOT, "exact_io_aware_45_b200", "csrc", kernel_file)
    if not (os.path.exists(p) and os.path.exists(src)):
        return None
    try:
        recs = json.load(open(p))
    except Exception:
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    for r in recs:
        if r.get("kernel_file") == kernel_file and r.get("source_sha256") == sha and \
                r.get("workload") == workload:
            return r.get("dram_bytes_per_launch")
    return None


def run_e2e(args, fa, w, dev, stream, bufs, mask, step_flops, world, barrier, wfa=None,
            wba=None):
    """The same step end to end through the public C ABI (fa_fwd / fa_bwd, or
    the window entry points): every step copies Q, K, V, dO in from pinned
    host memory and O, LSE, dQ, dK, dV out to it. The batch is cut into
    one-sequence chunks whose copy-in, compute and copy-out run on three
    streams, so chunk c's compute overlaps chunk c+1's copy-in and chunk
    c-1's copy-out (one cudaMemcpyAsync per tensor and chunk)."""
    import torch
    q, k, v, do, o, lse, dq, dk, dv = bufs
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    hin = [t.cpu().pin_memory() for t in (q, k, v, do)]
    hout = [torch.empty_like(t, device="cpu").pin_memory() for t in (o, lse, dq, dk, dv)]
    h2d = sum(t.numel() * t.element_size() for t in hin)
    d2h = sum(t.numel() * t.element_size() for t in hout)
    dins, douts = (q, k, v, do), (o, lse, dq, dk, dv)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    s_cmp = stream
    wsb = fa.fa_bwd_workspace_size(1, Hq, N, d)
    ws = fa.new_workspace(wsb, dev)
    P = lambda t: 0 if t is None else t.data_ptr()  # noqa: E731
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done = [ev() for _ in range(B)]
    cmp_done = [ev() for _ in range(B)]
    out_done = [None] * B   # chunk c's previous outputs have left the device

    def chunk_compute(c):
        qc, kc, vc, doc_, oc, lc, dqc, dkc, dvc = (t[c] for t in (q, k, v, do, o, lse, dq, dk, dv))
        if wfa is not None:
            fargs = (P(qc), P(kc), P(vc), P(oc), P(lc), 1, Hq, Hkv, N, d) + wfa[10:16] + \
                (P(ws), s_cmp.cuda_stream)
            st = fa.fa_fwd_window(*fargs)
        else:
            st = fa.fa_fwd(P(qc), P(kc), P(vc), P(oc), P(lc), 1, Hq, Hkv, N, d, float(w.scale),
                           int(w.causal), P(mask), fa.FA_BF16, P(ws), s_cmp.cuda_stream)
        if st != fa.FA_OK:
            raise RuntimeError(fa.status_string(st))
        if wba is not None:
            bargs = (P(qc), P(kc), P(vc), P(oc), P(doc_), P(lc), P(dqc), P(dkc), P(dvc), 1, Hq,
                     Hkv, N, d) + wba[14:21] + (P(ws), wsb, s_cmp.cuda_stream)
            st = fa.fa_bwd_window(*bargs)
        else:
            bargs = (P(qc), P(kc), P(vc), P(oc), P(doc_), P(lc), P(dqc), P(dkc), P(dvc), 1, Hq,
                     Hkv, N, d, float(w.scale), int(w.causal), P(mask), fa.FA_BF16, fa.FA_F32,
                     P(ws), wsb, s_cmp.cuda_stream)
            st = fa.fa_bwd_deterministic(*bargs, fa.PATH_AUTO) if args.deterministic \
                else fa.fa_bwd(*bargs)
        if st != fa.FA_OK:
            raise RuntimeError(fa.status_string(st))

    def e2e_step():
        for c in range(B):
            with torch.cuda.stream(s_in):
                # chunk c's inputs may be overwritten once its last compute is done
                s_in.wait_event(cmp_done[c])
                for dst, src in zip(dins, hin):
                    dst[c].copy_(src[c], non_blocking=True)
                in_done[c].record(s_in)
            s_cmp.wait_event(in_done[c])
            if out_done[c] is not None:
                s_cmp.wait_event(out_done[c])   # its outputs of the last step are out
            chunk_compute(c)
            cmp_done[c].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(cmp_done[c])
                for dst, src in zip(hout, douts):
                    dst[c].copy_(src[c], non_blocking=True)
                out_done[c] = ev()
                out_done[c].record(s_out)

    for c in range(B):
        cmp_done[c].record(s_cmp)
    e2e_step()
    torch.cuda.synchronize()
    barrier()
    a = torch.cuda.Event(enable_timing=True)
    b_ = torch.cuda.Event(enable_timing=True)
    a.record(s_cmp)
    s_in.wait_stream(s_cmp)
    s_out.wait_stream(s_cmp)
    for _ in range(args.e2e_steps):
        e2e_step()
    s_cmp.wait_stream(s_in)
    s_cmp.wait_stream(s_out)
    b_.record(s_cmp)
    torch.cuda.synchronize()
    barrier()
    ems = max_over_ranks(a.elapsed_time(b_), dev)
    if fa.device_error(ws) != fa.FA_OK:
        raise RuntimeError("device error word set during the end-to-end run")
    return {"value": job_tflops(step_flops, args.e2e_steps, world, ems), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
            "ms_per_step": ems / args.e2e_steps,
            "pipeline": f"{B} one-sequence chunks; copy-in, compute and copy-out on three streams"}


def run_ours(args):
    import torch
    import torch.distributed as dist
    from exact_io_aware_45_b200 import fa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    fa.lib()

    w = inputs.WORKLOADS[args.workload]
    x = inputs.make_inputs(w, seed=rank)
    bf = torch.bfloat16
    q, k, v, do = (torch.from_numpy(x[n]).to(dev, bf).contiguous() for n in ("q", "k", "v", "do"))
    mask = None if x["mask"] is None else torch.from_numpy(x["mask"]).to(dev)
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
    dk = torch.empty(k.shape, dtype=torch.float32, device=dev)
    dv = torch.empty(v.shape, dtype=torch.float32, device=dev)
    wsb = fa.fa_bwd_workspace_size(B, Hq, N, d)
    ws = fa.new_workspace(wsb, dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    P = lambda t: 0 if t is None else t.data_ptr()  # noqa: E731
    fwd_args = (P(q), P(k), P(v), P(o), P(lse), B, Hq, Hkv, N, d, float(w.scale), int(w.causal),
                P(mask), fa.FA_BF16, P(ws), sp, fa.PATH_AUTO)
    bwd_args = (P(q), P(k), P(v), P(o), P(do), P(lse), P(dq), P(dk), P(dv), B, Hq, Hkv, N, d,
                float(w.scale), int(w.causal), P(mask), fa.FA_BF16, fa.FA_F32, P(ws), wsb, sp,
                fa.PATH_AUTO)
    stages = [("fwd", lambda: fa.fa_fwd_ex(*fwd_args)),
              ("bwd_preprocess", lambda: fa.fa_bwd_preprocess(*bwd_args)),
              ("bwd_main", lambda: fa.fa_bwd_main(*bwd_args)),
              ("bwd_finalize", lambda: fa.fa_bwd_finalize(*bwd_args))]
    if args.window >= 0:
        # one stage each: fa_fwd_window, fa_bwd_window (preprocess, main, finalize)
        noop = lambda: fa.fa_exp2_fma(0, 0, 0, 0)  # noqa: E731
        wfa = (P(q), P(k), P(v), P(o), P(lse), B, Hq, Hkv, N, d, float(w.scale), int(w.causal),
               args.window, -1, P(mask), fa.FA_BF16, P(ws), sp)
        wba = (P(q), P(k), P(v), P(o), P(do), P(lse), P(dq), P(dk), P(dv), B, Hq, Hkv, N, d,
               float(w.scale), int(w.causal), args.window, -1, P(mask), fa.FA_BF16, fa.FA_F32,
               P(ws), wsb, sp)
        stages = [("fwd", lambda: fa.fa_fwd_window(*wfa)),
                  ("bwd_preprocess", noop),
                  ("bwd_main", lambda: fa.fa_bwd_window(*wba)),
                  ("bwd_finalize", noop)]
    if args.deterministic:
        # one stage: preprocess, main kernel without dQ, per-query-tile dQ kernel
        # (the empty stages make an ABI call that launches nothing, so the
        # launch count stays exact)
        noop = lambda: fa.fa_exp2_fma(0, 0, 0, 0)  # noqa: E731
        stages = [("fwd", lambda: fa.fa_fwd_ex(*fwd_args)),
                  ("bwd_preprocess", noop),
                  ("bwd_main", lambda: fa.fa_bwd_deterministic(*bwd_args)),
                  ("bwd_finalize", noop)]
    n_stage_ev = len(stages) + 1

    def step(evs=None):
        launches = 0
        if evs is not None:
            evs[0].record(stream)
        for i, (name, fn) in enumerate(stages):
            s = fn()
            if s != fa.FA_OK:
                raise RuntimeError(f"{name}: {fa.status_string(s)}")
            launches += fa.fa_last_launch_count()
            if evs is not None:
                evs[i + 1].record(stream)
        return launches

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    # clocks are sampled from before the warm-up to the end of the
    # end-to-end region, so the record covers every timed launch
    sampler = ClockSampler(local)
    sampler.start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fa.device_error(ws) != fa.FA_OK:
        raise RuntimeError("device error word set during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_stage_ev)]
           for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    launches = 0
    t_start.record(stream)
    for i in range(args.steps):
        launches += step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(t_start.elapsed_time(t_end), dev)
    err = fa.device_error(ws)
    if err != fa.FA_OK:
        raise RuntimeError(f"device error word set during timing: {fa.status_string(err)}")

    per_stage = {name: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1])
                                       for i in range(args.steps))
                 for j, (name, _) in enumerate(stages)}
    fwd_fl, bwd_fl = step_flops(w, x["mask"])
    if args.window >= 0:
        allowed = inputs.window_allowed_count(N, w.causal, args.window, -1) * B * Hq
        fwd_fl, bwd_fl = 4.0 * d * allowed, 10.0 * d * allowed
    value = job_tflops(fwd_fl + bwd_fl, args.steps, world, ms)

    # end to end through the C ABI with pinned host buffers
    e2e = None
    if args.e2e_steps > 0:
        e2e = run_e2e(args, fa, w, dev, stream, (q, k, v, do, o, lse, dq, dk, dv), mask,
                      fwd_fl + bwd_fl, world, barrier, wfa if args.window >= 0 else None,
                      wba if args.window >= 0 else None)
    clocks = sampler.stop()

    # dominant kernel: the stage with the longest mean duration
    dom = max(per_stage, key=per_stage.get)
    dom_fl = {"fwd": fwd_fl, "bwd_main": bwd_fl}.get(dom)
    peaks, kind = measured_peaks()
    peak_sel = select_bf16_peak(peaks, kind, ms, clocks)
    if dom_fl is not None:
        ach = dom_fl / (per_stage[dom] / 1e3) / 1e12
        kfile = "sm100_fwd.cu" if dom == "fwd" else "sm100_bwd.cu"
        roof = tensor_roofline(dom, ach, peak_sel, traffic_record(kfile, w.name))
    else:
        bytes_ = 4.0 * B * Hq * N * d * 2 + 8.0 * B * Hq * N
        peak = (peaks or {}).get("hbm_gbs", 6650.0)
        ach = bytes_ / (per_stage[dom] / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": dom, "achieved": ach, "peak": peak, "unit": "GB/s",
                "frac": ach / peak, "peak_kind": kind, "traffic": None}
    stage_frac = {}
    pk, _, pk_burst, _ = peak_sel
    stage_frac["fwd_tflops"] = fwd_fl / (per_stage["fwd"] / 1e3) / 1e12
    bwd_ms = per_stage["bwd_preprocess"] + per_stage["bwd_main"] + per_stage["bwd_finalize"]
    stage_frac["bwd_tflops"] = bwd_fl / (bwd_ms / 1e3) / 1e12
    stage_frac["fwd_frac_of_peak"] = stage_frac["fwd_tflops"] / pk
    stage_frac["bwd_frac_of_peak"] = stage_frac["bwd_tflops"] / pk
    stage_frac["fwd_frac_of_burst"] = stage_frac["fwd_tflops"] / pk_burst
    stage_frac["bwd_frac_of_burst"] = stage_frac["bwd_tflops"] / pk_burst

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, x)

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) rounded to bf16)",
            "config": workload_config(w, world, args.deterministic, args.window),
            "stages_ms": per_stage, "per_direction": stage_frac, "roofline": roof,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------- fp32 forward-only workload

# fp32 FMA throughput: 148 SMs x 128 fp32 lanes x 2 FLOP per FMA at the 1,965 MHz maximum SM clock
FP32_FMA_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def run_forward_only(args):
    """One step = one fp32 forward (fa_fwd, CUDA-core kernel) of a workload
    without a backward pass. Its inputs are far smaller than L2, so a 256 MB
    buffer is written before every timed launch and only the launches are
    timed (CUDA events around each); the step time is their sum."""
    import torch
    import torch.distributed as dist
    from exact_io_aware_45_b200 import fa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    fa.lib()

    w = inputs.WORKLOADS[args.workload]
    x = inputs.make_inputs(w, seed=rank)
    q, k, v = (torch.from_numpy(x[n]).to(dev).contiguous() for n in ("q", "k", "v"))
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    ws = fa.new_workspace(fa.fa_fwd_workspace_size(), dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    P = lambda t: t.data_ptr()  # noqa: E731
    fargs = (P(q), P(k), P(v), P(o), P(lse), B, Hq, Hkv, N, d, float(w.scale), int(w.causal), 0,
             fa.FA_F32, P(ws), sp)

    def fwd():
        s = fa.fa_fwd(*fargs)
        if s != fa.FA_OK:
            raise RuntimeError(f"fa_fwd: {fa.status_string(s)}")
        return fa.fa_last_launch_count()

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    sampler = ClockSampler(local)
    sampler.start()
    for _ in range(args.warmup):
        fwd()
    torch.cuda.synchronize()
    if fa.device_error(ws) != fa.FA_OK:
        raise RuntimeError("device error word set during warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    launches = 0
    for i in range(args.steps):
        flush.fill_(i & 255)
        ev[i][0].record(stream)
        launches += fwd()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), dev)
    if fa.device_error(ws) != fa.FA_OK:
        raise RuntimeError("device error word set during timing")
    fl = inputs.flops(w, mask=None, backward=False)
    value = job_tflops(fl, args.steps, world, ms)
    ach = fl / (ms / args.steps / 1e3) / 1e12
    roof = {"bound": "alu", "kernel": "fwd (fp32 CUDA cores)", "achieved": ach,
            "peak": FP32_FMA_PEAK_TFLOPS, "unit": "TFLOP/s", "frac": ach / FP32_FMA_PEAK_TFLOPS,
            "peak_kind": "derived: 148 SMs x 128 fp32 lanes x 2 FLOP x 1,965 MHz",
            "traffic": None}

    e2e = None
    if args.e2e_steps > 0:
        hq_, hk_, hv_ = (torch.from_numpy(x[n]).pin_memory() for n in ("q", "k", "v"))
        ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hq_, hk_, hv_))
        d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()

        def e2e_step():
            for dst, src in ((q, hq_), (k, hk_), (v, hv_)):
                dst.copy_(src, non_blocking=True)
            fwd()
            for dst, src in ((ho, o), (hl, lse)):
                dst.copy_(src, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        b_.record(stream)
        torch.cuda.synchronize()
        barrier()
        ems = max_over_ranks(a.elapsed_time(b_), dev)
        e2e = {"value": job_tflops(fl, args.e2e_steps, world, ems), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps}
    clocks = sampler.stop()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, x, budget_s=20.0)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (the lesson's NumPy draw: default_rng(0) normals, fp32)",
            "config": forward_only_config(w, world), "roofline": roof, "cpu_baseline": cpu,
            "e2e": e2e, "gpu_launches": launches, "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------- variable-length batch

VARLEN_NAME = "varlen_mix"
VARLEN = dict(total=32768, lo=256, hi=4096, Hq=32, Hkv=32, d=128, causal=True)


def run_varlen(args):
    """One step = fa_fwd_varlen + fa_bwd_varlen on a packed batch of seeded
    lengths (uniform in [256, 4096], 32768 tokens, 32 heads, d = 128, causal):
    a padding-free training batch. Not the headline workload; its own line."""
    import torch
    from exact_io_aware_45_b200 import fa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    fa.lib()
    c = VARLEN
    lengths = inputs.varlen_lengths(c["total"], c["lo"], c["hi"], seed=0)
    x = inputs.varlen_case(lengths, c["Hq"], c["Hkv"], c["d"], seed=rank)
    bf = torch.bfloat16
    q, k, v, do = (torch.from_numpy(x[n]).to(dev, bf).contiguous() for n in ("q", "k", "v", "do"))
    cu = torch.from_numpy(x["cu"]).to(dev)
    total, Hq, Hkv, d, B = c["total"], c["Hq"], c["Hkv"], c["d"], len(lengths)
    maxlen = x["max_seqlen"]
    scale = 1.0 / math.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty((Hq, total), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty(t.shape, dtype=torch.float32, device=dev) for t in (q, k, v))
    wsb = fa.fa_bwd_varlen_workspace_size(B, Hq, maxlen, total, d)
    ws = fa.new_workspace(wsb, dev)
    sp = torch.cuda.current_stream(dev).cuda_stream
    P = lambda t: t.data_ptr()  # noqa: E731
    fargs = (P(q), P(k), P(v), P(o), P(lse), P(cu), B, maxlen, total, Hq, Hkv, d, scale,
             int(c["causal"]), fa.FA_BF16, P(ws), sp)
    bargs = (P(q), P(k), P(v), P(o), P(do), P(lse), P(dq), P(dk), P(dv), P(cu), B, maxlen, total,
             Hq, Hkv, d, scale, int(c["causal"]), fa.FA_BF16, fa.FA_F32, P(ws), wsb, sp)
    stages = [("fwd", lambda: fa.fa_fwd_varlen(*fargs)), ("bwd", lambda: fa.fa_bwd_varlen(*bargs))]
    allowed = inputs.varlen_allowed_count(lengths, c["causal"]) * Hq
    fl = {"fwd": 4.0 * d * allowed, "bwd": 10.0 * d * allowed}
    launches = 0

    def step(evs=None):
        n = 0
        if evs is not None:
            evs[0].record()
        for i, (name, fn) in enumerate(stages):
            st = fn()
            if st != fa.FA_OK:
                raise RuntimeError(f"{name}: {fa.status_string(st)}")
            n += fa.fa_last_launch_count()
            if evs is not None:
                evs[i + 1].record()
        return n

    sampler = ClockSampler(local)
    sampler.start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(args.steps):
        launches += step(evs[i])
    t1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if fa.device_error(ws) != fa.FA_OK:
        raise RuntimeError("device error word set")
    ms = t0.elapsed_time(t1)
    per = {name: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs)
           for j, (name, _) in enumerate(stages)}
    value = (fl["fwd"] + fl["bwd"]) * args.steps * world / (ms / 1e3) / 1e12
    peaks, kind = measured_peaks()
    peak_sel = select_bf16_peak(peaks, kind, ms, clocks)
    dom = max(per, key=per.get)
    ach = fl[dom] / (per[dom] / 1e3) / 1e12
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) rounded to bf16; seeded lengths)",
            "config": {"workload": f"{VARLEN_NAME}: {B} sequences, lengths uniform in "
                                   f"[{c['lo']}, {c['hi']}], {total} tokens, Hq={Hq} Hkv={Hkv} "
                                   f"d={d} causal bf16 fwd+bwd (padding-free)",
                       "B": B, "total": total, "max_seqlen": maxlen, "Hq": Hq, "Hkv": Hkv,
                       "d": d, "causal": c["causal"], "grad_dtype": "f32",
                       "parallelism": f"replicas x{world} (independent batches)"},
            "stages_ms": per,
            "per_direction": {"fwd_tflops": fl["fwd"] / (per["fwd"] / 1e3) / 1e12,
                              "bwd_tflops": fl["bwd"] / (per["bwd"] / 1e3) / 1e12},
            "roofline": tensor_roofline(dom, ach, peak_sel, None),
            "cpu_baseline": None, "e2e": None, "gpu_launches": launches, "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        if args.workload == VARLEN_NAME:
            print(json.dumps({"impl": "reference", "unavailable": "the reference arm times the "
                              "oracle on the headline workloads only"}))
            return 0
        return run_reference(args)
    if args.workload == VARLEN_NAME:
        return run_varlen(args)
    if not inputs.WORKLOADS[args.workload].backward:
        return run_forward_only(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
