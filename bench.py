#!/usr/bin/env python
"""Benchmark of the SLA2 attention forward (router + linear totals + sparse
attention) on synthetic Wan2.1-shaped inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload wan13]
                    [--fp8] [--keep-ratio R] [--impl reference]

One process per GPU.  Under torchrun each process is one rank; `--gpus N`
with N > 1 outside a launcher starts N ranks of itself under torchrun.  Each
rank runs the whole hot path on its own batch (weak scaling; the heads of
different ranks never interact, so there is no collective on the data path),
the job's time is the maximum over ranks, and rank 0 prints one JSON line.

A step = sla_prepare + sla_route(SLA_ROUTE_KBAR_FROM_WS) + sla2_attn_fwd(
SLA_FLAG_PREPARED) on one batch already resident in HBM (bf16, d = 128: the
router takes the key-block means the prepass wrote; other inputs route
first).  Inputs (Q, K, V: 302 MB at the 1.3B shape) exceed the 126 MB L2, so
the timed loop does not flush L2 between steps.  `--fp8` (or an fp8_*
workload) runs the e4m3 sparse branch and reports its roofline against an
e4m3 tensor peak measured in the same run.  The e2e figure times
sla2_forward_host: pinned host inputs in, the output back to the host, one
C-ABI call per step.  `--impl reference` times the CPU oracle (the only
reference that exists) on a bounded sample of the same workload on rank 0,
without loading the library.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_linear_attention_b200 import dist_timing, inputs  # noqa: E402

# the library's binding, loaded only by the legs that run the GPU path (the
# reference arm times the CPU oracle alone and never maps libsla.so)
sla = None


def _load_binding():
    global sla
    if sla is None:
        from sparse_linear_attention_b200 import sla as binding
        sla = binding
    return sla

METRIC = "SLA2 attn fwd ms & effective TOPS @Wan-1.3B shape, 97% sparse; % tensor peak"
UNIT = "effective TOPS (4*N^2*d*H*B per forward / time)"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained"), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, 1400.0, "fallback"


def keep_of(w, count=None):
    """Kept blocks per query block: the workload's count, else its ratio through
    `count` (the library's sla_keep_count on the GPU legs, the oracle's
    keep_count on the CPU legs)."""
    if w.keep_count is not None:
        return w.keep_count
    return (count or sla.sla_keep_count)(w.keep_ratio, w.n_kv)


def oracle_keep_of(w):
    from oracle import sla_oracle as orc
    return keep_of(w, orc.keep_count)


def work_counts(w, kept_cpu):
    """Algorithmic work of one forward.

    full_ops   : 4*N^2*d per (b,h)  -- the dense attention the effective TOPS refers to
    sparse_flop: 4*d per (query row, kept valid key) -- QK^T and PV on kept tiles
    """
    N, d, bq, bkv = w.N, w.d, w.bq, w.bkv
    full = 4.0 * N * N * d * w.H * w.B
    # valid keys of each key block
    kv_valid = torch.clamp(N - torch.arange(w.n_kv) * bkv, max=bkv).to(torch.float64)
    q_rows = torch.clamp(N - torch.arange(w.n_q) * bq, max=bq).to(torch.float64)
    keys = kv_valid[kept_cpu.long()].sum(-1)  # [B,H,nq]
    pairs = float((keys * q_rows).sum())
    return full, 4.0 * d * pairs


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sms, mx, reasons = [], None, set()
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sms.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                 f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["no samples"]}
        loaded = [s for s in sms if mx is None or s > 0.3 * mx] or sms
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sms)}


def profile_traffic(kernel_src):
    """DRAM traffic per launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "sparse_fwd_kernel_wan13.md")
    try:
        txt = open(path).read()
    except OSError:
        return None
    m = re.search(r"source_sha256:\s*([0-9a-f]{64})", txt)
    t = re.search(r"traffic_bytes_per_launch:\s*([0-9.e+]+)", txt)
    if not m or not t:
        return None
    cur = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()
    return float(t.group(1)) if m.group(1) == cur else None


class OracleTimer:
    """The CPU oracle timed on a bounded sample of the workload: the whole
    router once, then single query blocks (random heads and positions), each
    extrapolated to the full forward."""

    def __init__(self, w, x):
        from oracle import sla_oracle as orc
        self.orc, self.w, self.x = orc, w, x
        q32, k32 = x["q"].to(torch.float32).numpy(), x["k"].to(torch.float32).numpy()
        t0 = time.perf_counter()
        self.kept, _, _ = orc.route(q32, k32, x["wq"].numpy(), x["wk"].numpy(), w.bq, w.bkv, "sla2", oracle_keep_of(w))
        self.t_route = time.perf_counter() - t0
        self.heads = {}
        self.blocks = 0
        self.t_att = 0.0
        import numpy as np
        self.rng = np.random.default_rng(0)

    def one_block(self):
        w, x = self.w, self.x
        h, i = int(self.rng.integers(0, w.H)), int(self.rng.integers(0, w.n_q))
        if h not in self.heads:
            self.heads[h] = tuple(x[n][:, h:h + 1].to(torch.float64).numpy() for n in ("q", "k", "v"))
        q64, k64, v64 = self.heads[h]
        t1 = time.perf_counter()
        self.orc.sla2_forward(q64, k64, v64, self.kept[:, h:h + 1], x["alpha"][:, h:h + 1].numpy(), w.bq, w.bkv,
                              blocks=[(0, 0, i)])
        t = time.perf_counter() - t1
        self.t_att += t
        self.blocks += 1
        return self.t_route + t * (w.B * w.H * w.n_q)

    def per_forward(self):
        w = self.w
        return self.t_route + self.t_att / max(self.blocks, 1) * (w.B * w.H * w.n_q)

    def describe(self):
        w = self.w
        return (f"CPU oracle (numpy fp64): router on the whole workload ({self.t_route:.2f} s) + attention "
                f"for {self.blocks} sampled query blocks of {w.B * w.H * w.n_q} ({self.t_att:.2f} s), "
                f"extrapolated per block")

    @staticmethod
    def threads():
        from threadpoolctl import threadpool_info
        return max([p.get("num_threads", 1) for p in threadpool_info()] or [1])


def soft_topk_leg(args, w, dev, stream):
    """SoftTop-k router forward [SLA2-deep §06] through sla_route_soft at the
    same workload: ms per call with Q, K resident, and its roofline.  The
    sigmoids run on the special-function unit (an exponential and a
    reciprocal each), so the bound is that unit: 16 operations per SM per clock
    = 8 sigmoids, times 148 SMs and the sampled SM clock.  Work per row =
    (bisection iterations + 1) x n_kv sigmoids; the fp32 bisection halves the
    bracket [-max(s/tau) - 40, -min(s/tau) + 40] until its midpoint stops
    moving, i.e. about log2(bracket / ulp(lambda)) times, counted from the
    scores and lambda the library returns."""
    import numpy as np
    x = inputs.make_inputs(w)
    q, kk = x["q"].to(dev), x["k"].to(dev)
    wq, wk = x["wq"].to(dev), x["wk"].to(dev)
    k, tau = keep_of(w), 0.1
    shape = sla.make_shape(q, w.bq, w.bkv)
    ws = torch.zeros(sla.sla_workspace_size(shape, sla.SLA_MODE_SLA2_TOPK), dtype=torch.uint8, device=dev)
    mask = torch.empty(w.B, w.H, w.n_q, w.n_kv, dtype=torch.float32, device=dev)
    lam = torch.empty(w.B, w.H, w.n_q, dtype=torch.float32, device=dev)
    kept = torch.empty(w.B, w.H, w.n_q, k, dtype=torch.int32, device=dev)
    scores = torch.empty(w.B, w.H, w.n_q, w.n_kv, dtype=torch.float32, device=dev)
    sla.sla_route(shape, q, kk, wq, wk, sla.SLA_MODE_SLA2_TOPK, k, 0, kept, None, scores, ws, stream)
    for _ in range(args.warmup):
        sla.sla_route_soft(shape, q, kk, wq, wk, k, tau, mask, lam, ws, stream)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(args.steps):
        sla.sla_route_soft(shape, q, kk, wq, wk, k, tau, mask, lam, ws, stream)
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if sla.sla_read_device_status(ws, stream) != 0:
        raise SystemExit("device-side error during the timed calls")
    ms = t0.elapsed_time(t1) / args.steps
    xs = (scores.cpu().numpy() / np.float32(tau)).astype(np.float32)
    width = (-xs.min(-1) + 40.0) - (-xs.max(-1) - 40.0)
    ulp = np.spacing(np.abs(lam.cpu().numpy()).astype(np.float32)).astype(np.float64)
    iters = np.ceil(np.log2(width / ulp))
    sig = float(((iters + 1.0) * w.n_kv).sum())
    mhz = clk.get("sm_mhz") or 1965.0
    peak = 148 * 8 * mhz * 1e6
    achieved = sig / (ms * 1e-3)
    print(json.dumps({
        "metric": "SoftTop-k router forward ms @Wan-1.3B shape (sla_route_soft, tau = 0.1)", "value": ms,
        "unit": "ms per call", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": False, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.d} bq={w.bq} bkv={w.bkv} "
                               f"budget={k}/{w.n_kv} key blocks"},
        "roofline": {"bound": "alu", "achieved": achieved / 1e9, "peak": peak / 1e9, "unit": "G sigmoid/s",
                     "frac": achieved / peak, "traffic": None,
                     "peak_source": "special-function unit: 16 ops per SM per clock, 2 per sigmoid, 148 SMs",
                     "algorithmic": "n_kv sigmoids per bisection probe and per row; mean probes per row "
                                    f"{float(iters.mean()):.1f}"},
        "gpu_launches": 2 * args.steps, "clocks": clk,
    }), flush=True)


def backward_oracle_ms(w, x, kept, do_cpu, budget_s, labels=None):
    """The oracle's backward (sla2_backward, or sla_backward when SLA labels
    are given) timed on sampled query blocks (random heads and positions, at
    least three, until budget_s seconds are spent), each block's time
    extrapolated to every block of the workload.  Returns (ms per backward,
    blocks timed, seconds spent)."""
    import numpy as np

    from oracle import sla_oracle as orc
    rng = np.random.default_rng(1)
    heads = {}
    spent, n = 0.0, 0
    while n < 3 or spent < budget_s:
        h, i = int(rng.integers(0, w.H)), int(rng.integers(0, w.n_q))
        if h not in heads:
            heads[h] = tuple(t[:, h:h + 1].to(torch.float64).numpy() for t in (x["q"], x["k"], x["v"], do_cpu))
        q64, k64, v64, do64 = heads[h]
        t1 = time.perf_counter()
        if labels is not None:
            orc.sla_backward(q64, k64, v64, labels[:, h:h + 1], x["wproj"].to(torch.float64).numpy(), do64, w.bq,
                             w.bkv, blocks=[(0, 0, i)])
        else:
            orc.sla2_backward(q64, k64, v64, kept[:, h:h + 1], x["alpha"][:, h:h + 1].to(torch.float64).numpy(),
                              do64, w.bq, w.bkv, blocks=[(0, 0, i)])
        spent += time.perf_counter() - t1
        n += 1
    return spent / n * (w.B * w.H * w.n_q) * 1e3, n, spent


def backward_leg(args, w, dev, stream):
    """SLA2 backward (sla2_attn_bwd), or for an SLA workload sla_attn_bwd, at
    the same workload: ms per call with every input resident, the kept
    (critical) blocks from the router, a seeded dO.  The work is dense
    contractions, so the roofline is the measured bf16 tensor peak; the
    algorithmic work is the FlashAttention-style backward of the sparse
    branch, 10 d FLOP per (query row, kept valid key): S recomputed,
    dP = dO V^T, dQ, dK and dV (the linear branch is not counted)."""
    x = inputs.make_inputs(w)
    sla_mode = w.mode == "sla"
    q, kk, v = x["q"].to(dev), x["k"].to(dev), x["v"].to(dev)
    wq, wk, alpha = x["wq"].to(dev), x["wk"].to(dev), x["alpha"].to(dev)
    k = sla.sla_keep_count(w.crit_ratio, w.n_kv) if sla_mode else keep_of(w)
    k_neg = sla.sla_keep_count(w.negl_ratio, w.n_kv) if sla_mode else 0
    mode = sla.SLA_MODE_SLA_3WAY if sla_mode else sla.SLA_MODE_SLA2_TOPK
    shape = sla.make_shape(q, w.bq, w.bkv)
    ws = torch.zeros(sla.sla_workspace_size(shape, mode), dtype=torch.uint8, device=dev)
    kept = torch.empty(w.B, w.H, w.n_q, k, dtype=torch.int32, device=dev)
    labels = torch.empty(w.B, w.H, w.n_q, w.n_kv, dtype=torch.int8, device=dev) if sla_mode else None
    sla.sla_route(shape, q, kk, wq, wk, mode, k, k_neg, kept, labels, None, ws, stream)
    g = torch.Generator().manual_seed(w.seed + 1000)
    do = torch.randn(q.shape, generator=g).to(q.dtype).to(dev)
    wsize = sla.sla_attn_bwd_workspace_size(shape) if sla_mode else sla.sla2_attn_bwd_workspace_size(shape)
    wsb = torch.zeros(wsize, dtype=torch.uint8, device=dev)
    dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
    dk, dv = torch.empty_like(dq), torch.empty_like(dq)
    dal = torch.empty(w.B, w.H, w.n_q, dtype=torch.float32, device=dev)
    phi = sla.SLA_PHI_ELU1 if args.phi == "elu1" else sla.SLA_PHI_SOFTMAX
    if sla_mode:
        wproj = x["wproj"].to(dev)
        dwp = torch.empty(w.d, w.d, dtype=torch.float32, device=dev)
        call = lambda: sla.sla_attn_bwd(shape, q, kk, v, labels, wproj, phi, do, dq, dk, dv, dwp, wsb, stream)
    else:
        call = lambda: sla.sla2_attn_bwd(shape, q, kk, v, kept, k, alpha, phi, do, dq, dk, dv, dal, wsb, stream)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(args.steps):
        call()
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if sla.sla_read_device_status(wsb, stream) != 0:
        raise SystemExit("device-side error during the timed calls")
    ms = t0.elapsed_time(t1) / args.steps
    kept_cpu = kept.cpu()
    _, executed = work_counts(w, kept_cpu)
    flops = executed / 4.0 * 10.0  # work_counts' executed count is 4 d per (row, kept valid key)
    cpu = None
    if not args.no_cpu_baseline:
        lab_cpu = labels.cpu().numpy() if sla_mode else None
        cpu_ms, nblk, t_cpu = backward_oracle_ms(w, x, kept_cpu.numpy(), do.cpu(), args.cpu_budget, lab_cpu)
        fn = "sla_backward" if sla_mode else "sla2_backward"
        cpu = {"value": cpu_ms, "unit": "ms per call", "cores": OracleTimer.threads(), "kind": "oracle",
               "sample": f"CPU oracle (numpy fp64) {fn} on {nblk} sampled query blocks of "
                         f"{w.B * w.H * w.n_q} ({t_cpu:.2f} s), extrapolated per block"}
    _, peak, _, src = peaks()
    achieved = flops / (ms * 1e-3) / 1e12
    # the SLA2 backward of bf16 inputs at d = 128, b_q = 128 runs on the tensor cores:
    # prepare (3), the attention kernel with its statistics epilogue, phi(Q), the
    # inverse lists, dQ, the dH reduction, the dH packing, dalpha, dK/dV
    tc_path = (not sla_mode) and w.dtype == "bf16" and w.d == 128 and w.bq == 128
    launches = 6 if sla_mode else (11 if tc_path else 3)
    metric = ("SLA backward ms @Wan-1.3B shape (sla_attn_bwd: dQ, dK, dV, dW_proj)" if sla_mode else
              "SLA2 backward ms @Wan-1.3B shape (sla2_attn_bwd: dQ, dK, dV, dalpha)")
    keep_txt = f"critical={k} negligible={k_neg}/{w.n_kv}" if sla_mode else f"keep={k}/{w.n_kv}"
    print(json.dumps({
        "metric": metric, "value": ms,
        "unit": "ms per call", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": False, "dtype": "bf16" if tc_path else "f32", "data": "synthetic",
        "config": {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.d} bq={w.bq} bkv={w.bkv} "
                               f"{keep_txt} key blocks, phi={args.phi}"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None, "peak_source": f"{src} bf16 dense (burst)",
                     "algorithmic": "10*d FLOP per (query row, kept valid key): the sparse branch's "
                                    "FlashAttention-style backward",
                     "path": "tensor cores (tcgen05)" if tc_path else "fp32 CUDA cores"},
        "gpu_launches": launches * args.steps, "clocks": clk, "cpu_baseline": cpu,
    }), flush=True)


def fp8_peak_tflops(dev, reps=10):
    """Dense e4m3 tensor-core throughput measured here, the way the bf16 peak
    is: torch._scaled_mm (cuBLASLt) on 8192^3 e4m3 operands with fp32 scales,
    2*N^3 FLOP, best of `reps` CUDA-event timings after warm-up."""
    n = 8192
    g = torch.Generator(device=dev).manual_seed(0)
    a = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
    one = torch.ones((), device=dev)
    mm = lambda: torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)  # noqa: E731
    for _ in range(3):
        mm()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mm()
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    del a, b
    return 2.0 * n ** 3 / (best * 1e-3) / 1e12


def hbm_roofline(name, bytes_, ms, hbm, src, what):
    achieved = bytes_ / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": name, "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "peak_source": f"{src} HBM copy", "algorithmic": what}


def reference_arm(args, w):
    """The CPU oracle (the only reference that exists) on a bounded sample of
    the workload, rank 0 only; the library is never loaded here."""
    rank, _, _ = dist_timing.world_info()
    if rank != 0:
        return
    x = inputs.make_inputs(w)
    ot = OracleTimer(w, x)
    for _ in range(args.warmup):
        ot.one_block()
    ot.t_att, ot.blocks = 0.0, 0
    vals = [ot.one_block() for _ in range(args.steps)]
    full = 4.0 * w.N * w.N * w.d * w.H * w.B
    t = statistics.median(vals)
    val = full / t / 1e12
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.d} bq={w.bq} bkv={w.bkv} "
                               f"keep={oracle_keep_of(w)}/{w.n_kv} key blocks"},
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": OracleTimer.threads(), "kind": "oracle",
                         "sample": ot.describe() + "; each step = one sampled query block"},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="wan13", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--phi", default="elu1", choices=["elu1", "softmax"],
                    help="linear-branch feature map (the pages' default for SLA2 is ELU+1)")
    ap.add_argument("--fp8", action="store_true",
                    help="the e4m3 (low-bit) sparse branch; implied by the fp8_* workloads")
    ap.add_argument("--int8", action="store_true",
                    help="the INT8 variant of the low-bit sparse branch (INT8 Q, K'; e4m3 P, V)")
    ap.add_argument("--keep-ratio", type=float, default=None,
                    help="SLA2 keep fraction instead of the workload's (the e4m3 sweep: 0.03, 0.05, 0.10)")
    ap.add_argument("--soft-topk", action="store_true",
                    help="time the SoftTop-k router (sla_route_soft) instead of the forward step")
    ap.add_argument("--backward", action="store_true",
                    help="time the SLA2 backward (sla2_attn_bwd) instead of the forward step")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")

    # --gpus N outside a launcher: start N ranks of this script under torchrun
    if args.gpus > 1 and not dist_timing.launched():
        raise SystemExit(dist_timing.run_ranks(os.path.abspath(__file__), sys.argv[1:], args.gpus))
    rank, world, local = dist_timing.world_info()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but the launcher started {world} ranks")

    w = inputs.WORKLOADS[args.workload]
    if args.keep_ratio is not None:
        w = dataclasses.replace(w, keep_ratio=args.keep_ratio, keep_count=None)
    int8 = args.int8
    fp8 = (args.fp8 or w.fp8) and not int8
    low = fp8 or int8
    if w.mode != "sla2" and (args.impl == "reference" or args.soft_topk or low):
        raise SystemExit("the reference arm, --fp8, --int8 and --soft-topk are SLA2 legs")
    if args.impl == "reference":
        reference_arm(args, w)
        return

    _load_binding()
    phi = sla.SLA_PHI_ELU1 if args.phi == "elu1" else sla.SLA_PHI_SOFTMAX
    sla_mode = w.mode == "sla"

    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    if args.soft_topk:
        if world == 1:
            soft_topk_leg(args, w, dev, stream)
        return
    if args.backward:
        if world == 1:
            backward_leg(args, w, dev, stream)
        return

    x = inputs.make_inputs(w)
    # SLA: k = critical blocks (+1), k_neg negligible (-1) [SLA 关键设计 2]; SLA2: k kept blocks
    k = sla.sla_keep_count(w.crit_ratio, w.n_kv) if sla_mode else keep_of(w)
    k_neg = sla.sla_keep_count(w.negl_ratio, w.n_kv) if sla_mode else 0
    mode = sla.SLA_MODE_SLA_3WAY if sla_mode else sla.SLA_MODE_SLA2_TOPK
    q, kk, v = x["q"].to(dev), x["k"].to(dev), x["v"].to(dev)
    wq, wk, alpha = x["wq"].to(dev), x["wk"].to(dev), x["alpha"].to(dev)
    wproj = x["wproj"].to(dev)
    shape = sla.make_shape(q, w.bq, w.bkv)
    ws = torch.zeros(sla.sla_workspace_size(shape, mode | (sla.SLA_WS_FP8 if low else 0)), dtype=torch.uint8,
                     device=dev)
    kept = torch.empty(w.B, w.H, w.n_q, k, dtype=torch.int32, device=dev)
    labels = torch.empty(w.B, w.H, w.n_q, w.n_kv, dtype=torch.int8, device=dev) if sla_mode else None
    out = torch.empty(w.B, w.H, w.N, w.d, dtype=torch.bfloat16, device=dev)
    low_flag = sla.SLA_FLAG_INT8 if int8 else (sla.SLA_FLAG_FP8 if fp8 else 0)
    attn_flags = sla.SLA_FLAG_PREPARED | low_flag
    # route 2, prepare 3 (+ Q conversion off the d = 128 bf16 grid), attention 1 (+ SLA label lists 1,
    # + e4m3 statistics and quantisation 2)
    launches_per_step = (2 + 3 + 1 + (1 if (w.d != 128 or w.dtype == "f32") else 0) + (1 if sla_mode else 0)
                         + (2 if low else 0))

    # bf16, d = 128: the prepass also writes the key-block means, so the router
    # runs after it and reads K only through the prepass (SLA_ROUTE_KBAR_FROM_WS)
    kbar_first = w.dtype == "bf16" and w.d == 128

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        if kbar_first:
            sla.sla_prepare(shape, kk, v, phi, ws, stream)
            if ev is not None:
                ev[1].record(stream)
            sla.sla_route(shape, q, kk, wq, wk, mode | sla.SLA_ROUTE_KBAR_FROM_WS, k, k_neg, kept, labels, None,
                          ws, stream)
        else:
            sla.sla_route(shape, q, kk, wq, wk, mode, k, k_neg, kept, labels, None, ws, stream)
            if ev is not None:
                ev[1].record(stream)
            sla.sla_prepare(shape, kk, v, phi, ws, stream)
        if ev is not None:
            ev[2].record(stream)
        if sla_mode:
            sla.sla_attn_fwd(shape, q, kk, v, labels, wproj, phi, sla.SLA_FLAG_PREPARED, out, ws, stream)
        else:
            sla.sla2_attn_fwd(shape, q, kk, v, kept, k, alpha, phi, attn_flags, out, ws, stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if sla.sla_read_device_status(ws, stream) != 0:
        raise SystemExit("device-side error during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index if world == 1 else local)
    clocks.start()
    time.sleep(0.3)
    dist_timing.barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    dist_timing.barrier()
    clk = clocks.stop()
    elapsed_ms = dist_timing.max_over_ranks(t_start.elapsed_time(t_end), dev)
    if sla.sla_read_device_status(ws, stream) != 0:
        raise SystemExit("device-side error during the timed steps")
    first_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    second_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    prep_ms, route_ms = (first_ms, second_ms) if kbar_first else (second_ms, first_ms)
    sparse_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)

    full_ops, sparse_flop = work_counts(w, kept.cpu())
    ms_step = elapsed_ms / args.steps
    value = dist_timing.job_throughput(full_ops, ms_step, world) / 1e12

    hbm, bf16_burst, bf16_sus, peak_src = peaks()
    achieved = sparse_flop / (sparse_ms * 1e-3) / 1e12
    if low:
        tc_peak, tc_src = fp8_peak_tflops(dev), "measured here: torch._scaled_mm e4m3 8192^3, best of 10 (burst)"
        if int8:
            tc_src += "; the INT8 variant's S runs kind::i8, whose nominal dense rate equals e4m3's"
    else:
        tc_peak, tc_src = bf16_burst, f"{peak_src} bf16 dense (burst)"
    traffic = None if low else profile_traffic(os.path.join(ROOT, "sparse_linear_attention_b200", "csrc",
                                                            "sparse_fwd.cu"))
    # HBM-bound stages by their algorithmic bytes: the prepass reads K and V, the
    # router reads Q (and K too unless the prepass handed it the key-block means)
    elt = 2 if w.dtype == "bf16" else 4
    tensor_bytes = w.B * w.H * w.N * w.d * elt
    hbm_lines = {
        "prepare": hbm_roofline("lin_prepass_tma_kernel + zsum/hsum", 2 * tensor_bytes, prep_ms, hbm, peak_src,
                                "read K, V once (2*B*H*N*d*elt bytes)"),
        "route": hbm_roofline("pool_project_kernel + score_select_kernel",
                              tensor_bytes * (1 if kbar_first else 2), route_ms, hbm, peak_src,
                              "read Q" + ("" if kbar_first else " and K") + " once"),
    }

    # end to end through the public API: pinned host buffers in, the output back
    # out, inside one C-ABI call per step (sla2_forward_host); SLA copies with torch
    hq, hk, hv = (t.pin_memory() for t in (x["q"], x["k"], x["v"]))
    hwq, hwk, hal, hwp = (t.pin_memory() for t in (x["wq"], x["wk"], x["alpha"], x["wproj"]))
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hwq, hwk, hwp if sla_mode else hal))
    d2h = hout.numel() * hout.element_size()
    if sla_mode:
        e2e_api = "torch copies around sla_route + sla_prepare + sla_attn_fwd"

        def e2e_step():
            for dst, src in ((q, hq), (kk, hk), (v, hv), (wq, hwq), (wk, hwk), (wproj, hwp)):
                dst.copy_(src, non_blocking=True)
            step()
            hout.copy_(out, non_blocking=True)
    else:
        e2e_api = "sla2_forward_host (host buffers in and out, one C-ABI call per step)"
        hflags = low_flag
        dbuf = torch.zeros(sla.sla2_forward_host_device_bytes(shape, k, sla.SLA_BF16, hflags), dtype=torch.uint8,
                           device=dev)
        del ws  # the host call carries its own workspace inside dbuf

        def e2e_step():
            sla.sla2_forward_host(shape, hq, hk, hv, hwq, hwk, hal, k, phi, hflags, hout, None, dbuf, stream)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    dist_timing.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    if not sla_mode and sla.sla_read_device_status(dbuf, stream) != 0:
        raise SystemExit("device-side error during the end-to-end steps")
    e2e_ms = dist_timing.max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, dev)
    e2e_val = dist_timing.job_throughput(full_ops, e2e_ms, world) / 1e12

    cpu = None
    if (rank == 0 and world == 1 and not args.no_cpu_baseline and not sla_mode and not low
            and phi == sla.SLA_PHI_ELU1):
        ot = OracleTimer(w, x)
        while ot.t_att < args.cpu_budget or ot.blocks < 4:
            ot.one_block()
        t_cpu = ot.per_forward()
        cpu = {"value": full_ops / t_cpu / 1e12, "unit": UNIT, "cores": OracleTimer.threads(), "kind": "oracle",
               "sample": ot.describe(), "ms_per_forward": t_cpu * 1e3}

    if world > 1:
        dist.destroy_process_group()
    if not dist_timing.reports(rank):
        return
    shape_names = {"wan13": "Wan2.1-1.3B-480P latent shape", "wan14": "Wan2.1-14B-720P latent shape",
                   "fp8_13": "Wan2.1-1.3B-480P latent shape, e4m3 sparse branch",
                   "fp8_14": "Wan2.1-14B-720P latent shape, e4m3 sparse branch"}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8+e4m3" if int8 else ("e4m3" if fp8 else "bf16"), "data": "synthetic",
        "config": {"workload": f"{w.name}: {shape_names[w.name]}" if w.name in shape_names else w.name,
                   "B": w.B, "H": w.H, "N": w.N, "d": w.d, "bq": w.bq, "bkv": w.bkv,
                   "kept_blocks": f"{k}/{w.n_kv} per query block ({100.0 * (1 - k / w.n_kv):.2f}% sparse)",
                   "phi": "elu+1" if phi == sla.SLA_PHI_ELU1 else "softmax over channels",
                   "method": "SLA (critical / marginal / negligible, O_s + Proj(O_l))" if sla_mode
                   else "SLA2 (top-k, alpha mix)" + (", e4m3 sparse branch" if fp8 else "")
                   + (", INT8 Q/K' with e4m3 P/V sparse branch" if int8 else ""),
                   "global_batch": w.B * world,
                   "l2": "no flush: Q,K,V = %.0f MB per rank > 126 MB L2" % (3 * q.numel() * 2 / 1e6)},
        "breakdown_ms": {"route": route_ms, "prepare": prep_ms, "sparse_attention": sparse_ms},
        "sparse_tflops_executed": achieved,
        "roofline": {"bound": "tensor", "kernel": "sparse_fwd_kernel", "achieved": achieved,
                     "peak": tc_peak, "unit": "TFLOP/s", "frac": achieved / tc_peak,
                     "peak_source": tc_src, "traffic": traffic,
                     "algorithmic": "4*d FLOP per (query row, kept valid key): QK^T + PV on kept tiles"
                                    + ("; the attention call includes the 8-bit quantisation" if low else "")},
        "hbm_rooflines": hbm_lines,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_val, "unit": UNIT, "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "api": e2e_api},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
