#!/usr/bin/env python
"""Benchmark of the frozen-NF4 QLoRA linear layer on B200.

Headline workload: the 65B-scale MLP pair, the up projection W 22016 x 8192
and the down projection W 8192 x 22016, each ~N(0, 0.015), M = 2048 tokens
(4 x 512), LoRA r = 64, alpha = 16, synthetic seeded inputs. One step is one
pass of the whole hot path over one batch, on inputs already resident in HBM,
for each of the two linears:
    quantize W (fp32 -> NF4 + double quant)
    -> forward (Y, sT; the weight dequantised inside the matmul)
    -> backward (dX through deq(W), dA, dB)
No bf16 copy of either weight is written (weight bytes 4-bit only); the
standalone dequantiser is timed as its own row. Two input sets alternate
between steps (about 3.4 GB, far more than the 126 MB L2).

Metric value: fwd+bwd algorithmic TFLOP/s = sum over the two linears of
(4MNK + 6Mr(N+K)) / step time, whole job (all ranks). Under torchrun every
rank runs an independent replica (weak scaling, no collective on the data
path); timing is the max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --case step|fwd:<workload>|bwd:<workload>|quantize:<workload>|
                           dequantize:<workload>|merge:<workload> [--reps R]
        (one call repeated, for profiler captures; prints nothing else)
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
sys.path.insert(0, ROOT)

_CORES = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
for _v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
    os.environ.setdefault(_v, str(_CORES))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "QLoRA linear fwd+bwd TFLOP/s and tokens/s; NF4 dequant GB/s (% of roofline)"
HEADLINE = synth.L65B[1:]  # MLP up 22016 x 8192, down 8192 x 22016; M 2048, r 64
WORKLOAD = "65b_mlp_up22016x8192_down8192x22016_m2048_r64"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_BF16_TFLOPS = 2250.0  # dense bf16, spec sheet (context only)


def peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


def fwd_bwd_flops(M, N, K, r):
    return 4 * M * N * K + 6 * M * r * (N + K)


def step_flops(cfgs):
    return sum(fwd_bwd_flops(c.M, c.N, c.K, c.r) for c in cfgs)


def workload_config():
    """The workload named identically by both arms."""
    return {"workload": WORKLOAD,
            "linears": [{"name": c.name, "N": c.N, "K": c.K} for c in HEADLINE],
            "M": HEADLINE[0].M, "r": HEADLINE[0].r, "alpha": HEADLINE[0].alpha, "w_std": HEADLINE[0].w_std,
            "step": "per linear: quantize(W fp32 -> NF4 + double quant) + forward + backward "
                    "(no bf16 weight written)",
            "l2": "inputs larger than L2: two alternating input sets, ~3.4 GB"}


# ------------------------------------------------------------- clocks ------

class ClockSampler:
    """nvidia-smi sampled every 100 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        target = str(device)
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            if uuid:
                target = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:  # noqa: BLE001 - fall back to the ordinal
            pass
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", target], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError, TypeError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "power_w_max": max(power) if power else None, "samples": len(sm)}


# ------------------------------------------------------- CPU oracle leg ----

class OracleSample:
    """The CPU oracle on a proportional slice of the workload: for each
    linear, m_s tokens forward+backward in fp64 against the oracle's
    dequantised W, plus the quantisation of m_s rows of W (the share of the
    once-per-step weight work that m_s of the M tokens carry)."""

    def __init__(self, cfgs):
        import oracle
        self.o = oracle
        self.cfgs = cfgs
        self.layers = []
        for cfg in cfgs:
            W = synth.weight(cfg).numpy()
            z = oracle.quantize_nf4(W)
            What = oracle.bf16_bits_to_f64(
                oracle.dequant_bf16_bits(z["codes"], z["qabsmax"], z["s2"], z["mean"], cfg.N, cfg.K))
            f64 = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
            self.layers.append(dict(cfg=cfg, W=W, What=What, X=f64(synth.activations(cfg)),
                                    dY=f64(synth.grad_output(cfg)), A=f64(synth.lora_a(cfg)), B=f64(synth.lora_b(cfg))))
        self.threads = oracle.num_threads()

    def step(self, m_s: int, offset: int = 0):
        for L in self.layers:
            c = L["cfg"]
            lo = offset % (c.M - m_s + 1)
            rows = slice(lo, lo + m_s)
            w0 = lo % (c.N - m_s + 1) if m_s <= c.N else 0
            self.o.quantize_nf4(L["W"][w0:w0 + min(m_s, c.N)])
            X, dY = L["X"][rows], L["dY"][rows]
            self.o.forward(X, L["What"], L["A"], L["B"], c.alpha, c.r)
            self.o.backward(dY, X, L["What"], L["A"], L["B"], c.alpha, c.r)

    def flops(self, m_s):
        return sum(fwd_bwd_flops(m_s, c.N, c.K, c.r) for c in self.cfgs)

    def calibrate(self, target_s: float) -> int:
        t0 = time.perf_counter()
        self.step(16)
        dt = max(time.perf_counter() - t0, 1e-4)
        m = int(16 * target_s / dt)
        m_s = 1
        while m_s * 2 <= max(m, 1) and m_s * 2 <= min(c.M for c in self.cfgs):
            m_s *= 2
        return m_s

    def describe(self, m_s):
        return (f"{m_s} tokens of fwd+bwd per linear (fp64 numpy) + quantisation of {m_s} rows of each W "
                f"(C oracle), on {self.threads} host threads")

    def sample_line(self, seconds: float = 10.0):
        m_s = self.calibrate(1.0)
        n = 0
        t0 = time.perf_counter()
        while True:
            self.step(m_s, offset=n * m_s)
            n += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                break
        value = self.flops(m_s) * n / el / 1e12
        return {"value": value, "unit": "TFLOP/s", "cores": self.threads, "kind": "oracle",
                "sample": f"{n} slices of {self.describe(m_s)}, {el:.1f} s"}


# ---------------------------------------------------------------- ranks ----

def max_over_ranks(x: float, pg, dev) -> float:
    """The largest of every rank's x (a time): the job takes as long as its
    slowest replica. pg is torch.distributed (any backend) or None."""
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_step_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job rate: every replica does the same step (weak scaling), so
    the job does world steps' work per (max over ranks) step time."""
    return flops_per_step_per_rank * world / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------ reference ----

def run_reference(args, rank, world):
    if rank != 0:
        return
    s = OracleSample(HEADLINE)
    budget = 150.0 / max(args.steps + args.warmup, 1)  # whole run within ~2.5 minutes
    m_s = s.calibrate(budget)
    for i in range(args.warmup):
        s.step(m_s, offset=i * m_s)
    t0 = time.perf_counter()
    for i in range(args.steps):
        s.step(m_s, offset=(args.warmup + i) * m_s)
    el = time.perf_counter() - t0
    value = s.flops(m_s) * args.steps / el / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": s.threads, "kind": "oracle",
                             "sample": "per step: " + s.describe(m_s)},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ ours ---

# DRAM bytes (read + write) of one launch of the dominant kernel, from one ncu
# capture of its current build on this workload (per kernel key). A kernel
# without a capture of its current version reports null.
NCU_TRAFFIC: dict = {
    # one step's four launches of fused_nf4_gemm_pair (up forward, up dX, down
    # forward, down dX): dram read + write 258.1, 307.4, 305.6, 257.6 MB
    "fused_nf4_gemm": 282.2e6,
}


def timed(fn, n=20):
    """Mean ms per call of fn(i), i = 0..n-1, replayed from one CUDA graph."""
    fn(0)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / n


def assert_device_ok(q, workspaces, where):
    """Every bounded wait of the pipelined kernels ended in time: a wait that
    ran out leaves its tile unwritten and sets the workspace status word."""
    for ws in workspaces:
        st = q.device_status(ws)
        if st != 0:
            raise RuntimeError(f"{where}: device status {q.STATUS.get(st, st)}")


class Linear:
    """Device buffers of one linear of the workload: two input sets (W fp32,
    X, A, B, dY), the packed weight, outputs and workspaces."""

    def __init__(self, q, cfg, dev, sets=2, w_fp32=True):
        self.q, self.cfg = q, cfg
        c = cfg
        host = []
        for s in range(sets):
            cs = c if s == 0 else synth.custom(N=c.N, K=c.K, M=c.M, r=c.r, alpha=c.alpha,
                                               seed_base=77 + 10 * c.layer_id + s, w_std=c.w_std,
                                               outliers=c.outliers)
            h = dict(X=synth.activations(cs), A=synth.lora_a(cs), B=synth.lora_b(cs), dY=synth.grad_output(cs))
            if w_fp32:
                h["W"] = synth.weight(cs)
            host.append(h)
        self.host = host
        self.sets = [{k: v.to(dev) for k, v in h.items()} for h in host]
        M, N, K, r = c.M, c.N, c.K, c.r
        self.w = q.NF4Weight.empty(N, K, dev)
        if not w_fp32:
            q.quantize_nf4(synth.weight(c).to(dev), out=self.w)
        self.Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        self.sT = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
        self.dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
        self.dA = torch.empty(r, K, dtype=torch.float32, device=dev)
        self.dB = torch.empty(N, r, dtype=torch.float32, device=dev)
        self.ws_q = torch.empty(q.workspace_bytes(q.OP_QUANTIZE, 0, N, K, 0), dtype=torch.uint8, device=dev)
        # zeroed, so the status word reads clean before the first call too
        self.ws_f = torch.zeros(q.workspace_bytes(q.OP_FWD, M, N, K, r), dtype=torch.uint8, device=dev)
        self.ws_b = torch.zeros(q.workspace_bytes(q.OP_BWD, M, N, K, r), dtype=torch.uint8, device=dev)

    def quantize(self, i):
        self.q.quantize_nf4(self.sets[i % len(self.sets)]["W"], out=self.w, ws=self.ws_q)

    def fwd(self, i, prof=None):
        s = self.sets[i % len(self.sets)]
        if prof is not None:
            self.q.profile_next_launch(self.q.KERNEL_FUSED_FWD, *prof)
        self.q.linear_fwd(s["X"], self.w, s["A"], s["B"], self.cfg.alpha, Y=self.Y, sT=self.sT, ws=self.ws_f)

    def bwd(self, i, prof=None):
        s = self.sets[i % len(self.sets)]
        if prof is not None:
            self.q.profile_next_launch(self.q.KERNEL_FUSED_DX, *prof)
        self.q.linear_bwd(s["dY"], s["X"], self.w, s["A"], s["B"], self.cfg.alpha, sT=self.sT, dX=self.dX,
                          dA=self.dA, dB=self.dB, ws=self.ws_b)

    def step(self, i, prof=None):
        self.quantize(i)
        self.fwd(i, None if prof is None else prof[0])
        self.bwd(i, None if prof is None else prof[1])

    def workspaces(self):
        return [self.ws_f, self.ws_b]

    def fused_flops(self):
        c = self.cfg
        return {"fwd": 2 * c.M * c.N * (c.K + c.r), "dx": 2 * c.M * c.K * (c.N + c.r)}


def fwd_bwd_rows(q, dev):
    """fwd+bwd of every other configuration's linears (weights quantised
    once, graph-timed): TFLOP/s and tokens/s per linear."""
    pk = peaks()[0]
    out = {}
    for cfg in [synth.TINY, synth.ATTN7B, *synth.MLP7B, synth.L65B[0]]:
        L = Linear(q, cfg, dev, sets=2, w_fp32=False)
        t = timed(lambda i: (L.fwd(i), L.bwd(i)), n=20)
        tf = timed(lambda i: L.fwd(i), n=20)
        assert_device_ok(q, L.workspaces(), cfg.name)
        fl = fwd_bwd_flops(cfg.M, cfg.N, cfg.K, cfg.r)
        out[cfg.name] = {"fwd_bwd_us": t * 1e3, "fwd_us": tf * 1e3, "TFLOPs": fl / (t * 1e-3) / 1e12,
                         "tokens_per_s": cfg.M / (t * 1e-3),
                         "frac_bf16_burst": fl / (t * 1e-3) / 1e12 / pk.get("bf16_tflops", 1590.0)}
        del L
        torch.cuda.empty_cache()
    return out


def other_rows(q, dev):
    """The other rows of the path on their own workloads (graph-timed): the
    quantiser and dequantiser on the large weights, the adapter merge and
    the small-batch forward sweep, each streaming from HBM (rotated weight
    copies)."""
    sweep = {}
    pk_hbm = peaks()[0].get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    by_shape = {}
    for c in synth.SWEEP:
        key = (c.N, c.K)
        if key not in by_shape:
            # enough packed copies that the rotation over them is larger
            # than twice the L2, so every timed call streams from HBM
            Wc = synth.weight(c).to(dev)
            ncopy = max(2, math.ceil(2 * l2 / (c.N * c.K * (0.5 + 1 / 64))))
            wcs = [q.quantize_nf4(Wc) for _ in range(ncopy)]
            Wbc = torch.empty(c.N, c.K, dtype=torch.bfloat16, device=dev)
            tq = timed(lambda i: q.quantize_nf4(Wc, out=wcs[i % ncopy]), n=10)
            td = timed(lambda i: q.dequantize_nf4(wcs[i % ncopy], out=Wbc), n=10)
            # the same weight stored in bf16 (a scratch packed copy: the rotated
            # copies keep the fp32 weight's codes for the sweep below)
            Wc16 = Wc.to(torch.bfloat16)
            scratch = q.NF4Weight.empty(c.N, c.K, dev)
            tq16 = timed(lambda i: q.quantize_nf4(Wc16, out=scratch), n=10)
            q16b = c.N * c.K * (2 + 0.5 + 1 / 64)
            sweep[f"quantize_bf16_{c.N}x{c.K}"] = {"us": tq16 * 1e3, "GBs": q16b / tq16 / 1e6,
                                                   "frac_hbm": q16b / tq16 / 1e6 / pk_hbm}
            del Wc16, scratch
            qb, db = c.N * c.K * (4 + 0.5 + 1 / 64), c.N * c.K * (0.5 + 1 / 64 + 4 / 16384 + 2)
            sweep[f"quantize_{c.N}x{c.K}"] = {"us": tq * 1e3, "GBs": qb / tq / 1e6, "frac_hbm": qb / tq / 1e6 / pk_hbm}
            sweep[f"dequantize_{c.N}x{c.K}"] = {"us": td * 1e3, "GBs": db / td / 1e6, "frac_hbm": db / td / 1e6 / pk_hbm}
            # the same weight stored without double quantisation (the rotated
            # copies' codes, rewritten with identical values, and fp32 constants)
            nodq = [q.NF4Weight(wcs[i].codes, None, None, None, c.N, c.K,
                                absmax=torch.empty(c.N * c.K // 64, dtype=torch.float32, device=dev))
                    for i in range(ncopy)]
            tqn = timed(lambda i: q.quantize_nf4_nodq(Wc, out=nodq[i % ncopy]), n=10)
            tdn = timed(lambda i: q.dequantize_nf4(nodq[i % ncopy], out=Wbc), n=10)
            qnb, dnb = c.N * c.K * (4 + 0.5 + 4 / 64), c.N * c.K * (0.5 + 4 / 64 + 2)
            sweep[f"quantize_nodq_{c.N}x{c.K}"] = {"us": tqn * 1e3, "GBs": qnb / tqn / 1e6,
                                                   "frac_hbm": qnb / tqn / 1e6 / pk_hbm}
            sweep[f"dequantize_nodq_{c.N}x{c.K}"] = {"us": tdn * 1e3, "GBs": dnb / tdn / 1e6,
                                                     "frac_hbm": dnb / tdn / 1e6 / pk_hbm}
            del nodq
            # adapter merge into the bf16 weight
            for rm in (16, 64):
                cm = synth.custom(N=c.N, K=c.K, M=1, r=rm)
                Am, Bm = synth.lora_a(cm).to(dev), synth.lora_b(cm).to(dev)
                tm = timed(lambda i: q.merge_lora(wcs[i % ncopy], Am, Bm, cm.alpha, out=Wbc), n=10)
                mb = c.N * c.K * (0.5 + 1 / 64 + 4 / 16384 + 2) + 2 * rm * (c.N + c.K)
                sweep[f"merge_r{rm}_{c.N}x{c.K}"] = {"us": tm * 1e3, "GBs": mb / tm / 1e6,
                                                     "frac_hbm": mb / tm / 1e6 / pk_hbm}
            del Wbc, Wc
            by_shape[key] = wcs
        wcs = by_shape[key]
        ncopy = len(wcs)
        Xc, Ac, Bc = synth.activations(c).to(dev), synth.lora_a(c).to(dev), synth.lora_b(c).to(dev)
        Yc = torch.empty(c.M, c.N, dtype=torch.bfloat16, device=dev)
        sTc = torch.empty(c.M, c.r, dtype=torch.bfloat16, device=dev)
        wsc = torch.empty(q.workspace_bytes(q.OP_FWD, c.M, c.N, c.K, c.r), dtype=torch.uint8, device=dev)
        tf = timed(lambda i: q.linear_fwd(Xc, wcs[i % ncopy], Ac, Bc, c.alpha, Y=Yc, sT=sTc, ws=wsc))
        # the weight-streaming kernel alone (events around it; a profiled
        # call launches it in plain stream order)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(20)]
        for e in evs:
            e[0].record()
            e[1].record()
        for i, e in enumerate(evs):
            q.profile_next_launch(q.KERNEL_FUSED_FWD, e[0], e[1])
            q.linear_fwd(Xc, wcs[i % ncopy], Ac, Bc, c.alpha, Y=Yc, sT=sTc, ws=wsc)
        torch.cuda.synchronize()
        assert_device_ok(q, [wsc], c.name)
        # mean, not median: single-launch event times come in steps of about
        # 2 us here, and the mean of many launches resolves below that step
        tk = statistics.mean(e[0].elapsed_time(e[1]) for e in evs[3:])
        gb = c.N * c.K * (0.5 + 1 / 64 + 4 / 16384) + 2 * c.M * (c.N + c.K) + 2 * c.r * (c.N + c.K)
        wb = c.N * c.K * (0.5 + 1 / 64 + 4 / 16384)
        sweep[c.name] = {"us": tf * 1e3, "GBs": gb / tf / 1e6, "frac_hbm": gb / tf / 1e6 / pk_hbm,
                         "weight_kernel_us": tk * 1e3, "weight_kernel_GBs": wb / tk / 1e6,
                         "weight_kernel_frac_hbm": wb / tk / 1e6 / pk_hbm}
    by_shape.clear()
    torch.cuda.empty_cache()
    return sweep


def run_ours(args, rank, world, local_rank):
    import bit_nf4_quantized_09_b200 as q

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    def barrier():
        if pg is not None:
            pg.barrier()

    layers = [Linear(q, c, dev) for c in HEADLINE]

    def step(i, prof=None):
        for j, L in enumerate(layers):
            L.step(i, None if prof is None else prof[j])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # ---- eager timing (host launches every kernel): reported for reference
    n_eager = min(args.steps, 50)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    h0 = time.perf_counter()
    for i in range(n_eager):
        step(i)
    host_ms = (time.perf_counter() - h0) * 1e3 / n_eager  # host enqueue time per step
    e1.record()
    torch.cuda.synchronize()
    eager_ms = e0.elapsed_time(e1) / n_eager

    # ---- timed region: the K steps, every kernel of every step, replayed from
    # one captured CUDA graph (no host launch gaps); each step records its own
    # events around the four fused matmuls (forward and dX of each linear)
    def ev():
        return torch.cuda.Event(enable_timing=True)
    prof = [[[(ev(), ev()) for _ in range(2)] for _ in layers] for _ in range(args.steps)]
    for per_step in prof:  # torch creates events lazily: make them exist before the library records them
        for per_layer in per_step:
            for a, b in per_layer:
                a.record()
                b.record()
    torch.cuda.synchronize()
    launches0 = q.launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(args.steps):
            step(i, prof[i])
    launches = q.launch_count() - launches0
    graph.replay()  # one untimed replay of the whole graph
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local_rank)
    time.sleep(0.15)
    barrier()
    torch.cuda.synchronize()
    start.record()
    graph.replay()
    stop.record()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    ms = max_over_ranks(start.elapsed_time(stop) / args.steps, pg, dev)
    for L in layers:
        assert_device_ok(q, L.workspaces(), "timed step")
    # per launch: (name, ms, flops) of the four fused matmuls of every step
    fused = []
    for per_step in prof:
        for j, L in enumerate(layers):
            fl = L.fused_flops()
            fused.append((f"fwd_{L.cfg.name}", per_step[j][0][0].elapsed_time(per_step[j][0][1]), fl["fwd"]))
            fused.append((f"dx_{L.cfg.name}", per_step[j][1][0].elapsed_time(per_step[j][1][1]), fl["dx"]))
    del graph

    # ---- per-row breakdown (outside the timed region, same inputs), each
    # graph-timed
    rows_ms = {}
    for L in layers:
        n = L.cfg.name
        rows_ms[f"quantize_{n}"] = timed(L.quantize)
        rows_ms[f"forward_{n}"] = timed(L.fwd)
        rows_ms[f"backward_{n}"] = timed(L.bwd)
    for L in layers:
        assert_device_ok(q, L.workspaces(), "rows")

    # ---- end to end through the public API with host buffers. Step i's
    # inputs go host -> device on a copy stream, its compute runs on the main
    # stream and its outputs go device -> host on a second copy stream, with
    # inputs and outputs double-buffered: the copies of neighbouring steps
    # overlap the compute, and every byte still crosses PCIe inside the timed
    # region.
    pins = [[{k: v.pin_memory() for k, v in h.items()} for h in L.host] for L in layers]
    outs = [[dict(Y=L.Y, dX=L.dX, dA=L.dA, dB=L.dB),
             dict(Y=torch.empty_like(L.Y), dX=torch.empty_like(L.dX), dA=torch.empty_like(L.dA),
                  dB=torch.empty_like(L.dB))] for L in layers]
    out_host = [[{k: torch.empty_like(v, device="cpu").pin_memory() for k, v in o.items()} for o in lo]
                for lo in outs]
    h2d = sum(v.numel() * v.element_size() for p in pins for v in p[0].values())
    d2h = sum(v.numel() * v.element_size() for lo in out_host for v in lo[0].values())
    main = torch.cuda.current_stream(dev)
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready, in_free = [torch.cuda.Event() for _ in range(2)], [torch.cuda.Event() for _ in range(2)]
    out_ready, out_free = [torch.cuda.Event() for _ in range(2)], [torch.cuda.Event() for _ in range(2)]
    for j in range(2):  # every buffer starts free
        in_free[j].record(main)
        out_free[j].record(main)

    def e2e_step(i):
        j = i % 2
        with torch.cuda.stream(h2d_s):
            h2d_s.wait_event(in_free[j])  # the step two back has finished reading set j
            for li, L in enumerate(layers):
                for k, v in L.sets[j].items():
                    v.copy_(pins[li][j][k], non_blocking=True)
            in_ready[j].record(h2d_s)
        main.wait_event(in_ready[j])
        main.wait_event(out_free[j])  # the step two back has left output set j
        for li, L in enumerate(layers):
            o = outs[li][j]
            s = L.sets[j]
            q.quantize_nf4(s["W"], out=L.w, ws=L.ws_q)
            q.linear_fwd(s["X"], L.w, s["A"], s["B"], L.cfg.alpha, Y=o["Y"], sT=L.sT, ws=L.ws_f)
            q.linear_bwd(s["dY"], s["X"], L.w, s["A"], s["B"], L.cfg.alpha, sT=L.sT, dX=o["dX"], dA=o["dA"],
                         dB=o["dB"], ws=L.ws_b)
        in_free[j].record(main)
        out_ready[j].record(main)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(out_ready[j])
            for li in range(len(layers)):
                for k, v in outs[li][j].items():
                    out_host[li][j][k].copy_(v, non_blocking=True)
            out_free[j].record(d2h_s)

    e2e_steps = max(3, min(args.steps, 20))
    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    h2d_s.wait_event(e0)
    d2h_s.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    main.wait_stream(h2d_s)
    main.wait_stream(d2h_s)
    e1.record(main)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, pg, dev)
    for L in layers:
        assert_device_ok(q, L.workspaces(), "end to end")
    del pins, out_host, outs

    # dequantise the headline weights (a3 standalone; not part of the step)
    deq = {}
    for L in layers:
        Wbf = torch.empty(L.cfg.N, L.cfg.K, dtype=torch.bfloat16, device=dev)
        t = timed(lambda i: q.dequantize_nf4(L.w, out=Wbf))
        deq[L.cfg.name] = (L.cfg.N * L.cfg.K * (0.5 + 1 / 64 + 4 / 16384 + 2)) / (t * 1e-3) / 1e9
        del Wbf
    flops_step = step_flops(HEADLINE)
    M = HEADLINE[0].M
    del layers
    torch.cuda.empty_cache()

    # ---- the other configurations' fwd+bwd and the other rows of the path
    # on their own workloads (graph-timed, outside the timed region)
    extra = {} if (args.no_sweep or rank != 0) else fwd_bwd_rows(q, dev)
    sweep = {} if (args.no_sweep or rank != 0) else other_rows(q, dev)

    value = job_tflops(flops_step, world, ms)
    pk, pk_kind = peaks()
    # dominant kernel: the fused matmul (every launch of it in the timed
    # region: forward and dX of both linears)
    f_ms = statistics.mean(t for _, t, _ in fused)
    f_flops = statistics.mean(f for _, _, f in fused)
    achieved = f_flops / (f_ms * 1e-3) / 1e12
    peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    by_launch = {}
    for name, t, f in fused:
        by_launch.setdefault(name, []).append((t, f))
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(),
        "tokens_per_s": M * world / (ms * 1e-3),
        "dequant_gbs": statistics.mean(deq.values()),
        "dequant_gbs_by_weight": deq,
        "rows_ms": rows_ms,
        "timing": "timed steps replayed from one CUDA graph holding all K steps",
        "eager_ms_per_step": eager_ms,
        "host_enqueue_ms_per_step": host_ms,
        "fused_launches_us": {k: statistics.mean(t for t, _ in v) * 1e3 for k, v in by_launch.items()},
        "roofline": {"kernel": "fused_nf4_gemm (forward and dX of both linears)", "bound": "tensor",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": NCU_TRAFFIC.get("fused_nf4_gemm"),
                     "traffic_source": "ncu capture of one step's four launches: mean of dram__bytes_read.sum + "
                                       "dram__bytes_write.sum per launch" if "fused_nf4_gemm" in NCU_TRAFFIC else None,
                     "peak_kind": f"bf16 burst ({pk_kind}; the timed graph lasts well under a second)",
                     "frac_of_sustained": achieved / pk.get("bf16_tflops_sustained", 1400.0),
                     "frac_of_datasheet_dense": achieved / DATASHEET_BF16_TFLOPS},
        "e2e": {"value": job_tflops(flops_step, world, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "overlap": "H2D of step i+1 and D2H of step i-1 on two copy streams beside step i's compute"},
        "gpu_launches": launches,
        "device_status": "ok",
        "fwd_bwd_rows": extra,
        "other_rows": sweep,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = OracleSample(HEADLINE).sample_line(args.cpu_seconds)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_case(args):
    """One call of the library repeated (for profiler captures): `step` is the
    headline step; `fwd:<workload>` etc. one entry point on one named
    workload (synth names), its weight quantised once beforehand."""
    import bit_nf4_quantized_09_b200 as q

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.case == "step":
        layers = [Linear(q, c, dev) for c in HEADLINE]
        for i in range(args.reps):
            for L in layers:
                L.step(i)
        torch.cuda.synchronize()
        for L in layers:
            assert_device_ok(q, L.workspaces(), "case step")
        return
    kind, _, name = args.case.partition(":")
    cfg = synth.by_name(name)
    L = Linear(q, cfg, dev, sets=1, w_fp32=kind == "quantize")
    if kind == "quantize":
        fn = L.quantize
    elif kind == "fwd":
        fn = L.fwd
    elif kind == "bwd":
        L.fwd(0)
        fn = L.bwd
    elif kind == "dequantize":
        Wbf = torch.empty(cfg.N, cfg.K, dtype=torch.bfloat16, device=dev)
        fn = lambda i: q.dequantize_nf4(L.w, out=Wbf)  # noqa: E731
    elif kind == "merge":
        Wbf = torch.empty(cfg.N, cfg.K, dtype=torch.bfloat16, device=dev)
        s = L.sets[0]
        fn = lambda i: q.merge_lora(L.w, s["A"], s["B"], cfg.alpha, out=Wbf)  # noqa: E731
    else:
        raise SystemExit(f"unknown case {args.case}")
    for i in range(args.reps):
        fn(i)
    torch.cuda.synchronize()
    assert_device_ok(q, L.workspaces(), f"case {args.case}")


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-sweep", action="store_true", help="skip the other configurations' rows")
    ap.add_argument("--rows-only", action="store_true",
                    help="only the small-batch / quantiser rows (one JSON line with other_rows), for profiling")
    ap.add_argument("--case", default=None, help="repeat one call for a profiler capture (see above)")
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
    elif args.case:
        run_case(args)
    elif args.rows_only:
        import bit_nf4_quantized_09_b200 as q
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        print(json.dumps({"fwd_bwd_rows": fwd_bwd_rows(q, dev), "other_rows": other_rows(q, dev)}), flush=True)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
