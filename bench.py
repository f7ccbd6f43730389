#!/usr/bin/env python3
"""Benchmark of the BitNet b1.58 BitLinear hot path on B200.

Default workload (the N=1 line): decode, M = 1 token, through the seven
linears of a 2B-class block (2560->6912 x2, 6912->2560, 2560->2560 x2,
2560->640 x2), x bf16 ~ N(0,1) with 1% outliers x20, fp32 y.  One step is
one pass of the per-token hot path over the block: per-token absmax int8
quantisation, ternary x int8 product with int32 accumulation and the
rescale, for all seven linears (weights are packed once beforehand, as a
model's weights are; packing is timed separately).  Metric: algorithmic
bytes (packed weights N*K/4 + bf16 x + fp32 y) per second.

The packed weights are replicated into enough copies that the rotating
working set exceeds 3x the L2 size, so every step streams its weights from
HBM.  Steps are replayed from CUDA graphs and timed with CUDA events on the
launching stream; multi-GPU runs are independent replicas (no collective on
the data path), timed as the max over ranks.

Other workloads (--workload): 7b (decode at 7B-class shapes, --m 1/4/16; from
two tokens up a step is the grouped call's workspace form: one quantiser
launch over the three linears, then one product launch on the codes),
prefill (M = 2048 tokens on the tensor cores; metric int8 TOPS), pack
(absmean quantise + 2-bit pack of the block's weights), sweep100b (one token
through 80 layers x 7 linears of a 100B-class model, 17.1 GB of packed
weights resident; weights drawn on the GPU by the counter-based generator).

--impl reference times the CPU oracle (oracle/, plain C) on the same
workload and metric, on this machine's host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "BitLinear decode weight GB/s (% of HBM peak); prefill int8 TOPS (% peak)"
NOMINAL_INT8_OVER_BF16 = 2.0     # dense int8 / dense bf16 tensor throughput (4.5 / 2.25 PFLOP/s)


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["block2b", "7b", "prefill", "pack", "sweep100b"], default="block2b")
    ap.add_argument("--m", type=int, default=1, help="tokens for --workload 7b")
    ap.add_argument("--mode", choices=["grouped", "fused", "separate"], default="grouped",
                    help="decode: grouped = one launch per step; fused = one launch per linear; "
                         "separate = quantise + product launches per linear")
    ap.add_argument("--decode-kernel", choices=["auto", "tensor", "dp4a", "tile", "lut"], default="auto",
                    help="decode kernel for M <= 16 (bitlinear_set_decode_kernel)")
    ap.add_argument("--rmsnorm", action="store_true",
                    help="decode: fuse SubLN (RMS normalisation with a gain per linear) into the quantiser prologue")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="oracle CPU-baseline budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill sub-measurement")
    return ap.parse_args()


# ----------------------------------------------------------------- utils
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "kind": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "kind": "fallback"}


class ClockSampler:
    """Polls SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _poll(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
        except Exception:
            pass

    def start(self):
        if self.nv is None:
            return
        self._sample()
        self._thr = threading.Thread(target=self._poll, daemon=True)
        self._thr.start()

    def stop(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml_unavailable"], "samples": 0}
        self._stop.set()
        if self._thr:
            self._thr.join()
        self._sample()
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


def decode_bytes(lin, M):
    """Algorithmic bytes of one decode pass: packed W + bf16 x + fp32 y."""
    return sum(L["N"] * L["K"] // 4 + M * L["K"] * 2 + M * L["N"] * 4 for L in lin)


# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu
# capture of the same launch configuration (profiles/ holds the summary and
# the command).  Valid only for the kernel source it was taken from: set an
# entry to None when that kernel changes.
MEASURED_TRAFFIC = {
    # stream_kernel<1, fused, bf16, fp32, 4>, 2B block, M = 1, grouped launch
    ("block2b", "stream_kernel", 1): 17_469_184,
    # gemm_tc_kernel<bf16>, M = 2048: mean of the step's two launches
    # (2560->6912: 9,722,368 B; 6912->2560: 18,645,504 B)
    ("prefill", "gemm_tc_kernel", 2048): 14_183_936,
}


def decode_kernel_name(args, M=1):
    """The kernel bitlinear_set_decode_kernel selects for the bench shapes:
    AUTO takes the dp4a streaming kernel up to 4 tokens, the tensor-core
    kernel above (both fit every bench shape except where noted by the
    library's fallbacks)."""
    if args.decode_kernel == "auto":
        return "stream_kernel" if M <= 4 else "dec_tc_kernel"
    return {"tensor": "dec_tc_kernel", "dp4a": "stream_kernel", "tile": "gemv_kernel",
            "lut": "lut_kernel"}[args.decode_kernel]


def max_over_ranks(ms, dist, dev):
    """The slowest rank's time: every rank contributes its own CUDA-event
    time and all take the maximum (dev=None reduces on the CPU, as with a
    gloo group)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], device=dev if dev is not None else "cpu", dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def linears_for(args):
    import synth
    if args.workload == "7b":
        M = args.m
        lin = []
        for i, (K, N, name) in enumerate(synth.SHAPES_7B):
            lin.append(dict(name=name, K=K, N=N, W=synth.weights(N, K, 10 + i),
                            x=synth.activations(M, K, 2000 + i, "bf16")))
        return lin, M, f"7b_decode_m{M}"
    if args.workload == "prefill":
        M = synth.M_PREFILL
        lin = []
        for i, (K, N, name) in enumerate(synth.PREFILL):
            lin.append(dict(name=name, K=K, N=N, W=synth.weights(N, K, 20 + i),
                            x=synth.activations(M, K, 3000 + i, "bf16")))
        return lin, M, "prefill_m2048"
    return synth.block2b_inputs(seed_base=0, M=1), 1, "block2b_decode_m1"


# ----------------------------------------------------- CPU (oracle) arm
def oracle_setup(lin):
    import numpy as np
    import oracle
    prepared = []
    for L in lin:
        g64 = oracle.absmean_gamma(L["W"])
        code, _, _ = oracle.ternary_codes(L["W"], g64, 1e-5)
        prepared.append(dict(x=L["x"], code=code, g32=float(np.float32(g64)), N=L["N"], K=L["K"]))
    return prepared


def oracle_pass(prepared, threads, row_frac=1.0):
    """One oracle pass over the linears (quantise, multiply, rescale); with
    row_frac < 1 only the first row_frac of each weight's output rows.
    Returns (algorithmic bytes, int ops) of the work done."""
    import oracle
    nbytes, ops = 0, 0
    for P in prepared:
        n = max(1, int(P["N"] * row_frac))
        oracle.forward_bf16_mt(P["x"], P["code"][:n], P["g32"], threads)
        M = P["x"].shape[0]
        nbytes += n * P["K"] // 4 + P["x"].size * 2 + M * n * 4
        ops += 2 * M * n * P["K"]
    return nbytes, ops


def cpu_baseline(lin, seconds, prefill=False):
    prepared = oracle_setup(lin)
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    total, passes = 0, 0
    frac = 1.0
    if prefill:   # a full prefill pass is minutes of scalar CPU work: sample rows
        frac = 0.01
    while True:
        b, o = oracle_pass(prepared, threads, frac)
        total += o if prefill else b
        passes += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    if prefill:
        return {"value": total / el / 1e12, "unit": "TOPS", "cores": threads, "kind": "oracle",
                "sample": f"{passes} oracle passes over 1% of the output rows of each prefill linear "
                          f"({el:.1f} s, {threads} threads)"}
    return {"value": total / el / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{passes} full oracle passes over the linears at M={lin[0]['x'].shape[0]} "
                      f"({el:.1f} s, {threads} threads, rows split across threads)"}


def run_reference(args, lin, M, config):
    """The oracle as the reference arm: rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    prefill = args.workload == "prefill"
    prepared = oracle_setup(lin)
    threads = os.cpu_count() or 1
    probe = 0.01 if prefill else 1.0
    t0 = time.perf_counter()
    oracle_pass(prepared, threads, probe)
    t_probe = (time.perf_counter() - t0) / probe
    budget = 120.0
    frac = min(1.0, budget / max(1e-9, t_probe * (args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_pass(prepared, threads, frac)
    t0 = time.perf_counter()
    nbytes, ops = 0, 0
    for _ in range(args.steps):
        b, o = oracle_pass(prepared, threads, frac)
        nbytes += b
        ops += o
    el = time.perf_counter() - t0
    value, unit = (ops / el / 1e12, "TOPS") if prefill else (nbytes / el / 1e9, "GB/s")
    sample = (f"each step: oracle pass over {frac * 100:.3g}% of every linear's output rows "
              f"(quantise + multiply + rescale), {threads} threads")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
            "data": "synthetic", "config": config,
            "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# --------------------------------------------------------------- GPU arm
class Graphs:
    """CUDA graphs of `copies` consecutive steps and of single steps."""

    def __init__(self, torch, stream, step, copies):
        self.copies = copies
        with torch.cuda.stream(stream):
            self.all = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.all, stream=stream):
                for i in range(copies):
                    step(i)
            self.one = []
            for i in range(copies):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    step(i)
                self.one.append(g)

    def run(self, n):
        full, rem = divmod(n, self.copies)
        for _ in range(full):
            self.all.replay()
        for i in range(rem):
            self.one[i].replay()


def time_region(torch, stream, fn, dist, dev):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0.record(stream)
    fn()
    e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    return max_over_ranks(e0.elapsed_time(e1), dist, dev)


def setup_problems(torch, bl, lin, M, dev, want_bytes, out_dtype):
    """Packs every weight once (GPU packer), then replicates weights, x and y
    into `copies` sets so that one pass over all copies touches > want_bytes."""
    import numpy as np
    packed0, g32s = [], []
    for L in lin:
        p, _, g = bl.pack(torch.from_numpy(L["W"]).to(dev))
        packed0.append(p)
        g32s.append(g)
    torch.cuda.synchronize()
    if bl.bitlinear_get_status() != bl.BL_OK:
        raise RuntimeError("non-finite weights")
    per_copy = sum(p.numel() for p in packed0) + sum(M * L["K"] * 2 + M * L["N"] * 4 for L in lin)
    copies = max(2, math.ceil(want_bytes / per_copy))
    packed = [[p.clone() for p in packed0] for _ in range(copies)]
    xs = [[torch.from_numpy(L["x"].view(np.int16)).to(dev).view(torch.bfloat16) for L in lin]
          for _ in range(copies)]
    ys = [[torch.empty((M, L["N"]), dtype=out_dtype, device=dev) for L in lin] for _ in range(copies)]
    return dict(packed=packed, g32=g32s, xs=xs, ys=ys, copies=copies, per_copy=per_copy,
                Ns=[L["N"] for L in lin], Ks=[L["K"] for L in lin])


def run_decode(torch, bl, args, lin, M, dev, stream, dist, l2):
    S = setup_problems(torch, bl, lin, M, dev, 3 * l2, torch.float32)
    copies, Ns, Ks = S["copies"], S["Ns"], S["Ks"]
    mode = args.mode
    if mode == "grouped" and not all(bl.bitlinear_forward_x_supported(M, K) for K in Ks):
        mode = "separate"
    qs = [torch.empty((M, bl.bitlinear_padded_k(K)), dtype=torch.int8, device=dev) for K in Ks]
    gains = [(1.0 + 0.25 * torch.randn(K, generator=torch.Generator().manual_seed(K))).to(dev) for K in Ks]
    ss = [torch.empty(M, dtype=torch.float32, device=dev) for _ in Ks]

    # the workspace form: for M >= 2 one quantiser launch over all linears,
    # then the product kernel on the codes
    ws = bl.decode_workspace(M, Ks, dev) if mode == "grouped" else None
    grouped_launches = 2 if M >= 2 else 1

    def step(i):
        c = i % copies
        if mode == "grouped" and args.rmsnorm:
            bl.bitlinear_forward_x_rmsnorm_grouped(S["xs"][c], gains, 1e-6, S["packed"][c], S["g32"], Ns, Ks,
                                                   S["ys"][c], stream, workspace=ws)
            return grouped_launches
        if mode == "grouped":
            bl.bitlinear_forward_x_grouped(S["xs"][c], S["packed"][c], S["g32"], Ns, Ks, S["ys"][c], stream,
                                           workspace=ws)
            return grouped_launches
        if mode == "fused":
            for j in range(len(lin)):
                bl.bitlinear_forward_x(S["xs"][c][j], S["packed"][c][j], S["g32"][j], Ns[j], Ks[j],
                                       S["ys"][c][j], stream)
            return len(lin)
        for j in range(len(lin)):
            bl.bitlinear_quant_act(S["xs"][c][j], qs[j], ss[j], stream)
            bl.bitlinear_forward(qs[j], ss[j], S["packed"][c][j], S["g32"][j], M, Ns[j], Ks[j],
                                 S["ys"][c][j], None, stream)
        return 2 * len(lin)

    try:
        launches = step(0)
    except bl.BitLinearError as e:
        # a forced decode kernel that cannot take the grouped fused form
        if mode != "grouped" or e.status != bl.BL_ERR_SHAPE:
            raise
        mode = "separate"
        launches = step(0)
    torch.cuda.synchronize()
    G = Graphs(torch, stream, step, copies)
    G.run(max(3, args.warmup))
    sampler = ClockSampler(dev.index)
    sampler.start()
    ms = time_region(torch, stream, lambda: G.run(args.steps), dist, dev)
    clocks = sampler.stop()
    if bl.bitlinear_get_status() != bl.BL_OK:
        raise RuntimeError("device status word set during the timed region")
    nbytes = decode_bytes(lin, M)

    # dominant kernel: the product kernel (the whole step in grouped mode)
    if mode == "grouped" and M == 1:
        kern_ms, kern_bytes, kname = ms / args.steps, nbytes, f"{decode_kernel_name(args, M)} (fused quantise, {len(lin)} linears, 1 launch)"
    elif mode == "grouped":
        # the whole step (quantiser + product kernel) against the product's
        # bytes: a lower bound on the product kernel's own rate
        kern_ms, kern_bytes, kname = ms / args.steps, nbytes, f"quant_kernel + {decode_kernel_name(args, M)} (product on the codes, {len(lin)} linears, 2 launches; both timed)"
    else:
        def kstep(i):
            c = i % copies
            for j in range(len(lin)):
                if mode == "fused":
                    bl.bitlinear_forward_x(S["xs"][c][j], S["packed"][c][j], S["g32"][j], Ns[j], Ks[j],
                                           S["ys"][c][j], stream)
                else:
                    bl.bitlinear_forward(qs[j], ss[j], S["packed"][c][j], S["g32"][j], M, Ns[j], Ks[j],
                                         S["ys"][c][j], None, stream)
        GK = Graphs(torch, stream, kstep, copies)
        GK.run(copies)
        reps = max(copies, args.steps)
        kms = time_region(torch, stream, lambda: GK.run(reps), dist, dev)
        kern_ms = kms / (reps * len(lin))
        kern_bytes = nbytes / len(lin)
        kname = f"{decode_kernel_name(args, M)} (product, one launch per linear)"
    return dict(S=S, mode=mode, ms=ms, launches=launches, clocks=clocks, nbytes=nbytes,
                kern_ms=kern_ms, kern_bytes=kern_bytes, kname=kname)


def run_e2e(torch, bl, lin, M, dev, stream, S, steps, dist):
    """Pinned host x -> H2D -> grouped C-ABI call -> D2H y, every step."""
    import numpy as np
    Ns, Ks, copies = S["Ns"], S["Ks"], S["copies"]
    hx = torch.empty(sum(M * K for K in Ks), dtype=torch.bfloat16).pin_memory()
    hy = torch.empty(sum(M * N for N in Ns), dtype=torch.float32).pin_memory()
    off = 0
    for L in lin:
        hx[off:off + M * L["K"]].copy_(torch.from_numpy(L["x"].view(np.int16).ravel()).view(torch.bfloat16))
        off += M * L["K"]
    dx = torch.empty_like(hx, device=dev)
    dy = torch.empty_like(hy, device=dev)
    xv, yv, ox, oy = [], [], 0, 0
    for K, N in zip(Ks, Ns):
        xv.append(dx[ox:ox + M * K].view(M, K))
        yv.append(dy[oy:oy + M * N].view(M, N))
        ox += M * K
        oy += M * N

    # one prepared grouped call per weight copy (the pointer arrays are built
    # once, as a decode loop would)
    calls = [bl.GroupedDecode(xv, S["packed"][c], S["g32"], Ns, Ks, yv) for c in range(copies)]

    def e2e_step(i):
        dx.copy_(hx, non_blocking=True)
        calls[i % copies](stream)
        hy.copy_(dy, non_blocking=True)

    for i in range(3):
        e2e_step(i)
    n = max(1, min(steps, 2000))
    ems = time_region(torch, stream, lambda: [e2e_step(i) for i in range(n)], dist, dev)
    return ems, n, hx.numel() * hx.element_size(), hy.numel() * hy.element_size()


def run_prefill(torch, bl, args, dev, stream, dist, l2, steps):
    import synth
    lin = []
    for i, (K, N, name) in enumerate(synth.PREFILL):
        lin.append(dict(name=name, K=K, N=N, W=synth.weights(N, K, 20 + i),
                        x=synth.activations(synth.M_PREFILL, K, 3000 + i, "bf16")))
    M = synth.M_PREFILL
    S = setup_problems(torch, bl, lin, M, dev, 3 * l2, torch.bfloat16)
    copies, Ns, Ks = S["copies"], S["Ns"], S["Ks"]
    qs = [[torch.empty((M, bl.bitlinear_padded_k(K)), dtype=torch.int8, device=dev) for K in Ks]
          for _ in range(copies)]
    ss = [[torch.empty(M, dtype=torch.float32, device=dev) for _ in Ks] for _ in range(copies)]

    def step(i):
        c = i % copies
        for j in range(len(lin)):
            bl.bitlinear_quant_act(S["xs"][c][j], qs[c][j], ss[c][j], stream)
            bl.bitlinear_forward(qs[c][j], ss[c][j], S["packed"][c][j], S["g32"][j], M, Ns[j], Ks[j],
                                 S["ys"][c][j], None, stream)

    def gstep(i):
        c = i % copies
        for j in range(len(lin)):
            bl.bitlinear_forward(qs[c][j], ss[c][j], S["packed"][c][j], S["g32"][j], M, Ns[j], Ks[j],
                                 S["ys"][c][j], None, stream)

    step(0)
    torch.cuda.synchronize()
    G = Graphs(torch, stream, step, copies)
    GK = Graphs(torch, stream, gstep, copies)
    G.run(max(3, min(args.warmup, 20)))
    ms = time_region(torch, stream, lambda: G.run(steps), dist, dev)
    GK.run(copies)
    kms = time_region(torch, stream, lambda: GK.run(steps), dist, dev)
    ops = sum(2 * M * N * K for N, K in zip(Ns, Ks))
    peaks = load_peaks()
    int8_peak = peaks["bf16_tflops"] * NOMINAL_INT8_OVER_BF16
    achieved = ops / (kms / steps / 1e3) / 1e12
    # measured int8 ceiling of the library GEMM (cuBLASLt via torch._int_mm), context only
    ref_tops = None
    try:
        a = torch.randint(-127, 128, (8192, 8192), dtype=torch.int8, device=dev)
        b = torch.randint(-127, 128, (8192, 8192), dtype=torch.int8, device=dev)
        for _ in range(3):
            torch._int_mm(a, b)
        n = 10
        tms = time_region(torch, stream, lambda: [torch._int_mm(a, b) for _ in range(n)], None, dev)
        ref_tops = 2 * 8192 ** 3 / (tms / n / 1e3) / 1e12
        del a, b
    except Exception:
        pass
    return {"workload": "prefill_m2048 (2560->6912, 6912->2560), bf16 x, bf16 y",
            "value": ops / (ms / steps / 1e3) / 1e12, "unit": "TOPS", "ms_per_step": ms / steps,
            "steps": steps, "launches_per_step": 2 * len(lin),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": int8_peak, "unit": "TFLOP/s",
                         "frac": achieved / int8_peak,
                         "traffic": MEASURED_TRAFFIC.get(("prefill", "gemm_tc_kernel", M)),
                         "kernel": "gemm_tc_kernel (tcgen05 kind::i8, weights expanded into TMEM)",
                         "peak_kind": f"{peaks['kind']} bf16 burst x nominal int8/bf16 ratio 2",
                         "avg_launch_us": kms / steps / len(lin) * 1e3,
                         "cublaslt_int8_8192cubed_tops": ref_tops},
            "l2_policy": f"{copies} rotating copies of x, q, weights and y (> 3x L2)"}


def run_pack(torch, bl, args, dev, stream, dist, l2):
    import synth
    lin = synth.block2b_inputs(0, 1)
    Ws = [torch.from_numpy(L["W"]).to(dev) for L in lin]
    wbytes = sum(w.numel() * 4 for w in Ws)
    copies = max(1, math.ceil(3 * l2 / wbytes))
    Wc = [[w.clone() for w in Ws] for _ in range(copies)]
    outs = [(torch.empty(bl.bitlinear_packed_bytes(L["N"], L["K"]), dtype=torch.uint8, device=dev),
             torch.empty(1, dtype=torch.float64, device=dev), torch.empty(1, dtype=torch.float32, device=dev),
             torch.empty(bl.bitlinear_pack_workspace_bytes(L["N"], L["K"]), dtype=torch.uint8, device=dev))
            for L in lin]

    def step(i):
        for j, L in enumerate(lin):
            p, g64, g32, ws = outs[j]
            bl.bitlinear_pack_weights(Wc[i % copies][j], 1e-5, p, g64, g32, ws, stream)

    step(0)
    torch.cuda.synchronize()
    G = Graphs(torch, stream, step, copies)
    G.run(3)
    steps = max(copies, min(args.steps, 200))
    ms = time_region(torch, stream, lambda: G.run(steps), dist, dev)
    nweights = sum(L["N"] * L["K"] for L in lin)
    algo = nweights * 4 + nweights // 4   # read fp32 W once + write 2-bit codes
    return {"value": algo * steps / (ms / 1e3) / 1e9, "unit": "GB/s", "ms_per_step": ms / steps,
            "steps": steps, "algorithmic_bytes_per_step": algo, "launches_per_step": 3 * len(lin),
            "note": "two passes over W (absmean, then codes); the second is served from L2 "
                    "for weights that fit there"}


SWEEP_SEED = 1234


def run_sweep(torch, bl, args, dev, stream, dist):
    """80 layers x 7 linears at M = 1; one grouped fused launch per layer."""
    import numpy as np
    import synth
    import synth.device as sd
    kmax = max(K * N for K, N, _ in synth.LAYER100B)
    wbuf = torch.empty(kmax, dtype=torch.float32, device=dev)
    layers = []
    t0 = time.perf_counter()
    for layer in range(synth.LAYERS100B):
        ps, gs, xs, ys = [], [], [], []
        for j, (K, N, name) in enumerate(synth.LAYER100B):
            g = layer * 7 + j
            W = wbuf[:N * K].view(N, K)
            sd.weights(W, SWEEP_SEED, g, 0, stream.cuda_stream)
            p = torch.empty(bl.bitlinear_packed_bytes(N, K), dtype=torch.uint8, device=dev)
            g64 = torch.empty(1, dtype=torch.float64, device=dev)
            g32 = torch.empty(1, dtype=torch.float32, device=dev)
            ws = torch.empty(bl.bitlinear_pack_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
            bl.bitlinear_pack_weights(W, 1e-5, p, g64, g32, ws, stream)
            x = synth.activations(1, K, 50_000 + g, "bf16")
            ps.append(p)
            gs.append(g32)
            xs.append(torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16))
            ys.append(torch.empty((1, N), dtype=torch.float32, device=dev))
        layers.append((xs, ps, gs, ys))
    torch.cuda.synchronize()
    setup_s = time.perf_counter() - t0
    del wbuf
    if bl.bitlinear_get_status() != bl.BL_OK:
        raise RuntimeError("non-finite weights")
    Ns = [N for K, N, _ in synth.LAYER100B]
    Ks = [K for K, N, _ in synth.LAYER100B]

    def step(i):
        for xs, ps, gs, ys in layers:
            bl.bitlinear_forward_x_grouped(xs, ps, gs, Ns, Ks, ys, stream)

    step(0)
    torch.cuda.synchronize()
    G = Graphs(torch, stream, step, 1)
    G.run(max(3, min(args.warmup, 10)))
    steps = max(3, min(args.steps, 50))
    sampler = ClockSampler(dev.index)
    sampler.start()
    ms = time_region(torch, stream, lambda: G.run(steps), dist, dev)
    clocks = sampler.stop()
    if bl.bitlinear_get_status() != bl.BL_OK:
        raise RuntimeError("device status word set during the timed region")
    lin = [dict(K=K, N=N) for K, N, _ in synth.LAYER100B]
    nbytes = decode_bytes(lin, 1) * synth.LAYERS100B
    packed_bytes = sum(p.numel() for _, ps, _, _ in layers for p in ps)
    return dict(ms=ms, steps=steps, nbytes=nbytes, packed_bytes=packed_bytes, clocks=clocks, setup_s=setup_s,
                launches=synth.LAYERS100B)


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    lin, M, wname = linears_for(args)
    config = {"workload": wname, "M": M, "linears": [f"{L['name']}:{L['K']}->{L['N']}" for L in lin],
              "x": "bf16 N(0,1)" + (", 1% outliers x20" if args.workload == "block2b" else ""),
              "y": "bf16" if args.workload == "prefill" else "fp32",
              "weights": "N(0,0.02) fp32, packed 2-bit", "parallelism": "replicas" if world > 1 else "single"}

    if args.impl == "reference":
        out = run_reference(args, lin, M, config)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    import torch
    import ternary_weight_linear_absmean_b200 as bl
    from ternary_weight_linear_absmean_b200 import _build
    _build.build()
    torch.cuda.set_device(local)
    bl.bitlinear_set_decode_kernel({"auto": bl.BL_DECODE_AUTO, "tensor": bl.BL_DECODE_TENSOR,
                                    "dp4a": bl.BL_DECODE_DP4A, "tile": bl.BL_DECODE_TILE,
                                    "lut": bl.BL_DECODE_LUT}[args.decode_kernel])
    config["decode_kernel"] = args.decode_kernel
    if args.rmsnorm:
        config["subln"] = "RMS normalisation with gain fused into every linear's quantiser prologue"
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    peaks = load_peaks()

    if args.workload == "prefill":
        sampler = ClockSampler(local)
        sampler.start()
        pf = run_prefill(torch, bl, args, dev, stream, dist, l2, max(8, args.steps // 100))
        clocks = sampler.stop()
        out = {"metric": METRIC, "value": pf["value"] * world, "unit": "TOPS", "n_gpus": world,
               "steps": pf["steps"], "warmup": args.warmup, "ms_per_step": pf["ms_per_step"],
               "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int32",
               "data": "synthetic", "config": dict(config, l2_policy=pf["l2_policy"]),
               "roofline": pf["roofline"], "gpu_launches": pf["launches_per_step"] * pf["steps"],
               "clocks": clocks}
        if rank == 0 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(lin, args.cpu_seconds, prefill=True)
    elif args.workload == "sweep100b":
        R = run_sweep(torch, bl, args, dev, stream, dist)
        per_step = R["ms"] / R["steps"]
        value = R["nbytes"] * R["steps"] * world / (R["ms"] / 1e3) / 1e9
        achieved = R["nbytes"] / (per_step / 1e3) / 1e9
        out = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": R["steps"],
               "warmup": args.warmup, "ms_per_step": per_step, "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "int32", "data": "synthetic",
               "config": {"workload": "sweep100b_decode_m1", "layers": 80,
                          "linears": [f"{K}->{N}" for K, N, _ in __import__("synth").LAYER100B],
                          "resident_packed_bytes": R["packed_bytes"], "setup_s": R["setup_s"],
                          "l2_policy": "inputs larger than L2 (17.1 GB resident, streamed once per step)"},
               "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                            "kernel": f"{decode_kernel_name(args, 1)} (80 grouped launches per step)",
                            "avg_launch_us": per_step / R["launches"] * 1e3},
               "gpu_launches": R["launches"] * R["steps"], "clocks": R["clocks"]}
    elif args.workload == "pack":
        pk = run_pack(torch, bl, args, dev, stream, dist, l2)
        out = {"metric": "absmean ternary quantise + 2-bit pack, GB/s", "value": pk["value"] * world,
               "unit": "GB/s", "n_gpus": world, "steps": pk["steps"], "warmup": 3,
               "ms_per_step": pk["ms_per_step"], "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "f64", "data": "synthetic",
               "config": {"workload": "pack_block2b", "note": pk["note"]},
               "roofline": {"bound": "hbm", "achieved": pk["value"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": pk["value"] / peaks["hbm_gbs"], "traffic": None},
               "gpu_launches": pk["launches_per_step"] * pk["steps"]}
    else:
        R = run_decode(torch, bl, args, lin, M, dev, stream, dist, l2)
        nbytes, ms = R["nbytes"], R["ms"]
        achieved = R["kern_bytes"] / (R["kern_ms"] / 1e3) / 1e9
        config.update({"weight_copies": R["S"]["copies"], "rotating_bytes": R["S"]["per_copy"] * R["S"]["copies"],
                       "l2_bytes": l2, "l2_policy": "inputs larger than L2: weights/x/y rotate over copies > 3x L2",
                       "mode": R["mode"]})
        out = {"metric": METRIC, "value": nbytes * args.steps * world / (ms / 1e3) / 1e9, "unit": "GB/s",
               "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
               "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int32",
               "data": "synthetic", "config": config,
               "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": achieved / peaks["hbm_gbs"],
                            "traffic": (MEASURED_TRAFFIC.get((args.workload, decode_kernel_name(args, M), M))
                                        if R["mode"] == "grouped" else None),
                            "kernel": R["kname"],
                            "peak_kind": f"{peaks['kind']} HBM copy bandwidth (burst)",
                            "algorithmic_bytes_per_launch": R["kern_bytes"],
                            "avg_launch_us": R["kern_ms"] * 1e3},
               "gpu_launches": R["launches"] * args.steps, "clocks": R["clocks"]}
        if not args.no_e2e and R["mode"] == "grouped":
            ems, n, hb, db = run_e2e(torch, bl, lin, M, dev, stream, R["S"], args.steps, dist)
            out["e2e"] = {"value": nbytes * n * world / (ems / 1e3) / 1e9, "unit": "GB/s",
                          "h2d_bytes_per_step": hb, "d2h_bytes_per_step": db, "ms_per_step": ems / n,
                          "path": "pinned host x -> H2D -> bitlinear_forward_x_grouped_ws (C ABI, prepared "
                                  "GroupedDecode call) -> D2H y"}
        if args.workload == "block2b" and not args.no_prefill:
            out["prefill"] = run_prefill(torch, bl, args, dev, stream, dist, l2, 20)
        if rank == 0 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(lin, args.cpu_seconds)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
