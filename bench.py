#!/usr/bin/env python3
"""Benchmark of the BitNet b1.58 BitLinear hot path on B200.

Default workload (N=1 line): decode, M = 1 token, through the seven linears
of a 2B-class block (2560->6912 x2, 6912->2560, 2560->2560 x2, 2560->640
x2), x bf16 ~ N(0,1) with 1% outliers x20, fp32 y.  One step = one pass of
the per-token hot path over the block: per-token absmax int8 quantisation,
ternary x int8 product with int32 accumulation and the rescale, for all
seven linears (the weights are packed once, before timing, as a model's
weights are).  Metric: algorithmic bytes (packed weights N*K/4 + bf16 x +
fp32 y) per second.

The packed weights of the block are replicated into enough copies that the
rotating working set exceeds 3x the L2 size, so every step streams its
weights from HBM.  Steps are replayed from CUDA graphs and timed with CUDA
events on the launching stream; multi-GPU runs are independent replicas
(no collective on the data path) timed as the max over ranks.

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


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--mode", choices=["grouped", "fused", "separate"], default="grouped",
                    help="grouped: one launch per step; fused: one launch per linear; "
                         "separate: quantise + product launches per linear")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="oracle CPU-baseline budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


# ----------------------------------------------------------------- utils
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


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


def block_bytes(lin, M):
    """Algorithmic bytes of one pass over the block: packed W + bf16 x + fp32 y."""
    return sum(L["N"] * L["K"] // 4 + M * L["K"] * 2 + M * L["N"] * 4 for L in lin)


# ----------------------------------------------------- CPU (oracle) arm
def oracle_block_setup(lin):
    import oracle
    prepared = []
    for L in lin:
        g64 = oracle.absmean_gamma(L["W"])
        code, _, _ = oracle.ternary_codes(L["W"], g64, 1e-5)
        prepared.append(dict(x=L["x"], code=code, g32=float(__import__("numpy").float32(g64)), N=L["N"], K=L["K"]))
    return prepared


def oracle_block_pass(prepared, threads, row_frac=1.0):
    """One oracle pass over the block (quantise, multiply, rescale); with
    row_frac < 1 only the first row_frac of each weight's rows."""
    import oracle
    nbytes = 0
    for P in prepared:
        n = max(1, int(P["N"] * row_frac))
        oracle.forward_bf16_mt(P["x"], P["code"][:n], P["g32"], threads)
        nbytes += n * P["K"] // 4 + P["x"].size * 2 + P["x"].shape[0] * n * 4
    return nbytes


def cpu_baseline(lin, seconds):
    prepared = oracle_block_setup(lin)
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    total, passes = 0, 0
    while True:
        total += oracle_block_pass(prepared, threads)
        passes += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": total / el / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{passes} full oracle passes over the 7-linear block at M=1 "
                      f"({el:.1f} s, {threads} threads, rows split across threads)"}


def run_reference(args, lin, M, config):
    """The oracle as the reference arm: rank 0 only."""
    import numpy as np  # noqa: F401
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    prepared = oracle_block_setup(lin)
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    oracle_block_pass(prepared, threads)
    t_full = time.perf_counter() - t0
    budget = 120.0
    frac = min(1.0, budget / max(1e-9, t_full * (args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_block_pass(prepared, threads, frac)
    t0 = time.perf_counter()
    nbytes = 0
    for _ in range(args.steps):
        nbytes += oracle_block_pass(prepared, threads, frac)
    el = time.perf_counter() - t0
    value = nbytes / el / 1e9
    sample = (f"each step: oracle pass over {frac * 100:.3g}% of every linear's output rows "
              f"(quantise + multiply + rescale), {threads} threads")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
            "data": "synthetic", "config": config,
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# --------------------------------------------------------------- GPU arm
def main():
    args = parse_args()
    import numpy as np
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    M = 1
    lin = synth.block2b_inputs(seed_base=0, M=M)
    config = {"workload": "block2b_decode_m1", "M": M,
              "linears": [f"{L['name']}:{L['K']}->{L['N']}" for L in lin],
              "x": "bf16 N(0,1), 1% outliers x20", "y": "fp32", "weights": "N(0,0.02) fp32, packed 2-bit",
              "parallelism": "replicas" if world > 1 else "single"}

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
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)

    # ---- pack the block's weights once, then replicate to > 3x L2
    packed0, g32s = [], []
    for L in lin:
        p, _, g = bl.pack(torch.from_numpy(L["W"]).to(dev))
        packed0.append(p)
        g32s.append(g)
    torch.cuda.synchronize()
    if bl.bitlinear_get_status() != bl.BL_OK:
        raise RuntimeError("non-finite weights")
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    wbytes = sum(p.numel() for p in packed0)
    copies = max(2, math.ceil(3 * l2 / wbytes))
    packed = [[p.clone() for p in packed0] for _ in range(copies)]
    xs = [[torch.from_numpy(L["x"].view(np.int16)).to(dev).view(torch.bfloat16) for L in lin] for _ in range(copies)]
    ys = [[torch.empty((M, L["N"]), dtype=torch.float32, device=dev) for L in lin] for _ in range(copies)]
    Ns = [L["N"] for L in lin]
    Ks = [L["K"] for L in lin]
    qs = [torch.empty((M, bl.bitlinear_padded_k(K)), dtype=torch.int8, device=dev) for K in Ks]
    ss = [torch.empty(M, dtype=torch.float32, device=dev) for _ in Ks]
    config.update({"weight_copies": copies, "rotating_weight_bytes": wbytes * copies,
                   "l2_bytes": l2, "l2_policy": "inputs larger than L2: weights rotate over copies > 3x L2",
                   "mode": args.mode})

    def step(i):
        c = i % copies
        if args.mode == "grouped":
            bl.bitlinear_forward_x_grouped(xs[c], packed[c], g32s, Ns, Ks, ys[c], stream)
            return 1
        if args.mode == "fused":
            for j in range(len(lin)):
                bl.bitlinear_forward_x(xs[c][j], packed[c][j], g32s[j], Ns[j], Ks[j], ys[c][j], stream)
            return len(lin)
        for j in range(len(lin)):
            bl.bitlinear_quant_act(xs[c][j], qs[j], ss[j], stream)
            bl.bitlinear_forward(qs[j], ss[j], packed[c][j], g32s[j], M, Ns[j], Ks[j], ys[c][j], None, stream)
        return 2 * len(lin)

    launches_per_step = step(0)
    torch.cuda.synchronize()

    # ---- CUDA graphs: one of `copies` steps, and single steps for the tail
    with torch.cuda.stream(stream):
        g_all = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_all, stream=stream):
            for i in range(copies):
                step(i)
        g_one = []
        for i in range(copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step(i)
            g_one.append(g)
    torch.cuda.synchronize()

    def run_steps(n):
        full, rem = divmod(n, copies)
        for _ in range(full):
            g_all.replay()
        for i in range(rem):
            g_one[i].replay()

    run_steps(max(3, args.warmup))
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    sampler = ClockSampler(local)
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0.record(stream)
    run_steps(args.steps)
    e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1)
    if dist:
        t = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    if bl.bitlinear_get_status() != bl.BL_OK:
        raise RuntimeError("device status word set during the timed region")

    nbytes = block_bytes(lin, M)
    value = nbytes * args.steps * world / (ms / 1e3) / 1e9
    ms_step = ms / args.steps

    # ---- dominant kernel: the product kernel (the whole step in grouped mode)
    peak, peak_kind = load_peaks()
    if args.mode == "grouped":
        kern_ms, kern_bytes = ms_step, nbytes
    else:
        # time the product launches alone (no quantisation) over the same rotation
        with torch.cuda.stream(stream):
            gk = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gk, stream=stream):
                for i in range(copies):
                    for j in range(len(lin)):
                        if args.mode == "fused":
                            bl.bitlinear_forward_x(xs[i][j], packed[i][j], g32s[j], Ns[j], Ks[j], ys[i][j], stream)
                        else:
                            bl.bitlinear_forward(qs[j], ss[j], packed[i][j], g32s[j], M, Ns[j], Ks[j], ys[i][j],
                                                 None, stream)
        reps = max(1, args.steps // copies)
        gk.replay()
        e0.record(stream)
        for _ in range(reps):
            gk.replay()
        e1.record(stream)
        e1.synchronize()
        kern_ms = e0.elapsed_time(e1) / (reps * copies * len(lin))
        kern_bytes = nbytes / len(lin)
    achieved = kern_bytes / (kern_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": None,
                "kernel": "gemv_kernel (fused quant prologue, grouped over the 7 linears)"
                if args.mode == "grouped" else "gemv_kernel",
                "peak_kind": f"{peak_kind} HBM copy bandwidth (burst)",
                "algorithmic_bytes_per_launch": kern_bytes, "avg_launch_us": kern_ms * 1e3}

    # ---- end to end through the public API: pinned host x in, host y out
    e2e = None
    if not args.no_e2e:
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
        e2e_steps = max(1, min(args.steps, 2000))

        def e2e_step(i):
            c = i % copies
            dx.copy_(hx, non_blocking=True)
            bl.bitlinear_forward_x_grouped(xv, packed[c], g32s, Ns, Ks, yv, stream)
            hy.copy_(dy, non_blocking=True)

        for i in range(3):
            e2e_step(i)
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(e2e_steps):
            e2e_step(i)
        e1.record(stream)
        e1.synchronize()
        ems = e0.elapsed_time(e1)
        if dist:
            t = torch.tensor([ems], device=dev, dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ems = float(t.item())
        e2e = {"value": nbytes * e2e_steps * world / (ems / 1e3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": hx.numel() * hx.element_size(),
               "d2h_bytes_per_step": hy.numel() * hy.element_size(),
               "ms_per_step": ems / e2e_steps,
               "path": "pinned host x -> H2D -> bitlinear_forward_x_grouped (C ABI) -> D2H y, per step"}

    out = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "int32", "data": "synthetic", "config": config,
           "roofline": roofline, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
           "clocks": clocks}
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(lin, args.cpu_seconds)
    if dist:
        dist.barrier()
        del g_all, g_one
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
