"""Benchmark of the grouped linear hot path on B200.

One step = gl_offsets + gl_fwd + gl_dgrad + gl_wgrad (accumulate into fp32
main_grad) over one batch of the ``bf16_g8`` workload (G=8 experts, K=4096,
N=14336, 16384 rows split Multinomial(Dirichlet(1))), stacked [G,N,K] bf16
weights resident in HBM.  ``value`` is whole-job TFLOP/s (the three GEMMs'
2*sum(m)*N*K flops each, over all ranks, divided by the max-over-ranks device
time of exactly ``--steps`` steps).

Contract: ``python bench.py --gpus N --steps K --warmup W`` (torchrun for
N > 1, one rank per GPU, every rank an independent replica: weak scaling);
rank 0 prints one JSON line.  ``--impl reference`` times the CPU oracle (fp64
numpy) on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from grouped_gemm_splits_b200 import gl, synth  # noqa: E402

METRIC = "grouped-GEMM TFLOPS fwd/dgrad/wgrad and % of B200 dense BF16/MXFP8 peak"
WORKLOAD = "bf16_g8"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


# ----------------------------------------------------------------------------
# clocks sampled during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# GPU step
# ----------------------------------------------------------------------------
class Step:
    """Device buffers and one pass of the hot path on the current stream."""

    def __init__(self, workload: str, seed_offset: int, device):
        wl = synth.WORKLOADS[workload]
        self.wl = wl
        self.m = synth.m_splits_for(workload)
        G, N, K, M = wl.G, wl.N, wl.K, wl.rows
        d = synth.operands(G, M, N, K, wl.seed + seed_offset, device=device, bias=wl.bias)
        self.x, self.w, self.dy, self.main_grad = d["x"], d["w"], d["dy"], d["main_grad"]
        self.bias = d.get("bias")
        self.m_dev = torch.tensor(self.m, device=device)
        self.offsets = torch.empty(G + 1, dtype=torch.int64, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.y = torch.empty(wl.out_rows, N, dtype=torch.bfloat16, device=device)
        self.dx = torch.empty(wl.out_rows, K, dtype=torch.bfloat16, device=device)
        self.flops = 2.0 * float(self.m.sum()) * N * K  # per GEMM
        # algorithmic bytes per launch (weights / main_grad of non-empty groups)
        ne = int((self.m > 0).sum())
        xb, dyb = M * K * 2, M * N * 2
        wb, mgb = ne * N * K * 2, ne * N * K * 4
        self.bytes = {"offsets": G * 8 + (G + 1) * 8 + 4,
                      "fwd": xb + wb + dyb, "dgrad": dyb + wb + xb, "wgrad": xb + dyb + 2 * mgb}
        self.launches = 4

    def run(self, ev=None):
        """One step; ``ev`` = list of 5 events recorded around the four ops."""
        if ev:
            ev[0].record()
        gl.gl_offsets(self.m_dev, self.wl.rows, self.wl.out_rows, self.offsets, self.status)
        if ev:
            ev[1].record()
        gl.gl_fwd(self.x, self.w, self.bias, self.offsets, self.status, self.y)
        if ev:
            ev[2].record()
        gl.gl_dgrad(self.dy, self.w, self.offsets, self.status, self.dx)
        if ev:
            ev[3].record()
        gl.gl_wgrad(self.x, self.dy, self.offsets, self.status, self.main_grad, accumulate=True)
        if ev:
            ev[4].record()


def e2e_measure(step: Step, steps: int, warmup: int):
    """Same step through the public API with the step's inputs (x, dy, split
    sizes) copied from pinned host memory and the status word read back."""
    hx = step.x.cpu().pin_memory()
    hdy = step.dy.cpu().pin_memory()
    hm = torch.tensor(step.m).pin_memory()
    hst = torch.empty(1, dtype=torch.int32).pin_memory()
    h2d = hx.numel() * 2 + hdy.numel() * 2 + hm.numel() * 8
    d2h = 4

    def one():
        step.x.copy_(hx, non_blocking=True)
        step.dy.copy_(hdy, non_blocking=True)
        step.m_dev.copy_(hm, non_blocking=True)
        step.run()
        hst.copy_(step.status, non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        one()
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    return ms, h2d, d2h, int(hst.item())


# ----------------------------------------------------------------------------
# CPU oracle on a bounded sample
# ----------------------------------------------------------------------------
def oracle_sample(workload: str = WORKLOAD, seed_offset: int = 0, rows_per_group: int = 96, groups=(0, 1)):
    """fwd + dgrad + wgrad of the oracle on ``rows_per_group`` rows of two
    groups of the workload.  Returns (flops, seconds, threads, description)."""
    from oracle import gl_oracle as orc
    from threadpoolctl import threadpool_info

    wl = synth.WORKLOADS[workload]
    G, N, K = wl.G, wl.N, wl.K
    gsel = [g for g in groups if g < G]
    M = rows_per_group * len(gsel)
    d = synth.operands(len(gsel), M, N, K, wl.seed + seed_offset, device="cpu", bias=False)
    m = [rows_per_group] * len(gsel)
    f = lambda t: orc.bf16_to_f64(synth.bf16_bits(t)) if t.dtype == torch.bfloat16 else t.double().numpy()
    t0 = time.perf_counter()
    x, w, dy, mg = f(d["x"]), f(d["w"]), f(d["dy"]), f(d["main_grad"])
    orc.fwd(x, w, None, m)
    orc.dgrad(dy, w, m)
    orc.wgrad(x, dy, m, mg, True)
    sec = time.perf_counter() - t0
    flops = 3 * 2.0 * M * N * K
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    desc = (f"{len(gsel)} groups x {rows_per_group} rows of the {workload} workload "
            f"(K={K}, N={N}); fwd+dgrad+wgrad in fp64 numpy, including bf16->fp64 conversion")
    return flops, sec, threads, desc


# ----------------------------------------------------------------------------
def dist_setup(gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD, choices=[w for w in synth.WORKLOADS if w != "mxfp8_g8"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()

    world, rank, local = dist_setup(args.gpus)
    wl = synth.WORKLOADS[args.workload]
    config = {"workload": f"{args.workload}: G={wl.G} K={wl.K} N={wl.N} rows={wl.rows}"
                          f"{' (output buffers ' + str(wl.out_rows) + ' rows)' if wl.out_rows > wl.rows else ''}, "
                          f"split sizes as in the workload table, stacked bf16 weights{', bias' if wl.bias else ''}, "
                          "fwd + dgrad + wgrad(accumulate into fp32 main_grad)",
              "l2": "no flush: every step streams > 3 GB of operands (W 0.9 GiB, dy 0.45 GiB, "
                    "main_grad 1.75 GiB), far larger than the 126 MB L2",
              "parallelism": f"replicas x{world}"}

    if args.impl == "reference":
        if rank != 0:
            return
        steps = max(1, min(args.steps, 3))
        samples = []
        for i in range(max(0, min(args.warmup, 1)) + steps):
            fl, sec, thr, desc = oracle_sample(args.workload)
            if i >= min(args.warmup, 1):
                samples.append((fl, sec))
        fl = sum(s[0] for s in samples)
        sec = sum(s[1] for s in samples)
        v = fl / sec / 1e12
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
                "steps": steps, "warmup": min(args.warmup, 1), "ms_per_step": 1e3 * sec / steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config,
                "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": thr, "kind": "oracle", "sample": desc},
                "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    gl.load()
    step = Step(args.workload, seed_offset=rank, device=dev)
    pk = peaks()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    sampler.start()  # sample clocks through warm-up and the timed region
    for _ in range(max(args.warmup, 3)):
        step.run()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for i in range(args.steps):
        step.run(evs[i])
    t_end.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    ms_total = t_start.elapsed_time(t_end)
    if world > 1:
        t = torch.tensor([ms_total], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms_total = float(t.item())
    ms_step = ms_total / args.steps
    status = int(step.status.item())

    names = ["offsets", "fwd", "dgrad", "wgrad"]
    op_ms = {n: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps))
             for j, n in enumerate(names)}
    timed_s = ms_total / 1e3
    peak_tf = pk["bf16_tflops_sustained"] if timed_s > 1.0 else pk["bf16_tflops"]
    peak_kind = "sustained" if timed_s > 1.0 else "burst"
    ops = {}
    for n in names:
        s = op_ms[n] / 1e3
        if n == "offsets":
            ops[n] = {"ms": op_ms[n], "gbs": step.bytes[n] / s / 1e9}
            continue
        tflops = step.flops / s / 1e12
        t_roof = max(step.flops / (peak_tf * 1e12), step.bytes[n] / (pk["hbm_gbs"] * 1e9))
        ops[n] = {"ms": op_ms[n], "tflops": tflops, "gbs": step.bytes[n] / s / 1e9,
                  "frac_of_roofline": t_roof / s, "frac_of_bf16_peak": tflops / peak_tf}
    dom = max(["fwd", "dgrad", "wgrad"], key=lambda n: op_ms[n])
    dom_tf = ops[dom]["tflops"]
    value = 3 * step.flops * world / (ms_step / 1e3) / 1e12

    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config, "status_word": status,
            "roofline": {"bound": "tensor", "kernel": f"grouped_gemm_kernel ({dom})", "achieved": dom_tf,
                         "peak": peak_tf, "unit": "TFLOP/s", "frac": dom_tf / peak_tf,
                         "peak_source": f"{pk['source']} bf16 ({peak_kind})", "traffic": None},
            "ops": ops, "gpu_launches": step.launches * args.steps, "clocks": clocks}

    if rank == 0:
        ms_e2e, h2d, d2h, st2 = e2e_measure(step, max(3, args.steps // 2), 2)
        line["e2e"] = {"value": 3 * step.flops * world / (ms_e2e / 1e3) / 1e12, "unit": "TFLOP/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e}
        if world == 1 and not args.no_cpu_baseline:
            fl, sec, thr, desc = oracle_sample(args.workload)
            line["cpu_baseline"] = {"value": fl / sec / 1e12, "unit": "TFLOP/s", "cores": thr,
                                    "kind": "oracle", "sample": desc, "seconds": sec}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
