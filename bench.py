"""Benchmark of the grouped linear hot path on B200.

One step = the whole path over one batch of the ``bf16_g8`` workload (G=8
experts, K=4096, N=14336, 16384 rows split Multinomial(Dirichlet(1))), with
stacked [G,N,K] bf16 weights and the fp32 main_grad resident in HBM:
gl_offsets, bf16 gl_fwd / gl_dgrad / gl_wgrad (accumulate), then the MXFP8
half on the ``mxfp8_g8`` splits (multiples of 128): group_quantize_mxfp8 of
x, W and dy (rowwise + columnwise) and the three block-scaled GEMMs.
``value`` is whole-job TFLOP/s: the six GEMMs' 2*sum(m)*N*K flops each, over
all ranks, divided by the max-over-ranks device time of exactly ``--steps``
steps.  ``--workload`` runs the same step at another workload's sizes and
split sizes (its MXFP8 half on the same splits).

Per-op times are medians over at least 50 steps (the timed ones, then untimed
ones right after the timed region when ``--steps`` < 50), each op bracketed by
CUDA events on the launching stream.

Contract: ``python bench.py --gpus N --steps K --warmup W`` (torchrun for
N > 1, one rank per GPU, every rank an independent replica: weak scaling);
rank 0 prints one JSON line.  ``--impl reference`` times the CPU oracle (fp64
numpy) on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from grouped_gemm_splits_b200 import gl, synth  # noqa: E402

METRIC = "grouped-GEMM TFLOPS fwd/dgrad/wgrad and % of B200 dense BF16/MXFP8 peak"
WORKLOAD = "bf16_g8"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
OP_SAMPLES = 50  # per-op medians are taken over at least this many steps

# DRAM bytes (read + write) per launch of each kernel at a workload, from one
# ncu capture (dram__bytes_read.sum + dram__bytes_write.sum), with the digest
# of the CUDA sources the capture ran.  When the sources have changed since,
# the figures describe other kernels: the line then reports traffic as null.
MEASURED_TRAFFIC = {
    "csrc_digest": "f037632f4168708d",
    # the second step of `bench.py --steps 2 --warmup 3` under ncu (one pass,
    # gpu__time_duration / dram__bytes_read / dram__bytes_write per launch)
    "bf16_g8": {"fwd": 1825746432, "dgrad": 2820858368, "wgrad": 5747676928,
                "quant_x": 219182592, "quant_w": 1877729792, "quant_dy": 914067200,
                "fwd_mx": 1006835200, "dgrad_mx": 1405178880, "wgrad_mx": 3657736704},
    # `bench.py --workload stacked_g128_ragged --steps 1 --warmup 1` under ncu
    # (the timed step's kernels; the MXFP8 wgrad from the warm-up step)
    "stacked_g128_ragged": {"fwd": 5596950272, "dgrad": 4619833600, "wgrad": 15660184320,
                            "quant_x": 1890677760, "quant_w": 7898937856, "quant_dy": 493870336,
                            "fwd_mx": 2672948224, "dgrad_mx": 2815816448, "wgrad_mx": 14946737664},
}


def csrc_digest() -> str:
    """Digest of the library's CUDA sources (names and contents)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "grouped_gemm_splits_b200", "csrc")
    for f in sorted(glob.glob(os.path.join(d, "*.cu")) + glob.glob(os.path.join(d, "*.cuh"))
                    + glob.glob(os.path.join(d, "*.h"))):
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload: str, op: str):
    """(bytes, source note) for a kernel, or (None, why not)."""
    cap = MEASURED_TRAFFIC.get("csrc_digest")
    if cap is None:
        return None, "no ncu capture recorded for the current kernels"
    if cap != csrc_digest():
        return None, f"stale: the CUDA sources changed since the ncu capture ({cap})"
    v = MEASURED_TRAFFIC.get(workload, {}).get(op)
    if v is None:
        return None, f"no ncu capture of this kernel at {workload}"
    return v, f"ncu capture of sources {cap}"


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
class MxStep:
    """The MXFP8 half of the step: cast x, W, dy (rowwise + columnwise), then
    the three block-scaled GEMMs, on the MXFP8 workload (same shapes, splits
    in multiples of 128)."""

    NAMES = ["quant_x", "quant_w", "quant_dy", "fwd_mx", "dgrad_mx", "wgrad_mx"]

    def __init__(self, seed_offset: int, device, x=None, w=None, dy=None, main_grad=None,
                 workload: str = "mxfp8_g8"):
        wl = synth.WORKLOADS[workload]
        self.wl = wl
        self.m = synth.m_splits_for(workload)
        G, N, K, M = wl.G, wl.N, wl.K, wl.rows
        if x is None:
            d = synth.operands(G, M, N, K, wl.seed + seed_offset, device=device, bias=False)
            x, w, dy, main_grad = d["x"], d["w"], d["dy"], d["main_grad"]
        self.x, self.w, self.dy, self.main_grad = x, w, dy, main_grad
        self.m_dev = torch.tensor(self.m, device=device)
        self.offsets = torch.empty(G + 1, dtype=torch.int64, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        gl.gl_offsets(self.m_dev, M, M, self.offsets, self.status)
        self.y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
        self.dx = torch.empty(M, K, dtype=torch.bfloat16, device=device)
        self.qx, self.qw, self.qdy = {}, {}, {}
        self.flops = 2.0 * float(self.m.sum()) * N * K
        ne = int((self.m > 0).sum())
        code_b = lambda n: n + n // 32  # codes + scales per copy
        self.bytes = {
            "quant_x": M * K * 2 + 2 * code_b(M * K),
            "quant_w": G * N * K * 2 + 2 * code_b(G * N * K),
            "quant_dy": M * N * 2 + 2 * code_b(M * N),
            "fwd_mx": code_b(M * K) + code_b(ne * N * K) + M * N * 2,
            "dgrad_mx": code_b(M * N) + code_b(ne * N * K) + M * K * 2,
            "wgrad_mx": code_b(M * K) + code_b(M * N) + 2 * ne * N * K * 4,
        }
        self.launches = 7  # offsets, three casts, three GEMMs

    def run_offsets(self):
        gl.gl_offsets(self.m_dev, self.wl.rows, self.wl.rows, self.offsets, self.status)

    def run(self, ev=None, i0=0):
        """The casts and GEMMs (after ``run_offsets``); events ev[i0..i0+6]."""
        wl = self.wl
        G, N, K = wl.G, wl.N, wl.K
        if ev:
            ev[i0].record()
        gl.group_quantize_mxfp8(self.x, self.offsets, rowwise=True, colwise=True, status=self.status,
                                out=self.qx, mma_scales=True)
        if ev:
            ev[i0 + 1].record()
        gl.group_quantize_mxfp8(self.w, rowwise=True, colwise=True, out=self.qw, mma_scales=True)
        if ev:
            ev[i0 + 2].record()
        gl.group_quantize_mxfp8(self.dy, self.offsets, rowwise=True, colwise=True, status=self.status,
                                out=self.qdy, mma_scales=True)
        if ev:
            ev[i0 + 3].record()
        gl.gl_fwd_mxfp8(self.qx["codes_r"], self.qx["scales_r"], self.qw["codes_r"].view(G, N, K),
                        self.qw["scales_r"], None, self.offsets, self.status, self.y)
        if ev:
            ev[i0 + 4].record()
        gl.gl_dgrad_mxfp8(self.qdy["codes_r"], self.qdy["scales_r"], self.qw["codes_c"].view(G, N, K),
                          self.qw["scales_c"], self.offsets, self.status, self.dx)
        if ev:
            ev[i0 + 5].record()
        gl.gl_wgrad_mxfp8(self.qx["codes_c"], self.qx["scales_c"], self.qdy["codes_c"], self.qdy["scales_c"],
                          self.offsets, self.status, self.main_grad, accumulate=True)
        if ev:
            ev[i0 + 6].record()


class Step:
    """Device buffers and one pass of the whole hot path on the current stream:
    offsets, bf16 fwd / dgrad / wgrad(accumulate), then the MXFP8 half
    (cast of x, W, dy and the three block-scaled GEMMs)."""

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
        flops = 2.0 * float(self.m.sum()) * N * K  # per GEMM
        ne = int((self.m > 0).sum())
        xb, dyb = M * K * 2, M * N * 2
        wb, mgb = ne * N * K * 2, ne * N * K * 4
        # the MXFP8 half: the MXFP8 workload's splits on the bf16 workload's
        # tensors (same shapes), else this workload's own splits
        mx_workload = "mxfp8_g8" if workload == "bf16_g8" else workload
        self.mx = MxStep(seed_offset, device, self.x, self.w, self.dy, self.main_grad, workload=mx_workload)
        self.names = ["offsets", "fwd", "dgrad", "wgrad"] + MxStep.NAMES
        self.flops = {"fwd": flops, "dgrad": flops, "wgrad": flops,
                      "fwd_mx": self.mx.flops, "dgrad_mx": self.mx.flops, "wgrad_mx": self.mx.flops}
        Gm = self.mx.wl.G
        self.bytes = {"offsets": G * 8 + (G + 1) * 8 + 4 + Gm * 8 + (Gm + 1) * 8 + 4,
                      "fwd": xb + wb + dyb, "dgrad": dyb + wb + xb, "wgrad": xb + dyb + 2 * mgb}
        self.bytes.update(self.mx.bytes)
        self.dtype = {"fwd": "bf16", "dgrad": "bf16", "wgrad": "bf16",
                      "fwd_mx": "mxfp8", "dgrad_mx": "mxfp8", "wgrad_mx": "mxfp8"}
        self.launches = 4 + self.mx.launches  # offsets, fwd, dgrad, wgrad + the MXFP8 half
        self.total_flops = sum(self.flops.values())

    def run(self, ev=None):
        """One step; ``ev`` = list of len(names)+1 events recorded around the ops."""
        if ev:
            ev[0].record()
        gl.gl_offsets(self.m_dev, self.wl.rows, self.wl.out_rows, self.offsets, self.status)
        self.mx.run_offsets()  # the MXFP8 half's split sizes
        if ev:
            ev[1].record()
        gl.gl_fwd(self.x, self.w, self.bias, self.offsets, self.status, self.y)
        if ev:
            ev[2].record()
        gl.gl_dgrad(self.dy, self.w, self.offsets, self.status, self.dx)
        if ev:
            ev[3].record()
        gl.gl_wgrad(self.x, self.dy, self.offsets, self.status, self.main_grad, accumulate=True)
        self.mx.run(ev, 4)


def e2e_measure(steps_ab, steps: int, warmup: int):
    """Same step through the public API with every step's inputs (x, dy, split
    sizes) copied from pinned host memory and its status word read back.

    Two device buffer sets (``steps_ab``) alternate: while step i computes on
    one, a copy stream fills the other with step i+1's inputs; events order
    each buffer's reuse.  Every copy and readback stays inside the timed
    region."""
    A = steps_ab[0]
    hx = A.x.cpu().pin_memory()
    hdy = A.dy.cpu().pin_memory()
    hm = torch.tensor(A.m).pin_memory()
    hm2 = torch.tensor(A.mx.m).pin_memory()
    hst = [torch.empty(1, dtype=torch.int32).pin_memory() for _ in range(2)]
    h2d = hx.numel() * 2 + hdy.numel() * 2 + hm.numel() * 8 + hm2.numel() * 8
    d2h = 4
    comp = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    copied = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]

    def one(i):
        b = i % 2
        S = steps_ab[b]
        with torch.cuda.stream(copy):
            copy.wait_event(done[b])  # the buffer's previous step has finished with it
            S.x.copy_(hx, non_blocking=True)
            S.dy.copy_(hdy, non_blocking=True)
            S.m_dev.copy_(hm, non_blocking=True)
            S.mx.m_dev.copy_(hm2, non_blocking=True)
            copied[b].record(copy)
        comp.wait_event(copied[b])
        S.run()
        hst[b].copy_(S.status, non_blocking=True)
        done[b].record(comp)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    copy.wait_event(t0)  # no copy of the timed steps starts before t0
    for i in range(steps):
        one(i)
    t1.record(comp)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    return ms, h2d, d2h, int(hst[0].item()) | int(hst[1].item())


# ----------------------------------------------------------------------------
# CPU oracle on a bounded sample
# ----------------------------------------------------------------------------
def oracle_sample(workload: str = WORKLOAD, seed_offset: int = 0, rows_per_group: int = 64, groups=(0, 1)):
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
    # the MXFP8 half: quantize (rowwise + columnwise), then the three products
    Gs = len(gsel)
    xq, xs = orc.quantize_rowwise(x)
    xcq, xcs = orc.quantize_colwise(x, m)
    dyq, dys = orc.quantize_rowwise(dy)
    dycq, dycs = orc.quantize_colwise(dy, m)
    wq, ws = orc.quantize_rowwise(w.reshape(Gs * N, K))
    wcq, wcs = orc.quantize_colwise(w.reshape(Gs * N, K), [N] * Gs)
    orc.fwd_mxfp8(xq, xs, wq.reshape(Gs, N, K), ws.reshape(Gs, N, K // 32), None, m)
    orc.dgrad_mxfp8(dyq, dys, wcq.reshape(Gs, N, K), wcs, m)
    orc.wgrad_mxfp8(xcq, xcs, dycq, dycs, m, mg, True)
    sec = time.perf_counter() - t0
    flops = 6 * 2.0 * M * N * K
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    desc = (f"{len(gsel)} groups x {rows_per_group} rows of the {workload} workload "
            f"(K={K}, N={N}); bf16 fwd+dgrad+wgrad and MXFP8 quantize+fwd+dgrad+wgrad in fp64 numpy, "
            "including bf16->fp64 conversion")
    return flops, sec, threads, desc


# ----------------------------------------------------------------------------
def rank_env():
    """(world size, rank, local rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def dist_setup(world: int, local: int) -> None:
    """One process per GPU: a NCCL process group (short timeout) when N > 1.
    The path has no exchange step, so the group only carries the barrier and
    the max-over-ranks reduction of the timed region."""
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))


def max_over_ranks(ms: float, device) -> float:
    """The job's time for a timed region: the slowest rank's (an all-reduce
    MAX over the process group); the value itself on a single process."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank_step: float, world: int, ms_step: float) -> float:
    """Whole-job throughput: every replica's flops over the slowest rank's time."""
    return flops_per_rank_step * world / (ms_step / 1e3) / 1e12


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD, choices=[w for w in synth.WORKLOADS if w != "mxfp8_g8"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()

    world, rank, local = rank_env()
    wl = synth.WORKLOADS[args.workload]
    config = {"workload": f"{args.workload}: G={wl.G} K={wl.K} N={wl.N} rows={wl.rows}"
                          f"{' (output buffers ' + str(wl.out_rows) + ' rows)' if wl.out_rows > wl.rows else ''}, "
                          f"split sizes as in the workload table, stacked bf16 weights{', bias' if wl.bias else ''}; "
                          "one step = offsets + bf16 fwd/dgrad/wgrad(accumulate into fp32 main_grad), then "
                          "MXFP8 cast of x, W, dy (rowwise + columnwise) and MXFP8 fwd/dgrad/wgrad"
                          + (" on the mxfp8_g8 splits (G=8, rows in multiples of 128)" if args.workload == "bf16_g8"
                             else " on the same splits"),
              "l2": "no flush: every step streams > 3 GB of operands (W 0.9 GiB, dy 0.45 GiB, "
                    "main_grad 1.75 GiB), far larger than the 126 MB L2",
              "parallelism": f"replicas x{world}"}

    if args.impl == "reference":
        if rank != 0:
            return
        steps = max(1, min(args.steps, 2))
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

    dist_setup(world, local)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    gl.load()
    step = Step(args.workload, seed_offset=rank, device=dev)
    pk = peaks()

    nev = len(step.names) + 1
    # per-op samples: the timed steps, plus untimed steps right after them
    # until there are at least OP_SAMPLES (per-op medians)
    n_samples = max(args.steps, OP_SAMPLES)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(n_samples)]
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
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), dev)
    ms_step = ms_total / args.steps
    for i in range(args.steps, n_samples):  # outside the timed region
        step.run(evs[i])
    torch.cuda.synchronize()
    status = int(step.status.item()) | int(step.mx.status.item())

    samples = {n: [evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(n_samples)]
               for j, n in enumerate(step.names)}
    op_ms = {n: statistics.median(v) for n, v in samples.items()}
    timed_s = ms_total / 1e3
    sustained = timed_s > 1.0
    peak_bf16 = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
    peak_kind = "sustained" if sustained else "burst"
    # MXFP8 tensor peak: the measured bf16 peak x 2 (dense fp8 / bf16 nominal ratio 4.5 / 2.25)
    peak_of = {"bf16": peak_bf16, "mxfp8": 2.0 * peak_bf16}
    ops = {}
    for n in step.names:
        sec = op_ms[n] / 1e3
        by = step.bytes[n]
        fl = step.flops.get(n, 0.0)
        e = {"ms": op_ms[n], "ms_mean": statistics.mean(samples[n]), "samples": n_samples,
             "gbs": by / sec / 1e9, "algorithmic_bytes": by}
        tr, tr_src = measured_traffic(args.workload, n)
        e["dram_traffic_bytes"] = tr
        if tr:
            e["traffic_over_algorithmic"] = tr / by
        if fl:
            pkt = peak_of[step.dtype[n]]
            t_flops, t_bytes = fl / (pkt * 1e12), by / (pk["hbm_gbs"] * 1e9)
            e.update({"tflops": fl / sec / 1e12, "dtype": step.dtype[n], "peak_tflops": pkt,
                      "bound": "tensor" if t_flops >= t_bytes else "hbm",
                      "frac_of_roofline": max(t_flops, t_bytes) / sec, "frac_of_tensor_peak": fl / sec / 1e12 / pkt})
        else:
            e.update({"bound": "hbm", "frac_of_hbm": by / sec / 1e9 / pk["hbm_gbs"]})
        ops[n] = e
    dom = max(step.names, key=lambda n: op_ms[n])
    tr, tr_src = measured_traffic(args.workload, dom)
    if ops[dom]["bound"] == "tensor":
        roof = {"bound": "tensor", "kernel": dom, "achieved": ops[dom]["tflops"],
                "peak": peak_of[step.dtype[dom]], "unit": "TFLOP/s",
                "frac": ops[dom]["tflops"] / peak_of[step.dtype[dom]],
                "peak_source": f"{pk['source']} bf16 ({peak_kind})" + (" x2 for fp8" if step.dtype[dom] == "mxfp8" else "")}
    else:
        roof = {"bound": "hbm", "kernel": dom, "achieved": ops[dom]["gbs"], "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": ops[dom]["gbs"] / pk["hbm_gbs"],
                "peak_source": f"{pk['source']} copy bandwidth"}
    roof.update({"traffic": tr, "traffic_source": tr_src, "algorithmic_bytes": step.bytes[dom],
                 "ms": op_ms[dom], "samples": n_samples})
    value = job_tflops(step.total_flops, world, ms_step)

    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16+mxfp8", "data": "synthetic",
            "config": config, "status_word": status, "roofline": roof,
            "ops": ops, "gpu_launches": step.launches * args.steps, "clocks": clocks}

    # Outside the step: the bias gradient (the column sums of each group's
    # rows of dy), an HBM-bound pass over dy measured on its own.
    db = torch.empty(step.wl.G, step.wl.N, dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        gl.gl_dbias(step.dy, step.offsets, step.status, db)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(20):
        gl.gl_dbias(step.dy, step.offsets, step.status, db)
    e1.record()
    torch.cuda.synchronize()
    db_ms = e0.elapsed_time(e1) / 20
    db_bytes = step.dy.numel() * 2 + db.numel() * 2 + (step.wl.G + 1) * 8
    line["extras"] = {"dbias": {"ms": db_ms, "gbs": db_bytes / (db_ms / 1e3) / 1e9,
                                "frac_of_hbm": db_bytes / (db_ms / 1e3) / 1e9 / pk["hbm_gbs"],
                                "bytes": db_bytes, "note": "not part of the step"}}

    # Also outside the step: the cast of dy fused with its bias gradient (one
    # pass over dy; group_quantize_mxfp8_dbias) on the MXFP8 half's splits,
    # against that half's cast of dy plus gl_dbias on the same splits.
    mx = step.mx

    def timed(f, n=20):
        for _ in range(3):
            f()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        for _ in range(n):
            f()
        a1.record()
        torch.cuda.synchronize()
        return a0.elapsed_time(a1) / n

    ws = torch.empty(gl.dbias_workspace_bytes(mx.wl.rows, mx.wl.N, mx.wl.G), dtype=torch.uint8, device=dev)
    qd, dbm = {}, torch.empty(mx.wl.G, mx.wl.N, dtype=torch.bfloat16, device=dev)
    fused_ms = timed(lambda: gl.group_quantize_mxfp8_dbias(mx.dy, mx.offsets, mx.status, out=qd, mma_scales=True,
                                                           dbias=dbm, workspace=ws))
    sep_db_ms = timed(lambda: gl.gl_dbias(mx.dy, mx.offsets, mx.status, dbm))
    cd_bytes = mx.bytes["quant_dy"] + dbm.numel() * 2
    line["extras"]["cast_dbias"] = {
        "ms": fused_ms, "gbs": cd_bytes / (fused_ms / 1e3) / 1e9,
        "frac_of_hbm": cd_bytes / (fused_ms / 1e3) / 1e9 / pk["hbm_gbs"], "bytes": cd_bytes,
        "separate_ms": ops["quant_dy"]["ms"] + sep_db_ms,
        "note": "MXFP8 cast of dy (rowwise + columnwise) with its bias gradient in one pass; separate_ms = the "
                "step's cast of dy + gl_dbias on the same splits; not part of the step"}

    # The whole step captured once as a CUDA graph and replayed (every entry
    # point is asynchronous, allocates nothing and never syncs the host), its
    # device time beside the eager step's.
    try:
        g_stream = torch.cuda.Stream()
        graph = torch.cuda.CUDAGraph()
        torch.cuda.synchronize()
        with torch.cuda.stream(g_stream):
            with torch.cuda.graph(graph, stream=g_stream):
                step.run()
        graph_ms = timed(graph.replay)
        eager_ms = timed(step.run)  # the same 20-step burst, eager, right after
        line["extras"]["graph_step"] = {"ms": graph_ms, "eager_ms": eager_ms,
                                        "note": "one captured step replayed 20 times against 20 eager steps "
                                                "right after (short bursts: clocks differ from the timed "
                                                "region's); not the headline"}
        del graph
    except RuntimeError as exc:  # report, keep the line
        line["extras"]["graph_step"] = {"unavailable": str(exc).splitlines()[0][:200]}

    # end to end on every rank (host buffers in, status out), slowest rank's time
    if world > 1:
        torch.distributed.barrier()
    step_b = Step(args.workload, seed_offset=rank + 1000, device=dev)  # second buffer set
    ms_e2e, h2d, d2h, st2 = e2e_measure((step, step_b), max(20, args.steps), 3)
    del step_b
    ms_e2e = max_over_ranks(ms_e2e, dev)
    line["e2e"] = {"value": job_tflops(step.total_flops, world, ms_e2e), "unit": "TFLOP/s",
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
                   "status_word": st2, "copies": "next step's inputs copied on a second stream while "
                                                 "the current step computes (two device buffer sets)"}
    if rank == 0:
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
