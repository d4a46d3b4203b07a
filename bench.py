#!/usr/bin/env python
"""Throughput of the SRFT-int4 KV codec on B200: quantize + dequantize GB/s.

One *step* is one pass of the whole hot path over one batch of synthetic
input: lambda calibration (first n_cal rows of every slice), fused
rotate-and-quantize of the whole cache, and fused dequantize-and-unrotate of
the whole cache. The default workload is the Qwen2.5-1.5B-shaped cache
(28 layers x {K,V}, 2 KV heads, d=128, 32768 tokens; int4, group 16).

value       algorithmic bytes of quantize + dequantize per step (fp16 in +
            codes + fp16 scales, for each) / device time per step, summed
            over ranks (weak scaling: every rank runs its own full cache).
e2e         the same metric through the C ABI with the input in pinned host
            memory copied to the device and the dequantized cache copied
            back inside every timed step.
roofline    the dominant kernel's algorithmic bytes per launch / its average
            CUDA-event duration, against the measured HBM copy bandwidth.
cpu_baseline  the float64 CPU oracle, as it stands, on a bounded sample.

`--impl reference` times that oracle as the reference arm instead.
"""

from __future__ import annotations

import argparse
import hashlib
import glob
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import kv_synth  # noqa: E402

METRIC = "SRFT-int4 KV quantize+dequantize GB/s vs B200 HBM peak; vectors/sec"
FALLBACK_HBM_GBS = 6650.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen_like_d128",
                    choices=[k for k, w in kv_synth.WORKLOADS.items() if w.d <= 128 and w.S * w.N * w.H < 2**28])
    ap.add_argument("--rotation", type=int, default=0, choices=[0, 1])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample", type=int, default=8192,
                    help="vectors per oracle step for the CPU baseline / reference arm")
    return ap.parse_args(argv)


def read_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def csrc_hash():
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(ROOT, "rotate_then_quantize_b200", "csrc", "*"))):
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def read_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken
    on the current kernel sources; null otherwise."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(p) as f:
            data = json.load(f)
    except Exception:
        return None
    ent = data.get(f"{kernel}:{workload}")
    if not ent or ent.get("csrc_sha") != csrc_hash():
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [r.split(",") for r in self.out.read().strip().splitlines() if r.count(",") >= 8]
        os.unlink(self.out.name)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        loaded = [r for r in rows if _num(r[4]) is not None and _num(r[4]) >= 50] or rows
        sm = [_num(r[1]) for r in loaded if _num(r[1]) is not None]
        mx = [_num(r[2]) for r in loaded if _num(r[2]) is not None]
        reasons = sorted({names[i] for r in loaded for i in range(4) if "Active" == r[5 + i].strip()})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(loaded),
                "power_w_max": max((_num(r[3]) or 0.0) for r in loaded) if loaded else None}


def _num(s):
    try:
        return float(s)
    except Exception:
        return None


# ---------------------------------------------------------------------------
# CPU oracle leg
# ---------------------------------------------------------------------------

def oracle_step(w, x16, signs, rot):
    """One oracle pass on a sample: calibrate, quantize, dequantize."""
    import oracle

    lam = oracle.calibrate_lambda(x16, signs, min(w.n_cal, x16.shape[1]), rot).astype(np.float32)
    q = oracle.quantize(x16, signs, lam, w.group, w.bits, rot)
    oracle.dequantize(q["codes"], q["scales"], signs, lam, w.d, w.group, w.bits, rot)


def oracle_sample(w, n_vectors, seed=0):
    rows = max(1, n_vectors // w.H)
    x16 = kv_synth.make_x_numpy(w, seed=seed, n_rows=rows, slices=range(1))
    signs = kv_synth.rademacher_signs(1, w.H, w.d, seed=1)
    return x16, signs, rows * w.H


def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] or [1])
    except Exception:
        return 1


def cpu_baseline(w, n_vectors, rot, steps=1):
    x16, signs, nv = oracle_sample(w, n_vectors)
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle_step(w, x16, signs, rot)
    dt = time.perf_counter() - t0
    gbs = 2 * nv * w.bytes_per_vector() * steps / dt / 1e9
    return {"value": gbs, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
            "vectors_per_s": nv * steps / dt, "seconds": dt,
            "sample": f"{nv} vectors of slice 0 ({w.name}), calibrate+quantize+dequantize x{steps}; "
                      f"float64 numpy, matrix products on {blas_threads()} BLAS threads, "
                      f"elementwise steps single-threaded"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = kv_synth.WORKLOADS[args.workload]
    x16, signs, nv = oracle_sample(w, args.cpu_sample)
    for _ in range(args.warmup):
        oracle_step(w, x16, signs, args.rotation)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(w, x16, signs, args.rotation)
    dt = time.perf_counter() - t0
    gbs = 2 * nv * w.bytes_per_vector() * args.steps / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(w, args, extra={"sample_vectors_per_step": nv}),
        "vectors_per_s": nv * args.steps / dt,
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{nv} vectors of slice 0 per step ({w.name})"},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _config(w, args, extra=None):
    c = {"workload": w.name, "slices": w.S, "rows": w.N, "heads": w.H, "d": w.d,
         "bits": w.bits, "group": w.group, "rotation": "SRFT" if args.rotation == 0 else "SRHT",
         "vectors": w.vectors, "n_cal": w.n_cal,
         "parallelism": f"replicas x{args.gpus} (independent caches, no collective)",
         "l2": "inputs larger than L2 (fp16 cache %.0f MB, codes+scales %.0f MB)" % (
             w.vectors * 2 * w.d / 1e6, w.vectors * (w.bytes_per_vector() - 2 * w.d) / 1e6)}
    if extra:
        c.update(extra)
    return c


# ---------------------------------------------------------------------------
# GPU leg
# ---------------------------------------------------------------------------

def run_ours(args):
    import torch

    import rotate_then_quantize_b200 as rq

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    w = kv_synth.WORKLOADS[args.workload]
    rot = args.rotation
    rq.load_library()
    x = kv_synth.make_x_torch(w, dev, seed=1000 * rank)
    signs = torch.from_numpy(kv_synth.rademacher_signs(w.S, w.H, w.d, seed=1 + rank)).to(dev)
    lam = torch.empty((w.S, w.H, w.d), dtype=torch.float32, device=dev)
    codes = torch.empty((w.S, w.N, w.H, w.d * w.bits // 8), dtype=torch.uint8, device=dev)
    scales = torch.empty((w.S, w.N, w.H, w.d // w.group), dtype=torch.float16, device=dev)
    xhat = torch.empty_like(x)
    desc = rq.make_desc(w.d, w.H, w.group, w.bits, rot)

    def step(ev=None):
        rq.srftq_calibrate_lambda(desc, x, signs, lam, w.n_cal)
        if ev is not None:
            ev[0].record()
        rq.srftq_quantize(desc, x, signs, lam, codes, scales)
        if ev is not None:
            ev[1].record()
        rq.srftq_dequantize(desc, codes, scales, signs, lam, xhat)
        if ev is not None:
            ev[2].record()

    def barrier():
        torch.cuda.synchronize()
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    if rq.srftq_check_device() != 0:
        raise RuntimeError("device guard fired during warm-up")

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    start.record()
    for k in range(K):
        step(evs[k])
    end.record()
    barrier()
    clk = clocks.stop()
    ms = start.elapsed_time(end)
    q_ms = [evs[k][0].elapsed_time(evs[k][1]) for k in range(K)]
    d_ms = [evs[k][1].elapsed_time(evs[k][2]) for k in range(K)]
    if pg is not None:
        t = torch.tensor([ms], device=dev, dtype=torch.float64)
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
        ms = float(t.item())
    if rq.srftq_check_device() != 0:
        raise RuntimeError("device guard fired during the timed steps")

    bytes_launch = w.vectors * w.bytes_per_vector()
    step_bytes = 2 * bytes_launch
    value = step_bytes * K * world / (ms / 1e3) / 1e9
    peak, peak_src = read_peak()
    q_avg, d_avg = statistics.mean(q_ms), statistics.mean(d_ms)
    dom = "quantize" if q_avg >= d_avg else "dequantize"
    dom_ms = max(q_avg, d_avg)
    achieved = bytes_launch / (dom_ms / 1e3) / 1e9
    kname = "quantize_kernel" if dom == "quantize" else "dequantize_kernel"

    e2e = None
    if not args.no_e2e:
        x_host = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
        x_host.copy_(x)
        xhat_host = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)

        def e2e_step():
            x.copy_(x_host, non_blocking=True)
            step()
            xhat_host.copy_(xhat, non_blocking=True)

        e2e_step()
        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record()
        for _ in range(args.e2e_steps):
            e2e_step()
        e2.record()
        barrier()
        ems = s2.elapsed_time(e2)
        if pg is not None:
            t = torch.tensor([ems], device=dev, dtype=torch.float64)
            pg.all_reduce(t, op=pg.ReduceOp.MAX)
            ems = float(t.item())
        e2e = {"value": step_bytes * args.e2e_steps * world / (ems / 1e3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": x.numel() * x.element_size(),
               "d2h_bytes_per_step": xhat.numel() * xhat.element_size(),
               "ms_per_step": ems / args.e2e_steps, "steps": args.e2e_steps,
               "path": "pinned host -> device copy, srftq_calibrate_lambda + srftq_quantize + "
                       "srftq_dequantize, device -> pinned host copy of the dequantized cache"}

    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": _config(w, args),
        "vectors_per_s": w.vectors * K * world / (ms / 1e3),
        "kernels": {"quantize_ms": q_avg, "dequantize_ms": d_avg,
                    "quantize_GBps": bytes_launch / (q_avg / 1e3) / 1e9,
                    "dequantize_GBps": bytes_launch / (d_avg / 1e3) / 1e9,
                    "calibrate_ms_est": ms / K - q_avg - d_avg},
        "roofline": {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else "fallback 6.65 TB/s",
                     "algorithmic_bytes_per_launch": bytes_launch,
                     "traffic": read_traffic(kname, w.name)},
        "gpu_launches": 3 * K,
        "clocks": clk,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_sample, rot)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
