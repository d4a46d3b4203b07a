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
import dataclasses
import hashlib
import json
import math
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
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen_like_d128", choices=list(kv_synth.WORKLOADS))
    ap.add_argument("--rotation", type=int, default=0, choices=[0, 1])
    ap.add_argument("--slices", type=int, default=None,
                    help="run the workload on its first SLICES slices only (smaller captures)")
    ap.add_argument("--reflectors", type=int, default=None,
                    help="run the workload through the dense-rotation calls with this many "
                         "(>= 1) Householder reflectors on its base rotation")
    ap.add_argument("--dense", action="store_true",
                    help="run the workload's base rotation itself (the SRFT / SRHT matrix, "
                         "no reflectors) through the dense tensor-core calls")
    ap.add_argument("--tokens", type=int, default=None,
                    help="decode_stream_d128: cached tokens per sequence (default 32768; "
                         "smaller captures)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--e2e-chunks", type=int, default=28,
                    help="chunks of whole slices the end-to-end step is pipelined over "
                         "(28 measured best on the Qwen-shaped step: 119 GB/s against 115 at 8)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the other_configs object (the other workloads' kernels, "
                         "measured after the headline)")
    ap.add_argument("--cpu-sample", type=int, default=8192,
                    help="vectors per oracle step of the reference arm")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU time the cpu_baseline leg spends (whole oracle steps on a "
                         "65536-vector sample, repeated)")
    return ap.parse_args(argv)


def read_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# Sources each timed kernel is compiled from: a committed DRAM-traffic figure
# is used only while these files are unchanged.
KERNEL_SOURCES = {
    "quantize_kernel": ("codec.cuh", "transform.cuh", "common.cuh", "ptx.cuh", "launch.cuh",
                        "launch_impl.cuh"),
    "dequantize_kernel": ("codec.cuh", "transform.cuh", "common.cuh", "ptx.cuh", "launch.cuh",
                          "launch_impl.cuh"),
    "quantize_split_kernel": ("codec_split.cuh", "codec.cuh", "transform.cuh", "common.cuh",
                              "ptx.cuh", "launch.cuh", "launch_impl.cuh", "launch_split.cuh",
                              "launch_d256.cu"),
    "dequantize_split_kernel": ("codec_split.cuh", "codec.cuh", "transform.cuh", "common.cuh",
                                "ptx.cuh", "launch.cuh", "launch_impl.cuh", "launch_split.cuh",
                                "launch_d256.cu"),
    "quantize_dense_mma_kernel": ("dense_mma.cuh", "tc.cuh", "codec.cuh", "transform.cuh",
                                  "common.cuh", "ptx.cuh", "launch.cuh", "launch_impl.cuh",
                                  "launch_dense.cu", "dense.cuh", "dense_mma_dequant.cuh"),
    "dequantize_dense_mma_kernel": ("dense_mma_dequant.cuh", "tc.cuh", "codec.cuh",
                                    "transform.cuh", "common.cuh", "ptx.cuh", "launch.cuh",
                                    "launch_impl.cuh", "launch_dense.cu", "dense.cuh",
                                    "dense_mma.cuh"),
}


def codec_kernel(kind: str, d: int, dense: bool = False) -> str:
    """Name of the kernel that runs `kind` ("quantize" / "dequantize") for a
    head dimension: d = 256 runs on the two-warp kernels; a dense rotation
    on the dense kernels."""
    if dense:
        return f"{kind}_dense_mma_kernel"
    return f"{kind}{'_split' if d == 256 else ''}_kernel"


def codec_calls(rq, w, desc, signs, seed, dev):
    """(table, (calibrate, quantize, dequantize)) of a workload: the FFT/WHT
    calls with the sign table, or, when the workload runs dense, the dense
    calls with the operand of R = H(v_1)...H(v_k) B (k = 0: B itself)."""
    import torch

    if not w.dense:
        return signs, (rq.srftq_calibrate_lambda, rq.srftq_quantize, rq.srftq_dequantize)
    V = None
    if w.reflectors:
        V = torch.from_numpy(kv_synth.householder_reflectors(w.S, w.H, w.reflectors, w.d,
                                                             seed=seed)).to(dev)
    op = rq.dense_operand(rq.householder_rotation(V, signs, rotation=desc.rotation))
    return op, (rq.srftq_calibrate_lambda_dense, rq.srftq_quantize_dense,
                rq.srftq_dequantize_dense)


def dense_flops_per_vector(kind: str, d: int) -> float:
    """Tensor-core flops per vector of the dense-rotation kernels: the
    quantiser computes R x as two fp16 products (x exact, R = hi + lo); the
    dequantiser computes R^T a as three (a = a_hi + a_lo: a_hi hi, a_lo hi,
    a_hi lo)."""
    return (4.0 if kind == "quantize" else 6.0) * d * d


def read_tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return (float(json.load(f)["bf16_tflops"]),
                    "measured (MEASURED_PEAKS.json bf16_tflops; fp16 runs at the same rate)")
    except Exception:
        return 1590.0, "fallback 1.59 PFLOP/s"


def dense_roofline(w, kind, ms, kname):
    """Roofline of a dense-rotation kernel: whichever of the tensor-core time
    (flops / measured dense fp16 peak) and the HBM time (algorithmic bytes /
    measured copy bandwidth) is longer bounds it; the other is reported
    beside it."""
    flops = dense_flops_per_vector(kind, w.d) * w.vectors
    nbytes = w.vectors * w.bytes_per_vector()
    tpeak, tsrc = read_tensor_peak()
    hpeak, hsrc = read_peak()
    t_tc, t_hbm = flops / (tpeak * 1e12), nbytes / (hpeak * 1e9)
    tc = {"bound": "tensor", "achieved": flops / (ms / 1e3) / 1e12, "peak": tpeak,
          "unit": "TFLOP/s", "peak_source": tsrc, "algorithmic_flops_per_launch": flops}
    hb = {"bound": "hbm", "achieved": nbytes / (ms / 1e3) / 1e9, "peak": hpeak, "unit": "GB/s",
          "peak_source": f"{hsrc} (MEASURED_PEAKS.json hbm_gbs)" if hsrc == "measured"
          else "fallback 6.65 TB/s", "algorithmic_bytes_per_launch": nbytes}
    for r in (tc, hb):
        r["frac"] = r["achieved"] / r["peak"]
    main, other = (tc, hb) if t_tc >= t_hbm else (hb, tc)
    out = {"bound": main["bound"], "kernel": kname, "launch": kind}
    out.update({k: v for k, v in main.items() if k != "bound"})
    out["traffic"] = read_traffic(kname, w.name)
    out["other_bound"] = other
    return out


def csrc_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for name in sorted(KERNEL_SOURCES.get(kernel, ())):
        with open(os.path.join(ROOT, "rotate_then_quantize_b200", "csrc", name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def read_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken
    on the current sources of that kernel; null otherwise."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(p) as f:
            data = json.load(f)
    except Exception:
        return None
    ent = data.get(f"{kernel}:{workload}")
    if not ent or ent.get("sources_sha") != csrc_hash(kernel):
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
    """One oracle pass on a sample: calibrate, quantize, dequantize (with the
    workload's dense rotation, reflectors or none, when it runs dense)."""
    import oracle

    n_cal = min(w.n_cal, x16.shape[1])
    if w.dense:
        V = kv_synth.householder_reflectors(1, w.H, w.reflectors, w.d, seed=1)
        R = oracle.householder_rotations(V, signs, rot)
        lam = oracle.calibrate_lambda_dense(x16, R, n_cal).astype(np.float32)
        q = oracle.quantize_dense(x16, R, lam, w.group, w.bits)
        oracle.dequantize_dense(q["codes"], q["scales"], R, lam, w.d, w.group, w.bits)
        return
    lam = oracle.calibrate_lambda(x16, signs, n_cal, rot).astype(np.float32)
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


def cpu_baseline(w, rot, seconds, n_vectors=65536):
    """The oracle, as it stands, on a 65536-vector sample of the workload,
    repeated (whole steps) until `seconds` of wall time have passed."""
    x16, signs, nv = oracle_sample(w, n_vectors)
    steps = 0
    t0 = time.perf_counter()
    while True:
        oracle_step(w, x16, signs, rot)
        steps += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            break
    gbs = 2 * nv * w.bytes_per_vector() * steps / dt / 1e9
    return {"value": gbs, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
            "vectors_per_s": nv * steps / dt, "seconds": dt,
            "sample": f"{nv} vectors of slice 0 ({w.name}), calibrate+quantize+dequantize, "
                      f"{steps} repetitions; float64 numpy, matrix products on "
                      f"{blas_threads()} BLAS threads, elementwise steps single-threaded"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = workload(args)
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

def _setup_ranks():
    """One process per GPU; NCCL only for the barrier and the max over ranks."""
    import torch

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
    return rank, world, local, dev, pg


def job_gbps(bytes_per_rank_step: float, steps: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's bytes over the slowest rank's time."""
    return bytes_per_rank_step * steps * world / (ms_max / 1e3) / 1e9


def rank_seeds(rank: int) -> tuple:
    """(data seed, sign seed) of a replica: every rank codes its own cache."""
    return 1000 * rank, 1 + rank


def _max_over_ranks(pg, dev, ms):
    import torch

    if pg is None:
        return ms
    t = torch.tensor([ms], device=dev, dtype=torch.float64)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())

def workload(args):
    """The named workload, cut to its first --slices slices if given."""

    w = kv_synth.WORKLOADS[args.workload]
    if args.slices is not None:
        if not 1 <= args.slices <= w.S:
            raise SystemExit(f"--slices must be in 1..{w.S}")
        w = dataclasses.replace(w, S=args.slices)
    if getattr(args, "reflectors", None) is not None:
        if args.workload == "decode_stream_d128" or w.d not in (64, 128, 256) or args.reflectors < 1:
            raise SystemExit("--reflectors needs a codec workload with d in {64, 128, 256}")
        w = dataclasses.replace(w, reflectors=args.reflectors, name=w.name + "+dense")
    if getattr(args, "dense", False):
        if args.workload == "decode_stream_d128" or w.d not in (64, 128, 256) or w.reflectors:
            raise SystemExit("--dense needs a codec workload with d in {64, 128, 256} and no "
                             "reflectors")
        w = dataclasses.replace(w, dense_base=True, name=w.name + "+dense0")
    if getattr(args, "tokens", None) is not None:
        if args.workload != "decode_stream_d128" or not 512 <= args.tokens <= 32768:
            raise SystemExit("--tokens applies to decode_stream_d128, 512..32768")
        w = dataclasses.replace(w, N=args.tokens * 32)
    return w


def run_ours(args):
    import torch

    import rotate_then_quantize_b200 as rq

    rank, world, local, dev, pg = _setup_ranks()
    w = workload(args)
    rot = args.rotation
    rq.load_library()
    data_seed, sign_seed = rank_seeds(rank)
    x = kv_synth.make_x_torch(w, dev, seed=data_seed)
    signs = torch.from_numpy(kv_synth.rademacher_signs(w.S, w.H, w.d, seed=sign_seed)).to(dev)
    lam = torch.empty((w.S, w.H, w.d), dtype=torch.float32, device=dev)
    codes = torch.empty((w.S, w.N, w.H, w.d * w.bits // 8), dtype=torch.uint8, device=dev)
    scales = torch.empty((w.S, w.N, w.H, w.d // w.group), dtype=torch.float16, device=dev)
    xhat = torch.empty_like(x)
    desc = rq.make_desc(w.d, w.H, w.group, w.bits, rot)
    # the per-(slice, head) table the calls read: the signs, or for a dense
    # rotation the operand of R = H(v_1) ... H(v_k) B (built once, before timing)
    table, fns = codec_calls(rq, w, desc, signs, sign_seed, dev)
    f_cal, f_q, f_dq = fns

    def step(ev=None):
        f_cal(desc, x, table, lam, w.n_cal)
        if ev is not None:
            ev[0].record()
        f_q(desc, x, table, lam, codes, scales)
        if ev is not None:
            ev[1].record()
        f_dq(desc, codes, scales, table, lam, xhat)
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
    ms = _max_over_ranks(pg, dev, start.elapsed_time(end))
    q_ms = [evs[k][0].elapsed_time(evs[k][1]) for k in range(K)]
    d_ms = [evs[k][1].elapsed_time(evs[k][2]) for k in range(K)]
    if rq.srftq_check_device() != 0:
        raise RuntimeError("device guard fired during the timed steps")

    quality = round_trip_error(x, xhat)

    bytes_launch = w.vectors * w.bytes_per_vector()
    step_bytes = 2 * bytes_launch
    value = job_gbps(step_bytes, K, world, ms)
    peak, peak_src = read_peak()
    q_avg, d_avg = statistics.mean(q_ms), statistics.mean(d_ms)
    dom = "quantize" if q_avg >= d_avg else "dequantize"
    dom_ms = max(q_avg, d_avg)
    achieved = bytes_launch / (dom_ms / 1e3) / 1e9
    kname = codec_kernel(dom, w.d, dense=w.dense)
    roof = {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": peak,
            "unit": "GB/s", "frac": achieved / peak,
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
            else "fallback 6.65 TB/s",
            "algorithmic_bytes_per_launch": bytes_launch,
            "traffic": read_traffic(kname, w.name)}
    if w.dense:
        roof = dense_roofline(w, dom, dom_ms, kname)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, rq, desc, w, x, table, lam, codes, scales, xhat, barrier, pg, dev,
                      step_bytes, world, fns)

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
        "roofline": roof,
        "gpu_launches": 3 * K,
        "clocks": clk,
        "quality": quality,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if (world == 1 and not args.no_other_configs and args.slices is None
            and args.workload == "qwen_like_d128"):
        del x, codes, scales, xhat
        torch.cuda.empty_cache()
        line["other_configs"] = other_configs(rq, dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, rot, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def _time_launches(fn, iters: int, warmup: int = 3) -> float:
    """Mean CUDA-event duration (ms) of fn() on the current stream."""
    import torch

    for _ in range(warmup):
        fn()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(iters)]
    torch.cuda.synchronize()
    for a, b in evs:
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in evs)


def _codec_figures(rq, w, rot, dev, iters):
    """Quantise and dequantise GB/s of one workload at full size (one launch each)."""
    import torch

    x = kv_synth.make_x_torch(w, dev, seed=0)
    signs = torch.from_numpy(kv_synth.rademacher_signs(w.S, w.H, w.d, seed=1)).to(dev)
    desc = rq.make_desc(w.d, w.H, w.group, w.bits, rot)
    table, (f_cal, f_q, f_dq) = codec_calls(rq, w, desc, signs, 1, dev)
    lam = torch.empty((w.S, w.H, w.d), dtype=torch.float32, device=dev)
    f_cal(desc, x, table, lam, w.n_cal)
    codes = torch.empty((w.S, w.N, w.H, w.d * w.bits // 8), dtype=torch.uint8, device=dev)
    scales = torch.empty((w.S, w.N, w.H, w.d // w.group), dtype=torch.float16, device=dev)
    xhat = torch.empty_like(x)
    q_ms = _time_launches(lambda: f_q(desc, x, table, lam, codes, scales), iters)
    d_ms = _time_launches(lambda: f_dq(desc, codes, scales, table, lam, xhat), iters)
    if rq.srftq_check_device() != 0:
        raise RuntimeError(f"device guard fired in {w.name}")
    peak = read_peak()[0]
    b = w.vectors * w.bytes_per_vector()
    out = {"rotation": "SRFT" if rot == 0 else "SRHT", "vectors": w.vectors,
           "bytes_per_launch": b, "launches_timed": iters,
           "quantize_ms": q_ms, "quantize_GBps": b / q_ms / 1e6,
           "quantize_frac": b / q_ms / 1e6 / peak,
           "dequantize_ms": d_ms, "dequantize_GBps": b / d_ms / 1e6,
           "dequantize_frac": b / d_ms / 1e6 / peak,
           "kernels": [codec_kernel("quantize", w.d, w.dense),
                       codec_kernel("dequantize", w.d, w.dense)],
           "rel_l2_error": round_trip_error(x, xhat)}
    del x, codes, scales, xhat
    torch.cuda.empty_cache()
    return out


def _attention_figures(rq, dev, iters):
    """The fused decode attention on one decode-stream layer: 32 sequences x 8
    KV heads over 32,768 cached int4 tokens (K and V), one query per KV head."""
    import torch

    w = kv_synth.WORKLOADS["decode_stream_d128"]
    B = 32
    n_ctx = w.N // B
    x = kv_synth.make_x_torch(w, dev, seed=0, slices=range(2))
    signs = torch.from_numpy(kv_synth.rademacher_signs(2, w.H, w.d, seed=1)).to(dev)
    desc = rq.make_desc(w.d, w.H, w.group, w.bits, 0)
    lam = torch.empty((2, w.H, w.d), dtype=torch.float32, device=dev)
    rq.srftq_calibrate_lambda(desc, x, signs, lam, w.n_cal)
    codes = torch.empty((2, w.N, w.H, w.d * w.bits // 8), dtype=torch.uint8, device=dev)
    scales = torch.empty((2, w.N, w.H, w.d // w.group), dtype=torch.float16, device=dev)
    rq.srftq_quantize(desc, x, signs, lam, codes, scales)
    fp16_ms = _time_launches(lambda: torch.sum(x, dtype=torch.float32), iters)
    del x
    torch.cuda.empty_cache()
    q = torch.randn((B, w.H, w.d), device=dev).to(torch.float16)
    out = torch.empty((B, w.H, w.d), dtype=torch.float32, device=dev)
    a_ms = _time_launches(lambda: rq.srftq_decode_attention(
        desc, q, codes[0], scales[0], signs[0], lam[0], codes[1], scales[1], signs[1], lam[1],
        n_ctx, B, 1, 1.0 / math.sqrt(w.d), out), iters)
    if rq.srftq_check_device() != 0:
        raise RuntimeError("device guard fired in the fused attention")
    b = 2 * w.N * w.H * (w.d * w.bits // 8 + 2 * (w.d // w.group))
    peak = read_peak()[0]
    del codes, scales
    torch.cuda.empty_cache()
    return {"layer": "32 sequences x 8 KV heads x 32768 cached tokens, int4 G16 K and V, "
                     "one query per KV head (srftq_decode_attention: 3 launches)",
            "ms_per_layer": a_ms, "codes_and_scales_bytes": b, "GBps": b / a_ms / 1e6,
            "frac": b / a_ms / 1e6 / peak, "launches_timed": iters,
            "fp16_read_ms_per_layer": fp16_ms,
            "over_fp16_read": a_ms / fp16_ms,
            "fp16_read": "torch.sum over the layer's fp16 K and V (the same tokens)"}


def parity_report():
    """Counts from the committed full-data parity report (written by
    tests/test_gpu_full_data.py), or None."""
    p = os.path.join(ROOT, "profiles", "parity_full_data.json")
    try:
        with open(p) as f:
            data = json.load(f)
    except Exception:
        return None
    keep = ("vectors", "codes", "code_mismatch_in_band", "code_violations",
            "scale_mismatch_in_band", "scale_violations", "zero_scale_groups",
            "dequant_violations", "dequant_max_err_over_tol")
    return {"source": "profiles/parity_full_data.json (tests/test_gpu_full_data.py, every "
                      "vector against the oracle)",
            **{k: {f: v[f] for f in keep if f in v} for k, v in data.items()
               if isinstance(v, dict) and "vectors" in v}}


def other_configs(rq, dev, iters=50):
    """The other workloads' kernels at full size, measured after the headline
    and outside its timed region: long-context int8 (SRFT and SRHT side by
    side, with their round-trip errors), the Gemma-shaped d = 256 cache, the
    Householder workload, the headline shape's SRFT as a dense tensor-core
    product (the matrix itself, beside the FFT kernels of the headline) and
    the fused decode attention of one decode-stream layer."""
    out = {}
    lc = kv_synth.WORKLOADS["longctx_int8_d128"]
    srft = _codec_figures(rq, lc, 0, dev, iters)
    srht = _codec_figures(rq, lc, 1, dev, iters)
    out["longctx_int8_d128"] = {"SRFT": srft, "SRHT": srht,
                                "rel_l2_mean_srft_vs_srht": [srft["rel_l2_error"]["rel_l2_mean"],
                                                             srht["rel_l2_error"]["rel_l2_mean"]]}
    out["gemma_like_d256"] = _codec_figures(rq, kv_synth.WORKLOADS["gemma_like_d256"], 0, dev,
                                            iters)
    hh = kv_synth.WORKLOADS["householder_d256"]
    out["householder_d256"] = _codec_figures(rq, hh, 0, dev, iters)
    flops = {k: dense_flops_per_vector(k, hh.d) * hh.vectors for k in ("quantize", "dequantize")}
    for kind, f in flops.items():
        out["householder_d256"][f"{kind}_TFLOPs"] = f / out["householder_d256"][f"{kind}_ms"] / 1e9
    out["householder_d256"]["flops_per_launch"] = flops
    qd = dataclasses.replace(kv_synth.WORKLOADS["qwen_like_d128"], dense_base=True,
                             name="qwen_like_d128+dense0")
    out["qwen_like_d128_srft_tensor_core"] = _codec_figures(rq, qd, 0, dev, iters)
    out["decode_stream_d128_fused_attention"] = _attention_figures(rq, dev, iters)
    rep = parity_report()
    if rep is not None:
        out["parity_full_data"] = rep
    return out


def e2e_chunks(n_slices: int, target: int = 8) -> list:
    """Slice ranges [a, b) of the pipelined end-to-end step: about `target`
    chunks of whole slices (calibration is per slice, so chunks never split
    one)."""
    n = max(1, min(target, n_slices))
    bounds = [round(i * n_slices / n) for i in range(n + 1)]
    return [(bounds[i], bounds[i + 1]) for i in range(n) if bounds[i + 1] > bounds[i]]


def run_e2e(args, rq, desc, w, x, signs, lam, codes, scales, xhat, barrier, pg, dev,
            step_bytes, world, fns) -> dict:
    """The step end to end through the C ABI: the fp16 cache comes from pinned
    host memory and the dequantised cache goes back to it, every step. The
    step is pipelined over chunks of whole slices on three streams (copy in,
    compute, copy out, ordered by events), so that host->device copies,
    kernels and device->host copies of different chunks overlap; PCIe
    carries both directions at once."""
    import torch

    x_host = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    x_host.copy_(x)
    xhat_host = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    chunks = e2e_chunks(w.S, args.e2e_chunks)
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    main = torch.cuda.current_stream()

    def e2e_step():
        start_ev = torch.cuda.Event()
        start_ev.record(main)
        done = []
        for a, b in chunks:
            e_in, e_cmp = torch.cuda.Event(), torch.cuda.Event()
            with torch.cuda.stream(s_in):
                s_in.wait_event(start_ev)
                x[a:b].copy_(x_host[a:b], non_blocking=True)
                e_in.record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(e_in)
                f_cal, f_q, f_dq = fns
                f_cal(desc, x[a:b], signs[a:b], lam[a:b], w.n_cal, s_cmp)
                f_q(desc, x[a:b], signs[a:b], lam[a:b], codes[a:b], scales[a:b], s_cmp)
                f_dq(desc, codes[a:b], scales[a:b], signs[a:b], lam[a:b], xhat[a:b], s_cmp)
                e_cmp.record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(e_cmp)
                xhat_host[a:b].copy_(xhat[a:b], non_blocking=True)
                e_out = torch.cuda.Event()
                e_out.record(s_out)
            done.append(e_out)
        for e in done:
            main.wait_event(e)

    e2e_step()
    barrier()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(main)
    for _ in range(args.e2e_steps):
        e2e_step()
    e2.record(main)
    barrier()
    ems = _max_over_ranks(pg, dev, s2.elapsed_time(e2))
    if rq.srftq_check_device() != 0:
        raise RuntimeError("device guard fired during the end-to-end steps")

    # The bound of this path: the same host->device and device->host copies
    # alone, concurrently on the copy streams, timed the same way (the data
    # copied are the step's own buffers, so nothing changes).
    def copy_step():
        start_ev = torch.cuda.Event()
        start_ev.record(main)
        e_in, e_out = torch.cuda.Event(), torch.cuda.Event()
        with torch.cuda.stream(s_in):
            s_in.wait_event(start_ev)
            x.copy_(x_host, non_blocking=True)
            e_in.record(s_in)
        with torch.cuda.stream(s_out):
            s_out.wait_event(start_ev)
            xhat_host.copy_(xhat, non_blocking=True)
            e_out.record(s_out)
        main.wait_event(e_in)
        main.wait_event(e_out)

    copy_step()
    barrier()
    s3, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s3.record(main)
    for _ in range(args.e2e_steps):
        copy_step()
    e3.record(main)
    barrier()
    cms = _max_over_ranks(pg, dev, s3.elapsed_time(e3))
    io_bytes = (x.numel() * x.element_size() + xhat.numel() * xhat.element_size())
    return {"value": step_bytes * args.e2e_steps * world / (ems / 1e3) / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": x.numel() * x.element_size(),
            "d2h_bytes_per_step": xhat.numel() * xhat.element_size(),
            "ms_per_step": ems / args.e2e_steps, "steps": args.e2e_steps,
            "chunks": len(chunks),
            "copy_only": {"ms_per_step": cms / args.e2e_steps,
                          "pcie_GBps": io_bytes * args.e2e_steps / (cms / 1e3) / 1e9,
                          "frac": (cms / args.e2e_steps) / (ems / args.e2e_steps),
                          "what": "the step's host->device and device->host copies alone, "
                                  "concurrently; frac = copy-only time / end-to-end time"},
            "path": "pinned host -> device copy, srftq_calibrate_lambda + srftq_quantize + "
                    "srftq_dequantize, device -> pinned host copy of the dequantized cache; "
                    f"pipelined over {len(chunks)} chunks of slices on three streams"}


def round_trip_error(x, xhat, chunk_rows: int = 4096) -> dict:
    """Per-vector relative L2 error ||xhat - x|| / ||x|| of the last step's
    round trip (quantize then dequantize), outside the timed region:
    mean, median, 99th percentile and maximum over every vector with a
    non-zero norm. Computed in float32 slice by slice."""
    import torch

    errs = []
    d = x.shape[-1]
    xf, hf = x.reshape(-1, d), xhat.reshape(-1, d)
    for i in range(0, xf.shape[0], chunk_rows * 64):
        a = xf[i:i + chunk_rows * 64].float()
        b = hf[i:i + chunk_rows * 64].float()
        n = a.norm(dim=1)
        keep = n > 0
        errs.append(((b - a).norm(dim=1)[keep] / n[keep]).cpu())
    e = torch.cat(errs)
    if e.numel() == 0:
        return {"rel_l2_mean": None}
    q = torch.quantile(e[torch.randperm(e.numel())[:1 << 24]] if e.numel() > (1 << 24) else e,
                       torch.tensor([0.5, 0.99]))
    return {"rel_l2_mean": float(e.mean()), "rel_l2_p50": float(q[0]),
            "rel_l2_p99": float(q[1]), "rel_l2_max": float(e.max()), "vectors": int(e.numel()),
            "what": "per-vector ||xhat - x|| / ||x|| of the last timed step"}


# ---------------------------------------------------------------------------
# Decode-style streaming
# ---------------------------------------------------------------------------

def run_decode(args):
    """Decode steps over an int4 cache of 32768 tokens x 32 sequences.

    Cache layout per slice (layer x {K, V}): row = token * 32 + sequence, so
    one decode step's new tokens are 32 consecutive rows. A step, per layer:
    quantize the 32 new (K, V) tokens into the cache at the next row block,
    then dequantize that layer's whole cache (both slices) into one fp16
    scratch buffer of a layer's shape, as an attention kernel would consume
    it. The comparator reads an fp16 cache of the same shape once per layer
    (torch.sum over the scratch buffer)."""
    import torch

    import rotate_then_quantize_b200 as rq

    rank, world, local, dev, pg = _setup_ranks()
    w = workload(args)
    B = 32
    T0 = w.N // B
    L = w.S // 2
    rot = args.rotation
    n_steps = args.warmup + 3 * args.steps + args.e2e_steps + 8
    cap = (T0 + n_steps) * B
    rq.load_library()
    desc = rq.make_desc(w.d, w.H, w.group, w.bits, rot)
    signs = torch.from_numpy(kv_synth.rademacher_signs(w.S, w.H, w.d, seed=1 + rank)).to(dev)
    lam = torch.empty((w.S, w.H, w.d), dtype=torch.float32, device=dev)
    codes = torch.empty((w.S, cap, w.H, w.d * w.bits // 8), dtype=torch.uint8, device=dev)
    scales = torch.empty((w.S, cap, w.H, w.d // w.group), dtype=torch.float16, device=dev)
    scratch = torch.empty((2, cap, w.H, w.d), dtype=torch.float16, device=dev)
    # the existing cache: seeded fp16 N(0,1) per slice, calibrated and quantized
    for s_ in range(w.S):
        xs = kv_synth.make_x_torch(w, dev, seed=1000 * rank, n_rows=T0 * B,
                                   slices=range(s_, s_ + 1), out=scratch[0:1, :T0 * B])
        rq.srftq_calibrate_lambda(desc, xs, signs[s_:s_ + 1], lam[s_:s_ + 1], w.n_cal)
        rq.srftq_quantize(desc, xs, signs[s_:s_ + 1], lam[s_:s_ + 1],
                          codes[s_:s_ + 1, :T0 * B], scales[s_:s_ + 1, :T0 * B])
    new_tok = kv_synth.make_x_torch(w, dev, seed=7 + 1000 * rank, n_rows=B)
    torch.cuda.synchronize()
    if rq.srftq_check_device() != 0:
        raise RuntimeError("device guard fired while filling the cache")

    state = {"t": 0}
    vec_bytes = w.bytes_per_vector()

    def step(ev=None):
        r0 = (T0 + state["t"]) * B
        n = r0 + B
        for l in range(L):
            sl = slice(2 * l, 2 * l + 2)
            rq.srftq_quantize(desc, new_tok[sl], signs[sl], lam[sl], codes[sl, r0:n],
                              scales[sl, r0:n])
            if ev is not None:
                ev[l][0].record()
            rq.srftq_dequantize(desc, codes[sl, :n], scales[sl, :n], signs[sl], lam[sl],
                                scratch[:, :n])
            if ev is not None:
                ev[l][1].record()
        state["t"] += 1
        return (w.S * B * w.H + w.S * n * w.H) * vec_bytes, w.S * n * w.H

    def barrier():
        torch.cuda.synchronize()
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    K = args.steps
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(L)]
           for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    start.record()
    tot_bytes = tot_vec = 0
    for k in range(K):
        b_, v_ = step(evs[k])
        tot_bytes += b_
        tot_vec += v_
    end.record()
    barrier()
    clk = clocks.stop()
    ms = _max_over_ranks(pg, dev, start.elapsed_time(end))
    if rq.srftq_check_device() != 0:
        raise RuntimeError("device guard fired during the timed steps")
    d_ms = [evs[k][l][0].elapsed_time(evs[k][l][1]) for k in range(K) for l in range(L)]
    n_last = (T0 + state["t"]) * B
    deq_bytes = 2 * n_last * w.H * vec_bytes
    d_avg = statistics.mean(d_ms)

    # comparator: the same decode steps reading a contiguous fp16 cache of one
    # layer's (K, V) shape instead, once per layer
    fp16_layer = scratch[:, :n_last].contiguous()
    fp16_bytes = 0
    acc = torch.zeros((), dtype=torch.float32, device=dev)
    for _ in range(2):
        for l in range(L):
            acc += torch.sum(fp16_layer, dtype=torch.float32)
    barrier()
    s3, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s3.record()
    for k in range(K):
        for l in range(L):
            acc += torch.sum(fp16_layer, dtype=torch.float32)
            fp16_bytes += fp16_layer.numel() * 2
    e3.record()
    barrier()
    fp16_ms = _max_over_ranks(pg, dev, s3.elapsed_time(e3))
    del fp16_layer

    # The same decode steps in the rotated domain (R orthogonal: (R q) . (R x)
    # = q . x): the layer's K and V dequantised without the inverse transform,
    # the step's 32 x H queries rotated with K's signs and the 32 x H attention
    # outputs unrotated with V's signs.
    q_tok = new_tok[0:1]
    q_rot = torch.empty((1, B, w.H, w.d), dtype=torch.float32, device=dev)
    o_rot = torch.randn((1, B, w.H, w.d), dtype=torch.float32, device=dev)
    o_out = torch.empty_like(o_rot)

    def step_rot(ev=None):
        r0 = (T0 + state["t"]) * B
        n = r0 + B
        for l in range(L):
            sl = slice(2 * l, 2 * l + 2)
            rq.srftq_quantize(desc, new_tok[sl], signs[sl], lam[sl], codes[sl, r0:n],
                              scales[sl, r0:n])
            rq.srftq_rotate(desc, q_tok, signs[2 * l:2 * l + 1], q_rot)
            if ev is not None:
                ev[l][0].record()
            rq.srftq_dequantize_rotated(desc, codes[sl, :n], scales[sl, :n], lam[sl],
                                        scratch[:, :n])
            if ev is not None:
                ev[l][1].record()
            rq.srftq_unrotate(desc, o_rot, signs[2 * l + 1:2 * l + 2], o_out)
        state["t"] += 1

    for _ in range(2):
        step_rot()
    barrier()
    evr = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(L)]
           for _ in range(K)]
    s4, e4 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s4.record()
    for k in range(K):
        step_rot(evr[k])
    e4.record()
    barrier()
    rot_ms = _max_over_ranks(pg, dev, s4.elapsed_time(e4))
    if rq.srftq_check_device() != 0:
        raise RuntimeError("device guard fired during the rotated-domain steps")
    r_avg = statistics.mean(evr[k][l][0].elapsed_time(evr[k][l][1])
                            for k in range(K) for l in range(L))
    n_rot = (T0 + state["t"]) * B
    rot_bytes = 2 * n_rot * w.H * vec_bytes
    # The same decode steps with attention fused into the dequantisation: one
    # query per (sequence, KV head) attends over the layer's K and V codes;
    # no fp16 cache is written and no inverse transform runs per token.
    q_dec = torch.randn((B, w.H, w.d), device=dev).to(torch.float16)
    att_out = torch.empty((B, w.H, w.d), dtype=torch.float32, device=dev)
    cbw, ngw = w.d * w.bits // 8, w.d // w.group

    def step_attn(ev=None):
        r0 = (T0 + state["t"]) * B
        n = r0 + B
        for l in range(L):
            sl = slice(2 * l, 2 * l + 2)
            rq.srftq_quantize(desc, new_tok[sl], signs[sl], lam[sl], codes[sl, r0:n],
                              scales[sl, r0:n])
            if ev is not None:
                ev[l][0].record()
            k, v = 2 * l, 2 * l + 1
            rq.srftq_decode_attention(desc, q_dec, codes[k, :n], scales[k, :n], signs[k], lam[k],
                                      codes[v, :n], scales[v, :n], signs[v], lam[v], n // B, B, 1,
                                      1.0 / math.sqrt(w.d), att_out)
            if ev is not None:
                ev[l][1].record()
        state["t"] += 1

    for _ in range(2):
        step_attn()
    barrier()
    eva = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(L)]
           for _ in range(K)]
    s5, e5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s5.record()
    for k in range(K):
        step_attn(eva[k])
    e5.record()
    barrier()
    att_ms = _max_over_ranks(pg, dev, s5.elapsed_time(e5))
    if rq.srftq_check_device() != 0:
        raise RuntimeError("device guard fired during the fused-attention steps")
    a_avg = statistics.mean(eva[k][l][0].elapsed_time(eva[k][l][1])
                            for k in range(K) for l in range(L))
    n_att = (T0 + state["t"]) * B
    att_bytes = 2 * n_att * w.H * (cbw + 2 * ngw)   # K and V codes and scales read
    fused = {"ms_per_step": att_ms / K,
             "attention_ms_per_layer": a_avg,
             "attention_GBps": att_bytes / (a_avg / 1e3) / 1e9,
             "attention_frac_of_peak": att_bytes / (a_avg / 1e3) / 1e9 / read_peak()[0],
             "step_over_fp16_read_time": (att_ms / K) / (fp16_ms / K),
             "attention_over_fp16_read_per_layer": a_avg / (fp16_ms / K / L),
             "step": "per layer: quantize 32 new K and V tokens, then one query per sequence "
                     "and KV head attends over the layer's int4 K and V codes "
                     "(srftq_decode_attention, rotated domain, float32 out)"}

    rotated = {"ms_per_step": rot_ms / K,
               "dequantize_rotated_ms_per_layer": r_avg,
               "dequantize_rotated_GBps": rot_bytes / (r_avg / 1e3) / 1e9,
               "dequantize_rotated_frac_of_peak": rot_bytes / (r_avg / 1e3) / 1e9 / read_peak()[0],
               "step_over_fp16_read_time": (rot_ms / K) / (fp16_ms / K),
               "step": "per layer: quantize 32 new K and V tokens, rotate 32 x H queries, "
                       "dequantize the layer's K and V cache in the rotated domain into an "
                       "fp16 scratch, unrotate 32 x H outputs"}

    e2e = None
    if not args.no_e2e:
        tok_host = torch.empty(new_tok.shape, dtype=new_tok.dtype, pin_memory=True)
        tok_host.copy_(new_tok)
        out_host = torch.empty((2, B, w.H, w.d), dtype=torch.float16, pin_memory=True)

        def e2e_step():
            new_tok.copy_(tok_host, non_blocking=True)
            r0 = (T0 + state["t"]) * B
            step()
            # the step's result: the last layer's appended tokens, dequantized
            out_host.copy_(scratch[:, r0:r0 + B], non_blocking=True)

        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record()
        e_bytes = 0
        for _ in range(args.e2e_steps):
            n = (T0 + state["t"] + 1) * B
            e_bytes += (w.S * B * w.H + w.S * n * w.H) * vec_bytes
            e2e_step()
        e2.record()
        barrier()
        ems = _max_over_ranks(pg, dev, s2.elapsed_time(e2))
        e2e = {"value": e_bytes * world / (ems / 1e3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": new_tok.numel() * new_tok.element_size(),
               "d2h_bytes_per_step": 2 * B * w.H * w.d * 2,
               "ms_per_step": ems / args.e2e_steps, "steps": args.e2e_steps,
               "path": "new tokens pinned host -> device, the step's quantize+dequantize "
                       "launches, the appended tokens' dequantized rows device -> host"}

    peak, peak_src = read_peak()
    achieved = deq_bytes / (d_avg / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": tot_bytes * world / (ms / 1e3) / 1e9, "unit": "GB/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": _config(w, args, extra={
            "sequences": B, "cached_tokens": T0, "layers": L,
            "step": "per layer: quantize 32 new K and V tokens into the cache, then "
                    "dequantize the layer's whole K and V cache into an fp16 scratch"}),
        "vectors_per_s": tot_vec * world / (ms / 1e3),
        "fp16_read": {"GBps": fp16_bytes / (fp16_ms / 1e3) / 1e9,
                      "ms_per_step": fp16_ms / K,
                      "bytes_per_step": fp16_bytes // K,
                      "how": "torch.sum over an fp16 buffer of one layer's K and V cache "
                             "shape, once per layer"},
        "int4_step_over_fp16_read_time": (ms / K) / (fp16_ms / K),
        "rotated_domain": rotated,
        "fused_attention": fused,
        "int4_step_over_fp16_read_at_peak": (ms / K) / (fp16_bytes / K / (read_peak()[0] * 1e6)),
        "kernels": {"dequantize_ms_per_layer": d_avg,
                    "dequantize_GBps": achieved,
                    "launches_per_step": 2 * L},
        "roofline": {"bound": "hbm", "kernel": codec_kernel("dequantize", w.d),
                     "achieved": achieved,
                     "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_src == "measured" else "fallback 6.65 TB/s",
                     "algorithmic_bytes_per_launch": deq_bytes,
                     "traffic": read_traffic(codec_kernel("dequantize", w.d), w.name)},
        "gpu_launches": 2 * L * K,
        "clocks": clk,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, rot, args.cpu_seconds)
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
    if args.workload == "decode_stream_d128":
        return run_decode(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
