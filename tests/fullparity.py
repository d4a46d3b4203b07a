"""Every-vector comparison of a GPU codec run with the CPU oracle.

The GPU side has already quantised and dequantised a whole workload in the
launch configuration the benchmark times. Here its inputs and outputs are
copied back chunk by chunk and checked in a pool of worker processes (started
with the `spawn` method, so no worker inherits the parent's CUDA context):

* codes and scales against ``oracle.quantize`` of the same fp16 inputs with
  the same signs and lambda (the tolerances of ``parity.check_codes``);
* the dequantised fp16 output against ``oracle.dequantize`` of the GPU's own
  codes and scales (``parity.check_dequant``), so a boundary-band code flip
  is not counted twice and every vector is compared.

The per-chunk statistics are summed into one record per workload, which the
tests write to ``profiles/parity_full_data.json``: the count of codes
compared, the boundary-band mismatches, the scale midpoint cases, the
sigma = 0 groups, the largest dequantisation error and every violation
count (all of which must be zero).
"""

from __future__ import annotations

import json
import multiprocessing as mp
import os
import time

import numpy as np

import oracle
import parity

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
REPORT = os.path.join(ROOT, "profiles", "parity_full_data.json")

_SUM_KEYS = ("codes", "code_mismatch_in_band", "code_violations", "scale_mismatch_in_band",
             "scale_violations", "groups_excluded", "zero_scale_groups", "zero_scale_violations",
             "dequant_values", "dequant_violations", "dequant_overflow_to_inf", "vectors")
_MAX_KEYS = ("dequant_max_abs_err", "dequant_max_err_over_tol")


def check_chunk(job: tuple) -> dict:
    """Worker: oracle quantise + dequantise of one chunk against the GPU's output.

    job = (x16 [1, n, H, d], signs [1, H, d], lam [1, H, d] float32,
           codes [1, n, H, cb], scales bits [1, n, H, ng], xhat bits [1, n, H, d],
           d, group, bits, rotation)."""
    x16, signs, lam, codes, scales, xhat, d, group, bits, rot = job
    with np.errstate(all="ignore"):
        ref = oracle.quantize(x16, signs, lam, group, bits, rot)
        st = parity.check_codes(ref, codes, scales, bits, group)
        deq = oracle.dequantize(codes, scales, signs, lam, d, group, bits, rot)
        dq = parity.check_dequant(xhat, deq["bits"])
    out = dict(st)
    out["dequant_values"] = int(xhat.size)
    out["dequant_violations"] = dq["violations"]
    out["dequant_overflow_to_inf"] = dq["overflow_to_inf"]
    out["dequant_max_abs_err"] = dq["max_abs_err"]
    out["dequant_max_err_over_tol"] = dq["max_err_over_tol"]
    out["vectors"] = int(np.prod(x16.shape[:3]))
    return out


def check_chunk_dense(job: tuple) -> dict:
    """Worker for the dense-rotation codec: as check_chunk, with the oracle's
    rotation matrices R [1, H, d, d] in place of the sign rows."""
    x16, R, lam, codes, scales, xhat, d, group, bits = job
    with np.errstate(all="ignore"):
        ref = oracle.quantize_dense(x16, R, lam, group, bits)
        st = parity.check_codes(ref, codes, scales, bits, group, parity.DENSE_SCALE_BAND,
                                parity.dense_code_band(ref, lam, group))
        deq = oracle.dequantize_dense(codes, scales, R, lam, d, group, bits)
        dq = parity.check_dequant(xhat, deq["bits"])
    out = dict(st)
    out["dequant_values"] = int(xhat.size)
    out["dequant_violations"] = dq["violations"]
    out["dequant_overflow_to_inf"] = dq["overflow_to_inf"]
    out["dequant_max_abs_err"] = dq["max_abs_err"]
    out["dequant_max_err_over_tol"] = dq["max_err_over_tol"]
    out["vectors"] = int(np.prod(x16.shape[:3]))
    return out


def merge(total: dict, part: dict) -> dict:
    for k in _SUM_KEYS:
        total[k] = total.get(k, 0) + part.get(k, 0)
    for k in _MAX_KEYS:
        total[k] = max(total.get(k, 0.0), part.get(k, 0.0))
    return total


def workers() -> int:
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 4
    return max(1, n)


class Checker:
    """A spawn pool with a bounded number of chunks in flight."""

    def __init__(self, n_workers: int | None = None):
        self.n = n_workers or workers()
        # one BLAS thread per worker (the pool supplies the parallelism); the
        # workers read this from the environment they are spawned with
        keys = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")
        saved = {k: os.environ.get(k) for k in keys}
        for k in keys:
            os.environ[k] = "1"
        try:
            self.pool = mp.get_context("spawn").Pool(self.n)
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        self.pending = []
        self.total: dict = {}
        self.t0 = time.time()

    def submit(self, job: tuple, fn=check_chunk) -> None:
        while len(self.pending) >= 2 * self.n:
            self._drain_one()
        self.pending.append(self.pool.apply_async(fn, (job,)))

    def _drain_one(self) -> None:
        merge(self.total, self.pending.pop(0).get())

    def result(self) -> dict:
        while self.pending:
            self._drain_one()
        out = dict(self.total)
        self.total = {}
        out["oracle_seconds"] = round(time.time() - self.t0, 1)
        out["oracle_workers"] = self.n
        self.t0 = time.time()
        return out

    def close(self) -> None:
        self.pool.close()
        self.pool.join()


def violations(stats: dict) -> dict:
    return {k: v for k, v in stats.items() if "violation" in k and v}


def write_report(key: str, record: dict, path: str = REPORT) -> None:
    """Adds (or replaces) one workload's record in the JSON report."""
    data = {}
    if os.path.exists(path):
        try:
            with open(path) as f:
                data = json.load(f)
        except (OSError, ValueError):
            data = {}
    data[key] = record
    os.makedirs(os.path.dirname(path), exist_ok=True)
    with open(path, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
        f.write("\n")
