"""Seeded synthetic KV-cache inputs shaped like the paper's workloads.

This module only draws random numbers: fp16 key/value tensors, Rademacher sign
tables and outlier masks. It holds none of the codec's arithmetic, so both the
CPU oracle (tests) and the CUDA library (tests, bench) can take their inputs
from it without sharing any of the method.

No public dataset or model is used: the "Qwen2.5-1.5B-like" and "Gemma-3-like"
names only fix shapes (layers, KV heads, head dim, sequence length) and the
value distributions described per workload below.

Two backends draw the values:

* ``numpy``: ``numpy.random.default_rng`` seeded per (seed, slice[, head]); used
  for the small workloads and for any input the oracle checks in full.
* ``torch``: a seeded ``torch.Generator`` on the target device, one stream
  per slice; used for the multi-GB workloads. The two backends give
  different (each reproducible) values.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    S: int           # slices (layers x {K, V})
    N: int           # rows per slice (tokens, or token x batch)
    H: int           # KV heads
    d: int           # head dim
    bits: int
    group: int
    dist: str        # "normal" or "student_t4"
    outlier: str     # "none", "coord", "channel"
    outlier_p: float
    outlier_scale: float
    n_cal: int = 512
    rotations: tuple = (0,)
    note: str = ""
    reflectors: int = 0   # Householder reflectors on the base rotation (dense codec)
    dense_base: bool = False   # the base rotation itself as a dense product (k = 0)

    @property
    def dense(self) -> bool:
        """The rotation runs as a dense d x d product (the tensor-core codec):
        always with reflectors, and for the plain SRFT / SRHT matrix when
        dense_base is set."""
        return self.reflectors > 0 or self.dense_base

    @property
    def vectors(self) -> int:
        return self.S * self.N * self.H

    def bytes_per_vector(self) -> int:
        """fp16 vector + codes + fp16 scales: the bytes one quantize (or one
        dequantize) moves per vector."""
        return 2 * self.d + self.d * self.bits // 8 + 2 * (self.d // self.group)


WORKLOADS = {
    "tiny_d64": Workload(
        "tiny_d64", S=1, N=4096, H=1, d=64, bits=4, group=16, dist="normal",
        outlier="coord", outlier_p=0.01, outlier_scale=20.0,
        note="4096 vectors, d=64, N(0,1) seed 0 with 1% of coordinates x20; "
             "Rademacher signs seed 1; lambda from the first 512 vectors; int4 G16"),
    "qwen_like_d128": Workload(
        "qwen_like_d128", S=56, N=32768, H=2, d=128, bits=4, group=16, dist="normal",
        outlier="channel", outlier_p=4, outlier_scale=30.0,
        note="28 layers x {K,V}, 2 KV heads, d=128, seq 32768, batch 1; N(0,1) plus "
             "4 fixed channels per (layer, K/V, head) x30; int4 G16"),
    "longctx_int8_d128": Workload(
        "longctx_int8_d128", S=2, N=131072, H=8, d=128, bits=8, group=16,
        dist="student_t4", outlier="none", outlier_p=0.0, outlier_scale=1.0,
        rotations=(0, 1),
        note="1 layer x {K,V}, 8 KV heads, d=128, seq 131072; Student-t(4)/sqrt(2); "
             "int8 G16; SRFT and SRHT"),
    "gemma_like_d256": Workload(
        "gemma_like_d256", S=4, N=32768, H=4, d=256, bits=4, group=32, dist="normal",
        outlier="coord", outlier_p=0.005, outlier_scale=25.0,
        note="2 layers x {K,V}, 4 KV heads, d=256, batch 4 x seq 8192 rows; N(0,1) "
             "with 0.5% of coordinates x25; int4 G32"),
    "householder_d256": Workload(
        "householder_d256", S=4, N=32768, H=4, d=256, bits=4, group=32, dist="normal",
        outlier="coord", outlier_p=0.005, outlier_scale=25.0, reflectors=128,
        note="the gemma_like_d256 shape with a dense rotation: k = d/2 = 128 Householder "
             "reflectors (seeded N(0,1) vectors standing in for learned ones) on the SRFT "
             "base; int4 G32"),
    "decode_stream_d128": Workload(
        "decode_stream_d128", S=64, N=32768 * 32, H=8, d=128, bits=4, group=16,
        dist="normal", outlier="none", outlier_p=0.0, outlier_scale=1.0,
        note="32 layers x {K,V}, batch 32, 8 KV heads, d=128, int4 cache of 32768 "
             "tokens per sequence (rows = token*32 + batch); each step appends one "
             "token per sequence and layer, then dequantizes the whole cache"),
}


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, *key]))


def rademacher_signs(S: int, H: int, d: int, seed: int) -> np.ndarray:
    """int8 +-1 sign table [S, H, d], one independent row per (slice, head)."""
    out = np.empty((S, H, d), dtype=np.int8)
    for s in range(S):
        for h in range(H):
            out[s, h] = np.where(_rng(seed, s, h).random(d) < 0.5, -1, 1)
    return out


def householder_reflectors(S: int, H: int, k: int, d: int, seed: int) -> np.ndarray:
    """float32 reflector vectors [S, H, k, d] drawn N(0, 1), one independent
    set per (slice, head). The pages' reflectors are learned from data; these
    stand in for them (they only need to be nonzero)."""
    out = np.empty((S, H, k, d), dtype=np.float32)
    for s in range(S):
        for h in range(H):
            out[s, h] = _rng(seed, s, h, 11).standard_normal((k, d))
    return out


def _values_numpy(w: Workload, s: int, seed: int, n_rows: int) -> np.ndarray:
    rng = _rng(seed, s)
    shape = (n_rows, w.H, w.d)
    if w.dist == "normal":
        x = rng.standard_normal(shape)
    elif w.dist == "student_t4":
        x = rng.standard_t(4.0, size=shape) / math.sqrt(2.0)   # unit variance
    else:
        raise ValueError(w.dist)
    if w.outlier == "coord":
        x = np.where(rng.random(shape) < w.outlier_p, x * w.outlier_scale, x)
    elif w.outlier == "channel":
        for h in range(w.H):
            ch = _rng(seed, s, h, 7).choice(w.d, size=int(w.outlier_p), replace=False)
            x[:, h, ch] *= w.outlier_scale
    return x


def make_x_numpy(w: Workload, seed: int = 0, n_rows: int | None = None,
                 slices: range | None = None) -> np.ndarray:
    """fp16 x [len(slices), n_rows, H, d] drawn with numpy."""
    n_rows = w.N if n_rows is None else n_rows
    slices = range(w.S) if slices is None else slices
    out = np.empty((len(slices), n_rows, w.H, w.d), dtype=np.float16)
    for i, s in enumerate(slices):
        out[i] = _values_numpy(w, s, seed, n_rows).astype(np.float16)
    return out


def tiny_inputs():
    """The tiny codec check exactly as specified: values from seed 0 (then the
    1% outlier mask from the same stream), signs from seed 1."""
    w = WORKLOADS["tiny_d64"]
    rng = np.random.default_rng(0)
    x = rng.standard_normal((w.N, w.d))
    x = np.where(rng.random((w.N, w.d)) < w.outlier_p, x * w.outlier_scale, x)
    signs = np.where(np.random.default_rng(1).random(w.d) < 0.5, -1, 1).astype(np.int8)
    return x.astype(np.float16).reshape(1, w.N, 1, w.d), signs.reshape(1, 1, w.d)


def make_x_torch(w: Workload, device, seed: int = 0, n_rows: int | None = None,
                 slices: range | None = None, out=None):
    """fp16 x [len(slices), n_rows, H, d] drawn on `device` with torch.

    Student-t(4) is drawn as Z / sqrt(chi2_4 / 4) from five normals; outlier
    masks come from the same per-slice generator.
    """
    import torch

    n_rows = w.N if n_rows is None else n_rows
    slices = range(w.S) if slices is None else slices
    if out is None:
        out = torch.empty((len(slices), n_rows, w.H, w.d), dtype=torch.float16, device=device)
    g = torch.Generator(device=device)
    for i, s in enumerate(slices):
        g.manual_seed(int(np.random.SeedSequence([seed, s]).generate_state(1)[0]))
        shape = (n_rows, w.H, w.d)
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        if w.dist == "student_t4":
            chi = torch.zeros(shape, device=device, dtype=torch.float32)
            for _ in range(4):
                chi += torch.randn(shape, generator=g, device=device, dtype=torch.float32) ** 2
            x = x / torch.sqrt(chi / 4.0) / math.sqrt(2.0)
        if w.outlier == "coord":
            m = torch.rand(shape, generator=g, device=device) < w.outlier_p
            x = torch.where(m, x * w.outlier_scale, x)
        elif w.outlier == "channel":
            for h in range(w.H):
                ch = _rng(seed, s, h, 7).choice(w.d, size=int(w.outlier_p), replace=False)
                x[:, h, torch.as_tensor(ch, device=device)] *= w.outlier_scale
        out[i].copy_(x.to(torch.float16))
        del x
    return out
