"""Plain float64 statement of the codec with a dense rotation matrix.

Test infrastructure only, like ``srft_oracle``: nothing in the library imports
it. It covers the Householder-rotation variant of "When Quantization Is
Free" (technical summary, Methodology 3, "Householder rotations": at d = 256,
k = d/2 reflectors give practically lossless quantisation; Key Results,
"lossless regime"), and any other rotation given as an explicit matrix.

Readings taken where the pages leave a step open (listed again in the design
notes of the repository):

H1. A Householder reflector of a nonzero vector v is H(v) = I - 2 v v^T /
    (v^T v) (the textbook reflector; v need not be normalised).
H2. The learned rotation sits on top of the fixed random base rotation: the
    pages compare learning a rotation *with* and *without* the SRFT base
    (Methodology 3, learned rotations), so the rotation of a vector is
    R x = H(v_1) H(v_2) ... H(v_k) B x, with B = the SRFT (or SRHT) matrix of
    ``srft_oracle.rotation_matrix`` including its sign diagonal. H(v_k) acts
    first. k = 0 gives B itself.
H3. The pages' reflectors are learned from data, which is not available
    here: the tests draw them from a seeded normal distribution.
H4. Everything after the rotation is the codec of ``srft_oracle``: the same
    lambda rescale, group absmax, binary16 scale, rounding, packing; the
    dequantiser applies R^T.

Layouts: rotation matrices are [S, H, d, d] float64 (y = R x, row n of R
gives output coordinate n); reflectors [S, H, k, d].
"""

from __future__ import annotations

import numpy as np

from .srft_oracle import (
    binary16_bits_to_float,
    float_to_binary16_bits,
    pack_codes,
    quantize_vectors,
    rotation_matrix,
    unpack_codes,
)


def reflector(v: np.ndarray) -> np.ndarray:
    """H(v) = I - 2 v v^T / (v^T v), float64 (reading H1)."""
    v = np.asarray(v, dtype=np.float64)
    vv = float(v @ v)
    if vv == 0.0:
        raise ValueError("a reflector vector must be nonzero")
    return np.eye(v.shape[0]) - (2.0 / vv) * np.outer(v, v)


def householder_matrix(reflectors: np.ndarray, signs_row: np.ndarray, kind: int) -> np.ndarray:
    """R = H(v_1) H(v_2) ... H(v_k) B for one (slice, head), float64 (reading H2).

    reflectors [k, d] (k may be 0); B = rotation_matrix(d, signs_row, kind)."""
    reflectors = np.asarray(reflectors, dtype=np.float64)
    d = np.asarray(signs_row).shape[0]
    R = rotation_matrix(d, signs_row, kind)
    for i in range(reflectors.shape[0] - 1, -1, -1):   # H(v_k) first
        R = reflector(reflectors[i]) @ R
    return R


def householder_rotations(reflectors: np.ndarray, signs: np.ndarray, kind: int) -> np.ndarray:
    """[S, H, d, d] rotation matrices from reflectors [S, H, k, d] and signs [S, H, d]."""
    S, H, _, d = np.asarray(reflectors).shape
    out = np.empty((S, H, d, d), dtype=np.float64)
    for s in range(S):
        for h in range(H):
            out[s, h] = householder_matrix(reflectors[s, h], signs[s, h], kind)
    return out


def rotate_dense(x: np.ndarray, R: np.ndarray) -> np.ndarray:
    """y = R_{s,h} x for every vector of x [S, N, H, d]; float64."""
    x = np.asarray(x)
    S, N, H, d = x.shape
    y = np.empty((S, N, H, d), dtype=np.float64)
    for s in range(S):
        for h in range(H):
            y[s, :, h, :] = x[s, :, h, :].astype(np.float64) @ np.asarray(R[s, h]).T
    return y


def unrotate_dense(y: np.ndarray, R: np.ndarray) -> np.ndarray:
    """x = R_{s,h}^T y for every vector; float64."""
    y = np.asarray(y, dtype=np.float64)
    S, N, H, d = y.shape
    out = np.empty((S, N, H, d), dtype=np.float64)
    for s in range(S):
        for h in range(H):
            out[s, :, h, :] = y[s, :, h, :] @ np.asarray(R[s, h])
    return out


def quantize_dense(x: np.ndarray, R: np.ndarray, lam: np.ndarray, group: int,
                   bits: int) -> dict:
    """The codec's quantiser with the rotation R (reading H4): y = R x, then
    ``quantize_vectors`` and nibble packing, as ``srft_oracle.quantize``."""
    y = rotate_dense(x, R)
    out = quantize_vectors(y, np.asarray(lam, dtype=np.float32)[:, None, :, :], group, bits)
    out["codes"] = pack_codes(out["q"], bits)
    out["scales"] = out["scale_bits"]
    out["y"] = y
    return out


def dequantize_dense(codes: np.ndarray, scales: np.ndarray, R: np.ndarray, lam: np.ndarray,
                     d: int, group: int, bits: int) -> dict:
    """xhat = R^T (lambda * sigma * q), rounded to binary16 (ties to even)."""
    q = unpack_codes(codes, bits)
    if q.shape[-1] != d:
        raise ValueError("codes do not match d")
    sig = binary16_bits_to_float(scales)
    S, N, H, _ = q.shape
    yhat = (q.reshape(S, N, H, d // group, group).astype(np.float64) * sig[..., None])
    yhat = yhat.reshape(S, N, H, d) * np.asarray(lam, np.float32).astype(np.float64)[:, None]
    xhat64 = unrotate_dense(yhat, R)
    return {"bits": float_to_binary16_bits(xhat64), "xhat64": xhat64, "yhat": yhat}


def calibrate_lambda_dense(x: np.ndarray, R: np.ndarray, n_cal: int) -> np.ndarray:
    """lambda [S, H, d]: RMS of rotated coordinate j over the first n_cal rows
    (1 where the sum of squares is zero), as ``srft_oracle.calibrate_lambda``."""
    x = np.asarray(x)
    if n_cal < 1 or n_cal > x.shape[1]:
        raise ValueError("n_cal must be in [1, N]")
    y = rotate_dense(x[:, :n_cal], R)
    ss = np.sum(y * y, axis=1)
    return np.where(ss == 0.0, 1.0, np.sqrt(ss / n_cal))


def split_operand(R32: np.ndarray) -> tuple:
    """(hi, lo) binary16 bit patterns of a float32 matrix: hi = binary16(R),
    lo = binary16(R - hi), both rounded to nearest even; hi + lo carries
    about 22 significant bits of R."""
    R32 = np.asarray(R32, dtype=np.float32).astype(np.float64)
    hi = float_to_binary16_bits(R32)
    lo = float_to_binary16_bits(R32 - binary16_bits_to_float(hi))
    return hi, lo
