"""Comparison of CUDA results with the CPU oracle, with the stated tolerances.

Tolerances (fixed before any kernel ran):

* rotated values (float32): |y_gpu - y_ref| <= 1e-5 * max(|y_ref|, rms of the
  reference vector); the floor keeps coordinates near zero from failing on
  absolute noise.
* group scales (binary16): bit-equal, except where the oracle's
  absmax / qmax lies within 1e-6 (relative) of the rounding midpoint between
  the two binary16 values the sides chose; such groups are counted and their
  codes left out of the code comparison.
* codes: bit-equal, except where the oracle's pre-rounding value w / sigma
  lies within 1e-4 code units of a rounding boundary (k + 1/2, or the clamp
  edge qmax + 1/2); such codes must differ by exactly one step and are
  counted.
* dequantised output: |xhat_gpu - xhat_ref| <= 1e-3 * max(1, |xhat_ref|),
  both sides dequantising the oracle's codes and scales (or, for a GPU
  round trip, the vectors whose GPU codes and scales equal the oracle's);
  values beyond the binary16 range round to the same infinity on both sides
  and count as equal.
* lambda (calibration): relative 1e-5.
* dense-rotation codec: both bands follow from the rotation tolerance
  instead. Its rotation is a float32 product summing d terms per coordinate
  (on the tensor cores, d fp16 products per half of the operand): the FFT's
  rotated values carry ~1e-7 relative error, the dense product's ~1e-6 at
  d = 256. A rotated value within the 1e-5 rotation tolerance moves
  absmax / qmax by at most 1e-5 relative (scale band 1e-5), and moves
  w_j / sigma_g by at most 1e-5 max(|y_j|, rms(y)) / (lambda_j sigma_g)
  code units (code band: that, or 1e-4 where it is smaller). The latter
  matters for int8 (127 levels), whose code unit is 18 times finer than
  int4's.
"""

from __future__ import annotations

import numpy as np

import oracle

CODE_BAND = 1e-4
SCALE_BAND = 1e-6
ROT_TOL = 1e-5
DEQ_TOL = 1e-3
LAM_TOL = 1e-5
DENSE_SCALE_BAND = 1e-5


def check_rotation(y_gpu: np.ndarray, y_ref: np.ndarray) -> dict:
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    rms = np.sqrt(np.mean(y_ref * y_ref, axis=-1, keepdims=True))
    floor = np.maximum(np.abs(y_ref), rms)
    err = np.abs(y_gpu - y_ref) / np.where(floor > 0, floor, 1.0)
    bad = int(np.sum(err > ROT_TOL))
    return {"max_rel_err": float(err.max(initial=0.0)), "violations": bad}


def dense_code_band(ref: dict, lam: np.ndarray, group: int) -> np.ndarray:
    """Per-coordinate code band of the dense codec (see the module docstring):
    max(1e-4, 1e-5 max(|y_j|, rms(y)) / (lambda_j sigma_g)) in code units,
    from the oracle's rotated values y and scales; lam [S, H, d]."""
    y = np.asarray(ref["y"], np.float64)
    rms = np.sqrt(np.mean(y * y, axis=-1, keepdims=True))
    sig = oracle.binary16_bits_to_float(ref["scale_bits"]).repeat(group, axis=-1)
    lam_b = np.asarray(lam, np.float32).astype(np.float64)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        band = ROT_TOL * np.maximum(np.abs(y), rms) / (lam_b * sig)
    return np.maximum(CODE_BAND, np.nan_to_num(band, nan=CODE_BAND, posinf=CODE_BAND))


def check_codes(ref: dict, codes_gpu: np.ndarray, scales_gpu: np.ndarray, bits: int,
                group: int, scale_band: float = SCALE_BAND, code_band=None) -> dict:
    """ref: output of oracle.quantize (or quantize_vectors + pack) on the same inputs.

    Groups whose oracle scale is zero (sigma = 0: the group's absmax rounds
    to zero) must have all-zero codes on both sides; they are counted and any
    nonzero code there is a violation. Every other group is compared as the
    tolerances above say."""
    qmax = oracle.qmax_for(bits)
    q_gpu = oracle.unpack_codes(codes_gpu, bits)
    q_ref = ref["q"]
    s_ref = np.asarray(ref["scale_bits"]).astype(np.int64)
    s_gpu = np.asarray(scales_gpu).view(np.uint16).astype(np.int64)
    shape_g = s_ref.shape
    # scale mismatches: adjacent binary16 values, oracle value near their midpoint
    smis = s_ref != s_gpu
    v_ref = oracle.binary16_bits_to_float(s_ref)
    v_gpu = oracle.binary16_bits_to_float(s_gpu)
    mid = 0.5 * (v_ref + v_gpu)
    pre_s = ref["scale_pre"]
    near_mid = np.abs(pre_s - mid) <= scale_band * np.maximum(np.abs(pre_s), 1e-30)
    scale_ok = (~smis) | (near_mid & (np.abs(s_ref - s_gpu) == 1))
    scale_viol = int(np.sum(~scale_ok))
    qg_ref = q_ref.reshape(shape_g + (group,))
    qg_gpu = q_gpu.reshape(shape_g + (group,))
    # sigma = 0 groups (equal on both sides): every code must be zero
    zero = (~smis) & (v_ref == 0)
    zero_viol = int(np.sum(zero[..., None] & ((qg_gpu != 0) | (qg_ref != 0))))
    # codes of the other groups whose scales agree
    cmp = (~smis & ~zero)[..., None] & np.ones_like(qg_ref, dtype=bool)
    cmis = cmp & (qg_ref != qg_gpu)
    pre = np.abs(ref["pre"].reshape(shape_g + (group,)))
    pre = np.where(zero[..., None], 0.0, pre)    # w / 0 is not a rounding position
    frac = pre - np.floor(pre)
    cb = CODE_BAND if code_band is None else np.asarray(code_band).reshape(pre.shape)
    near_half = np.abs(frac - 0.5) < cb
    near_clamp = np.abs(pre - (qmax + 0.5)) < cb
    one_step = np.abs(qg_ref - qg_gpu) == 1
    allowed = (near_half | near_clamp) & one_step
    code_viol = int(np.sum(cmis & ~allowed))
    return {
        "codes": int(np.sum(cmp)),
        "code_mismatch_in_band": int(np.sum(cmis & allowed)),
        "code_violations": code_viol,
        "scale_mismatch_in_band": int(np.sum(smis & scale_ok)),
        "scale_violations": scale_viol,
        "groups_excluded": int(np.sum(smis)),
        "zero_scale_groups": int(np.sum(zero)),
        "zero_scale_violations": zero_viol,
    }


def check_dequant(xhat_gpu_bits: np.ndarray, xhat_ref_bits: np.ndarray) -> dict:
    a = oracle.binary16_bits_to_float(np.asarray(xhat_gpu_bits).view(np.uint16))
    r = oracle.binary16_bits_to_float(np.asarray(xhat_ref_bits).view(np.uint16))
    same_inf = np.isinf(a) & np.isinf(r) & (np.sign(a) == np.sign(r))
    finite = np.isfinite(a) & np.isfinite(r)
    a0, r0 = np.where(finite, a, 0.0), np.where(finite, r, 0.0)
    err = np.abs(a0 - r0)
    tol = DEQ_TOL * np.maximum(1.0, np.abs(r0))
    ok = same_inf | (finite & (err <= tol))
    return {"max_abs_err": float(err.max(initial=0.0)),
            "max_err_over_tol": float((err / tol).max(initial=0.0)),
            "overflow_to_inf": int(np.sum(same_inf)),
            "violations": int(np.sum(~ok))}


def check_lambda(lam_gpu: np.ndarray, lam_ref: np.ndarray) -> dict:
    # lambda_j^2 is the mean of y_j^2, and each rotated y_j carries an absolute
    # error of about ROT_TOL times the vector's RMS (see check_rotation). So
    # lambda_j inherits an absolute error of about ROT_TOL times the RMS of its
    # (slice, head) row of lambdas; with few calibration rows a coordinate can
    # sit near zero, and the relative test uses that RMS as its floor.
    rms = np.sqrt(np.mean(lam_ref * lam_ref, axis=-1, keepdims=True))
    floor = np.maximum(np.abs(lam_ref), rms)
    rel = np.abs(np.asarray(lam_gpu, np.float64) - lam_ref) / np.where(floor > 0, floor, 1.0)
    return {"max_rel_err": float(rel.max(initial=0.0)), "violations": int(np.sum(rel > LAM_TOL))}


def assert_clean(stats: dict, what: str) -> None:
    bad = {k: v for k, v in stats.items() if "violation" in k and v}
    assert not bad, f"{what}: {stats}"
