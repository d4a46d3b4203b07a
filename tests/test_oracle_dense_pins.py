"""Pins of the dense-rotation oracle (oracle/dense_oracle.py): the
Householder variant of "When Quantization Is Free" (Methodology 3) and the
codec with a rotation given as an explicit matrix.

Each pin is something the mathematics or a hand-worked example fixes, not a
retyping of the oracle's own formula: reflector identities, orthogonality,
the order of the product against a plain loop that applies the reflectors
one at a time, hand-worked d = 4 matrices, the reduction to the pinned SRFT /
SRHT codec when there are no reflectors, and the orthogonal error bound.
"""

import json
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def _refl(rng, S, H, k, d):
    return rng.standard_normal((S, H, k, d))


def _signs(rng, S, H, d):
    return np.where(rng.random((S, H, d)) < 0.5, -1, 1).astype(np.int8)


@pytest.mark.parametrize("d", [4, 16, 128])
def test_reflector_is_a_symmetric_involution_that_flips_v(d):
    rng = np.random.default_rng(d)
    v = rng.standard_normal(d)
    Hm = oracle.reflector(v)
    assert np.abs(Hm - Hm.T).max() <= 1e-14
    assert np.abs(Hm @ Hm - np.eye(d)).max() <= 1e-13
    assert np.abs(Hm @ v + v).max() <= 1e-12 * np.linalg.norm(v)
    u = rng.standard_normal(d)
    u -= (u @ v) / (v @ v) * v                     # u orthogonal to v
    assert np.abs(Hm @ u - u).max() <= 1e-12 * np.linalg.norm(u)
    # the scale of v does not matter
    assert np.abs(oracle.reflector(3.5 * v) - Hm).max() <= 1e-14
    with pytest.raises(ValueError):
        oracle.reflector(np.zeros(d))


@pytest.mark.parametrize("kind", [0, 1])
@pytest.mark.parametrize("d,k", [(4, 2), (16, 8), (64, 32), (256, 128), (256, 1)])
def test_householder_rotation_is_orthogonal(kind, d, k):
    rng = np.random.default_rng(d * 3 + k + kind)
    R = oracle.householder_rotations(_refl(rng, 1, 1, k, d), _signs(rng, 1, 1, d), kind)[0, 0]
    assert np.abs(R.T @ R - np.eye(d)).max() <= 1e-12
    x = rng.standard_normal(d)
    assert abs(np.linalg.norm(R @ x) - np.linalg.norm(x)) <= 1e-12 * np.linalg.norm(x)


@pytest.mark.parametrize("kind", [0, 1])
def test_product_order_against_one_reflector_at_a_time(kind):
    """R x must equal: rotate by the signed base, then reflect by v_k, v_{k-1},
    ..., v_1 in turn, each reflection written as x - 2 v (v.x) / (v.v)."""
    rng = np.random.default_rng(11 + kind)
    d, k = 32, 16
    V = _refl(rng, 1, 1, k, d)
    s = _signs(rng, 1, 1, d)
    R = oracle.householder_rotations(V, s, kind)[0, 0]
    B = oracle.rotation_matrix(d, s[0, 0], kind)
    for _ in range(5):
        x = rng.standard_normal(d)
        y = B @ x
        for i in range(k - 1, -1, -1):
            v = V[0, 0, i]
            y = y - 2.0 * v * (v @ y) / (v @ v)
        assert np.abs(R @ x - y).max() <= 1e-12


def test_hand_worked_d4_householder_rows():
    with open(os.path.join(HERE, "golden", "householder_d4.json")) as f:
        g = json.load(f)
    signs = np.asarray(g["signs"], np.int8)
    for case in g["cases"]:
        V = np.asarray(case["reflectors"], np.float64).reshape(-1, 4)
        R = oracle.householder_matrix(V, signs, g["kind"])
        assert np.abs(R - np.asarray(case["rows"])).max() <= 1e-15, case


@pytest.mark.parametrize("kind", [0, 1])
def test_no_reflectors_is_the_pinned_base_codec(kind):
    """With k = 0 the dense codec is the SRFT / SRHT codec of srft_oracle,
    which its own pins fix: identical codes, scales and dequantisation."""
    rng = np.random.default_rng(5 + kind)
    S, N, H, d, group, bits = 2, 9, 3, 64, 16, 4
    x16 = rng.standard_normal((S, N, H, d)).astype(np.float16)
    signs = _signs(rng, S, H, d)
    lam = np.exp(rng.uniform(-1, 1, (S, H, d))).astype(np.float32)
    R = oracle.householder_rotations(np.zeros((S, H, 0, d)), signs, kind)
    a = oracle.quantize_dense(x16, R, lam, group, bits)
    b = oracle.quantize(x16, signs, lam, group, bits, kind)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])
    da = oracle.dequantize_dense(a["codes"], a["scales"], R, lam, d, group, bits)
    db = oracle.dequantize(b["codes"], b["scales"], signs, lam, d, group, bits, kind)
    assert np.array_equal(da["bits"], db["bits"])
    la = oracle.calibrate_lambda_dense(x16, R, N)
    lb = oracle.calibrate_lambda(x16, signs, N, kind)
    assert np.abs(la - lb).max() <= 1e-12 * np.abs(lb).max()


def test_dense_roundtrip_and_error_bound():
    """Unrotate inverts rotate exactly (R orthogonal), and the dequantised
    vector is within ||lambda * sigma / 2|| of x (orthogonality), before the
    binary16 output rounding."""
    rng = np.random.default_rng(8)
    S, N, H, d, k, group, bits = 1, 200, 2, 256, 128, 32, 4
    x16 = (rng.standard_normal((S, N, H, d)) *
           np.where(rng.random((S, N, H, d)) < 0.005, 25.0, 1.0)).astype(np.float16)
    R = oracle.householder_rotations(_refl(rng, S, H, k, d), _signs(rng, S, H, d), 0)
    y = oracle.rotate_dense(x16, R)
    back = oracle.unrotate_dense(y, R)
    assert np.abs(back - x16.astype(np.float64)).max() <= 1e-12 * float(np.abs(x16).max())
    lam = oracle.calibrate_lambda_dense(x16, R, 128).astype(np.float32)
    q = oracle.quantize_dense(x16, R, lam, group, bits)
    dq = oracle.dequantize_dense(q["codes"], q["scales"], R, lam, d, group, bits)
    sig = oracle.binary16_bits_to_float(q["scales"]).repeat(group, axis=-1)
    bound = np.linalg.norm(sig * lam[:, None].astype(np.float64) / 2, axis=-1)
    err = np.linalg.norm(dq["xhat64"] - x16.astype(np.float64), axis=-1)
    assert np.all(err <= bound * (1 + 1e-9) + 1e-9)


def test_calibration_of_a_dense_rotation_closed_form():
    """A single calibration row x gives lambda_j = |(R x)_j| (1 where it is 0)."""
    rng = np.random.default_rng(2)
    d = 16
    R = oracle.householder_rotations(_refl(rng, 1, 1, 8, d), _signs(rng, 1, 1, d), 1)
    x = rng.standard_normal((1, 1, 1, d)).astype(np.float16)
    lam = oracle.calibrate_lambda_dense(x, R, 1)[0, 0]
    y = R[0, 0] @ x[0, 0, 0].astype(np.float64)
    assert np.abs(lam - np.where(y == 0, 1.0, np.abs(y))).max() <= 1e-15


def test_operand_split_is_two_binary16_roundings():
    """hi is the binary16 rounding of R (numpy's float16 conversion is a
    special case of it), lo the binary16 rounding of the remainder, and
    hi + lo reproduces R to about 2^-22 of its magnitude."""
    rng = np.random.default_rng(4)
    R32 = (rng.standard_normal((2, 3, 16, 16)) / 4).astype(np.float32)
    hi, lo = oracle.split_operand(R32)
    assert np.array_equal(hi, R32.astype(np.float16).view(np.uint16))
    rem = R32.astype(np.float64) - R32.astype(np.float16).astype(np.float64)
    assert np.array_equal(lo, rem.astype(np.float16).view(np.uint16))
    back = oracle.binary16_bits_to_float(hi) + oracle.binary16_bits_to_float(lo)
    assert np.abs(back - R32).max() <= 2.0 ** -22 * np.abs(R32).max()
