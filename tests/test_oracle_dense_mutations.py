"""Planted mistakes in copies of the dense-rotation oracle's steps: each must
fail one of the pins of tests/test_oracle_dense_pins.py (on the CPU)."""

import json
import os

import numpy as np

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden_errors(build):
    """Largest deviation of build(reflectors [k, d], signs, kind) from the
    hand-worked d = 4 rows."""
    with open(os.path.join(HERE, "golden", "householder_d4.json")) as f:
        g = json.load(f)
    signs = np.asarray(g["signs"], np.int8)
    return max(float(np.abs(build(np.asarray(c["reflectors"], float).reshape(-1, 4), signs,
                                  g["kind"]) - np.asarray(c["rows"])).max())
               for c in g["cases"])


def _loop_error(build, kind=0, d=16, k=6, seed=3):
    """Deviation of build(...) x from reflecting the base-rotated x by v_k .. v_1."""
    rng = np.random.default_rng(seed)
    V = rng.standard_normal((k, d))
    s = np.where(rng.random(d) < 0.5, -1, 1).astype(np.int8)
    R = build(V, s, kind)
    x = rng.standard_normal(d)
    y = oracle.rotation_matrix(d, s, kind) @ x
    for i in range(k - 1, -1, -1):
        y = y - 2.0 * V[i] * (V[i] @ y) / (V[i] @ V[i])
    return float(np.abs(R @ x - y).max())


def _orth_error(build, kind=1, d=16, k=8):
    rng = np.random.default_rng(7)
    R = build(rng.standard_normal((k, d)), np.ones(d, np.int8), kind)
    return float(np.abs(R.T @ R - np.eye(d)).max())


def test_the_oracle_itself_passes():
    assert _golden_errors(oracle.householder_matrix) <= 1e-15
    assert _loop_error(oracle.householder_matrix) <= 1e-12
    assert _orth_error(oracle.householder_matrix) <= 1e-12


def test_reflectors_in_the_wrong_order_are_caught():
    def build(V, s, kind):
        R = oracle.rotation_matrix(V.shape[1] if V.size else len(s), s, kind)
        for i in range(V.shape[0]):              # H(v_1) first: wrong
            R = oracle.reflector(V[i]) @ R
        return R
    assert _golden_errors(build) > 0.1
    assert _loop_error(build) > 1e-3


def test_a_reflector_without_its_factor_two_is_caught():
    def build(V, s, kind):
        R = oracle.rotation_matrix(len(s), s, kind)
        for i in range(V.shape[0] - 1, -1, -1):
            v = V[i]
            R = (np.eye(len(v)) - np.outer(v, v) / (v @ v)) @ R   # a projector
        return R
    assert _orth_error(build) > 1e-3


def test_reflectors_without_the_base_rotation_are_caught():
    def build(V, s, kind):
        R = np.eye(len(s))
        for i in range(V.shape[0] - 1, -1, -1):
            R = oracle.reflector(V[i]) @ R
        return R
    assert _golden_errors(build) > 0.1
    assert _loop_error(build) > 1e-3


def test_dequantising_with_the_forward_matrix_is_caught():
    """Applying R instead of R^T on the way back breaks the round trip."""
    rng = np.random.default_rng(1)
    d = 16
    R = oracle.householder_rotations(rng.standard_normal((1, 1, 8, d)),
                                     np.ones((1, 1, d), np.int8), 0)
    x = rng.standard_normal((1, 3, 1, d))
    y = oracle.rotate_dense(x, R)
    wrong = oracle.rotate_dense(y, R)            # R R x instead of R^T R x
    assert np.abs(wrong - x).max() > 1e-3
    assert np.abs(oracle.unrotate_dense(y, R) - x).max() <= 1e-12
