"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test ties an oracle function to a closed form, a textbook or library
special case, a brute-force computation on tiny inputs, or a hand-worked
example stored under tests/golden/ with its citation. The checks are written as
helpers that take the function under test, so tests/test_oracle_mutations.py
can feed them deliberately broken variants and show that each plausible
mistake is caught.
"""

import cmath
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg

import oracle
from oracle import srft_oracle as so

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
DIMS = [2, 4, 8, 16, 32, 64, 128, 256]


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _parse(expr):
    table = {"1/2": 0.5, "-1/2": -0.5, "0": 0.0,
             "1/sqrt2": 1 / math.sqrt(2), "-1/sqrt2": -1 / math.sqrt(2)}
    return table[expr]


def _rand_signs(rng, d):
    return np.where(rng.random(d) < 0.5, -1, 1).astype(np.int8)


# ---------------------------------------------------------------------------
# Helpers that measure one property of a given implementation
# ---------------------------------------------------------------------------

def orthogonality_error(matrix_fn, d):
    R = matrix_fn(d)
    return float(np.max(np.abs(R.T @ R - np.eye(d))))


def rfft_special_case_error(matrix_fn, d, seed=0):
    """SRFT against numpy.fft.rfft(s*x, norm='ortho') packed by reading 1."""
    rng = np.random.default_rng(seed)
    s = _rand_signs(rng, d)
    x = rng.standard_normal((5, d))
    X = np.fft.rfft(s * x, norm="ortho")
    packed = np.empty((5, d))
    packed[:, 0] = X[:, 0].real
    packed[:, 1] = X[:, d // 2].real
    packed[:, 2::2] = math.sqrt(2) * X[:, 1:d // 2].real
    packed[:, 3::2] = math.sqrt(2) * X[:, 1:d // 2].imag
    R = matrix_fn(d) * np.where(s < 0, -1.0, 1.0)[None, :]
    return float(np.max(np.abs(x @ R.T - packed)))


def brute_force_dft_error(matrix_fn, d):
    """Columns of P.F from a pure-Python complex DFT summation + pack."""
    R = matrix_fn(d)
    worst = 0.0
    for n in range(d):
        e = [0.0] * d
        e[n] = 1.0
        X = []
        for k in range(d // 2 + 1):
            acc = 0j
            for m in range(d):
                acc += e[m] * cmath.exp(-2j * math.pi * k * m / d)
            X.append(acc / math.sqrt(d))
        col = [X[0].real, X[d // 2].real]
        for k in range(1, d // 2):
            col += [math.sqrt(2) * X[k].real, math.sqrt(2) * X[k].imag]
        worst = max(worst, max(abs(col[j] - R[j, n]) for j in range(d)))
    return worst


def hadamard_special_case_error(matrix_fn, d, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((5, d))
    H = scipy.linalg.hadamard(d) / math.sqrt(d)
    return float(np.max(np.abs(x @ matrix_fn(d).T - x @ H.T)))


def golden_quant_mismatches(quant_fn):
    bad = []
    for case in _load("group_quant.json")["cases"]:
        w = np.array([case["w"]], dtype=np.float64)
        out = quant_fn(w, np.ones_like(w), 4, case["bits"])
        sig = int(out["scale_bits"][0, 0])
        if sig != int(case["sigma_bits"], 16) or list(out["q"][0]) != case["q"]:
            bad.append((case["note"], hex(sig), list(out["q"][0])))
    return bad


def golden_pack_mismatches(pack_fn):
    bad = []
    for case in _load("int4_packing.json")["cases"]:
        b = int(pack_fn(np.array([case["q"]]), 4)[0, 0])
        if b != int(case["byte"], 16):
            bad.append((case["q"], hex(b)))
    return bad


def lossless_roundtrip_error(quantize_fn, dequantize_fn, kind, d=32, group=8, bits=4, seed=3):
    """Vectors whose rotation lies exactly on the code grid must come back exactly."""
    rng = np.random.default_rng(seed)
    S, N, H = 2, 6, 3
    qmax = oracle.qmax_for(bits)
    signs = np.where(rng.random((S, H, d)) < 0.5, -1, 1).astype(np.int8)
    lam = np.exp2(rng.integers(-2, 3, size=(S, H, d))).astype(np.float32)
    q = rng.integers(-qmax, qmax + 1, size=(S, N, H, d // group, group))
    q[..., 0] = qmax                                  # absmax = qmax * sigma
    sig_bits = oracle.float_to_binary16_bits(
        np.exp2(rng.integers(-6, 4, size=(S, N, H, d // group))) * rng.choice([1.0, 1.25, 1.5], size=(S, N, H, d // group)))
    sig = oracle.binary16_bits_to_float(sig_bits)
    y = (q * sig[..., None]).reshape(S, N, H, d) * lam[:, None].astype(np.float64)
    x = so.unrotate(y, signs, kind)
    out = quantize_fn(x, signs, lam, group, bits, kind)
    code_err = int(np.sum(out["q"] != q.reshape(S, N, H, d)))
    back = dequantize_fn(out["codes"], out["scales"], signs, lam, d, group, bits, kind)
    return code_err, float(np.max(np.abs(back["xhat64"] - x)))


# ---------------------------------------------------------------------------
# Rotation pins
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d", DIMS)
@pytest.mark.parametrize("fn", [oracle.srft_matrix, oracle.srht_matrix], ids=["srft", "srht"])
def test_rotation_is_orthogonal(fn, d):
    assert orthogonality_error(fn, d) <= 1e-12


@pytest.mark.parametrize("kind", [oracle.SRFT, oracle.SRHT])
@pytest.mark.parametrize("d", [4, 16, 64, 256])
def test_parseval_and_roundtrip(kind, d):
    rng = np.random.default_rng(d + 7 * kind)
    S, N, H = 2, 9, 3
    x = rng.standard_normal((S, N, H, d))
    signs = np.where(rng.random((S, H, d)) < 0.5, -1, 1).astype(np.int8)
    y = oracle.rotate(x, signs, kind)
    nx = np.linalg.norm(x, axis=-1)
    ny = np.linalg.norm(y, axis=-1)
    assert np.max(np.abs(ny - nx) / nx) <= 1e-12
    back = oracle.unrotate(y, signs, kind)
    assert np.max(np.abs(back - x)) <= 1e-12 * np.max(nx)


def test_d4_rows_hand_worked():
    g = _load("srft_d4_rows.json")
    want = np.array([[_parse(e) for e in row] for row in g["rows"]])
    assert np.max(np.abs(oracle.srft_matrix(4) - want)) <= 1e-15


@pytest.mark.parametrize("d", [4, 8])
def test_brute_force_complex_dft(d):
    assert brute_force_dft_error(oracle.srft_matrix, d) <= 1e-14


@pytest.mark.parametrize("d", [2, 4, 8, 32, 128, 256])
def test_numpy_rfft_special_case(d):
    assert rfft_special_case_error(oracle.srft_matrix, d) <= 1e-12


@pytest.mark.parametrize("d", [2, 4, 8, 32, 128, 256])
def test_scipy_hadamard_special_case(d):
    assert hadamard_special_case_error(oracle.srht_matrix, d) <= 1e-13


def test_signs_apply_to_input_coordinates():
    """R diag(s) x == R (s*x): the sign vector multiplies the input (Methodology 1)."""
    rng = np.random.default_rng(11)
    d = 16
    x = rng.standard_normal((1, 4, 1, d))
    s = _rand_signs(rng, d)[None, None, :]
    y = oracle.rotate(x, s, oracle.SRFT)
    y2 = x[0, :, 0, :] @ (oracle.srft_matrix(d) @ np.diag(np.where(s[0, 0] < 0, -1.0, 1.0))).T
    assert np.max(np.abs(y[0, :, 0, :] - y2)) <= 1e-13
    # zero entries of the sign table count as +1
    s0 = np.zeros_like(s)
    assert np.allclose(oracle.rotate(x, s0, oracle.SRFT)[0, :, 0, :],
                       x[0, :, 0, :] @ oracle.srft_matrix(d).T, atol=1e-13)


@pytest.mark.parametrize("kind", [oracle.SRFT, oracle.SRHT])
def test_isotropy_on_gaussian_input(kind):
    """x ~ N(0, I) rotates to N(0, I): every packed coordinate has variance 1."""
    rng = np.random.default_rng(5)
    d, n = 64, 200_000
    x = rng.standard_normal((1, n, 1, d))
    signs = _rand_signs(rng, d)[None, None, :]
    y = oracle.rotate(x, signs, kind)[0, :, 0, :]
    var = np.mean(y * y, axis=0)
    assert np.max(np.abs(var - 1.0)) <= 0.02


# ---------------------------------------------------------------------------
# binary16 pins
# ---------------------------------------------------------------------------

def test_binary16_matches_numpy_on_random_ties_and_subnormals():
    rng = np.random.default_rng(0)
    n = 1_000_000
    wide = rng.standard_normal(n) * np.exp2(rng.uniform(-30, 17, n))
    E = rng.integers(-14, 16, n // 4)
    k = rng.integers(1024, 2048, n // 4)
    ties = (2 * k + 1) * np.exp2(E - 11.0) * rng.choice([-1, 1], n // 4)
    sub_ties = (2 * rng.integers(0, 1024, n // 4) + 1) * 2.0 ** -25
    edge = np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9,
                     2.0 ** -24, 2.0 ** -25, 2.0 ** -26, 2.0 ** -14, np.inf, -np.inf])
    v = np.concatenate([wide, ties, sub_ties, edge])
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    got = oracle.float_to_binary16_bits(v)
    assert int(np.sum(got != ref)) == 0
    assert int(oracle.float_to_binary16_bits(np.array([np.nan]))[0]) & 0x7C00 == 0x7C00


def test_binary16_decode_matches_numpy():
    allbits = np.arange(65536, dtype=np.uint16)
    ref = allbits.view(np.float16).astype(np.float64)
    got = oracle.binary16_bits_to_float(allbits)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))


def test_binary16_saturation():
    assert int(oracle.float_to_binary16_bits(np.array([1e6]), saturate=True)[0]) == 0x7BFF
    assert int(oracle.float_to_binary16_bits(np.array([-1e6]), saturate=True)[0]) == 0xFBFF


# ---------------------------------------------------------------------------
# Quantiser pins
# ---------------------------------------------------------------------------

def test_int4_packing_hand_worked():
    assert golden_pack_mismatches(oracle.pack_codes) == []


@pytest.mark.parametrize("bits", [4, 8])
def test_pack_unpack_roundtrip(bits):
    rng = np.random.default_rng(bits)
    qmax = oracle.qmax_for(bits)
    q = rng.integers(-qmax - 1, qmax + 1, size=(3, 5, 64))
    assert np.array_equal(oracle.unpack_codes(oracle.pack_codes(q, bits), bits), q)


def test_group_quantisation_hand_worked():
    assert golden_quant_mismatches(oracle.quantize_vectors) == []


def test_group_membership_brute_force():
    """Per-group absmax over G consecutive coordinates, checked with plain loops."""
    rng = np.random.default_rng(2)
    d, G, bits = 16, 4, 4
    w = rng.standard_normal((7, d)) * np.exp2(rng.integers(-3, 4, (7, d)))
    out = oracle.quantize_vectors(w, np.ones(d), G, bits)
    for r in range(7):
        for g in range(d // G):
            a = max(abs(float(np.float32(w[r, j]))) for j in range(g * G, (g + 1) * G))
            sig = float(oracle.binary16_bits_to_float(out["scale_bits"][r, g]))
            want_bits = int(oracle.float_to_binary16_bits(np.float64(np.float32(a) / np.float32(7))))
            assert int(out["scale_bits"][r, g]) == want_bits
            for j in range(g * G, (g + 1) * G):
                v = float(np.float32(np.float32(w[r, j]) / np.float32(sig)))
                assert out["q"][r, j] == max(-7, min(7, round(v)))


def test_lambda_divides_on_quantise():
    """Scaling y and lambda by the same power of two leaves every decision unchanged,
    and lambda = 2 gives the same codes as y / 2 with lambda = 1."""
    rng = np.random.default_rng(4)
    d = 32
    y = rng.standard_normal((50, d))
    a = oracle.quantize_vectors(y, np.full(d, 2.0), 16, 4)
    b = oracle.quantize_vectors(y / 2.0, np.ones(d), 16, 4)
    assert np.array_equal(a["q"], b["q"])
    assert np.array_equal(a["scale_bits"], b["scale_bits"])
    c = oracle.quantize_vectors(y, np.ones(d), 16, 4)
    sa = oracle.binary16_bits_to_float(a["scale_bits"])
    sc = oracle.binary16_bits_to_float(c["scale_bits"])
    assert np.allclose(sa * 2.0, sc, rtol=2e-3)


@pytest.mark.parametrize("kind", [oracle.SRFT, oracle.SRHT])
@pytest.mark.parametrize("bits,group", [(4, 8), (8, 16), (4, 32)])
def test_on_grid_vectors_roundtrip_exactly(kind, bits, group):
    code_err, xerr = lossless_roundtrip_error(oracle.quantize, oracle.dequantize, kind,
                                              d=32, group=group, bits=bits)
    assert code_err == 0
    assert xerr <= 1e-12


@pytest.mark.parametrize("kind", [oracle.SRFT, oracle.SRHT])
def test_error_bound_by_orthogonality(kind):
    """Where no clamp fires |w_hat - w| <= sigma/2 per coordinate, so
    ||xhat - x||_2 <= ||lambda * sigma / 2||_2 (before binary16 output rounding)."""
    rng = np.random.default_rng(6)
    S, N, H, d, G = 2, 64, 2, 64, 16
    x = rng.standard_normal((S, N, H, d)).astype(np.float16)
    signs = np.where(rng.random((S, H, d)) < 0.5, -1, 1).astype(np.int8)
    lam = oracle.calibrate_lambda(x, signs, 32, kind).astype(np.float32)
    out = oracle.quantize(x, signs, lam, G, 4, kind)
    back = oracle.dequantize(out["codes"], out["scales"], signs, lam, d, G, 4, kind)
    sig = oracle.binary16_bits_to_float(out["scales"])
    bound = np.sqrt(np.sum((np.repeat(sig, G, axis=-1) * lam[:, None] / 2.0) ** 2, axis=-1))
    err = np.linalg.norm(back["xhat64"] - x.astype(np.float64), axis=-1)
    assert np.all(err <= bound * (1 + 1e-6))
    # per coordinate in the rotated domain
    w = out["y"] / lam[:, None].astype(np.float64)
    what = back["yhat"] / lam[:, None].astype(np.float64)
    assert np.all(np.abs(what - w) <= np.repeat(sig, G, axis=-1) * (0.5 + 1e-5))


# ---------------------------------------------------------------------------
# Calibration pins
# ---------------------------------------------------------------------------

def test_calibration_closed_form_unit_vector():
    """Rows all equal to e_0: y = column 0 of R, so lambda_j = |R_j0|, and the
    channels where R_j0 = 0 (the Im rows) take the lambda = 1 rule."""
    d = 16
    x = np.zeros((1, 8, 1, d))
    x[..., 0] = 1.0
    signs = np.ones((1, 1, d), dtype=np.int8)
    lam = oracle.calibrate_lambda(x, signs, 8, oracle.SRFT)[0, 0]
    c = 1 / math.sqrt(d)
    want = np.array([c, c] + [math.sqrt(2) * c, 1.0] * (d // 2 - 1))
    assert np.max(np.abs(lam - want)) <= 1e-15


@pytest.mark.parametrize("kind", [oracle.SRFT, oracle.SRHT])
def test_calibration_energy_invariant(kind):
    """sum_j lambda_j^2 = mean over rows of ||x||^2 (Parseval), and only the first
    n_cal rows matter."""
    rng = np.random.default_rng(8)
    x = rng.standard_normal((2, 40, 3, 32))
    signs = np.where(rng.random((2, 3, 32)) < 0.5, -1, 1).astype(np.int8)
    lam = oracle.calibrate_lambda(x, signs, 24, kind)
    energy = np.mean(np.sum(x[:, :24] ** 2, axis=-1), axis=1)
    assert np.max(np.abs(np.sum(lam ** 2, axis=-1) - energy) / energy) <= 1e-12
    x2 = x.copy()
    x2[:, 24:] *= 100.0
    assert np.array_equal(oracle.calibrate_lambda(x2, signs, 24, kind), lam)


@pytest.mark.parametrize("kind", [oracle.SRFT, oracle.SRHT])
def test_rotated_domain_attention_equals_plain_attention(kind):
    """Orthogonality ("When Quantization Is Free", Methodology 1) carried
    through decode attention: with K and V quantised, scoring the rotated
    query against the rotated-domain cache gives the scores of the plain query
    against the dequantised cache, and undoing the rotation of the
    rotated-domain output gives the plain output, to float64 rounding."""
    rng = np.random.default_rng(11)
    S, T, H, d, group, bits = 1, 37, 2, 64, 16, 4
    k16 = rng.standard_normal((S, T, H, d)).astype(np.float16)
    v16 = rng.standard_normal((S, T, H, d)).astype(np.float16)
    sk = np.where(rng.random((S, H, d)) < 0.5, -1, 1).astype(np.int8)
    sv = np.where(rng.random((S, H, d)) < 0.5, -1, 1).astype(np.int8)
    lk = np.exp(rng.uniform(-0.5, 0.5, (S, H, d))).astype(np.float32)
    lv = np.exp(rng.uniform(-0.5, 0.5, (S, H, d))).astype(np.float32)
    qk, qv = (oracle.quantize(k16, sk, lk, group, bits, kind),
              oracle.quantize(v16, sv, lv, group, bits, kind))
    kx = oracle.dequantize(qk["codes"], qk["scales"], sk, lk, d, group, bits, kind)["xhat64"]
    vx = oracle.dequantize(qv["codes"], qv["scales"], sv, lv, d, group, bits, kind)["xhat64"]
    ky = oracle.dequantize_rotated(qk["codes"], qk["scales"], lk, d, group, bits)["yhat"]
    vy = oracle.dequantize_rotated(qv["codes"], qv["scales"], lv, d, group, bits)["yhat"]
    q = rng.standard_normal((S, 1, H, d)).astype(np.float16)
    q_rot = oracle.rotate(q, sk, kind)                       # R_K q, float64
    for h in range(H):
        plain = kx[0, :, h, :] @ q[0, 0, h, :].astype(np.float64)
        rotated = ky[0, :, h, :] @ q_rot[0, 0, h, :]
        np.testing.assert_allclose(rotated, plain, rtol=1e-12, atol=1e-12)
        p = np.exp(plain - plain.max())
        p /= p.sum()
        out_plain = p @ vx[0, :, h, :]
        out_rot = (p @ vy[0, :, h, :])[None, None, None, :]
        sv_h = sv[:, h:h + 1, :]
        out = oracle.unrotate(out_rot, sv_h, kind)[0, 0, 0]
        np.testing.assert_allclose(out, out_plain, rtol=1e-12, atol=1e-12)


def test_rotated_dequantisation_is_the_scaled_codes():
    """Hand-worked: codes (-7, 3) in one byte, sigma = 0.5, lambda = (2, 4)
    give (-7 * 0.5 * 2, 3 * 0.5 * 4) = (-7, 6)."""
    codes = np.array([[[[0x39]]]], dtype=np.uint8)          # low nibble -7, high 3
    scales = oracle.float_to_binary16_bits(np.array([[[[0.5]]]]))
    lam = np.array([[[2.0, 4.0]]], dtype=np.float32)
    out = oracle.dequantize_rotated(codes, scales, lam, 2, 2, 4)
    np.testing.assert_array_equal(out["yhat"][0, 0, 0], [-7.0, 6.0])


def _attn_cache(rng, rows, H, d, group, bits, kind):
    x = rng.standard_normal((1, rows, H, d)).astype(np.float16)
    s = np.where(rng.random((1, H, d)) < 0.5, -1, 1).astype(np.int8)
    lam = np.exp(rng.uniform(-0.3, 0.3, (1, H, d))).astype(np.float32)
    qz = oracle.quantize(x, s, lam, group, bits, kind)
    return qz["codes"][0], qz["scales"][0], s[0], lam[0]


def attention_pin_errors(attn, kind: int = 0) -> dict:
    """The attention pins as numbers, for any implementation `attn` with the
    signature of ``oracle.decode_attention`` (the planted-mistake tests reuse
    this): the error of the one-token closed form, of the zero-query mean, of
    token-order invariance, and of the large-scale argmax limit."""
    rng = np.random.default_rng(31 + kind)
    H, d, group, bits, n_seq, n_ctx = 2, 16, 8, 4, 2, 6
    rows = n_ctx * n_seq
    kc, ks, ksg, kl = _attn_cache(rng, rows, H, d, group, bits, kind)
    vc, vs, vsg, vl = _attn_cache(rng, rows, H, d, group, bits, kind)
    q = rng.standard_normal((n_seq, H, d))
    args = (d, group, bits, kind)
    kx = oracle.dequantize(kc[None], ks[None], ksg[None], kl[None], *args)["xhat64"][0]
    vx = oracle.dequantize(vc[None], vs[None], vsg[None], vl[None], *args)["xhat64"][0]
    err = {}
    one = attn(q, kc, ks, ksg, kl, vc, vs, vsg, vl, *args, 1, n_seq, 1, 0.3)
    err["one_token"] = float(np.abs(one - vx[:n_seq]).max())
    zero = attn(np.zeros_like(q), kc, ks, ksg, kl, vc, vs, vsg, vl, *args, n_ctx, n_seq, 1, 0.3)
    mean = np.stack([vx[np.arange(n_ctx) * n_seq + b].mean(axis=0) for b in range(n_seq)])
    err["zero_query"] = float(np.abs(zero - mean).max())
    a = attn(q, kc, ks, ksg, kl, vc, vs, vsg, vl, *args, n_ctx, n_seq, 1, 0.3)
    rev = np.array([(n_ctx - 1 - t) * n_seq + b for t in range(n_ctx) for b in range(n_seq)])
    a_rev = attn(q, kc[rev], ks[rev], ksg, kl, vc[rev], vs[rev], vsg, vl, *args, n_ctx, n_seq,
                 1, 0.3)
    err["order"] = float(np.abs(a - a_rev).max())
    hard = attn(q, kc, ks, ksg, kl, vc, vs, vsg, vl, *args, n_ctx, n_seq, 1, 1e4)
    e = 0.0
    for b in range(n_seq):
        r = np.arange(n_ctx) * n_seq + b
        for h in range(H):
            top = int(np.argmax(kx[r, h] @ q[b, h]))
            e = max(e, float(np.abs(hard[b, h] - vx[r[top], h]).max()))
    err["argmax"] = e
    return err


@pytest.mark.parametrize("kind", [0, 1])
def test_attention_pins_hold_for_the_oracle(kind):
    err = attention_pin_errors(oracle.decode_attention, kind)
    assert max(err.values()) < 1e-9, err


@pytest.mark.parametrize("kind", [0, 1])
def test_decode_attention_is_order_free_and_tends_to_the_argmax(kind):
    """Two more properties of the attention reference. Attention is a sum
    over tokens, so reversing the token order of the K and V rows together
    leaves every output unchanged (a mismatched K/V row or a wrong stride
    breaks this). With the softmax scale large, the weights concentrate on
    the token of the largest score, and the output tends to that token's
    dequantised value."""
    rng = np.random.default_rng(23)
    H, d, group, bits, n_seq, n_ctx = 2, 16, 8, 4, 2, 6
    rows = n_ctx * n_seq
    kc, ks, ksg, kl = _attn_cache(rng, rows, H, d, group, bits, kind)
    vc, vs, vsg, vl = _attn_cache(rng, rows, H, d, group, bits, kind)
    q = rng.standard_normal((n_seq, H, d))
    a = oracle.decode_attention(q, kc, ks, ksg, kl, vc, vs, vsg, vl, d, group, bits, kind,
                                n_ctx, n_seq, 1, 0.3)
    rev = np.array([(n_ctx - 1 - t) * n_seq + b for t in range(n_ctx) for b in range(n_seq)])
    a_rev = oracle.decode_attention(q, kc[rev], ks[rev], ksg, kl, vc[rev], vs[rev], vsg, vl, d,
                                    group, bits, kind, n_ctx, n_seq, 1, 0.3)
    np.testing.assert_allclose(a, a_rev, rtol=1e-12, atol=1e-12)
    kx = oracle.dequantize(kc[None], ks[None], ksg[None], kl[None], d, group, bits,
                           kind)["xhat64"][0]
    vx = oracle.dequantize(vc[None], vs[None], vsg[None], vl[None], d, group, bits,
                           kind)["xhat64"][0]
    hard = oracle.decode_attention(q, kc, ks, ksg, kl, vc, vs, vsg, vl, d, group, bits, kind,
                                   n_ctx, n_seq, 1, 1e4)
    for b in range(n_seq):
        r = np.arange(n_ctx) * n_seq + b
        for h in range(H):
            scores = kx[r, h] @ q[b, h]
            top = np.argsort(scores)[-2:]
            assert scores[top[1]] - scores[top[0]] > 1e-2   # a clear maximum here
            np.testing.assert_allclose(hard[b, h], vx[r[top[1]], h], rtol=1e-9, atol=1e-9)


@pytest.mark.parametrize("kind", [oracle.SRFT, oracle.SRHT])
def test_decode_attention_special_cases(kind):
    """Closed forms of the attention reference: one token gives that
    token's dequantised value; a zero query weights every token equally (the
    mean of the values); the two layouts of the same rows agree."""
    rng = np.random.default_rng(17)
    H, d, group, bits, n_seq = 2, 16, 8, 4, 3
    kc, ks, ksg, kl = _attn_cache(rng, 12, H, d, group, bits, kind)
    vc, vs, vsg, vl = _attn_cache(rng, 12, H, d, group, bits, kind)
    q = rng.standard_normal((n_seq, 2 * H, d))
    vx = oracle.dequantize(vc[None], vs[None], vsg[None], vl[None], d, group, bits,
                           kind)["xhat64"][0]
    one = oracle.decode_attention(q, kc, ks, ksg, kl, vc, vs, vsg, vl, d, group, bits, kind,
                                  1, n_seq, 1, 0.25)
    for b in range(n_seq):
        for hq in range(2 * H):
            np.testing.assert_allclose(one[b, hq], vx[b, hq // 2], rtol=1e-12, atol=1e-12)
    zero = oracle.decode_attention(np.zeros_like(q), kc, ks, ksg, kl, vc, vs, vsg, vl, d, group,
                                   bits, kind, 4, n_seq, 1, 0.25)
    for b in range(n_seq):
        rows = np.arange(4) * n_seq + b
        for hq in range(2 * H):
            np.testing.assert_allclose(zero[b, hq], vx[rows, hq // 2].mean(axis=0), rtol=1e-12,
                                       atol=1e-12)
    # sequence-major rows (row = b * 4 + t) hold the same tokens as token-major
    # rows (row = t * 3 + b) after a permutation of the cache
    perm = np.array([t * n_seq + b for b in range(n_seq) for t in range(4)])
    a1 = oracle.decode_attention(q, kc, ks, ksg, kl, vc, vs, vsg, vl, d, group, bits, kind, 4,
                                 n_seq, 1, 0.25)
    a2 = oracle.decode_attention(q, kc[perm], ks[perm], ksg, kl, vc[perm], vs[perm], vsg, vl, d,
                                 group, bits, kind, 4, 1, 4, 0.25)
    np.testing.assert_allclose(a1, a2, rtol=1e-12, atol=1e-12)
