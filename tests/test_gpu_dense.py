"""GPU parity of the dense-rotation codec (the Householder variant of "When
Quantization Is Free", Methodology 3) against oracle/dense_oracle.py,
through the C ABI.

The rotation builder is compared with the oracle's float64 matrices (float32
storage: 2e-6 absolute on entries of unit-norm rows); the operand split bit
for bit; the codec stages with the tolerances of tests/parity.py (the dense
path's bands follow from the rotation tolerance), each stage fed the oracle's own inputs: the quantiser and
the calibration get the operand of the oracle's matrix (rounded to float32),
the dequantiser the oracle's codes.
"""

import numpy as np
import pytest

import kv_synth
import oracle
import parity

torch = pytest.importorskip("torch")
import rotate_then_quantize_b200 as rq  # noqa: E402

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
ROT_ENTRY_TOL = 2e-6


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    rq.load_library()
    yield
    assert rq.srftq_check_device() == 0, "a device-side guard fired"


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _np16(t):
    return t.cpu().numpy().view(np.uint16)


def _case(rng, S, N, H, d, k, kind, outlier_p=0.01, scale=20.0):
    x = rng.standard_normal((S, N, H, d))
    x = np.where(rng.random(x.shape) < outlier_p, x * scale, x).astype(np.float16)
    signs = np.where(rng.random((S, H, d)) < 0.5, -1, 1).astype(np.int8)
    V = rng.standard_normal((S, H, k, d)).astype(np.float32)
    R = oracle.householder_rotations(V, signs, kind)
    return x, signs, V, R


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kind", [0, 1])
@pytest.mark.parametrize("k_frac", [0, 1, 2])
def test_householder_rotation_matches_oracle(d, kind, k_frac):
    """k = 0 (the base matrix alone), one reflector, and k = d/2."""
    k = {0: 0, 1: 1, 2: d // 2}[k_frac]
    rng = np.random.default_rng(d + 10 * kind + k)
    S, H = 2, 3
    signs = np.where(rng.random((S, H, d)) < 0.5, -1, 1).astype(np.int8)
    V = rng.standard_normal((S, H, k, d)).astype(np.float32)
    R = oracle.householder_rotations(V, signs, kind)
    got = rq.householder_rotation(_t(V) if k else None, _t(signs), rotation=kind).cpu().numpy()
    err = np.abs(got - R).max()
    assert err <= ROT_ENTRY_TOL, err
    # and it is orthogonal to float32 accuracy
    g = got.astype(np.float64)
    assert np.abs(np.einsum("shij,shik->shjk", g, g) - np.eye(d)).max() < 1e-5


def test_operand_split_is_bit_exact():
    rng = np.random.default_rng(1)
    R32 = (rng.standard_normal((2, 3, 128, 128)) / 11.3).astype(np.float32)
    R32[0, 0, 0, :8] = [0.0, -0.0, 1e-9, -3e-6, 6.1e-5, 65504.0, 1.0, -1.0]  # zero, subnormals
    op = rq.dense_operand(_t(R32)).cpu().numpy().view(np.uint16)
    hi, lo = oracle.split_operand(R32)
    assert np.array_equal(op[:, :, 0], hi)
    assert np.array_equal(op[:, :, 1], lo)


def _quant_check(x16, R, lam, d, group, bits, what):
    op = rq.dense_operand(_t(R.astype(np.float32)))
    lt = _t(lam)
    codes, scales = rq.quantize_dense(_t(x16), op, lt, group, bits)
    ref = oracle.quantize_dense(x16, R, lam, group, bits)
    c_np, s_np = codes.cpu().numpy(), _np16(scales)
    stats = parity.check_codes(ref, c_np, s_np, bits, group, parity.DENSE_SCALE_BAND,
                               parity.dense_code_band(ref, lam, group))
    parity.assert_clean(stats, f"{what} codes")
    # dequantiser on the oracle's codes, and the GPU round trip on its own codes
    deq = oracle.dequantize_dense(ref["codes"], ref["scales"], R, lam, d, group, bits)
    xhat = rq.dequantize_dense(_t(ref["codes"]), _t(ref["scales"].view(np.float16)), op, lt, d,
                               group, bits)
    parity.assert_clean(parity.check_dequant(_np16(xhat), deq["bits"]), f"{what} dequant")
    xrt = rq.dequantize_dense(codes, scales, op, lt, d, group, bits)
    deq_own = oracle.dequantize_dense(c_np, s_np, R, lam, d, group, bits)
    parity.assert_clean(parity.check_dequant(_np16(xrt), deq_own["bits"]), f"{what} round trip")
    return stats


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("kind", [0, 1])
def test_dense_codec_matches_oracle(d, bits, kind):
    """Every group size 8..d, ragged rows (several 64-row tiles and a partial
    one), several slices and heads, k = d/2 reflectors."""
    rng = np.random.default_rng(3 * d + bits + kind)
    S, N, H = 2, 150, 3
    x16, signs, V, R = _case(rng, S, N, H, d, d // 2, kind)
    lam = oracle.calibrate_lambda_dense(x16, R, 64).astype(np.float32)
    g = 8
    while g <= d:
        _quant_check(x16, R, lam, d, g, bits, f"d{d} b{bits} g{g} base{kind}")
        g *= 2


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("n_cal", [1, 63, 64, 200, 1100])
def test_dense_calibration_matches_oracle(d, n_cal):
    """One cluster per (slice, head) whose blocks take every 8th 64-row
    tile: fewer rows than blocks, a partial tile, and (1100 rows) more tiles
    than blocks."""
    rng = np.random.default_rng(d + n_cal)
    x16, signs, V, R = _case(rng, 2, max(n_cal, 8), 3, d, d // 2, 0)
    op = rq.dense_operand(_t(R.astype(np.float32)))
    lam = rq.calibrate_lambda_dense(_t(x16), op, n_cal).cpu().numpy()
    parity.assert_clean(parity.check_lambda(lam, oracle.calibrate_lambda_dense(x16, R, n_cal)),
                        f"dense lambda d{d} n_cal{n_cal}")


def test_dense_codec_with_the_gpu_built_rotation():
    """End to end on the GPU's own rotation (built from the same reflectors):
    the codes agree with the oracle's within the boundary band, since the
    two matrices differ only by float32 rounding."""
    rng = np.random.default_rng(77)
    d, group, bits = 256, 32, 4
    x16, signs, V, R = _case(rng, 2, 100, 2, d, d // 2, 0, outlier_p=0.005, scale=25.0)
    lam = oracle.calibrate_lambda_dense(x16, R, 64).astype(np.float32)
    op = rq.dense_operand(rq.householder_rotation(_t(V), _t(signs)))
    codes, scales = rq.quantize_dense(_t(x16), op, _t(lam), group, bits)
    ref = oracle.quantize_dense(x16, R, lam, group, bits)
    parity.assert_clean(parity.check_codes(ref, codes.cpu().numpy(), _np16(scales), bits, group,
                                           parity.DENSE_SCALE_BAND,
                                           parity.dense_code_band(ref, lam, group)),
                        "gpu-built rotation")


def test_dense_strided_windows_keep_their_guard_bands():
    rng = np.random.default_rng(5)
    d, group, bits, S, T, H, N, off = 128, 16, 4, 2, 90, 2, 37, 21
    big = rng.standard_normal((S, T, H, d)).astype(np.float16)
    signs = np.where(rng.random((S, H, d)) < 0.5, -1, 1).astype(np.int8)
    R = oracle.householder_rotations(rng.standard_normal((S, H, 8, d)), signs, 0)
    lam = np.exp(rng.uniform(-0.5, 0.5, (S, H, d))).astype(np.float32)
    op, lt = rq.dense_operand(_t(R.astype(np.float32))), _t(lam)
    codes = torch.full((S, T, H, d // 2), 0xAB, dtype=torch.uint8, device=DEV)
    scales = torch.full((S, T, H, d // group), 7.0, dtype=torch.float16, device=DEV)
    desc = rq.make_desc(d, H, group, bits)
    rq.srftq_quantize_dense(desc, _t(big)[:, off:off + N], op, lt, codes[:, off:off + N],
                            scales[:, off:off + N])
    ref = oracle.quantize_dense(big[:, off:off + N], R, lam, group, bits)
    c_np, s_np = codes.cpu().numpy(), _np16(scales)
    parity.assert_clean(parity.check_codes(ref, c_np[:, off:off + N], s_np[:, off:off + N], bits,
                                           group, parity.DENSE_SCALE_BAND,
                                           parity.dense_code_band(ref, lam, group)),
                        "strided dense codes")
    outside = np.ones(T, bool)
    outside[off:off + N] = False
    assert np.all(c_np[:, outside] == 0xAB)
    assert np.all(s_np[:, outside] == np.float16(7.0).view(np.uint16))
    xh = torch.full((S, T, H, d), -3.0, dtype=torch.float16, device=DEV)
    rq.srftq_dequantize_dense(desc, codes[:, off:off + N], scales[:, off:off + N], op, lt,
                              xh[:, off:off + N])
    deq = oracle.dequantize_dense(c_np[:, off:off + N], s_np[:, off:off + N], R, lam, d, group,
                                  bits)
    xh_np = _np16(xh)
    parity.assert_clean(parity.check_dequant(xh_np[:, off:off + N], deq["bits"]),
                        "strided dense dequant")
    assert np.all(xh_np[:, outside] == np.float16(-3.0).view(np.uint16))


def test_dense_degenerate_values():
    """Zero vectors (sigma = 0), tiny and huge values, extreme lambda."""
    rng = np.random.default_rng(9)
    d, group = 128, 16
    x = rng.standard_normal((1, 64, 1, d))
    x[:, 0] = 0.0
    x[:, 1] = 1e-7 * rng.standard_normal(d)
    x[:, 2] = 6e4 * np.sign(rng.standard_normal(d))
    x16 = x.astype(np.float16)
    signs = np.where(rng.random((1, 1, d)) < 0.5, -1, 1).astype(np.int8)
    R = oracle.householder_rotations(rng.standard_normal((1, 1, 64, d)), signs, 0)
    for lam_val in (1.0, 1e-3, 3e3):
        lam = np.full((1, 1, d), lam_val, np.float32)
        for bits in (4, 8):
            _quant_check(x16, R, lam, d, group, bits, f"degenerate lam={lam_val} b{bits}")


@pytest.mark.parametrize("d,group,bits", [(64, 16, 4), (128, 16, 4), (128, 128, 8),
                                          (256, 32, 4), (256, 256, 4)])
def test_dense_quantiser_ranges_cross_slices_and_heads(d, group, bits):
    """More 128-row blocks than the GPU has SMs, so every CTA of the
    quantiser takes a range of several blocks that crosses (slice, head)
    boundaries: the operand is reloaded (d <= 128) or streamed (d = 256)
    for each, and a partial last block per (slice, head). Every vector is
    compared with the oracle."""
    rng = np.random.default_rng(d + group + bits)
    S, N, H = 3, 1000, 5                       # 8 blocks per (slice, head), 120 in all ...
    if d < 256:
        S, N = 4, 2600                         # ... or 21 x 20 = 420
    x16, signs, V, R = _case(rng, S, N, H, d, d // 2, 0, outlier_p=0.005, scale=25.0)
    lam = oracle.calibrate_lambda_dense(x16, R, 128).astype(np.float32)
    op = rq.dense_operand(_t(R.astype(np.float32)))
    codes, scales = rq.quantize_dense(_t(x16), op, _t(lam), group, bits)
    ref = oracle.quantize_dense(x16, R, lam, group, bits)
    parity.assert_clean(parity.check_codes(ref, codes.cpu().numpy(), _np16(scales), bits, group,
                                           parity.DENSE_SCALE_BAND,
                                           parity.dense_code_band(ref, lam, group)),
                        f"d{d} g{group} b{bits} many blocks")


def _random_codes(rng, S, N, H, d, group, bits, lo_exp, hi_exp):
    """Arbitrary code bytes (every nibble / byte value, the quantiser's unused
    -8 and -128 included) and fp16 scales log-uniform over 2^lo_exp ..
    2^hi_exp, so that the rows of one block span several binades."""
    codes = rng.integers(0, 256, (S, N, H, d * bits // 8), dtype=np.uint8)
    sig = np.exp2(rng.uniform(lo_exp, hi_exp, (S, N, H, d // group)))
    scales = np.minimum(sig, 65504.0).astype(np.float16).view(np.uint16)
    return codes, scales


def _assert_dequant_scale_free(gpu_bits, xhat64, what):
    """The dequantiser against the oracle's float64 xhat, at any magnitude:
    each finite output within one binary16 ulp of the exact value (its own
    rounding) plus 1e-5 of the vector's largest |xhat| (the float32
    accumulation of 3 d tensor-core products, for an output that cancels);
    an infinite output only where the exact value is at the overflow
    threshold (65520) within that same error, with its sign."""
    a = oracle.binary16_bits_to_float(np.asarray(gpu_bits).view(np.uint16))
    r = np.asarray(xhat64, np.float64)
    vmax = np.max(np.abs(r), axis=-1, keepdims=True)
    band = 1e-5 * vmax
    mag = np.abs(r)
    ulp = np.where(mag < 2.0 ** -14, 2.0 ** -24,
                   np.exp2(np.floor(np.log2(np.maximum(mag, 2.0 ** -14))) - 10))
    ulp = np.minimum(ulp, 32.0)
    fin = np.isfinite(a)
    ok_f = fin & (np.abs(np.where(fin, a, 0.0) - r) <= ulp + band)
    ok_i = np.isinf(a) & (np.sign(a) == np.sign(r)) & (mag >= 65520.0 - band)
    ok = ok_f | ok_i
    assert ok.all(), (f"{what}: {int((~ok).sum())} of {ok.size} outputs off, "
                      f"{int(np.isnan(a).sum())} NaN")


@pytest.mark.parametrize("d,group,bits", [(64, 8, 8), (128, 16, 4), (128, 128, 8),
                                          (256, 32, 4), (256, 8, 8), (256, 256, 4)])
def test_dense_dequantiser_ranges_cross_slices_and_heads(d, group, bits):
    """The tensor-core dequantiser with more 128-row blocks than SMs: every
    CTA walks a range that crosses (slice, head) boundaries (operand
    reloaded for d <= 128, streamed for d = 256), with a partial last block
    per (slice, head); codes are arbitrary bytes and the scales of a vector
    span 2^-7 .. 2^-3, so each row takes its own power-of-two range scale.
    Every output is compared with the oracle."""
    rng = np.random.default_rng(7 * d + group + bits)
    S, N, H = 3, 1000, 5
    if d < 256:
        S, N = 4, 2600
    signs = np.where(rng.random((S, H, d)) < 0.5, -1, 1).astype(np.int8)
    R = oracle.householder_rotations(rng.standard_normal((S, H, 16, d)), signs, 1)
    lam = np.exp(rng.uniform(-2.0, 2.0, (S, H, d))).astype(np.float32)
    codes, scales = _random_codes(rng, S, N, H, d, group, bits, -7.0, -3.0)
    op = rq.dense_operand(_t(R.astype(np.float32)))
    xhat = rq.dequantize_dense(_t(codes), _t(scales.view(np.float16)), op, _t(lam), d, group,
                               bits)
    deq = oracle.dequantize_dense(codes, scales, R, lam, d, group, bits)
    what = f"d{d} g{group} b{bits} many blocks dequant"
    parity.assert_clean(parity.check_dequant(_np16(xhat), deq["bits"]), what)
    _assert_dequant_scale_free(_np16(xhat), deq["xhat64"], what)


@pytest.mark.parametrize("bits", [4, 8])
def test_dense_dequantiser_extreme_magnitudes(bits):
    """lambda sigma q far outside fp16's range in both directions: sigma up
    to 65504 with lambda up to 1e4 (|a| ~ 1e10: outputs overflow to inf),
    fp16-subnormal sigma with lambda down to 1e-6 (outputs far below fp16's
    normal range), and vectors mixing both. The row scale keeps every A
    element inside fp16 before the split, so the outputs stay within the
    scale-free bound of the exact values."""
    rng = np.random.default_rng(11 + bits)
    d, group, S, N, H = 128, 16, 2, 300, 2
    signs = np.where(rng.random((S, H, d)) < 0.5, -1, 1).astype(np.int8)
    R = oracle.householder_rotations(rng.standard_normal((S, H, 8, d)), signs, 0)
    op = rq.dense_operand(_t(R.astype(np.float32)))
    for lam_lo, lam_hi, e_lo, e_hi in ((1e2, 1e4, 8.0, 15.9), (1e-6, 1e-4, -24.0, -14.0),
                                       (1e-3, 1e3, -24.0, 15.9)):
        lam = np.exp(rng.uniform(np.log(lam_lo), np.log(lam_hi), (S, H, d))).astype(np.float32)
        codes, scales = _random_codes(rng, S, N, H, d, group, bits, e_lo, e_hi)
        xhat = rq.dequantize_dense(_t(codes), _t(scales.view(np.float16)), op, _t(lam), d, group,
                                   bits)
        deq = oracle.dequantize_dense(codes, scales, R, lam, d, group, bits)
        _assert_dequant_scale_free(
            _np16(xhat), deq["xhat64"],
            f"b{bits} lambda {lam_lo:g}..{lam_hi:g} sigma 2^{e_lo:g}..2^{e_hi:g}")


@pytest.mark.parametrize("d,bits,group,kind", [(128, 4, 16, 0), (128, 8, 16, 1), (256, 4, 32, 0),
                                               (64, 4, 8, 0)])
def test_dense_form_of_the_base_rotation_is_the_fft_codec(d, bits, group, kind):
    """The tensor-core codec run with the signed SRFT / SRHT matrix itself
    (k = 0, built on the GPU) against the FFT codec's oracle
    (oracle.quantize / dequantize, which rotate by the transform): the same
    codes and scales within the dense bands, and the oracle's dequantised
    values from the oracle's codes."""
    rng = np.random.default_rng(d + bits + kind)
    S, N, H = 2, 300, 3
    x16, signs, _, _ = _case(rng, S, N, H, d, 1, kind)
    lam = oracle.calibrate_lambda(x16, signs, 64, kind).astype(np.float32)
    op = rq.dense_operand(rq.householder_rotation(None, _t(signs), rotation=kind))
    codes, scales = rq.quantize_dense(_t(x16), op, _t(lam), group, bits)
    ref = oracle.quantize(x16, signs, lam, group, bits, kind)
    parity.assert_clean(parity.check_codes(ref, codes.cpu().numpy(), _np16(scales), bits, group,
                                           parity.DENSE_SCALE_BAND,
                                           parity.dense_code_band(ref, lam, group)),
                        f"dense base d{d} b{bits} rot{kind}")
    xhat = rq.dequantize_dense(_t(ref["codes"]), _t(ref["scales"].view(np.float16)), op, _t(lam),
                               d, group, bits)
    deq = oracle.dequantize(ref["codes"], ref["scales"], signs, lam, d, group, bits, kind)
    parity.assert_clean(parity.check_dequant(_np16(xhat), deq["bits"]),
                        f"dense base d{d} b{bits} rot{kind} dequant")


@pytest.mark.parametrize("d,bits,group,kind", [(128, 4, 16, 0), (256, 4, 32, 1)])
def test_dense_base_codes_decode_with_the_fft_dequantiser(d, bits, group, kind):
    """The tensor-core quantiser run with the SRFT / SRHT matrix itself and the
    FFT / WHT dequantiser implement one codec: codes and scales from the first
    decode with the second to the oracle's dequantisation of those codes."""
    rng = np.random.default_rng(5 * d + bits + kind)
    S, N, H = 2, 200, 2
    x16, signs, _, _ = _case(rng, S, N, H, d, 1, kind)
    lam = oracle.calibrate_lambda(x16, signs, 64, kind).astype(np.float32)
    op = rq.dense_operand(rq.householder_rotation(None, _t(signs), rotation=kind))
    codes, scales = rq.quantize_dense(_t(x16), op, _t(lam), group, bits)
    xhat = rq.dequantize(codes, scales, _t(signs), _t(lam), d, group=group, bits=bits,
                         rotation=kind)
    deq = oracle.dequantize(codes.cpu().numpy(), _np16(scales), signs, lam, d, group, bits, kind)
    parity.assert_clean(parity.check_dequant(_np16(xhat), deq["bits"]),
                        f"dense-quantised, FFT-dequantised d{d} rot{kind}")
