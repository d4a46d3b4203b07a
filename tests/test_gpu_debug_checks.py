"""The debug build (libsrftq_debug.so, -DSRFTQ_DEBUG_CHECKS): every kernel
checks each global-memory index it computes against the call's extents and
records a failure in the device guard word instead of making the access.

The index check itself is exercised on the device without a fault (a probe
checks an index outside its range and records it); then the small-case
sweeps of every entry point run on the debug build, which must report no
violation and produce the oracle's results.
"""

import math
import os

import numpy as np
import pytest

import oracle
import parity

torch = pytest.importorskip("torch")
import rotate_then_quantize_b200 as rq  # noqa: E402
from rotate_then_quantize_b200 import binding as b  # noqa: E402

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _debug_library():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    if not os.path.exists(b.LIB_DEBUG_PATH):
        from rotate_then_quantize_b200 import build
        build.build(debug=True)
    rq.load_library(b.LIB_DEBUG_PATH)
    yield
    with rq.debug_checks():
        assert rq.srftq_check_device() == 0


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _np16(t):
    return t.cpu().numpy().view(np.uint16)


def test_index_check_is_recorded_in_the_debug_build_only():
    with rq.debug_checks():
        assert rq.srftq_debug_checks()
        assert rq.srftq_check_device() == 0
        assert rq.srftq_probe_index_check(3, 4) == 0
        assert rq.srftq_check_device() == 0            # inside the range: nothing recorded
        assert rq.srftq_probe_index_check(4, 4) == 0
        assert rq.srftq_check_device() == b.SRFTQ_ERR_DEVICE_CHECK
        assert rq.srftq_probe_index_check(-1, 4) == 0
        assert rq.srftq_check_device() == b.SRFTQ_ERR_DEVICE_CHECK
        assert rq.srftq_check_device() == 0            # the check cleared the word
    assert not rq.srftq_debug_checks()                 # the release build compiles it away
    assert rq.srftq_probe_index_check(4, 4) == 0
    assert rq.srftq_check_device() == 0


def _codec_case(d, bits, group, rot, S=2, N=45, H=3, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((S, N, H, d))
    x16 = np.where(rng.random(x.shape) < 0.01, 20 * x, x).astype(np.float16)
    signs = np.where(rng.random((S, H, d)) < 0.5, -1, 1).astype(np.int8)
    lam = oracle.calibrate_lambda(x16, signs, 32, rot).astype(np.float32)
    return x16, signs, lam


@pytest.mark.parametrize("d", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("rot", [0, 1])
def test_codec_sweep_under_index_checks(d, bits, rot):
    """Quantise, dequantise, calibrate, rotate, unrotate and the rotated-domain
    dequantiser for the smallest, a middle and the largest group, ragged rows
    and several heads: no index check fails, and the results match the
    oracle."""
    with rq.debug_checks():
        for group in sorted({8, min(32, d), d}):
            x16, signs, lam = _codec_case(d, bits, group, rot, seed=d + bits + group + rot)
            xt, st, lt = _t(x16), _t(signs), _t(lam)
            codes, scales = rq.quantize(xt, st, lt, group, bits, rot)
            ref = oracle.quantize(x16, signs, lam, group, bits, rot)
            parity.assert_clean(parity.check_codes(ref, codes.cpu().numpy(), _np16(scales), bits,
                                                   group), f"d{d} g{group} codes")
            xh = rq.dequantize(codes, scales, st, lt, d, group, bits, rot)
            deq = oracle.dequantize(codes.cpu().numpy(), _np16(scales), signs, lam, d, group, bits,
                                    rot)
            parity.assert_clean(parity.check_dequant(_np16(xh), deq["bits"]), f"d{d} dequant")
            rd = rq.dequantize_rotated(codes, scales, lt, d, group, bits)
            want = oracle.dequantize_rotated(codes.cpu().numpy(), _np16(scales), lam, d, group,
                                             bits)
            parity.assert_clean(parity.check_dequant(_np16(rd), want["bits"]), f"d{d} rotated")
        lam_gpu = rq.calibrate_lambda(xt, st, 32, rotation=rot).cpu().numpy()
        parity.assert_clean(parity.check_lambda(lam_gpu, oracle.calibrate_lambda(x16, signs, 32,
                                                                                 rot)), "lambda")
        y = rq.rotate(xt, st, lt, rotation=rot).cpu().numpy()
        parity.assert_clean(parity.check_rotation(y, oracle.rotate(x16, signs, rot) /
                                                  lam[:, None].astype(np.float64)), "rotate")
        yy = rq.rotate(xt, st, rotation=rot)
        back = rq.unrotate(yy, st, rotation=rot).cpu().numpy()
        parity.assert_clean(parity.check_rotation(back, x16.astype(np.float64)), "unrotate")
        assert rq.srftq_check_device() == 0


@pytest.mark.parametrize("bits,group,q_per_kv", [(4, 16, 1), (8, 32, 2), (4, 128, 8)])
def test_attention_under_index_checks(bits, group, q_per_kv):
    rng = np.random.default_rng(bits + group + q_per_kv)
    H, d, n_seq, n_ctx = 2, 128, 3, 129
    rows = n_ctx * n_seq
    parts = []
    for _ in range(2):
        x = rng.standard_normal((1, rows, H, d)).astype(np.float16)
        s = np.where(rng.random((1, H, d)) < 0.5, -1, 1).astype(np.int8)
        lam = oracle.calibrate_lambda(x, s, 64).astype(np.float32)
        qz = oracle.quantize(x, s, lam, group, bits)
        parts.append((qz["codes"][0], qz["scales"][0], s[0], lam[0]))
    (kc, ks, ksg, kl), (vc, vs, vsg, vl) = parts
    q = rng.standard_normal((n_seq, H * q_per_kv, d)).astype(np.float16)
    scale = 1.0 / math.sqrt(d)
    with rq.debug_checks():
        out = rq.decode_attention(_t(q), _t(kc), _t(ks.view(np.float16)), _t(ksg), _t(kl),
                                  _t(vc), _t(vs.view(np.float16)), _t(vsg), _t(vl), group, bits,
                                  0, n_ctx=n_ctx, tok_stride_rows=n_seq, seq_stride_rows=1,
                                  scale=scale).cpu().numpy()
        assert rq.srftq_check_device() == 0
    ref = oracle.decode_attention(q, kc, ks, ksg, kl, vc, vs, vsg, vl, d, group, bits, 0, n_ctx,
                                  n_seq, 1, scale)
    assert (np.abs(out - ref) / np.maximum(1.0, np.abs(ref))).max() < 2e-5


@pytest.mark.parametrize("d,group,bits", [(64, 16, 4), (128, 128, 8), (256, 32, 4)])
def test_dense_codec_under_index_checks(d, group, bits):
    rng = np.random.default_rng(d + group)
    S, N, H = 2, 300, 3                        # several 128-row blocks and a partial one
    x16 = rng.standard_normal((S, N, H, d)).astype(np.float16)
    signs = np.where(rng.random((S, H, d)) < 0.5, -1, 1).astype(np.int8)
    V = rng.standard_normal((S, H, d // 2, d)).astype(np.float32)
    R = oracle.householder_rotations(V, signs, 0)
    lam = oracle.calibrate_lambda_dense(x16, R, 64).astype(np.float32)
    with rq.debug_checks():
        rot = rq.householder_rotation(_t(V), _t(signs))
        op = rq.dense_operand(_t(R.astype(np.float32)))
        codes, scales = rq.quantize_dense(_t(x16), op, _t(lam), group, bits)
        xh = rq.dequantize_dense(codes, scales, op, _t(lam), d, group, bits)
        lam_gpu = rq.calibrate_lambda_dense(_t(x16), op, 64).cpu().numpy()
        assert rq.srftq_check_device() == 0
    assert np.abs(rot.cpu().numpy() - R).max() < 2e-6
    ref = oracle.quantize_dense(x16, R, lam, group, bits)
    parity.assert_clean(parity.check_codes(ref, codes.cpu().numpy(), _np16(scales), bits, group,
                                           parity.DENSE_SCALE_BAND,
                                           parity.dense_code_band(ref, lam, group)), "dense codes")
    deq = oracle.dequantize_dense(codes.cpu().numpy(), _np16(scales), R, lam, d, group, bits)
    parity.assert_clean(parity.check_dequant(_np16(xh), deq["bits"]), "dense dequant")
    parity.assert_clean(parity.check_lambda(lam_gpu, oracle.calibrate_lambda_dense(x16, R, 64)),
                        "dense lambda")
