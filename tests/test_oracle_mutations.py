"""Planted mistakes: each broken variant of an oracle step must fail a pin.

The variants are built here, on the CPU, from the oracle's own definitions with
one plausible error each (a dropped factor, a wrong sign, a transposed
operand, a swapped index, a different rounding). Nothing here touches the GPU.
"""

import math

import numpy as np

import oracle
from oracle import srft_oracle as so
from test_oracle_pins import (
    attention_pin_errors,
    brute_force_dft_error,
    golden_pack_mismatches,
    golden_quant_mismatches,
    hadamard_special_case_error,
    lossless_roundtrip_error,
    orthogonality_error,
    rfft_special_case_error,
)


def _srft_variant(d, *, im_sign=-1.0, sqrt2=math.sqrt(2.0), swap_re_im=False, nyquist_alt=True):
    c = 1.0 / math.sqrt(d)
    n = np.arange(d)
    R = np.empty((d, d))
    R[0] = c
    R[1] = c * (np.where(n % 2 == 0, 1.0, -1.0) if nyquist_alt else 1.0)
    for k in range(1, d // 2):
        th = 2 * math.pi * ((k * n) % d) / d
        re, im = sqrt2 * c * np.cos(th), im_sign * sqrt2 * c * np.sin(th)
        if swap_re_im:
            re, im = im, re
        R[2 * k], R[2 * k + 1] = re, im
    return R


def test_wrong_sign_of_imaginary_rows_is_caught():
    fn = lambda d: _srft_variant(d, im_sign=+1.0)
    assert orthogonality_error(fn, 16) <= 1e-12          # still orthogonal ...
    assert rfft_special_case_error(fn, 16) > 1e-3        # ... but not the DFT
    assert brute_force_dft_error(fn, 8) > 1e-3


def test_dropped_sqrt2_is_caught():
    fn = lambda d: _srft_variant(d, sqrt2=1.0)
    assert orthogonality_error(fn, 16) > 1e-3


def test_swapped_pack_order_is_caught():
    fn = lambda d: _srft_variant(d, swap_re_im=True)
    assert rfft_special_case_error(fn, 16) > 1e-3


def test_wrong_nyquist_row_is_caught():
    fn = lambda d: _srft_variant(d, nyquist_alt=False)
    assert orthogonality_error(fn, 16) > 1e-3


def test_wrong_hadamard_parity_is_caught():
    def fn(d):
        i = np.arange(d)[:, None]
        j = np.arange(d)[None, :]
        v, parity = i | j, np.zeros((d, d), dtype=np.int64)
        while np.any(v):
            parity ^= v & 1
            v >>= 1
        return np.where(parity == 1, -1.0, 1.0) / math.sqrt(d)
    assert hadamard_special_case_error(fn, 16) > 1e-3


def test_transposed_rotation_is_caught():
    fn = lambda d: oracle.srft_matrix(d).T
    assert rfft_special_case_error(fn, 16) > 1e-3


def test_round_half_away_from_zero_is_caught():
    def quant(y, lam, group, bits):
        out = so.quantize_vectors(y, lam, group, bits)
        sig = so.binary16_bits_to_float(out["scale_bits"]).astype(np.float32)
        qmax = so.qmax_for(bits)
        v = (y.astype(np.float32) / np.float32(1.0)).reshape(sig.shape + (group,)) / sig[..., None]
        q = np.clip(np.sign(v) * np.floor(np.abs(v) + 0.5), -qmax, qmax)
        out["q"] = np.where(sig[..., None] == 0, 0, np.nan_to_num(q)).astype(np.int64).reshape(y.shape)
        return out
    assert golden_quant_mismatches(quant) != []


def test_asymmetric_int4_range_is_caught():
    def quant(y, lam, group, bits):
        orig = so.qmax_for
        so.qmax_for = lambda b: 8 if b == 4 else 127
        try:
            return so.quantize_vectors(y, lam, group, bits)
        finally:
            so.qmax_for = orig
    assert golden_quant_mismatches(quant) != []


def test_swapped_nibbles_are_caught():
    def pack(q, bits):
        q = np.asarray(q).astype(np.int64)
        return ((q[..., 1::2] & 0xF) | ((q[..., 0::2] & 0xF) << 4)).astype(np.uint8)
    assert golden_pack_mismatches(pack) != []


def test_truncating_binary16_is_caught():
    def quant(y, lam, group, bits):
        out = so.quantize_vectors(y, lam, group, bits)
        r = (np.max(np.abs(np.asarray(y, np.float32)).reshape(out["scale_bits"].shape + (group,)), axis=-1)
             / np.float32(so.qmax_for(bits)))
        out["scale_bits"] = r.astype(np.float64).astype(np.float16).view(np.uint16) & np.uint16(0xFFFE)
        return out
    assert golden_quant_mismatches(quant) != []


def test_dequantise_with_forward_rotation_is_caught():
    def deq(codes, scales, signs, lam, d, group, bits, kind):
        orig = so.unrotate
        so.unrotate = lambda y, s, k: so.rotate(y, s, k)
        try:
            return so.dequantize(codes, scales, signs, lam, d, group, bits, kind)
        finally:
            so.unrotate = orig
    _, xerr = lossless_roundtrip_error(oracle.quantize, deq, oracle.SRFT)
    assert xerr > 1e-3


def test_lambda_multiplied_on_quantise_is_caught():
    def quantize(x, signs, lam, group, bits, kind):
        return so.quantize(x, signs, 1.0 / np.asarray(lam, dtype=np.float32), group, bits, kind)
    code_err, _ = lossless_roundtrip_error(quantize, oracle.dequantize, oracle.SRFT)
    assert code_err > 0


def _attention_variant(*, v_lambda=True, v_signs_of_k=False, v_shift=0, use_scale=True):
    """decode_attention written out from the oracle's own steps, with one
    plausible error switched on."""
    def attn(q, k_codes, k_scales, k_signs, k_lam, v_codes, v_scales, v_signs, v_lam, d, group,
             bits, kind, n_ctx, tok_stride_rows, seq_stride_rows, scale):
        q = np.asarray(q, dtype=np.float64)
        n_seq, HQ, _ = q.shape
        H = k_codes.shape[1]
        Q = HQ // H
        out = np.empty((n_seq, HQ, d))
        vs_used = k_signs if v_signs_of_k else v_signs
        vl_used = v_lam if v_lambda else np.ones_like(v_lam)
        for b in range(n_seq):
            rows = np.arange(n_ctx) * tok_stride_rows + b * seq_stride_rows
            vrows = rows[(np.arange(n_ctx) + v_shift) % n_ctx]
            kx = oracle.dequantize(k_codes[None, rows], k_scales[None, rows], k_signs[None],
                                   k_lam[None], d, group, bits, kind)["xhat64"][0]
            vx = oracle.dequantize(v_codes[None, vrows], v_scales[None, vrows], vs_used[None],
                                   vl_used[None], d, group, bits, kind)["xhat64"][0]
            for h in range(H):
                for g in range(Q):
                    s_ = (scale if use_scale else 1.0) * (kx[:, h, :] @ q[b, h * Q + g])
                    p = np.exp(s_ - s_.max())
                    out[b, h * Q + g] = (p / p.sum()) @ vx[:, h, :]
        return out
    return attn


def test_unchanged_attention_variant_passes_the_pins():
    assert max(attention_pin_errors(_attention_variant()).values()) < 1e-9


def test_attention_values_without_lambda_are_caught():
    assert attention_pin_errors(_attention_variant(v_lambda=False))["one_token"] > 1e-3


def test_attention_values_with_the_key_signs_are_caught():
    assert attention_pin_errors(_attention_variant(v_signs_of_k=True))["one_token"] > 1e-3


def test_attention_values_one_token_off_are_caught():
    err = attention_pin_errors(_attention_variant(v_shift=1))
    assert err["zero_query"] < 1e-9      # the same set of values, so the mean holds ...
    assert err["order"] > 1e-3           # ... but the K/V pairing does not


def test_attention_without_the_softmax_scale_is_caught():
    assert attention_pin_errors(_attention_variant(use_scale=False))["argmax"] > 1e-3
