"""Plain float64 CPU statement of the SRFT / SRHT rotate-then-quantize codec.

Test infrastructure only: the library never imports this module (see the
package docstring for who may). Every step is the definition written out, in
the order the paper's fused kernel applies them; there is no blocking, fusion
or fast transform here. The rotation is an explicit d x d matrix applied with a
matrix product, so a reader can check each row against the formula.

Layouts (shared with the C ABI, described in ``include/srftq.h``):

* ``x``       [S, N, H, d]   float16 or any float (converted exactly to float64)
* ``signs``   [S, H, d]      int8; a negative entry means -1, anything else +1
* ``lam``     [S, H, d]      float32 per-channel scale lambda
* ``codes``   [S, N, H, d*bits/8] uint8
* ``scales``  [S, N, H, d/G] uint16 holding IEEE binary16 bit patterns

Readings taken where the pages leave a step open (each one also listed in the
design notes of the repository):

1. pack order: interleaved [X_0, X_{d/2}, sqrt2*Re X_1, sqrt2*Im X_1, ...].
2. DFT kernel exp(-2*pi*i*k*n/d), normalised by 1/sqrt(d) (unitary).
3. d is a power of two (the pages' FFT is radix-2 over d/2 points).
5. lambda divides on quantize (w = y / lambda) and multiplies on dequantize.
6. lambda_j = RMS of rotated coordinate j over the first n_cal rows; 1 if 0.
7. symmetric integer range: int4 in [-7, 7], int8 in [-127, 127].
8. group scale sigma = binary16 round-to-nearest-even of (absmax / qmax); the
   codes are computed with that stored binary16 value, so dequantisation
   inverts the quantiser exactly; codes are clamped to +-qmax.
9. sigma that would overflow binary16 saturates to 65504; sigma == 0 gives
   all-zero codes for that group.
10. rounding ties go to even.
11. int4: element 2k in the low nibble of byte k, element 2k+1 in the high.
12. a group is G consecutive packed coordinates.
13. dequantised output is binary16 (round-to-nearest-even).
14. SRHT: Sylvester (natural) order Hadamard matrix, 1/sqrt(d), no packing.

Decision precision: where floating point decides an integer (the binary16
scale and the integer codes), the decision is taken in float32 -- the
precision the CUDA kernels compute in -- starting from the float64 rotation
rounded to float32. ``quantize`` also returns the float64 pre-rounding values
so a comparison can tell which codes sit within a hair of a rounding boundary.
"""

from __future__ import annotations

import math

import numpy as np

SRFT = 0
SRHT = 1

_SQRT2 = math.sqrt(2.0)


def _check_pow2(d: int) -> None:
    if d < 2 or (d & (d - 1)) != 0:
        raise ValueError(f"d must be a power of two >= 2, got {d}")


# ---------------------------------------------------------------------------
# Rotations
# ---------------------------------------------------------------------------

def srft_matrix(d: int) -> np.ndarray:
    """Real d x d matrix P.F of the SRFT without its sign diagonal (float64).

    "When Quantization Is Free", Methodology 1: SRFT(x) = pack(F diag(s) x),
    F the unitary DFT. F x for real x is Hermitian, so the d real numbers
    X_0 (real), X_{d/2} (real) and Re/Im X_k for 0 < k < d/2 carry all of it;
    "pack" lists them interleaved with sqrt(2) on the complex bins so that the
    packed map is orthogonal (reading 1). With theta = 2*pi*((k*n) mod d)/d
    (the product is reduced mod d first so the angle is formed exactly):

        row 0      : 1/sqrt(d)
        row 1      : (-1)^n / sqrt(d)
        row 2k     :  sqrt(2)/sqrt(d) * cos(theta)
        row 2k + 1 : -sqrt(2)/sqrt(d) * sin(theta)        (0 < k < d/2)
    """
    _check_pow2(d)
    c = 1.0 / math.sqrt(d)
    n = np.arange(d)
    R = np.empty((d, d), dtype=np.float64)
    R[0, :] = c
    R[1, :] = c * np.where(n % 2 == 0, 1.0, -1.0)
    for k in range(1, d // 2):
        theta = 2.0 * math.pi * ((k * n) % d) / d
        R[2 * k, :] = _SQRT2 * c * np.cos(theta)
        R[2 * k + 1, :] = -_SQRT2 * c * np.sin(theta)
    return R


def srht_matrix(d: int) -> np.ndarray:
    """Normalised Sylvester Hadamard matrix H_d / sqrt(d) (float64).

    "HyperQuant", Methodology 1: RHT(x) = H D x with H the Walsh-Hadamard
    matrix and D a random sign diagonal; entry (i, j) is
    (-1)^popcount(i AND j), scaled by 1/sqrt(d) so the map is orthogonal
    (reading 14).
    """
    _check_pow2(d)
    i = np.arange(d)[:, None]
    j = np.arange(d)[None, :]
    parity = np.zeros((d, d), dtype=np.int64)
    v = i & j
    while np.any(v):
        parity ^= v & 1
        v = v >> 1
    return np.where(parity == 1, -1.0, 1.0) / math.sqrt(d)


def _sign_values(signs: np.ndarray) -> np.ndarray:
    """+-1.0 from the int8 sign table: negative means -1, anything else +1."""
    return np.where(np.asarray(signs) < 0, -1.0, 1.0)


def rotation_matrix(d: int, signs_row: np.ndarray, kind: int = SRFT) -> np.ndarray:
    """The full rotation M . diag(s) for one (slice, head) sign row, float64."""
    base = srft_matrix(d) if kind == SRFT else srht_matrix(d)
    s = _sign_values(signs_row)
    if s.shape != (d,):
        raise ValueError("sign row must have d entries")
    return base * s[None, :]


def rotate(x: np.ndarray, signs: np.ndarray, kind: int = SRFT) -> np.ndarray:
    """y = R_{s,h} x for every vector of x [S, N, H, d]; returns float64.

    The product is the definition itself (an O(d^2) matrix product per
    vector), not a fast transform.
    """
    x = np.asarray(x)
    S, N, H, d = x.shape
    signs = np.asarray(signs)
    if signs.shape != (S, H, d):
        raise ValueError(f"signs must be [S, H, d] = {(S, H, d)}, got {signs.shape}")
    y = np.empty((S, N, H, d), dtype=np.float64)
    for s in range(S):
        for h in range(H):
            R = rotation_matrix(d, signs[s, h], kind)
            y[s, :, h, :] = x[s, :, h, :].astype(np.float64) @ R.T
    return y


def unrotate(yhat: np.ndarray, signs: np.ndarray, kind: int = SRFT) -> np.ndarray:
    """x = R_{s,h}^T y for every vector (the inverse rotation), float64."""
    yhat = np.asarray(yhat, dtype=np.float64)
    S, N, H, d = yhat.shape
    out = np.empty((S, N, H, d), dtype=np.float64)
    for s in range(S):
        for h in range(H):
            R = rotation_matrix(d, signs[s, h], kind)
            out[s, :, h, :] = yhat[s, :, h, :] @ R
    return out


# ---------------------------------------------------------------------------
# IEEE-754 binary16, written out from the format definition
# ---------------------------------------------------------------------------

def float_to_binary16_bits(v, saturate: bool = False) -> np.ndarray:
    """Round float64 values to binary16, ties to even; returns uint16 bits.

    binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
    Normal numbers with a in [2^E, 2^(E+1)), -14 <= E <= 15, have quantum
    2^(E-10); below 2^-14 the quantum is fixed at 2^-24 (subnormals).
    The magnitude divided by its quantum is exact in float64 (a power-of-two
    scaling), and rounding that to an integer ties-to-even is the whole
    rounding step; a carry to 2048 moves to the next binade on its own
    because exponent and fraction are added, not or-ed. Values whose rounded
    magnitude reaches 2^16 overflow to infinity, or to 65504 when
    ``saturate`` is set. NaN maps to 0x7E00.
    """
    v = np.asarray(v, dtype=np.float64)
    neg = np.signbit(v)
    a = np.abs(v)
    finite = np.isfinite(a)
    a_f = np.where(finite, a, 0.0)
    _, e = np.frexp(a_f)                     # a = m * 2^e, m in [0.5, 1)
    E = e.astype(np.int64) - 1               # a in [2^E, 2^(E+1))
    qexp = np.maximum(E, -14) - 10           # log2 of the quantum
    n = np.rint(np.ldexp(a_f, -qexp)).astype(np.int64)
    sub = E < -14
    bits = np.where(sub, n, ((E + 15) << 10) + (n - 1024))
    bits = np.where(a_f == 0.0, 0, bits)
    over = bits >= 0x7C00
    inf_bits = 0x7BFF if saturate else 0x7C00
    bits = np.where(over, inf_bits, bits)
    bits = np.where(np.isinf(a), inf_bits, bits)
    bits = np.where(np.isnan(v), 0x7E00, bits)
    bits = np.where(neg & ~np.isnan(v), bits | 0x8000, bits)
    return bits.astype(np.uint16)


def binary16_bits_to_float(bits) -> np.ndarray:
    """Exact float64 value of binary16 bit patterns."""
    b = np.asarray(bits).astype(np.int64) & 0xFFFF
    sign = np.where(b & 0x8000, -1.0, 1.0)
    field = (b >> 10) & 0x1F
    frac = b & 0x3FF
    val = np.where(field == 0, np.ldexp(frac.astype(np.float64), -24),
                   np.ldexp((frac + 1024).astype(np.float64), field - 25))
    val = np.where(field == 31, np.where(frac == 0, np.inf, np.nan), val)
    return sign * val


# ---------------------------------------------------------------------------
# Codes
# ---------------------------------------------------------------------------

def pack_codes(q: np.ndarray, bits: int) -> np.ndarray:
    """Pack integer codes [..., d] into bytes [..., d*bits/8].

    "When Quantization Is Free", Methodology 2, step 5: two int4 values share
    one byte. Reading 11: element 2k in the low nibble, element 2k+1 in the
    high nibble, each as a 4-bit two's complement field. int8 codes are
    stored one per byte as two's complement.
    """
    q = np.asarray(q).astype(np.int64)
    if bits == 8:
        return (q & 0xFF).astype(np.uint8)
    if bits != 4:
        raise ValueError("bits must be 4 or 8")
    lo = q[..., 0::2] & 0xF
    hi = q[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Inverse of ``pack_codes``: bytes -> signed integers (int64)."""
    c = np.asarray(codes).astype(np.int64)
    if bits == 8:
        return np.where(c >= 128, c - 256, c)
    if bits != 4:
        raise ValueError("bits must be 4 or 8")
    lo = c & 0xF
    hi = (c >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(c.shape[:-1] + (c.shape[-1] * 2,), dtype=np.int64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def qmax_for(bits: int) -> int:
    """Largest code magnitude: 7 for int4, 127 for int8 (reading 7)."""
    if bits not in (4, 8):
        raise ValueError("bits must be 4 or 8")
    return (1 << (bits - 1)) - 1


# ---------------------------------------------------------------------------
# Quantiser and dequantiser
# ---------------------------------------------------------------------------

def quantize_vectors(y: np.ndarray, lam: np.ndarray, group: int, bits: int) -> dict:
    """Quantise already-rotated vectors y [..., d] (float64) with lambda [..., d].

    "When Quantization Is Free", Methodology 2, step 4 and Methodology 3:
    rescale every coordinate by its own lambda, take the absolute maximum over
    each group of ``group`` consecutive coordinates, round to a signed
    integer. Steps (decisions in float32, see the module docstring):

        w     = fl32(y) / lambda                      (float32 division)
        a_g   = max_{j in g} |w_j|
        sigma = binary16_rne(fl32(a_g / qmax)), saturated at 65504
        q_j   = clamp(rint(w_j / sigma), -qmax, qmax)  (float32 division)
        q_j   = 0 for the whole group when sigma == 0

    Returns q (int64, [..., d]), sigma bits (uint16, [..., d/G]) and the
    float64 diagnostics ``pre`` = (y / lambda) / sigma (the pre-rounding value
    in code units) and ``scale_pre`` = max|y/lambda| / qmax per group.
    """
    y = np.asarray(y, dtype=np.float64)
    d = y.shape[-1]
    if d % group != 0:
        raise ValueError("group must divide d")
    qmax = qmax_for(bits)
    lam32 = np.broadcast_to(np.asarray(lam, dtype=np.float32), y.shape)
    y32 = y.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        w = y32 / lam32
        wg = w.reshape(y.shape[:-1] + (d // group, group))
        a = np.max(np.abs(wg), axis=-1)
        r = a / np.float32(qmax)
        sig_bits = float_to_binary16_bits(r.astype(np.float64), saturate=True)
        sig = binary16_bits_to_float(sig_bits).astype(np.float32)
        v = wg / sig[..., None]
        q = np.clip(np.rint(v), -qmax, qmax)
        q = np.where(sig[..., None] == 0, 0.0, q)
        q = np.nan_to_num(q, nan=0.0).astype(np.int64).reshape(y.shape)
        w64 = y / lam32.astype(np.float64)
        a64 = np.max(np.abs(w64.reshape(wg.shape)), axis=-1)
        pre = (w64.reshape(wg.shape) / sig.astype(np.float64)[..., None]).reshape(y.shape)
    return {"q": q, "scale_bits": sig_bits, "pre": pre, "scale_pre": a64 / qmax}


def quantize(x: np.ndarray, signs: np.ndarray, lam: np.ndarray, group: int,
             bits: int, kind: int = SRFT) -> dict:
    """Full quantiser: rotate (float64 definition) then ``quantize_vectors``.

    x [S, N, H, d], signs [S, H, d], lam [S, H, d]. Returns a dict with
    ``codes`` (uint8 [S, N, H, d*bits/8]), ``scales`` (uint16 binary16 bits,
    [S, N, H, d/G]), the rotated ``y`` (float64) and the diagnostics of
    ``quantize_vectors``.
    """
    y = rotate(x, signs, kind)
    lam_b = np.asarray(lam, dtype=np.float32)[:, None, :, :]
    out = quantize_vectors(y, lam_b, group, bits)
    out["codes"] = pack_codes(out["q"], bits)
    out["scales"] = out["scale_bits"]
    out["y"] = y
    return out


def dequantize(codes: np.ndarray, scales: np.ndarray, signs: np.ndarray,
               lam: np.ndarray, d: int, group: int, bits: int,
               kind: int = SRFT) -> dict:
    """Inverse of ``quantize``: unpack, descale, un-rotate, round to binary16.

    yhat_j = q_j * sigma_g * lambda_j; xhat = R^T yhat (float64, the exact
    inverse of an orthogonal R); the result is rounded to binary16 ties to
    even (reading 13). Returns ``bits`` (uint16 [S, N, H, d]) and the float64
    value before that rounding as ``xhat64``.
    """
    q = unpack_codes(codes, bits)
    if q.shape[-1] != d:
        raise ValueError("codes do not match d")
    sig = binary16_bits_to_float(scales)
    S, N, H, _ = q.shape
    qg = q.reshape(S, N, H, d // group, group).astype(np.float64)
    yhat = (qg * sig[..., None]).reshape(S, N, H, d)
    yhat = yhat * np.asarray(lam, dtype=np.float32).astype(np.float64)[:, None, :, :]
    xhat64 = unrotate(yhat, signs, kind)
    return {"bits": float_to_binary16_bits(xhat64), "xhat64": xhat64, "yhat": yhat}


def dequantize_rotated(codes: np.ndarray, scales: np.ndarray, lam: np.ndarray, d: int,
                       group: int, bits: int) -> dict:
    """The dequantised cache left in the rotated domain: yhat_j = q_j * sigma_g
    * lambda_j (the first half of ``dequantize``, before R^T), float64, and
    its binary16 rounding (ties to even) as ``bits``. Since R is orthogonal
    ("When Quantization Is Free", Methodology 1), (R q) . yhat = q . (R^T yhat)
    for any query q: attention can run on these vectors with a rotated query.
    """
    q = unpack_codes(codes, bits)
    if q.shape[-1] != d:
        raise ValueError("codes do not match d")
    sig = binary16_bits_to_float(scales)
    S, N, H, _ = q.shape
    qg = q.reshape(S, N, H, d // group, group).astype(np.float64)
    yhat = (qg * sig[..., None]).reshape(S, N, H, d)
    yhat = yhat * np.asarray(lam, dtype=np.float32).astype(np.float64)[:, None, :, :]
    return {"bits": float_to_binary16_bits(yhat), "yhat": yhat}


def decode_attention(q: np.ndarray, k_codes: np.ndarray, k_scales: np.ndarray,
                     k_signs: np.ndarray, k_lam: np.ndarray, v_codes: np.ndarray,
                     v_scales: np.ndarray, v_signs: np.ndarray, v_lam: np.ndarray, d: int,
                     group: int, bits: int, kind: int, n_ctx: int, tok_stride_rows: int,
                     seq_stride_rows: int, scale: float) -> np.ndarray:
    """One decode step of attention over the quantised caches, float64:
    out[b, h*Q + g] = sum_t softmax_t(scale * q[b, h*Q + g] . khat[t]) vhat[t]
    with khat, vhat = ``dequantize`` of the rows t*tok_stride + b*seq_stride
    (before the binary16 rounding). q [n_seq][H*Q][d]; caches [rows][H][...];
    signs and lambda [H][d] (one slice)."""
    q = np.asarray(q, dtype=np.float64)
    n_seq, HQ, _ = q.shape
    H = k_codes.shape[1]
    Q = HQ // H
    out = np.empty((n_seq, HQ, d), dtype=np.float64)
    for b in range(n_seq):
        rows = np.arange(n_ctx) * tok_stride_rows + b * seq_stride_rows
        kx = dequantize(k_codes[None, rows], k_scales[None, rows], k_signs[None], k_lam[None],
                        d, group, bits, kind)["xhat64"][0]
        vx = dequantize(v_codes[None, rows], v_scales[None, rows], v_signs[None], v_lam[None],
                        d, group, bits, kind)["xhat64"][0]
        for h in range(H):
            for g in range(Q):
                s = scale * (kx[:, h, :] @ q[b, h * Q + g])
                p = np.exp(s - s.max())
                out[b, h * Q + g] = (p / p.sum()) @ vx[:, h, :]
    return out


def calibrate_lambda(x: np.ndarray, signs: np.ndarray, n_cal: int,
                     kind: int = SRFT) -> np.ndarray:
    """Per-channel lambda [S, H, d] (float64) from the first n_cal rows.

    Reading 6 of "When Quantization Is Free", Methodology 2 step 4 (a
    calibrated per-channel scale): lambda_{s,h,j} is the root mean square of
    rotated coordinate j of head h over rows 0 .. n_cal-1 of slice s; a
    channel whose sum of squares is zero gets lambda = 1.
    """
    x = np.asarray(x)
    if n_cal < 1 or n_cal > x.shape[1]:
        raise ValueError("n_cal must be in [1, N]")
    y = rotate(x[:, :n_cal], signs, kind)
    ss = np.sum(y * y, axis=1)
    lam = np.sqrt(ss / n_cal)
    return np.where(ss == 0.0, 1.0, lam)
