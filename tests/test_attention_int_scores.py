"""Host checks of the integer key-score scheme of the fused attention
(csrc/attention.cuh, int4 keys with one query per KV head).

The kernel writes each query coordinate q_j of a 16-coordinate sub-group m
as Q_j = rint(q_j 2^(E_m + 16)) = B0 2^16 + B1 2^8 + B2 (balanced
base-256 digits), with E_m = 5 - floor(log2 max|q| on m), and takes
sum_j c_j Q_j from u8 x s8 tensor-core products whose accumulator starts
at -8 sum B. These tests restate that arithmetic in numpy and check the
claims the kernel relies on: every digit is a signed byte, the combined
integer fits in int32 for the worst int4 codes, the representation error
is at most 2^-22 of the sub-group maximum, and the documented
mma.m16n8k32 fragment layouts together with the kernel's k-order give
the exact integer dot products. The GPU kernel itself is compared with
the oracle in tests/test_gpu_parity.py.
"""
import numpy as np
import pytest


def _digits(q: np.ndarray, e: int):
    """Balanced base-256 digits of rint(q 2^(e + 16)) (ties to even, as
    __float2int_rn); q float32, one sub-group."""
    Q = np.rint(np.ldexp(q.astype(np.float64), e + 16)).astype(np.int64)
    b2 = ((Q + 128) & 255) - 128
    q1 = (Q - b2) >> 8
    b1 = ((q1 + 128) & 255) - 128
    b0 = (q1 - b1) >> 8
    return Q, np.stack([b0, b1, b2])


def _exponent(q: np.ndarray) -> int:
    a = float(np.max(np.abs(q)))
    return 5 - int(np.floor(np.log2(a))) if a > 0 else 0


@pytest.mark.parametrize("scale", [1e-30, 1e-3, 1.0, 3.0e4, 1e30])
def test_digits_are_signed_bytes_and_exact_to_2_pow_minus_22(scale):
    rng = np.random.default_rng(7)
    for _ in range(200):
        q = (rng.standard_normal(16) * scale).astype(np.float32)
        q[rng.integers(16)] = np.float32(scale) * np.float32(1.999999)  # near the top of a binade
        e = _exponent(q)
        Q, b = _digits(q, e)
        assert np.all(np.abs(b[0]) <= 65) and np.all(np.abs(b[1:]) <= 128)
        assert np.array_equal(b[0] * 65536 + b[1] * 256 + b[2], Q)
        err = np.abs(np.ldexp(Q.astype(np.float64), -(e + 16)) - q.astype(np.float64))
        assert err.max() <= 2.0 ** -22 * np.abs(q).max()


def test_combined_integer_fits_int32_for_the_worst_codes():
    # |c| <= 8 over 16 coordinates, with the largest digits of either sign
    b0, b12 = 65, 128
    worst = 16 * 8 * (b0 * 65536 + b12 * 256 + b12)
    assert worst < 2 ** 31
    # every partial sum the accumulator holds: u = c + 8 in [0, 15] times a
    # digit, over 16 coordinates, after a start of -8 sum B
    assert 16 * 15 * 128 + 8 * 16 * 128 < 2 ** 31


def _pack(codes: np.ndarray) -> np.ndarray:
    """int4 codes [32, 128] -> uint32 words [32, 16]; coordinate 2i in the
    low nibble of byte i."""
    lo = codes[:, 0::2] & 15
    hi = codes[:, 1::2] & 15
    return (lo | (hi << 4)).astype(np.uint8).view("<u4")


@pytest.mark.parametrize("group", [16, 32, 64, 128])
def test_fragment_k_order_gives_exact_integer_scores(group):
    """Lane (g, t) of k-step ks holds word 4t + ks of token rows g, g + 8:
    low nibbles are k = 4t + i, high nibbles k = 4t + 16 + i (A of
    m16n8k32, rows g and g + 8); B holds digit p of the same coordinates in
    column g when g is the word's sub-group. Rebuilding A and B from those
    per-lane registers by the documented fragment layouts must give, per
    (token, sub-group), exactly sum_j c_j Q_j."""
    rng = np.random.default_rng(group)
    q = (rng.standard_normal(128) * 3.0).astype(np.float32)
    codes = rng.integers(-8, 8, size=(32, 128))
    codes[0] = -8
    codes[1] = 7
    words = _pack(codes)
    E = [_exponent(q[16 * m:16 * m + 16]) for m in range(8)]
    Qs, B = zip(*[_digits(q[16 * m:16 * m + 16], E[m]) for m in range(8)])
    Q = np.concatenate(Qs)
    Bd = np.concatenate(B, axis=1)                       # [3, 128]
    S = np.array([[Bd[p, 16 * m:16 * m + 16].sum() for m in range(8)] for p in range(3)])
    for mt in range(2):
        acc = np.zeros((3, 16, 8), np.int64)
        for p in range(3):
            acc[p] += -8 * S[p][None, :]                 # accumulator start, per column
        for ks in range(4):
            A = np.zeros((16, 32), np.int64)
            Bm = np.zeros((3, 32, 8), np.int64)
            for lane in range(32):
                g, t = lane >> 2, lane & 3
                w = 4 * t + ks
                regs = []
                for row in (16 * mt + g, 16 * mt + g + 8):
                    wd = int(words[row, w])
                    regs.append((wd & 0x0F0F0F0F) ^ 0x08080808)
                    regs.append(((wd >> 4) & 0x0F0F0F0F) ^ 0x08080808)
                a = [regs[0], regs[2], regs[1], regs[3]]   # {row g lo, row g+8 lo, row g hi, row g+8 hi}
                for i in range(16):
                    row = g if (i < 4 or 8 <= i < 12) else g + 8
                    col = 4 * t + (i & 3) + (16 if i >= 8 else 0)
                    A[row, col] = (a[i // 4] >> (8 * (i & 3))) & 0xFF
                for p in range(3):
                    for i in range(8):
                        c = 8 * w + 2 * (i & 3) + (1 if i >= 4 else 0)
                        k = 4 * t + (i & 3) + (16 if i >= 4 else 0)
                        Bm[p, k, g] = Bd[p, c] if c // 16 == g else 0
            for p in range(3):
                acc[p] += A @ Bm[p]
        D = (acc[0] << 16) + (acc[1] << 8) + acc[2]
        for r in range(16):
            tok = 16 * mt + r
            for m in range(8):
                sl = slice(16 * m, 16 * m + 16)
                assert D[r, m] == int(np.dot(codes[tok, sl], Q[sl]))
                assert abs(D[r, m]) < 2 ** 31
