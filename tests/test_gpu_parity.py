"""GPU parity: the CUDA library against the CPU oracle, through the C ABI.

Small cases run every compiled configuration in full (several 32-row tiles,
a ragged last tile, several slices and heads). The paper-shaped workloads run
at full size in the same launch configuration the benchmark uses; the oracle
checks a sample of rows from every slice, and properties that hold for any
size are checked on every vector.
"""

import math

import numpy as np
import pytest

import kv_synth
import oracle
import parity

torch = pytest.importorskip("torch")
import rotate_then_quantize_b200 as rq  # noqa: E402

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    rq.load_library()
    yield
    assert rq.srftq_check_device() == 0, "a device-side guard fired"


def _signs(rng, S, H, d):
    return np.where(rng.random((S, H, d)) < 0.5, -1, 1).astype(np.int8)


def _x(rng, S, N, H, d, outlier_p=0.01, scale=20.0):
    x = rng.standard_normal((S, N, H, d))
    x = np.where(rng.random(x.shape) < outlier_p, x * scale, x)
    return x.astype(np.float16)


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _np16(t):
    return t.cpu().numpy().view(np.uint16)


def run_and_check(x16, signs, lam, d, group, bits, rot, what):
    """Rotation, quantisation and dequantisation of x16 on the GPU vs the oracle."""
    xt, st, lt = _t(x16), _t(signs), _t(lam)
    y = rq.rotate(xt, st, lt, rotation=rot).cpu().numpy()
    y_ref = oracle.rotate(x16, signs, rot) / lam[:, None].astype(np.float64)
    parity.assert_clean(parity.check_rotation(y, y_ref), f"{what} rotate")

    codes, scales = rq.quantize(xt, st, lt, group, bits, rot)
    ref = oracle.quantize(x16, signs, lam, group, bits, rot)
    c_np, s_np = codes.cpu().numpy(), _np16(scales)
    stats = parity.check_codes(ref, c_np, s_np, bits, group)
    parity.assert_clean(stats, f"{what} codes")

    # the dequantiser runs on the oracle's codes, so both sides see the same input
    deq = oracle.dequantize(ref["codes"], ref["scales"], signs, lam, d, group, bits, rot)
    xhat = rq.dequantize(_t(ref["codes"]), _t(ref["scales"].view(np.float16)), st, lt, d, group,
                         bits, rot)
    parity.assert_clean(parity.check_dequant(_np16(xhat), deq["bits"]), f"{what} dequant")
    # and the GPU round trip, where its codes equal the oracle's
    xhat_rt = rq.dequantize(codes, scales, st, lt, d, group, bits, rot)
    check_dequant_where_codes_match(_np16(xhat_rt), c_np, s_np, ref, deq, f"{what} round trip")
    return stats


def check_dequant_where_codes_match(xh_bits, c_np, s_np, ref, deq, what):
    """Dequantised vectors of the GPU's own codes against the oracle's
    dequantisation of the oracle's codes, on the vectors whose codes and
    scales are identical (all but the flagged rounding-boundary cases)."""
    same = np.all(c_np == ref["codes"], axis=-1) & np.all(s_np == ref["scales"], axis=-1)
    parity.assert_clean(parity.check_dequant(xh_bits[same], deq["bits"][same]), what)
    return int((~same).sum())


def _configs():
    out = []
    for d in (16, 32, 64, 128, 256):
        for bits in (4, 8):
            g = 8
            while g <= d:
                for rot in (rq.SRFT, rq.SRHT):
                    out.append((d, bits, g, rot))
                g *= 2
    return out


@pytest.mark.parametrize("d,bits,group,rot", _configs())
def test_small_sweep(d, bits, group, rot):
    rng = np.random.default_rng(1000 * d + 100 * bits + group + rot)
    S, N, H = 2, 45, 3
    x16 = _x(rng, S, N, H, d)
    signs = _signs(rng, S, H, d)
    lam = oracle.calibrate_lambda(x16, signs, 32, rot).astype(np.float32)
    run_and_check(x16, signs, lam, d, group, bits, rot, f"d{d} b{bits} g{group} r{rot}")
    lam_gpu = rq.calibrate_lambda(_t(x16), _t(signs), 32, rotation=rot).cpu().numpy()
    parity.assert_clean(parity.check_lambda(lam_gpu, oracle.calibrate_lambda(x16, signs, 32, rot)),
                        "lambda")


@pytest.mark.parametrize("N", [1, 31, 32, 33, 97])
@pytest.mark.parametrize("H", [1, 5])
def test_ragged_rows_and_heads(N, H):
    rng = np.random.default_rng(N * 7 + H)
    d, group, bits = 64, 16, 4
    x16 = _x(rng, 3, N, H, d)
    signs = _signs(rng, 3, H, d)
    lam = np.exp(rng.uniform(-1, 1, (3, H, d))).astype(np.float32)
    run_and_check(x16, signs, lam, d, group, bits, rq.SRFT, f"N{N} H{H}")


@pytest.mark.parametrize("H", [2, 4, 6, 8, 12, 16])
@pytest.mark.parametrize("d,bits,group", [(64, 4, 16), (128, 4, 16), (128, 8, 32), (128, 4, 64),
                                           (256, 4, 32), (256, 8, 64), (256, 4, 128),
                                           (256, 8, 256)])
def test_head_block_tiles(H, d, bits, group):
    """Tiles span up to 8 heads of 32 / heads-per-tile rows; cover every
    heads-per-tile value, several head blocks per slice and ragged rows."""
    rng = np.random.default_rng(100 * H + d)
    S, N = 2, 29
    x16 = _x(rng, S, N, H, d)
    signs = _signs(rng, S, H, d)
    lam = np.exp(rng.uniform(-1, 1, (S, H, d))).astype(np.float32)
    run_and_check(x16, signs, lam, d, group, bits, rq.SRFT, f"H{H} d{d}")


@pytest.mark.parametrize("n_cal", [1, 64, 100, 512, 700, 1100])
@pytest.mark.parametrize("d", [64, 256])
def test_calibration_row_counts(n_cal, d):
    """Calibration runs one 8-block cluster per (slice, head), block r taking
    the 64-row batches 64 (r + 8 b): cover fewer rows than one batch, ragged
    batches, exactly one batch per block and several batches per block."""
    rng = np.random.default_rng(n_cal + d)
    S, H = 2, 3
    x16 = _x(rng, S, max(n_cal, 8), H, d)
    signs = _signs(rng, S, H, d)
    for rot in (rq.SRFT, rq.SRHT):
        lam_gpu = rq.calibrate_lambda(_t(x16), _t(signs), n_cal, rotation=rot).cpu().numpy()
        parity.assert_clean(
            parity.check_lambda(lam_gpu, oracle.calibrate_lambda(x16, signs, n_cal, rot)),
            f"lambda n_cal={n_cal} d={d} rot={rot}")


@pytest.mark.parametrize("N", [1, 15, 16, 17, 47])
@pytest.mark.parametrize("rot", [0, 1])
@pytest.mark.parametrize("d,group", [(128, 16), (256, 32)])
def test_ragged_rows_d128_d256(N, rot, d, group):
    """Ragged row counts leave part of the last tile empty: at d = 128 (one
    thread per vector) and at d = 256 (two warps sharing a tile, both of
    which must skip the missing rows)."""
    rng = np.random.default_rng(N * 11 + rot + d)
    bits, H = 4, 3
    x16 = _x(rng, 2, N, H, d, outlier_p=0.005, scale=25.0)
    signs = _signs(rng, 2, H, d)
    lam = np.exp(rng.uniform(-1, 1, (2, H, d))).astype(np.float32)
    run_and_check(x16, signs, lam, d, group, bits, rot, f"d{d} N{N} r{rot}")


@pytest.mark.parametrize("group", [128, 256])
@pytest.mark.parametrize("rot", [0, 1])
@pytest.mark.parametrize("N", [1, 7, 40])
def test_groups_spanning_both_warps_d256(group, rot, N):
    """At d = 256 the codec splits each vector over two warps. A group of
    128 coordinates (SRFT) or 256 (either rotation; 256 is one scale per
    vector, the per-token baseline) has coordinates in both warps, whose
    partial absmaxes are combined before the scale is formed; an SRHT group
    of 128 lies inside one warp. Ragged rows, several heads, outliers."""
    rng = np.random.default_rng(N * 13 + group + rot)
    d, H = 256, 3
    x16 = _x(rng, 2, N, H, d, outlier_p=0.005, scale=25.0)
    signs = _signs(rng, 2, H, d)
    lam = np.exp(rng.uniform(-1, 1, (2, H, d))).astype(np.float32)
    for bits in (4, 8):
        run_and_check(x16, signs, lam, d, group, bits, rot, f"d256 g{group} r{rot} N{N} b{bits}")


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("bits", [4, 8])
def test_strided_views_and_guard_bands(bits, d):
    """Slices with a row stride larger than the rows used (a cache written at a
    row offset); rows outside the written window must keep their sentinel."""
    rng = np.random.default_rng(bits + d)
    S, T, H, group, N, off = 3, 100, 2, 16, 37, 41
    big = _x(rng, S, T, H, d)
    signs = _signs(rng, S, H, d)
    lam = np.exp(rng.uniform(-0.5, 0.5, (S, H, d))).astype(np.float32)
    xt, st, lt = _t(big), _t(signs), _t(lam)
    codes_big = torch.full((S, T, H, d * bits // 8), 0xAB, dtype=torch.uint8, device=DEV)
    scales_big = torch.full((S, T, H, d // group), 7.0, dtype=torch.float16, device=DEV)
    desc = rq.make_desc(d, H, group, bits)
    rq.srftq_quantize(desc, xt[:, off:off + N], st, lt, codes_big[:, off:off + N],
                      scales_big[:, off:off + N])
    ref = oracle.quantize(big[:, off:off + N], signs, lam, group, bits)
    c_np = codes_big.cpu().numpy()
    s_np = _np16(scales_big)
    parity.assert_clean(parity.check_codes(ref, c_np[:, off:off + N], s_np[:, off:off + N],
                                           bits, group), "strided codes")
    outside = np.ones(T, dtype=bool)
    outside[off:off + N] = False
    assert np.all(c_np[:, outside] == 0xAB)
    assert np.all(s_np[:, outside] == np.float16(7.0).view(np.uint16))
    # dequantise the oracle's codes, placed in the strided window, into a
    # strided view with a sentinel around it
    codes_big[:, off:off + N] = _t(ref["codes"])
    scales_big[:, off:off + N] = _t(ref["scales"].view(np.float16))
    xh_big = torch.full((S, T, H, d), -3.0, dtype=torch.float16, device=DEV)
    rq.srftq_dequantize(desc, codes_big[:, off:off + N], scales_big[:, off:off + N], st, lt,
                        xh_big[:, off:off + N])
    deq = oracle.dequantize(ref["codes"], ref["scales"], signs, lam, d, group, bits)
    xh = _np16(xh_big)
    parity.assert_clean(parity.check_dequant(xh[:, off:off + N], deq["bits"]), "strided dequant")
    assert np.all(xh[:, outside] == np.float16(-3.0).view(np.uint16))


def test_degenerate_values():
    """Zero vectors (sigma = 0), values driving sigma subnormal or saturated,
    and exact ties; all decided as the oracle decides them."""
    rng = np.random.default_rng(5)
    S, N, H, d, group = 1, 64, 1, 64, 16
    x = rng.standard_normal((S, N, H, d))
    x[:, 0] = 0.0                              # all-zero vector
    x[:, 1] = 1e-7 * rng.standard_normal(d)    # tiny: subnormal scales
    x[:, 2] = 6e4 * np.sign(rng.standard_normal(d))  # near fp16 max
    x[:, 3, :, 5] = 1.0                        # single spike
    x16 = x.astype(np.float16)
    signs = _signs(rng, S, H, d)
    for lam_val in (1.0, 1e-3, 3e3):
        lam = np.full((S, H, d), lam_val, dtype=np.float32)
        for bits in (4, 8):
            run_and_check(x16, signs, lam, d, group, bits, rq.SRFT, f"degenerate lam={lam_val}")


def test_non_finite_inputs_do_not_fault():
    rng = np.random.default_rng(9)
    x16 = _x(rng, 1, 40, 2, 128)
    x16[0, 3, 0, 7] = np.inf
    x16[0, 5, 1, 0] = np.nan
    signs = _signs(rng, 1, 2, 128)
    lam = np.ones((1, 2, 128), np.float32)
    codes, scales = rq.quantize(_t(x16), _t(signs), _t(lam), 16, 4)
    rq.dequantize(codes, scales, _t(signs), _t(lam), 128, 16, 4)
    torch.cuda.synchronize()
    assert rq.srftq_check_device() == 0
    # rows without non-finite values are still exact
    clean = [r for r in range(40) if r not in (3, 5)]
    ref = oracle.quantize(x16[:, clean], signs, lam, 16, 4)
    parity.assert_clean(parity.check_codes(ref, codes.cpu().numpy()[:, clean],
                                           _np16(scales)[:, clean], 4, 16), "finite rows")


def test_bounded_wait_that_runs_out_is_reported_and_the_context_stays_usable():
    """Failure detection without a fault: a wait on a barrier nothing arrives
    on gives up after its poll limit, records the timeout in the guard word
    (as every codec kernel's bounded wait does), and the next check reports
    it; the same context then runs a codec call cleanly."""
    assert rq.srftq_check_device() == 0
    assert rq.srftq_probe_wait_timeout(1 << 12) == 0
    assert rq.srftq_check_device() == rq.binding.SRFTQ_ERR_DEVICE_CHECK
    assert rq.srftq_check_device() == 0          # the check cleared the word
    rng = np.random.default_rng(5)
    x16 = _x(rng, 1, 40, 2, 128)
    signs = _signs(rng, 1, 2, 128)
    lam = np.exp(rng.uniform(-1, 1, (1, 2, 128))).astype(np.float32)
    run_and_check(x16, signs, lam, 128, 16, 4, rq.SRFT, "after timeout probe")
    assert rq.srftq_check_device() == 0


def test_empty_call_launches_nothing():
    x = torch.empty((2, 0, 3, 64), dtype=torch.float16, device=DEV)
    codes, scales = rq.quantize(x, torch.ones((2, 3, 64), dtype=torch.int8, device=DEV),
                                torch.ones((2, 3, 64), device=DEV), 16, 4)
    assert codes.numel() == 0 and scales.numel() == 0


# ---------------------------------------------------------------------------
# Paper-shaped workloads
# ---------------------------------------------------------------------------

def test_tiny_workload_full():
    """4096 vectors, d=64, seeded exactly as specified; every output checked."""
    w = kv_synth.WORKLOADS["tiny_d64"]
    x16, signs = kv_synth.tiny_inputs()
    lam64 = oracle.calibrate_lambda(x16, signs, w.n_cal)
    lam_gpu = rq.calibrate_lambda(_t(x16), _t(signs), w.n_cal).cpu().numpy()
    parity.assert_clean(parity.check_lambda(lam_gpu, lam64), "tiny lambda")
    stats = run_and_check(x16, signs, lam64.astype(np.float32), w.d, w.group, w.bits, rq.SRFT,
                          "tiny")
    print("tiny codes:", stats)


def _sample_rows(rng, N, k):
    rows = np.unique(np.concatenate([rng.choice(N, size=k, replace=False), [0, N - 1]]))
    return rows


def _workload_check(name, rot, k_rows=48):
    w = kv_synth.WORKLOADS[name]
    rng = np.random.default_rng(17)
    x = kv_synth.make_x_torch(w, DEV, seed=0)
    signs = kv_synth.rademacher_signs(w.S, w.H, w.d, seed=1)
    st = _t(signs)
    # lambda: the oracle's, from the first n_cal rows of every slice
    x_cal = x[:, :w.n_cal].cpu().numpy()
    lam64 = oracle.calibrate_lambda(x_cal, signs, w.n_cal, rot)
    lam = lam64.astype(np.float32)
    lt = _t(lam)
    lam_gpu = rq.calibrate_lambda(x, st, w.n_cal, rotation=rot).cpu().numpy()
    parity.assert_clean(parity.check_lambda(lam_gpu, lam64), f"{name} lambda")

    codes, scales = rq.quantize(x, st, lt, w.group, w.bits, rot)
    xhat = rq.dequantize(codes, scales, st, lt, w.d, w.group, w.bits, rot)
    torch.cuda.synchronize()

    totals = {}
    for s in range(w.S):
        rows = _sample_rows(rng, w.N, k_rows)
        xs = x[s:s + 1, rows].cpu().numpy()
        ref = oracle.quantize(xs, signs[s:s + 1], lam[s:s + 1], w.group, w.bits, rot)
        c_np = codes[s:s + 1, rows].cpu().numpy()
        s_np = _np16(scales[s:s + 1, rows])
        stats = parity.check_codes(ref, c_np, s_np, w.bits, w.group)
        parity.assert_clean(stats, f"{name} slice {s} codes")
        deq = oracle.dequantize(ref["codes"], ref["scales"], signs[s:s + 1], lam[s:s + 1], w.d,
                                w.group, w.bits, rot)
        # the full-size launch's output where its codes equal the oracle's ...
        check_dequant_where_codes_match(_np16(xhat[s:s + 1, rows]), c_np, s_np, ref, deq,
                                        f"{name} slice {s} dequant")
        # ... and the dequantiser on the oracle's own codes for the sampled rows
        xh_ref_in = rq.dequantize(_t(ref["codes"]), _t(ref["scales"].view(np.float16)),
                                  st[s:s + 1], lt[s:s + 1], w.d, w.group, w.bits, rot)
        parity.assert_clean(parity.check_dequant(_np16(xh_ref_in), deq["bits"]),
                            f"{name} slice {s} dequant of the oracle's codes")
        for key, v in stats.items():
            totals[key] = totals.get(key, 0) + v

    # every vector: range of codes, and the orthogonal error bound
    qmin_code = 0x8 if w.bits == 4 else 0x80
    if w.bits == 4:
        assert not bool(((codes & 0xF) == qmin_code).any() or ((codes >> 4) == qmin_code).any())
    else:
        assert not bool((codes == qmin_code).any())
    sig = scales.float().repeat_interleave(w.group, dim=-1)
    bound = torch.linalg.vector_norm(sig * lt[:, None] / 2, dim=-1)
    err = torch.linalg.vector_norm(xhat.float() - x.float(), dim=-1)
    slack = torch.linalg.vector_norm(xhat.float(), dim=-1) * 2.0 ** -11 + 1e-3 * bound + 1e-6
    assert bool((err <= bound + slack).all()), float((err - bound - slack).max())
    rel = (err / torch.linalg.vector_norm(x.float(), dim=-1).clamp_min(1e-12))
    print(f"{name} rot{rot}: sampled code stats {totals}; rel-L2 error mean "
          f"{float(rel.mean()):.4f} p99 {float(rel.quantile(0.99) if rel.numel() < 2**24 else rel[:2**24].quantile(0.99)):.4f}")
    del x, codes, scales, xhat
    torch.cuda.empty_cache()
    return totals


def test_qwen_like_workload_sampled():
    _workload_check("qwen_like_d128", rq.SRFT)


@pytest.mark.parametrize("rot", [0, 1])
def test_longctx_int8_workload_sampled(rot):
    _workload_check("longctx_int8_d128", rot)


def test_gemma_like_d256_workload_sampled():
    _workload_check("gemma_like_d256", rq.SRFT)


@pytest.mark.parametrize("rot", [0, 1])
def test_decode_streaming_appends(rot):
    """Decode-style use: a cache with spare capacity is filled, then each step
    appends one token for every sequence (rows token * B + sequence) and the
    whole cache is dequantized. Appended codes must equal a one-shot
    quantization of all tokens; untouched capacity keeps its sentinel."""
    rng = np.random.default_rng(31 + rot)
    S, B, T0, steps, H, d, group, bits = 4, 4, 20, 3, 2, 128, 16, 4
    cap = (T0 + steps + 2) * B
    x_all = _x(rng, S, (T0 + steps) * B, H, d, outlier_p=0.0)
    signs = _signs(rng, S, H, d)
    st = _t(signs)
    lam_np = oracle.calibrate_lambda(x_all[:, :T0 * B], signs, 16, rot).astype(np.float32)
    lam = _t(lam_np)
    codes = torch.full((S, cap, H, d * bits // 8), 0x5A, dtype=torch.uint8, device=DEV)
    scales = torch.full((S, cap, H, d // group), 9.0, dtype=torch.float16, device=DEV)
    xhat = torch.full((S, cap, H, d), 5.0, dtype=torch.float16, device=DEV)
    desc = rq.make_desc(d, H, group, bits, rot)
    rq.srftq_quantize(desc, _t(x_all[:, :T0 * B]), st, lam, codes[:, :T0 * B], scales[:, :T0 * B])
    for t in range(steps):
        r0 = (T0 + t) * B
        for layer in range(S // 2):
            sl = slice(2 * layer, 2 * layer + 2)
            rq.srftq_quantize(desc, _t(x_all[sl, r0:r0 + B]), st[sl], lam[sl], codes[sl, r0:r0 + B],
                              scales[sl, r0:r0 + B])
            rq.srftq_dequantize(desc, codes[sl, :r0 + B], scales[sl, :r0 + B], st[sl], lam[sl],
                                xhat[sl, :r0 + B])
    n = (T0 + steps) * B
    ref = oracle.quantize(x_all, signs, lam_np, group, bits, rot)
    c_np, s_np = codes.cpu().numpy(), _np16(scales)
    parity.assert_clean(parity.check_codes(ref, c_np[:, :n], s_np[:, :n], bits, group), "append codes")
    deq = oracle.dequantize(ref["codes"], ref["scales"], signs, lam_np, d, group, bits, rot)
    xh = _np16(xhat)
    check_dequant_where_codes_match(xh[:, :n], c_np[:, :n], s_np[:, :n], ref, deq,
                                    "streamed dequant")
    assert np.all(c_np[:, n:] == 0x5A)
    assert np.all(s_np[:, n:] == np.float16(9.0).view(np.uint16))
    assert np.all(xh[:, n:] == np.float16(5.0).view(np.uint16))


# ---------------------------------------------------------------------------
# Decode in the rotated domain: R orthogonal, so (R q) . (R x) = q . x
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d,bits,group", [(16, 4, 8), (64, 4, 16), (128, 4, 16), (128, 8, 32),
                                          (128, 4, 128), (256, 4, 32), (256, 8, 64)])
def test_dequantize_rotated_matches_oracle(d, bits, group):
    rng = np.random.default_rng(7 * d + bits + group)
    S, N, H = 2, 37, 3
    x16 = _x(rng, S, N, H, d)
    signs = _signs(rng, S, H, d)
    lam = np.exp(rng.uniform(-1, 1, (S, H, d))).astype(np.float32)
    ref = oracle.quantize(x16, signs, lam, group, bits)
    out = rq.dequantize_rotated(_t(ref["codes"]), _t(ref["scales"].view(np.float16)), _t(lam),
                                d, group, bits)
    want = oracle.dequantize_rotated(ref["codes"], ref["scales"], lam, d, group, bits)
    parity.assert_clean(parity.check_dequant(_np16(out), want["bits"]),
                        f"rotated dequant d{d} b{bits} g{group}")
    # a strided window of a larger cache leaves the rows around it untouched
    big = torch.full((S, N + 9, H, d), 7.0, dtype=torch.float16, device=DEV)
    desc = rq.make_desc(d, H, group, bits)
    rq.srftq_dequantize_rotated(desc, _t(ref["codes"]), _t(ref["scales"].view(np.float16)),
                                _t(lam), big[:, 4:4 + N])
    assert torch.equal(big[:, 4:4 + N], out)
    assert torch.all(big[:, :4] == 7.0) and torch.all(big[:, 4 + N:] == 7.0)


def test_dequantize_rotated_full_decode_stream_layer_sampled():
    """One decode-stream layer as the bench dequantises it in the rotated
    domain: 2 slices (K, V) x 1,048,576 rows (32,768 tokens x 32 sequences)
    x 8 heads, int4 G16, in one launch (the grid walks the slices in y and a
    slice's 134 M chunks in x). Codes in [-7, 7], fp16 scales in [0.01,
    0.3] and lambda in [0.5, 2] are drawn on the device; 4096 sampled rows
    are checked against the oracle."""
    import torch
    S, N, H, d, group, bits = 2, 32768 * 32, 8, 128, 16, 4
    gen = torch.Generator(device=DEV)
    gen.manual_seed(77)
    codes = torch.randint(0, 256, (S, N, H, d // 2), generator=gen, device=DEV,
                          dtype=torch.int32).to(torch.uint8)
    codes ^= ((codes & 0x0F) == 0x08).to(torch.uint8) * 0x08
    codes ^= ((codes >> 4) == 0x08).to(torch.uint8) * 0x80
    scales = (torch.rand((S, N, H, d // group), generator=gen, device=DEV) * 0.29
              + 0.01).to(torch.float16)
    lam = torch.rand((S, H, d), generator=gen, device=DEV) * 1.5 + 0.5
    out = rq.dequantize_rotated(codes, scales, lam, d, group, bits)
    torch.cuda.synchronize()
    rows = torch.randint(0, N, (4096,), generator=gen, device=DEV)
    rows[0], rows[-1] = 0, N - 1
    for s_ in range(S):
        c = codes[s_].index_select(0, rows).cpu().numpy()[None]
        sc = scales[s_].index_select(0, rows).cpu().numpy().view(np.uint16)[None]
        want = oracle.dequantize_rotated(c, sc, lam[s_:s_ + 1].cpu().numpy(), d, group, bits)
        got = out[s_].index_select(0, rows).cpu().numpy().view(np.uint16)[None]
        parity.assert_clean(parity.check_dequant(got, want["bits"]),
                            f"rotated dequant, full layer, slice {s_}")


@pytest.mark.parametrize("d", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("rot", [0, 1])
def test_unrotate_matches_oracle_and_inverts_rotate(d, rot):
    rng = np.random.default_rng(13 * d + rot)
    S, N, H = 2, 21, 3
    y = rng.standard_normal((S, N, H, d)).astype(np.float32)
    signs = _signs(rng, S, H, d)
    x = rq.unrotate(_t(y), _t(signs), rotation=rot).cpu().numpy()
    parity.assert_clean(parity.check_rotation(x, oracle.unrotate(y, signs, rot)), f"unrotate d{d}")
    x16 = _x(rng, S, N, H, d)
    back = rq.unrotate(rq.rotate(_t(x16), _t(signs), rotation=rot), _t(signs),
                       rotation=rot).cpu().numpy()
    parity.assert_clean(parity.check_rotation(back, x16.astype(np.float64)), f"round trip d{d}")


@pytest.mark.parametrize("rot", [0, 1])
def test_decode_attention_in_the_rotated_domain(rot):
    """One decode query per head against an int4 K/V cache, run entirely in
    the rotated domain on the GPU (rotate q with K's signs, score against the
    rotated-domain K cache, softmax, accumulate the rotated-domain V cache,
    unrotate the output with V's signs) and compared with float64 attention
    over the oracle's dequantised K and V."""
    rng = np.random.default_rng(21 + rot)
    T, H, d, group, bits = 300, 4, 128, 16, 4
    # the decode-stream cache's distribution: N(0, 1), no outliers
    k16 = _x(rng, 1, T, H, d, outlier_p=0.0)
    v16 = _x(rng, 1, T, H, d, outlier_p=0.0)
    sk, sv = _signs(rng, 1, H, d), _signs(rng, 1, H, d)
    lk = oracle.calibrate_lambda(k16, sk, 128, rot).astype(np.float32)
    lv = oracle.calibrate_lambda(v16, sv, 128, rot).astype(np.float32)
    qk = oracle.quantize(k16, sk, lk, group, bits, rot)
    qv = oracle.quantize(v16, sv, lv, group, bits, rot)
    q16 = _x(rng, 1, 1, H, d, outlier_p=0.0)

    q_rot = rq.rotate(_t(q16), _t(sk), rotation=rot)[0, 0]                      # [H, d]
    k_rot = rq.dequantize_rotated(_t(qk["codes"]), _t(qk["scales"].view(np.float16)), _t(lk),
                                  d, group, bits)[0].float()                     # [T, H, d]
    v_rot = rq.dequantize_rotated(_t(qv["codes"]), _t(qv["scales"].view(np.float16)), _t(lv),
                                  d, group, bits)[0].float()
    scores = torch.einsum("hd,thd->ht", q_rot, k_rot) / math.sqrt(d)
    p = torch.softmax(scores, dim=1)
    o_rot = torch.einsum("ht,thd->hd", p, v_rot)
    o = rq.unrotate(o_rot[None, None].contiguous(), _t(sv), rotation=rot)[0, 0].cpu().numpy()

    # (1) the same arithmetic in float64: attention over the oracle's own
    # fp16-rounded rotated-domain K and V (bit-equal to the GPU's, checked by
    # test_dequantize_rotated_matches_oracle), the rotated query, R^T of the
    # output; only float32 accumulation on the GPU differs (~1e-6 relative)
    ky16 = oracle.binary16_bits_to_float(
        oracle.dequantize_rotated(qk["codes"], qk["scales"], lk, d, group, bits)["bits"])[0]
    vy16 = oracle.binary16_bits_to_float(
        oracle.dequantize_rotated(qv["codes"], qv["scales"], lv, d, group, bits)["bits"])[0]
    qy = oracle.rotate(q16, sk, rot)[0, 0]
    # (2) exact attention over the dequantised cache (no fp16 storage)
    kx = oracle.dequantize(qk["codes"], qk["scales"], sk, lk, d, group, bits, rot)["xhat64"][0]
    vx = oracle.dequantize(qv["codes"], qv["scales"], sv, lv, d, group, bits, rot)["xhat64"][0]
    for h in range(H):
        s16 = ky16[:, h, :] @ qy[h] / math.sqrt(d)
        p16 = np.exp(s16 - s16.max())
        p16 /= p16.sum()
        o16 = oracle.unrotate((p16 @ vy16[:, h, :])[None, None, None, :], sv[:, h:h + 1, :],
                              rot)[0, 0, 0]
        err16 = np.abs(o[h] - o16) / np.maximum(1.0, np.abs(o16))
        assert err16.max() < 1e-4, ("same arithmetic", h, float(err16.max()))
        s_ref = kx[:, h, :] @ q16[0, 0, h, :].astype(np.float64) / math.sqrt(d)
        p_ref = np.exp(s_ref - s_ref.max())
        p_ref /= p_ref.sum()
        o_ref = p_ref @ vx[:, h, :]
        # fp16 storage of K and V moves the output by ~1e-4 on this unit-scale
        # data; 2e-3 only guards against gross disagreement
        err = np.abs(o[h] - o_ref) / np.maximum(1.0, np.abs(o_ref))
        assert err.max() < 2e-3, ("exact attention", h, float(err.max()))


# ---------------------------------------------------------------------------
# Fused decode attention over the quantised cache (rotated domain)
# ---------------------------------------------------------------------------

def _attn_case(rng, rows, H, d, group, bits, rot, outliers=0.0):
    x = _x(rng, 1, rows, H, d, outlier_p=outliers)
    s = _signs(rng, 1, H, d)
    lam = oracle.calibrate_lambda(x, s, min(rows, 64), rot).astype(np.float32)
    qz = oracle.quantize(x, s, lam, group, bits, rot)
    return qz["codes"][0], qz["scales"][0], s[0], lam[0]


@pytest.mark.parametrize("n_ctx", [1, 5, 128, 129, 1000])
@pytest.mark.parametrize("q_per_kv", [1, 2, 8])
@pytest.mark.parametrize("bits,group,rot", [(4, 16, 0), (8, 32, 1), (4, 128, 1), (4, 32, 0),
                                            (4, 64, 1)])
def test_decode_attention_matches_oracle(n_ctx, q_per_kv, bits, group, rot):
    """Token counts below the cluster's 8 CTAs (empty CTAs), ragged and
    exact tiles; grouped queries; both rotations. The GPU path is float32
    from codes to output (no fp16 cache), so it must agree with float64
    attention over the dequantised cache to ~1e-5 relative."""
    rng = np.random.default_rng(n_ctx * 31 + q_per_kv * 7 + bits + group + rot)
    H, d, n_seq = 2, 128, 3
    rows = n_ctx * n_seq
    kc, ks, ksg, kl = _attn_case(rng, rows, H, d, group, bits, rot)
    vc, vs, vsg, vl = _attn_case(rng, rows, H, d, group, bits, rot)
    q = rng.standard_normal((n_seq, H * q_per_kv, d)).astype(np.float16)
    scale = 1.0 / math.sqrt(d)
    out = rq.decode_attention(_t(q), _t(kc), _t(ks.view(np.float16)), _t(ksg), _t(kl), _t(vc),
                              _t(vs.view(np.float16)), _t(vsg), _t(vl), group, bits, rot,
                              n_ctx=n_ctx, tok_stride_rows=n_seq, seq_stride_rows=1,
                              scale=scale).cpu().numpy()
    ref = oracle.decode_attention(q, kc, ks, ksg, kl, vc, vs, vsg, vl, d, group, bits, rot, n_ctx,
                                  n_seq, 1, scale)
    err = np.abs(out - ref) / np.maximum(1.0, np.abs(ref))
    assert err.max() < 2e-5, float(err.max())


def test_decode_attention_full_decode_stream_size_sampled():
    """The launch configuration the decode-stream bench times: 32 sequences x
    8 KV heads (256 clusters) over 32,768 cached tokens, int4 G16, SRFT, one
    query per KV head, rows = token * 32 + sequence. The cache is drawn on
    the device (codes in [-7, 7], as the quantiser writes them, fp16 scales
    in [0.01, 0.3], lambda in [0.5, 2]); three (sequence, head) outputs are
    checked against float64 attention over the oracle's dequantisation of
    the same rows. Each lane sums about 1,000 float32 products per
    coordinate, so the bound is 1e-4 of max(1, |ref|) (the small cases
    above meet 2e-5)."""
    import torch
    n_seq, H, d, n_ctx, group, bits, rot = 32, 8, 128, 32768, 16, 4, 0
    rows = n_ctx * n_seq
    gen = torch.Generator(device=DEV)
    gen.manual_seed(2024)

    def codes():
        c = torch.randint(0, 256, (rows, H, d // 2), generator=gen, device=DEV,
                          dtype=torch.int32).to(torch.uint8)
        c ^= ((c & 0x0F) == 0x08).to(torch.uint8) * 0x08   # nibble -8 -> 0
        c ^= ((c >> 4) == 0x08).to(torch.uint8) * 0x80
        return c

    def scales():
        return (torch.rand((rows, H, d // group), generator=gen, device=DEV) * 0.29
                + 0.01).to(torch.float16)

    kc, ks, vc, vs = codes(), scales(), codes(), scales()
    sgn = (torch.randint(0, 2, (2, H, d), generator=gen, device=DEV) * 2 - 1).to(torch.int8)
    lam = torch.rand((2, H, d), generator=gen, device=DEV) * 1.5 + 0.5
    q = torch.randn((n_seq, H, d), generator=gen, device=DEV).to(torch.float16)
    scale = 1.0 / math.sqrt(d)
    out = rq.decode_attention(q, kc, ks, sgn[0], lam[0], vc, vs, sgn[1], lam[1], group, bits,
                              rot, n_ctx=n_ctx, tok_stride_rows=n_seq, seq_stride_rows=1,
                              scale=scale)
    torch.cuda.synchronize()
    assert rq.srftq_check_device() == 0
    out = out.cpu().numpy()
    sg, lm = sgn.cpu().numpy(), lam.cpu().numpy()
    for b, h in ((0, 0), (17, 5), (31, 7)):
        idx = torch.arange(n_ctx, device=DEV) * n_seq + b

        def rows_of(t):
            return t.index_select(0, idx)[:, h:h + 1].cpu().numpy()

        ref = oracle.decode_attention(
            q[b:b + 1, h:h + 1].cpu().numpy(), rows_of(kc), rows_of(ks).view(np.uint16),
            sg[0, h:h + 1], lm[0, h:h + 1], rows_of(vc), rows_of(vs).view(np.uint16),
            sg[1, h:h + 1], lm[1, h:h + 1], d, group, bits, rot, n_ctx, 1, 0, scale)[0, 0]
        err = np.abs(out[b, h] - ref) / np.maximum(1.0, np.abs(ref))
        assert err.max() < 1e-4, (b, h, float(err.max()))


def test_decode_attention_sequence_major_layout_and_outliers():
    """Rows = sequence * n_ctx + token (the other common layout), and a
    cache with x25 outliers, whose scores spread over a wide range."""
    rng = np.random.default_rng(99)
    H, d, n_seq, n_ctx, group, bits, rot = 4, 128, 2, 700, 16, 4, 0
    rows = n_seq * n_ctx
    kc, ks, ksg, kl = _attn_case(rng, rows, H, d, group, bits, rot, outliers=0.005)
    vc, vs, vsg, vl = _attn_case(rng, rows, H, d, group, bits, rot, outliers=0.005)
    q = _x(rng, 1, n_seq, H, d)[0]
    scale = 1.0 / math.sqrt(d)
    out = rq.decode_attention(_t(q), _t(kc), _t(ks.view(np.float16)), _t(ksg), _t(kl), _t(vc),
                              _t(vs.view(np.float16)), _t(vsg), _t(vl), group, bits, rot,
                              n_ctx=n_ctx, tok_stride_rows=1, seq_stride_rows=n_ctx,
                              scale=scale).cpu().numpy()
    ref = oracle.decode_attention(q, kc, ks, ksg, kl, vc, vs, vsg, vl, d, group, bits, rot, n_ctx,
                                  1, n_ctx, scale)
    err = np.abs(out - ref) / np.maximum(1.0, np.abs(ref))
    assert err.max() < 1e-4, float(err.max())
