"""CPU checks of the comparison rules in tests/parity.py: each planted
difference must be classified the way the stated tolerances say (accepted
inside its band, a violation outside it), so a GPU test cannot pass by a
comparison that lets real mismatches through."""

import numpy as np

import oracle
import parity


def _case(seed=0, N=64, d=64, group=16, bits=4):
    rng = np.random.default_rng(seed)
    x16 = rng.standard_normal((1, N, 1, d)).astype(np.float16)
    signs = np.where(rng.random((1, 1, d)) < 0.5, -1, 1).astype(np.int8)
    lam = np.ones((1, 1, d), np.float32)
    return oracle.quantize(x16, signs, lam, group, bits), signs, lam


def test_identical_outputs_are_clean():
    ref, _, _ = _case()
    st = parity.check_codes(ref, ref["codes"].copy(), ref["scales"].copy(), 4, 16)
    assert st["code_violations"] == st["scale_violations"] == st["zero_scale_violations"] == 0
    assert st["codes"] == 64 * 64


def test_a_code_off_by_one_away_from_a_boundary_is_a_violation():
    ref, _, _ = _case()
    q = ref["q"].copy()
    pre = np.abs(ref["pre"])
    frac = pre - np.floor(pre)
    idx = np.argwhere((np.abs(frac - 0.5) > 0.1) & (np.abs(q) < 7))[0]
    q[tuple(idx)] += 1
    st = parity.check_codes(ref, oracle.pack_codes(q, 4), ref["scales"], 4, 16)
    assert st["code_violations"] == 1


def test_a_code_off_by_one_inside_the_band_is_counted_not_failed():
    ref, _, _ = _case()
    ref = dict(ref)
    pre = ref["pre"].copy()
    q = ref["q"].copy()
    # move one pre-rounding value onto a rounding midpoint (within the band)
    i = tuple(np.argwhere(np.abs(q) < 6)[0])
    pre[i] = q[i] + 0.5 + 0.5e-4 * np.sign(q[i] + 0.1)
    ref["pre"] = pre
    q_gpu = q.copy()
    q_gpu[i] = q[i] + 1
    st = parity.check_codes(ref, oracle.pack_codes(q_gpu, 4), ref["scales"], 4, 16)
    assert st["code_violations"] == 0 and st["code_mismatch_in_band"] == 1
    q_gpu[i] = q[i] + 2            # two steps away: never allowed
    st = parity.check_codes(ref, oracle.pack_codes(q_gpu, 4), ref["scales"], 4, 16)
    assert st["code_violations"] == 1


def test_zero_scale_groups_must_have_zero_codes():
    ref, signs, lam = _case()
    x16 = np.zeros((1, 4, 1, 64), np.float16)
    x16[0, 1, 0, 3] = 1.0          # one nonzero vector; the others give sigma = 0 everywhere
    ref = oracle.quantize(x16, signs, lam, 16, 4)
    st = parity.check_codes(ref, ref["codes"], ref["scales"], 4, 16)
    assert st["zero_scale_groups"] >= 3 * 4 and st["zero_scale_violations"] == 0
    bad = ref["codes"].copy()
    bad[0, 0, 0, 0] = 0x01         # a nonzero code in a sigma = 0 group
    st = parity.check_codes(ref, bad, ref["scales"], 4, 16)
    assert st["zero_scale_violations"] == 1


def test_a_scale_one_step_off_counts_only_near_the_midpoint():
    ref, _, _ = _case()
    s_gpu = ref["scales"].copy()
    s_gpu[0, 0, 0, 0] += 1
    st = parity.check_codes(ref, ref["codes"], s_gpu, 4, 16)
    assert st["scale_violations"] == 1      # the oracle's value is nowhere near that midpoint
    ref2 = dict(ref)
    sp = ref["scale_pre"].copy()
    lo = oracle.binary16_bits_to_float(ref["scales"][0, 0, 0, 0])
    hi = oracle.binary16_bits_to_float(s_gpu[0, 0, 0, 0])
    sp[0, 0, 0, 0] = 0.5 * (lo + hi)
    ref2["scale_pre"] = sp
    st = parity.check_codes(ref2, ref["codes"], s_gpu, 4, 16)
    assert st["scale_violations"] == 0 and st["groups_excluded"] == 1


def test_dequant_tolerance_is_relative_above_one_and_absolute_below():
    r = oracle.float_to_binary16_bits(np.array([0.5, 100.0, -3.0]))
    ok = oracle.float_to_binary16_bits(np.array([0.5 + 0.9e-3, 100.0 * (1 + 0.9e-3), -3.0]))
    bad = oracle.float_to_binary16_bits(np.array([0.5 + 1.5e-3, 100.0 * (1 + 1.5e-3), -3.0]))
    assert parity.check_dequant(ok, r)["violations"] == 0
    assert parity.check_dequant(bad, r)["violations"] == 2


def test_full_data_checker_runs_in_spawned_workers():
    """The full-data harness (tests/fullparity.py) in two spawned workers:
    the oracle's own outputs are clean, and one planted code is found."""
    import fullparity

    rng = np.random.default_rng(3)
    d, group, bits, H = 64, 16, 4, 2
    x16 = rng.standard_normal((1, 40, H, d)).astype(np.float16)
    signs = np.where(rng.random((1, H, d)) < 0.5, -1, 1).astype(np.int8)
    lam = np.exp(rng.uniform(-1, 1, (1, H, d))).astype(np.float32)
    ref = oracle.quantize(x16, signs, lam, group, bits)
    deq = oracle.dequantize(ref["codes"], ref["scales"], signs, lam, d, group, bits)
    c = fullparity.Checker(2)
    try:
        for r0 in (0, 20):
            sl = slice(r0, r0 + 20)
            c.submit((x16[:, sl], signs, lam, ref["codes"][:, sl], ref["scales"][:, sl],
                      deq["bits"][:, sl], d, group, bits, 0))
        clean = c.result()
        bad = ref["codes"].copy()
        q = ref["q"]
        i = tuple(np.argwhere((np.abs(q) < 6) & (np.abs(np.abs(ref["pre"]) % 1 - 0.5) > 0.1))[0])
        q2 = q.copy()
        q2[i] += 1
        bad = oracle.pack_codes(q2, bits)
        c.submit((x16, signs, lam, bad, ref["scales"], deq["bits"], d, group, bits, 0))
        planted = c.result()
    finally:
        c.close()
    assert clean["vectors"] == 80 and not fullparity.violations(clean)
    assert planted["code_violations"] == 1


def test_dense_code_band_follows_the_rotation_tolerance():
    """The dense codec's code band is max(1e-4, 1e-5 max(|y|, rms)/(lambda
    sigma)): int8's finer code unit widens it, and a flip just outside 1e-4
    but inside that band is counted, not failed; two steps never pass."""
    rng = np.random.default_rng(12)
    d, group = 64, 16
    x16 = rng.standard_normal((1, 32, 1, d)).astype(np.float16)
    R = oracle.householder_rotations(rng.standard_normal((1, 1, 8, d)), np.ones((1, 1, d), np.int8),
                                     0)
    lam = np.ones((1, 1, d), np.float32)
    for bits, wider in ((4, False), (8, True)):
        ref = oracle.quantize_dense(x16, R, lam, group, bits)
        band = parity.dense_code_band(ref, lam, group)
        assert band.min() >= parity.CODE_BAND
        assert (band.max() > 2 * parity.CODE_BAND) == wider
    ref = dict(ref)                                    # int8
    band = parity.dense_code_band(ref, lam, group)
    i = tuple(np.argwhere((band > 3e-4) & (np.abs(ref["q"]) < 100))[0])
    pre, q = ref["pre"].copy(), ref["q"].copy()
    pre[i] = q[i] + 0.5 + 2e-4 * (1 if q[i] >= 0 else -1)
    ref["pre"] = pre
    q_gpu = q.copy()
    q_gpu[i] += 1 if q[i] >= 0 else -1
    st = parity.check_codes(ref, oracle.pack_codes(q_gpu, 8), ref["scales"], 8, group,
                            parity.DENSE_SCALE_BAND, band)
    assert st["code_violations"] == 0 and st["code_mismatch_in_band"] == 1
    st = parity.check_codes(ref, oracle.pack_codes(q_gpu, 8), ref["scales"], 8, group)
    assert st["code_violations"] == 1                  # the fixed 1e-4 band would fail it
