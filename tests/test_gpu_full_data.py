"""GPU parity on the full data of every workload, through the C ABI.

Each workload runs on the GPU exactly as the benchmark launches it (one
quantise and one dequantise launch over the whole cache; the decode stream's
per-layer appends and full-cache dequantisation), and then every vector is
compared with the CPU oracle (tests/fullparity.py): codes and scales against
the oracle's quantisation of the same fp16 inputs, and the dequantised output
against the oracle's dequantisation of the GPU's own codes. Both sides use the
oracle's lambda (its calibration over the first 512 rows of every slice,
rounded to float32), so each stage is checked on its own; the GPU calibration
is checked against the same lambda.

The counts (codes compared, boundary-band mismatches, scale midpoint cases,
sigma = 0 groups, largest dequantisation error) are written per workload to
profiles/parity_full_data.json; every violation count must be zero.

Decode stream: slices 0 and 63 of the 64-slice cache are checked in full
(1,048,576 cached rows plus the appended ones, 8 heads), and the appended
tokens of every slice.
"""

import numpy as np
import pytest

import fullparity
import kv_synth
import oracle
import parity

torch = pytest.importorskip("torch")
import rotate_then_quantize_b200 as rq  # noqa: E402

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
VECTORS_PER_CHUNK = 32768


@pytest.fixture(scope="module")
def checker():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    rq.load_library()
    c = fullparity.Checker()
    yield c
    c.close()
    assert rq.srftq_check_device() == 0, "a device-side guard fired"


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _bits16(t):
    return t.cpu().numpy().view(np.uint16)


def _submit_slice(checker, x, codes, scales, xhat, s, signs, lam, w, rot, rows=None,
                  x_rows=None):
    """Queues every vector of slice s (rows [0, n) of the GPU tensors) for the
    oracle, in chunks; x_rows(r0, r1) returns the fp16 inputs of those rows
    when they do not all come from x."""
    n = codes.shape[1] if rows is None else rows
    step = max(1, VECTORS_PER_CHUNK // w.H)
    for r0 in range(0, n, step):
        r1 = min(n, r0 + step)
        xs = x[s:s + 1, r0:r1].cpu().numpy() if x_rows is None else x_rows(r0, r1)
        checker.submit((xs, signs[s:s + 1], lam[s:s + 1], codes[s:s + 1, r0:r1].cpu().numpy(),
                        _bits16(scales[s:s + 1, r0:r1]), _bits16(xhat[s:s + 1, r0:r1]),
                        w.d, w.group, w.bits, rot))


def _rel_l2(x, xhat):
    """Per-vector ||xhat - x|| / ||x|| over the whole cache (on the GPU)."""
    vals = []
    for s in range(x.shape[0]):
        e = torch.linalg.vector_norm(xhat[s].float() - x[s].float(), dim=-1)
        n = torch.linalg.vector_norm(x[s].float(), dim=-1).clamp_min(1e-12)
        vals.append((e / n).flatten())
    r = torch.cat(vals)
    sample = r if r.numel() <= (1 << 24) else r[torch.randperm(r.numel(), device=r.device)[:1 << 24]]
    return {"mean": float(r.mean()), "p50": float(sample.quantile(0.5)),
            "p99": float(sample.quantile(0.99)), "max": float(r.max())}


def _oracle_lambda(x, signs, w, rot):
    x_cal = x[:, :w.n_cal].cpu().numpy()
    return oracle.calibrate_lambda(x_cal, signs, w.n_cal, rot)


def _workload(checker, name, rot):
    w = kv_synth.WORKLOADS[name]
    x = kv_synth.make_x_torch(w, DEV, seed=0)
    signs = kv_synth.rademacher_signs(w.S, w.H, w.d, seed=1)
    st = _t(signs)
    lam64 = _oracle_lambda(x, signs, w, rot)
    lam = lam64.astype(np.float32)
    lt = _t(lam)
    lam_gpu = rq.calibrate_lambda(x, st, w.n_cal, rotation=rot).cpu().numpy()
    lam_stats = parity.check_lambda(lam_gpu, lam64)
    parity.assert_clean(lam_stats, f"{name} lambda")
    # the benchmark's launches: one quantise and one dequantise over the whole cache
    codes, scales = rq.quantize(x, st, lt, w.group, w.bits, rot)
    xhat = rq.dequantize(codes, scales, st, lt, w.d, w.group, w.bits, rot)
    torch.cuda.synchronize()
    for s in range(w.S):
        _submit_slice(checker, x, codes, scales, xhat, s, signs, lam, w, rot)
    quality = _rel_l2(x, xhat)
    stats = checker.result()
    record = {"workload": name, "rotation": "SRFT" if rot == 0 else "SRHT",
              "shape": [w.S, w.N, w.H, w.d], "bits": w.bits, "group": w.group,
              "lambda_max_rel_err": lam_stats["max_rel_err"], "rel_l2_error": quality, **stats}
    fullparity.write_report(f"{name}:{record['rotation']}", record)
    print(name, record)
    assert not fullparity.violations(stats), stats
    assert stats["vectors"] == w.vectors
    del x, codes, scales, xhat
    torch.cuda.empty_cache()
    return record


def test_full_data_tiny(checker):
    w = kv_synth.WORKLOADS["tiny_d64"]
    x16, signs = kv_synth.tiny_inputs()
    lam64 = oracle.calibrate_lambda(x16, signs, w.n_cal)
    lam = lam64.astype(np.float32)
    x, st, lt = _t(x16), _t(signs), _t(lam)
    codes, scales = rq.quantize(x, st, lt, w.group, w.bits)
    xhat = rq.dequantize(codes, scales, st, lt, w.d, w.group, w.bits)
    _submit_slice(checker, x, codes, scales, xhat, 0, signs, lam, w, 0)
    stats = checker.result()
    fullparity.write_report("tiny_d64:SRFT", {"workload": "tiny_d64", "rotation": "SRFT",
                                               "shape": [1, w.N, 1, w.d], "bits": w.bits,
                                               "group": w.group, "rel_l2_error": _rel_l2(x, xhat),
                                               **stats})
    assert not fullparity.violations(stats), stats
    assert stats["vectors"] == w.vectors


def test_full_data_qwen_like(checker):
    _workload(checker, "qwen_like_d128", 0)


def test_full_data_longctx_int8_both_rotations(checker):
    """SRFT and SRHT on the same Student-t cache; the pages find the two
    rotations statistically indistinguishable ("When Quantization Is Free",
    Methodology 1), so their mean round-trip errors are reported side by side
    and must agree within a few percent."""
    srft = _workload(checker, "longctx_int8_d128", 0)
    srht = _workload(checker, "longctx_int8_d128", 1)
    a, b = srft["rel_l2_error"]["mean"], srht["rel_l2_error"]["mean"]
    fullparity.write_report("longctx_int8_d128:SRFT_vs_SRHT",
                            {"rel_l2_mean_srft": a, "rel_l2_mean_srht": b,
                             "relative_difference": abs(a - b) / max(a, b)})
    assert abs(a - b) / max(a, b) < 0.05, (a, b)


def test_full_data_gemma_like_d256(checker):
    _workload(checker, "gemma_like_d256", 0)


def test_full_data_decode_stream_slices_0_and_63(checker):
    """The decode-stream cache built as the benchmark builds it: 64 slices of
    32,768 tokens x 32 sequences x 8 heads, each slice calibrated and
    quantised in one launch; then decode steps that append one token per
    sequence to every slice (one quantise launch per layer into the cache at
    the next row block) and dequantise each layer's whole cache (one launch
    over its two slices). Slices 0 and 63 are then checked in full, and the
    appended tokens of all 64 slices."""
    w = kv_synth.WORKLOADS["decode_stream_d128"]
    B, steps = 32, 3
    T0, L = w.N // B, w.S // 2
    n = (T0 + steps) * B
    desc = rq.make_desc(w.d, w.H, w.group, w.bits, 0)
    signs = kv_synth.rademacher_signs(w.S, w.H, w.d, seed=1)
    st = _t(signs)
    lam = np.empty((w.S, w.H, w.d), np.float32)
    codes = torch.empty((w.S, n, w.H, w.d * w.bits // 8), dtype=torch.uint8, device=DEV)
    scales = torch.empty((w.S, n, w.H, w.d // w.group), dtype=torch.float16, device=DEV)
    scratch = torch.empty((2, n, w.H, w.d), dtype=torch.float16, device=DEV)
    for s in range(w.S):
        xs = kv_synth.make_x_torch(w, DEV, seed=0, n_rows=T0 * B, slices=range(s, s + 1),
                                   out=scratch[0:1, :T0 * B])
        lam[s] = oracle.calibrate_lambda(xs[:, :w.n_cal].cpu().numpy(), signs[s:s + 1],
                                         w.n_cal)[0]
        rq.srftq_quantize(desc, xs, st[s:s + 1], _t(lam[s:s + 1]), codes[s:s + 1, :T0 * B],
                          scales[s:s + 1, :T0 * B])
    lt = _t(lam)
    new_tok = kv_synth.make_x_torch(w, DEV, seed=7, n_rows=B)
    for t in range(steps):
        r0 = (T0 + t) * B
        for layer in range(L):
            sl = slice(2 * layer, 2 * layer + 2)
            rq.srftq_quantize(desc, new_tok[sl], st[sl], lt[sl], codes[sl, r0:r0 + B],
                              scales[sl, r0:r0 + B])
            rq.srftq_dequantize(desc, codes[sl, :r0 + B], scales[sl, :r0 + B], st[sl], lt[sl],
                                scratch[:, :r0 + B])
    torch.cuda.synchronize()
    assert rq.srftq_check_device() == 0

    # every appended token of every slice (the dequantised rows of slices 0
    # and 63 are checked with their slices below)
    tok = new_tok.cpu().numpy()
    app_codes = codes[:, T0 * B:].cpu().numpy()
    app_scales = _bits16(scales[:, T0 * B:])
    app = {}
    ref = oracle.quantize(tok, signs, lam, w.group, w.bits)   # the same tokens every step
    for t in range(steps):
        stt = parity.check_codes(ref, app_codes[:, t * B:(t + 1) * B],
                                 app_scales[:, t * B:(t + 1) * B], w.bits, w.group)
        parity.assert_clean(stt, f"appended tokens, step {t}")
        app = fullparity.merge(app, dict(stt, vectors=w.S * B * w.H))

    # slices 0 and 63 in full: layer 0's and layer 31's whole cache, each
    # dequantised by the benchmark's per-layer launch
    for s in (0, w.S - 1):
        layer = s // 2
        sl = slice(2 * layer, 2 * layer + 2)
        rq.srftq_dequantize(desc, codes[sl], scales[sl], st[sl], lt[sl], scratch)
        torch.cuda.synchronize()
        xs = kv_synth.make_x_torch(w, DEV, seed=0, n_rows=T0 * B, slices=range(s, s + 1))

        app_x = np.tile(tok[s:s + 1], (1, steps, 1, 1))    # rows T0*B .. n-1

        def rows(r0, r1, xs=xs, app_x=app_x):
            parts = []
            if r0 < T0 * B:
                parts.append(xs[:, r0:min(r1, T0 * B)].cpu().numpy())
            if r1 > T0 * B:
                parts.append(app_x[:, max(r0, T0 * B) - T0 * B:r1 - T0 * B])
            return np.concatenate(parts, axis=1)

        xh = scratch[s % 2:s % 2 + 1]
        _submit_slice(checker, xs, codes[s:s + 1], scales[s:s + 1], xh, 0, signs[s:s + 1],
                      lam[s:s + 1], w, 0, rows=n, x_rows=rows)
        del xs
    stats = checker.result()
    record = {"workload": "decode_stream_d128", "rotation": "SRFT",
              "checked": "slices 0 and 63 in full (32,771 tokens x 32 sequences x 8 heads "
                         "each, after 3 decode steps), and the appended tokens of all 64 slices",
              "shape": [w.S, n, w.H, w.d], "bits": w.bits, "group": w.group,
              "appended_tokens": app, **stats}
    fullparity.write_report("decode_stream_d128:SRFT", record)
    print(record)
    assert not fullparity.violations(stats), stats
    assert stats["vectors"] == 2 * n * w.H
    del codes, scales, scratch
    torch.cuda.empty_cache()


def test_full_data_householder_d256(checker):
    """The dense-rotation codec at the Gemma-shaped size (4 slices x 32768
    rows x 4 heads, d = 256, int4 G32) with k = 128 Householder reflectors
    on the SRFT base ("When Quantization Is Free", Methodology 3), as the
    benchmark launches it: every vector against the oracle, which uses its
    own float64 rotation; the GPU reads the operand of that rotation rounded
    to float32, and builds its own from the same reflectors for a second,
    end-to-end pass."""
    w = kv_synth.WORKLOADS["householder_d256"]
    x = kv_synth.make_x_torch(w, DEV, seed=0)
    signs = kv_synth.rademacher_signs(w.S, w.H, w.d, seed=1)
    V = kv_synth.householder_reflectors(w.S, w.H, w.reflectors, w.d, seed=1)
    R = oracle.householder_rotations(V, signs, 0)
    lam64 = oracle.calibrate_lambda_dense(x[:, :w.n_cal].cpu().numpy(), R, w.n_cal)
    lam = lam64.astype(np.float32)
    lt = _t(lam)
    op = rq.dense_operand(_t(R.astype(np.float32)))
    lam_gpu = rq.calibrate_lambda_dense(x, op, w.n_cal).cpu().numpy()
    lam_stats = parity.check_lambda(lam_gpu, lam64)
    parity.assert_clean(lam_stats, "householder lambda")
    codes, scales = rq.quantize_dense(x, op, lt, w.group, w.bits)
    xhat = rq.dequantize_dense(codes, scales, op, lt, w.d, w.group, w.bits)
    torch.cuda.synchronize()
    step = max(1, VECTORS_PER_CHUNK // w.H)
    for s in range(w.S):
        for r0 in range(0, w.N, step):
            r1 = min(w.N, r0 + step)
            checker.submit((x[s:s + 1, r0:r1].cpu().numpy(), R[s:s + 1], lam[s:s + 1],
                            codes[s:s + 1, r0:r1].cpu().numpy(), _bits16(scales[s:s + 1, r0:r1]),
                            _bits16(xhat[s:s + 1, r0:r1]), w.d, w.group, w.bits),
                           fullparity.check_chunk_dense)
    quality = _rel_l2(x, xhat)
    stats = checker.result()
    # the GPU-built rotation end to end: codes within the band of the oracle's
    op_gpu = rq.dense_operand(rq.householder_rotation(_t(V), _t(signs)))
    codes2, scales2 = rq.quantize_dense(x[:1], op_gpu[:1], lt[:1], w.group, w.bits)
    ref = oracle.quantize_dense(x[:1, :4096].cpu().numpy(), R[:1], lam[:1], w.group, w.bits)
    gpu_built = parity.check_codes(ref, codes2[:, :4096].cpu().numpy(),
                                   _bits16(scales2[:, :4096]), w.bits, w.group,
                                   parity.DENSE_SCALE_BAND,
                                   parity.dense_code_band(ref, lam[:1], w.group))
    parity.assert_clean(gpu_built, "GPU-built rotation")
    record = {"workload": w.name, "rotation": "Householder k=128 on SRFT",
              "shape": [w.S, w.N, w.H, w.d], "bits": w.bits, "group": w.group,
              "lambda_max_rel_err": lam_stats["max_rel_err"], "rel_l2_error": quality,
              "gpu_built_rotation_first_4096_rows": gpu_built, **stats}
    fullparity.write_report(f"{w.name}:householder", record)
    print(record)
    assert not fullparity.violations(stats), stats
    assert stats["vectors"] == w.vectors
