"""Host-side checks of libsrftq.so that need no GPU.

The library must load, export every entry point include/srftq.h declares, and
reject bad arguments on the host with the documented status before anything
would be launched (no call here reaches a kernel launch).
"""

import ctypes
import os
import re
import subprocess

import pytest

import rotate_then_quantize_b200 as rq
from rotate_then_quantize_b200 import binding as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "srftq.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(srftq_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(b.LIB_PATH):
        pytest.fail("libsrftq.so is not built; run python -m rotate_then_quantize_b200.build")
    return rq.load_library()


def test_header_declares_the_boundary():
    assert _declared() == sorted(b.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", b.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (srftq_\w+)", out))
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)


def test_timeout_probe_rejects_out_of_range_polls(lib):
    # validated before any launch: no GPU is touched
    assert lib.srftq_probe_wait_timeout(0, None) == b.SRFTQ_ERR_INVALID_ARG
    assert lib.srftq_probe_wait_timeout((1 << 22) + 1, None) == b.SRFTQ_ERR_INVALID_ARG


def test_version_and_status_strings(lib):
    assert rq.srftq_version() >= 100
    for st in (0, -1, -2, -3, -4, -5):
        assert rq.status_string(st) != "unknown status"
    assert rq.status_string(42) == "unknown status"


def _q(lib, desc, S=1, N=8, x=16, xs=8, sg=16, lam=16, codes=16, sc=16, os_=8):
    """srftq_quantize with fake (never dereferenced) addresses."""
    return lib.srftq_quantize(ctypes.byref(desc) if desc is not None else None, S, N,
                              x, xs, sg, lam, codes, sc, os_, None)


FAKE = 1 << 40  # a 16-byte-aligned address far from anything; never touched


def _addrs(n_bytes_apart=1 << 30):
    return [FAKE + i * n_bytes_apart for i in range(6)]


def test_quantize_rejects_bad_descriptors(lib):
    x, sg, lam, codes, sc, _ = _addrs()
    ok = dict(x=x, sg=sg, lam=lam, codes=codes, sc=sc)
    assert _q(lib, None, **ok) == b.SRFTQ_ERR_INVALID_ARG
    for d, heads, group, bits, rot, want in [
        (96, 2, 16, 4, 0, b.SRFTQ_ERR_UNSUPPORTED),    # d not a supported power of two
        (512, 2, 16, 4, 0, b.SRFTQ_ERR_UNSUPPORTED),
        (128, 0, 16, 4, 0, b.SRFTQ_ERR_INVALID_ARG),   # no heads
        (128, 2, 12, 4, 0, b.SRFTQ_ERR_UNSUPPORTED),   # group not a power of two
        (128, 2, 4, 4, 0, b.SRFTQ_ERR_UNSUPPORTED),    # group below 8
        (64, 2, 128, 4, 0, b.SRFTQ_ERR_UNSUPPORTED),   # group above d
        (256, 2, 512, 4, 0, b.SRFTQ_ERR_UNSUPPORTED),  # group above d
        (16, 2, 32, 8, 1, b.SRFTQ_ERR_UNSUPPORTED),
        (128, 2, 16, 3, 0, b.SRFTQ_ERR_UNSUPPORTED),   # bits
        (128, 2, 16, 4, 2, b.SRFTQ_ERR_UNSUPPORTED),   # rotation
    ]:
        assert _q(lib, rq.make_desc(d, heads, group, bits, rot), **ok) == want, (d, heads, group, bits, rot)


def test_quantize_rejects_bad_sizes_pointers_and_overlap(lib):
    desc = rq.make_desc(128, 2, 16, 4)
    x, sg, lam, codes, sc, _ = _addrs()
    ok = dict(x=x, sg=sg, lam=lam, codes=codes, sc=sc)
    assert _q(lib, desc, N=-1, **ok) == b.SRFTQ_ERR_INVALID_ARG
    assert _q(lib, desc, S=-1, **ok) == b.SRFTQ_ERR_INVALID_ARG
    assert _q(lib, desc, N=0, **ok) == b.SRFTQ_OK            # nothing to do, nothing launched
    assert _q(lib, desc, S=0, **ok) == b.SRFTQ_OK
    assert _q(lib, desc, S=2, N=8, xs=4, **ok) == b.SRFTQ_ERR_INVALID_ARG   # overlapping slices
    assert _q(lib, desc, S=2, N=8, os_=4, **ok) == b.SRFTQ_ERR_INVALID_ARG
    assert _q(lib, desc, **dict(ok, x=0)) == b.SRFTQ_ERR_INVALID_ARG
    assert _q(lib, desc, **dict(ok, sc=0)) == b.SRFTQ_ERR_INVALID_ARG
    assert _q(lib, desc, **dict(ok, x=x + 8)) == b.SRFTQ_ERR_MISALIGNED
    assert _q(lib, desc, **dict(ok, codes=codes + 4)) == b.SRFTQ_ERR_MISALIGNED
    # in-place: codes inside x
    assert _q(lib, desc, **dict(ok, codes=x + 256)) == b.SRFTQ_ERR_INVALID_ARG
    # scales overlapping codes
    assert _q(lib, desc, **dict(ok, sc=codes + 16)) == b.SRFTQ_ERR_INVALID_ARG


def test_dequantize_calibrate_rotate_validation(lib):
    desc = rq.make_desc(64, 3, 16, 8, 1)
    c, s, sg, lam, xh, y = _addrs()
    D = ctypes.byref(desc)
    assert lib.srftq_dequantize(D, 1, 8, c, s, 8, sg, lam, c, 8, None) == b.SRFTQ_ERR_INVALID_ARG
    assert lib.srftq_dequantize(D, 1, 8, c + 2, s, 8, sg, lam, xh, 8, None) == b.SRFTQ_ERR_MISALIGNED
    assert lib.srftq_dequantize(D, 1, 0, c, s, 8, sg, lam, xh, 8, None) == b.SRFTQ_OK
    assert lib.srftq_calibrate_lambda(D, 1, 0, c, 8, sg, lam, None) == b.SRFTQ_ERR_INVALID_ARG
    assert lib.srftq_calibrate_lambda(D, 1, 9, c, 8, sg, lam, None) == b.SRFTQ_ERR_INVALID_ARG
    assert lib.srftq_calibrate_lambda(D, 0, 4, c, 8, sg, lam, None) == b.SRFTQ_OK
    assert lib.srftq_calibrate_lambda(D, 1, 4, c, 8, sg, c, None) == b.SRFTQ_ERR_INVALID_ARG
    assert lib.srftq_rotate(D, 1, 8, c, 8, sg, None, c, None) == b.SRFTQ_ERR_INVALID_ARG
    assert lib.srftq_rotate(D, 1, 8, c, 8, sg, lam + 4, y, None) == b.SRFTQ_ERR_MISALIGNED
    assert lib.srftq_rotate(D, 1, 0, c, 8, sg, None, y, None) == b.SRFTQ_OK


def test_rotated_domain_calls_validate_before_launching(lib):
    desc = rq.make_desc(64, 3, 16, 8, 0)
    c, s, sg, lam, xh, y = _addrs()
    D = ctypes.byref(desc)
    R = lib.srftq_dequantize_rotated
    assert R(D, 1, 8, c, s, 8, lam, c, 8, None) == b.SRFTQ_ERR_INVALID_ARG      # out overlaps codes
    assert R(D, 1, 8, c, s, 8, None, xh, 8, None) == b.SRFTQ_ERR_INVALID_ARG   # no lambda
    assert R(D, 1, 8, c, s + 2, 8, lam, xh, 8, None) == b.SRFTQ_ERR_MISALIGNED
    assert R(D, 1, 8, c, s, 4, lam, xh, 8, None) == b.SRFTQ_ERR_INVALID_ARG    # stride < rows
    assert R(D, 0, 8, c, s, 8, lam, xh, 8, None) == b.SRFTQ_OK                 # nothing to do
    assert R(None, 1, 8, c, s, 8, lam, xh, 8, None) == b.SRFTQ_ERR_INVALID_ARG
    U = lib.srftq_unrotate
    assert U(D, 1, 8, y, 8, sg, y, 8, None) == b.SRFTQ_ERR_INVALID_ARG         # in place
    assert U(D, 1, 8, y, 8, sg, y + 16, 8, None) == b.SRFTQ_ERR_INVALID_ARG    # overlap
    assert U(D, 1, 8, y + 8, 8, sg, xh, 8, None) == b.SRFTQ_ERR_MISALIGNED
    assert U(D, 1, 8, y, 8, None, xh, 8, None) == b.SRFTQ_ERR_INVALID_ARG
    assert U(D, 1, 0, y, 8, sg, xh, 8, None) == b.SRFTQ_OK


def test_decode_attention_validates_before_launching(lib):
    c, s, sg, lam, xh, y = _addrs()
    A = lib.srftq_decode_attention

    def call(desc, n_seq=2, n_ctx=16, qpk=1, q=xh, kc=c, ks=s, ksg=sg, kl=lam, out=y, ts=2, ss=1):
        return A(ctypes.byref(desc), n_seq, n_ctx, qpk, q, kc, ks, ksg, kl, kc + (1 << 28),
                 ks + (1 << 28), ksg, kl, ts, ss, 0.1, out, None)

    ok = rq.make_desc(128, 4, 16, 4, 0)
    assert call(rq.make_desc(64, 4, 16, 4, 0)) == b.SRFTQ_ERR_UNSUPPORTED     # d = 128 only
    assert call(ok, qpk=3) == b.SRFTQ_ERR_UNSUPPORTED
    assert call(ok, n_ctx=0) == b.SRFTQ_ERR_INVALID_ARG
    assert call(ok, ts=-1) == b.SRFTQ_ERR_INVALID_ARG
    assert call(ok, q=0) == b.SRFTQ_ERR_INVALID_ARG
    assert call(ok, out=y + 4) == b.SRFTQ_ERR_MISALIGNED
    assert call(ok, out=xh) == b.SRFTQ_ERR_INVALID_ARG                         # out overlaps q
    assert call(ok, n_seq=0) == b.SRFTQ_OK                                     # nothing to do


def test_python_binding_rejects_bad_views():
    torch = pytest.importorskip("torch")
    x = torch.zeros((2, 8, 3, 64), dtype=torch.float16)
    with pytest.raises(ValueError):
        b._rows_layout(x.transpose(1, 2), 3, 64, "x")
    ptr, S, N, stride = b._rows_layout(x[:, 2:6], 3, 64, "x")
    assert (S, N, stride) == (2, 4, 8)


def test_python_binding_refuses_overlapping_slices():
    """An expanded view (slice stride 0) or any view whose slices sit closer
    than N rows would make the library walk S * N rows of a smaller
    allocation; the binding refuses it before the C ABI is called."""
    torch = pytest.importorskip("torch")
    x = torch.zeros((1, 8, 2, 64), dtype=torch.float16)
    with pytest.raises(ValueError, match="overlap"):
        b._rows_layout(x.expand(3, 8, 2, 64), 2, 64, "x")
    big = torch.zeros((16, 2, 64), dtype=torch.float16)
    overlapping = big.as_strided((2, 8, 2, 64), (4 * 128, 128, 64, 1))   # slice stride 4 < 8 rows
    with pytest.raises(ValueError, match="overlap"):
        b._rows_layout(overlapping, 2, 64, "x")
    # one slice: the stride is irrelevant and the rows are passed as the stride
    assert b._rows_layout(x.expand(1, 8, 2, 64), 2, 64, "x")[1:] == (1, 8, 8)
    desc = rq.make_desc(64, 2, 16, 4)
    codes = torch.zeros((1, 8, 2, 32), dtype=torch.uint8).expand(3, 8, 2, 32)
    scales = torch.zeros((1, 8, 2, 4), dtype=torch.float16).expand(3, 8, 2, 4)
    signs = torch.ones((3, 2, 64), dtype=torch.int8)
    lam = torch.ones((3, 2, 64))
    with pytest.raises(ValueError):
        rq.srftq_quantize(desc, x.expand(3, 8, 2, 64), signs, lam, codes, scales)
    with pytest.raises(ValueError):
        rq.srftq_dequantize(desc, codes, scales, signs, lam, x.expand(3, 8, 2, 64))


def test_python_binding_refuses_host_tensors_and_wrong_dtypes():
    """The binding passes data pointers to device code, so a host tensor or a
    tensor of another dtype (read as fp16, say) is refused with ValueError
    before the library is called."""
    torch = pytest.importorskip("torch")
    desc = rq.make_desc(64, 2, 16, 4)
    S, N, H, d = 2, 8, 2, 64
    good = dict(x=torch.zeros((S, N, H, d), dtype=torch.float16),
                signs=torch.ones((S, H, d), dtype=torch.int8),
                lam=torch.ones((S, H, d), dtype=torch.float32),
                codes=torch.zeros((S, N, H, d // 2), dtype=torch.uint8),
                scales=torch.zeros((S, N, H, d // 16), dtype=torch.float16))
    # host tensors of the right dtypes: refused for their device
    with pytest.raises(ValueError, match="CUDA"):
        rq.srftq_quantize(desc, **good)
    for name, wrong in (("x", torch.float32), ("x", torch.bfloat16), ("signs", torch.uint8),
                        ("lam", torch.float64), ("codes", torch.int8),
                        ("scales", torch.float32)):
        args = dict(good)
        args[name] = good[name].to(wrong)
        with pytest.raises(ValueError):
            rq.srftq_quantize(desc, **args)
        # the dtype is checked before the device
        with pytest.raises(ValueError, match="dtype"):
            b._check_tensor(args[name], good[name].dtype, name)
    with pytest.raises(ValueError):
        rq.srftq_dequantize(desc, good["codes"], good["scales"], good["signs"], good["lam"],
                            good["x"].float())
    with pytest.raises(ValueError):
        rq.srftq_rotate(desc, good["x"], good["signs"], torch.zeros((S, N, H, d)))
    with pytest.raises(ValueError):
        rq.srftq_unrotate(desc, torch.zeros((S, N, H, d)), good["signs"],
                          torch.zeros((S, N, H, d)))


def test_dense_calls_validate_before_launching(lib):
    c, s, sg, lam, xh, y = _addrs()
    ok = rq.make_desc(256, 2, 32, 4, 0)
    D = ctypes.byref(ok)
    Hh = lib.srftq_householder_rotation
    assert Hh(ctypes.byref(rq.make_desc(32, 2, 8, 4, 0)), 1, 4, y, sg, xh, None) == \
        b.SRFTQ_ERR_UNSUPPORTED                                      # d = 64, 128, 256 only
    assert Hh(ctypes.byref(rq.make_desc(256, 2, 8, 4, 5)), 1, 4, y, sg, xh, None) == \
        b.SRFTQ_ERR_UNSUPPORTED                                      # base rotation
    assert Hh(D, 1, -1, y, sg, xh, None) == b.SRFTQ_ERR_INVALID_ARG
    assert Hh(D, 1, 4, 0, sg, xh, None) == b.SRFTQ_ERR_INVALID_ARG     # no reflectors
    assert Hh(D, 1, 4, y, sg, y + 64, None) == b.SRFTQ_ERR_INVALID_ARG  # output over input
    assert Hh(D, 1, 4, y, sg, xh + 8, None) == b.SRFTQ_ERR_MISALIGNED
    assert Hh(D, 0, 4, y, sg, xh, None) == b.SRFTQ_OK
    Op = lib.srftq_dense_operand
    assert Op(D, 1, y, y + 16, None) == b.SRFTQ_ERR_INVALID_ARG
    assert Op(D, 1, y, 0, None) == b.SRFTQ_ERR_INVALID_ARG
    assert Op(D, 0, y, xh, None) == b.SRFTQ_OK
    Q = lib.srftq_quantize_dense
    assert Q(ctypes.byref(rq.make_desc(256, 2, 512, 4)), 1, 8, xh, 8, y, lam, c, s, 8, None) == \
        b.SRFTQ_ERR_UNSUPPORTED
    assert Q(D, 1, 8, xh, 8, y, lam, xh + 64, s, 8, None) == b.SRFTQ_ERR_INVALID_ARG  # in place
    assert Q(D, 2, 8, xh, 4, y, lam, c, s, 8, None) == b.SRFTQ_ERR_INVALID_ARG       # stride < N
    assert Q(D, 1, 8, xh, 8, y + 2, lam, c, s, 8, None) == b.SRFTQ_ERR_MISALIGNED
    assert Q(D, 1, 0, xh, 8, y, lam, c, s, 8, None) == b.SRFTQ_OK
    Dq = lib.srftq_dequantize_dense
    assert Dq(D, 1, 8, c, s, 8, y, lam, c + 16, 8, None) == b.SRFTQ_ERR_INVALID_ARG
    assert Dq(D, 1, 8, c, s, 8, None, lam, xh, 8, None) == b.SRFTQ_ERR_INVALID_ARG
    assert Dq(D, 1, 0, c, s, 8, y, lam, xh, 8, None) == b.SRFTQ_OK
    Cal = lib.srftq_calibrate_lambda_dense
    assert Cal(D, 1, 0, xh, 8, y, lam, None) == b.SRFTQ_ERR_INVALID_ARG
    assert Cal(D, 1, 9, xh, 8, y, lam, None) == b.SRFTQ_ERR_INVALID_ARG
    assert Cal(D, 1, 4, xh, 8, y, xh, None) == b.SRFTQ_ERR_INVALID_ARG      # lambda over x
    assert Cal(D, 0, 4, xh, 8, y, lam, None) == b.SRFTQ_OK


def test_debug_library_exports_the_boundary_and_reports_its_checks(lib):
    """The index-checking build (libsrftq_debug.so) exports every declared
    symbol too; srftq_debug_checks tells the two builds apart without a GPU."""
    if not os.path.exists(b.LIB_DEBUG_PATH):
        pytest.fail("libsrftq_debug.so is not built; run python -m rotate_then_quantize_b200.build "
                    "--debug")
    out = subprocess.run(["nm", "-D", "--defined-only", b.LIB_DEBUG_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (srftq_\w+)", out))
    for name in _declared():
        assert name in exported, name
    assert rq.load_library(b.LIB_DEBUG_PATH).srftq_debug_checks() == 1
    assert lib.srftq_debug_checks() == 0


def test_no_symbol_is_merged_across_libraries(lib):
    """libsrftq.so and libsrftq_debug.so may share a process. A symbol of
    type STB_GNU_UNIQUE (nm: "u"), as GCC emits for the local statics of
    template functions, would be merged between them by the dynamic linker
    even when both are loaded locally, and one library's kernel-attribute
    cache would then stand for the other's kernels."""
    for path in (b.LIB_PATH, b.LIB_DEBUG_PATH):
        if not os.path.exists(path):
            continue
        out = subprocess.run(["nm", "-D", path], capture_output=True, text=True, check=True).stdout
        unique = [ln for ln in out.splitlines() if " u " in ln]
        assert not unique, (path, unique[:5])
