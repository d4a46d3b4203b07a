"""ctypes binding of libsrftq.so (argument marshalling only).

Every function named ``srftq_*`` here calls the C entry point of the same
name declared in include/srftq.h; the arguments are torch tensors on a CUDA
device (PyTorch provides device memory and streams, nothing else). All of the
codec's work runs in the library's CUDA kernels: there is no fallback, and
loading fails loudly when the library has not been built.

Tensor views are accepted when each row's heads and elements are contiguous;
a slice stride larger than the row count (for example ``cache[:, t0:t1]`` of
a [S, T, H, d] buffer) is passed through as the slice stride in rows.
"""

from __future__ import annotations

import contextlib
import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libsrftq.so")
# the same library built with device-side index checks (SRFTQ_DEBUG_CHECKS)
LIB_DEBUG_PATH = os.path.join(PKG_DIR, "libsrftq_debug.so")

SRFTQ_OK = 0
SRFTQ_ERR_INVALID_ARG = -1
SRFTQ_ERR_UNSUPPORTED = -2
SRFTQ_ERR_MISALIGNED = -3
SRFTQ_ERR_CUDA = -4
SRFTQ_ERR_DEVICE_CHECK = -5

SRFT = 0
SRHT = 1

# Every symbol include/srftq.h declares (checked by the CPU test suite).
EXPORTED = ("srftq_quantize", "srftq_dequantize", "srftq_calibrate_lambda", "srftq_rotate",
            "srftq_dequantize_rotated", "srftq_unrotate", "srftq_decode_attention",
            "srftq_householder_rotation", "srftq_dense_operand", "srftq_calibrate_lambda_dense",
            "srftq_quantize_dense", "srftq_dequantize_dense", "srftq_status_string",
            "srftq_check_device", "srftq_probe_wait_timeout", "srftq_probe_index_check",
            "srftq_debug_checks", "srftq_version")


class SrftqDesc(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("heads", ctypes.c_int32), ("group", ctypes.c_int32),
                ("bits", ctypes.c_int32), ("rotation", ctypes.c_int32)]


class SrftqError(RuntimeError):
    def __init__(self, fn, status, text):
        super().__init__(f"{fn} failed: status {status} ({text})")
        self.status = status


_libs = {}            # path -> loaded library
_use_debug = False    # set inside debug_checks()


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Loads the in-tree libsrftq.so once (or, inside `debug_checks()`, the
    in-tree libsrftq_debug.so); raises if it is missing (no CPU fallback
    exists)."""
    if path is None:
        path = LIB_DEBUG_PATH if _use_debug else LIB_PATH
    if path in _libs:
        return _libs[path]
    if not os.path.exists(path):
        flag = " --debug" if path == LIB_DEBUG_PATH else ""
        raise FileNotFoundError(
            f"{path} not found: build it with `python -m rotate_then_quantize_b200.build{flag}`")
    lib = ctypes.CDLL(path)
    P, I64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    D = ctypes.POINTER(SrftqDesc)
    lib.srftq_quantize.argtypes = [D, I64, I64, P, I64, P, P, P, P, I64, P]
    lib.srftq_dequantize.argtypes = [D, I64, I64, P, P, I64, P, P, P, I64, P]
    lib.srftq_calibrate_lambda.argtypes = [D, I64, I64, P, I64, P, P, P]
    lib.srftq_rotate.argtypes = [D, I64, I64, P, I64, P, P, P, P]
    lib.srftq_dequantize_rotated.argtypes = [D, I64, I64, P, P, I64, P, P, I64, P]
    lib.srftq_unrotate.argtypes = [D, I64, I64, P, I64, P, P, I64, P]
    lib.srftq_decode_attention.argtypes = [D, I64, I64, I32, P, P, P, P, P, P, P, P, P, I64, I64,
                                           ctypes.c_float, P, P]
    lib.srftq_householder_rotation.argtypes = [D, I64, ctypes.c_int32, P, P, P, P]
    lib.srftq_dense_operand.argtypes = [D, I64, P, P, P]
    lib.srftq_calibrate_lambda_dense.argtypes = [D, I64, I64, P, I64, P, P, P]
    lib.srftq_quantize_dense.argtypes = [D, I64, I64, P, I64, P, P, P, P, I64, P]
    lib.srftq_dequantize_dense.argtypes = [D, I64, I64, P, P, I64, P, P, P, I64, P]
    lib.srftq_status_string.argtypes = [I32]
    lib.srftq_status_string.restype = ctypes.c_char_p
    lib.srftq_check_device.argtypes = [P]
    lib.srftq_probe_wait_timeout.argtypes = [ctypes.c_uint32, P]
    lib.srftq_probe_index_check.argtypes = [I64, I64, P]
    lib.srftq_debug_checks.argtypes = []
    lib.srftq_version.argtypes = []
    for name in EXPORTED:
        if name != "srftq_status_string":
            getattr(lib, name).restype = I32
    _libs[path] = lib
    return lib


@contextlib.contextmanager
def debug_checks():
    """Within the block every srftq_* call of this module goes to the in-tree
    debug build (libsrftq_debug.so, `python -m rotate_then_quantize_b200.build
    --debug`), whose kernels check every global-memory index against the
    call's extents and record a failure in the device guard word
    (srftq_check_device) instead of making the access."""
    global _use_debug
    load_library(LIB_DEBUG_PATH)
    prev = _use_debug
    _use_debug = True
    try:
        yield
    finally:
        _use_debug = prev


def status_string(status: int) -> str:
    return load_library().srftq_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != SRFTQ_OK:
        raise SrftqError(fn, status, status_string(status))


def make_desc(d: int, heads: int, group: int, bits: int, rotation: int = SRFT) -> SrftqDesc:
    return SrftqDesc(int(d), int(heads), int(group), int(bits), int(rotation))


def _stream_handle(stream) -> int:
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _rows_layout(t, H: int, row_elems: int, name: str):
    """(pointer, n_slices, n_rows, slice_stride_rows) of a [S, N, H, e] view.

    Each row's heads and elements must be contiguous; slices may sit further
    apart than N rows (a window of a larger cache) but must not overlap, so a
    view whose slice stride is below N rows (an expanded or overlapping
    view) is refused before anything reaches the library."""
    if t.dim() != 4 or t.shape[2] != H or t.shape[3] != row_elems:
        raise ValueError(f"{name}: expected [S, N, {H}, {row_elems}], got {tuple(t.shape)}")
    S, N = t.shape[0], t.shape[1]
    if N > 1 and t.stride(1) != H * row_elems:
        raise ValueError(f"{name}: heads and elements of a row must be contiguous")
    if t.stride(3) != 1 or t.stride(2) != row_elems:
        raise ValueError(f"{name}: heads and elements of a row must be contiguous")
    if S <= 1:
        return t.data_ptr(), S, N, N
    if t.stride(0) % (H * row_elems) != 0:
        raise ValueError(f"{name}: slice stride must be a whole number of rows")
    stride_rows = t.stride(0) // (H * row_elems)
    if stride_rows < N:
        raise ValueError(f"{name}: slices overlap (slice stride {stride_rows} rows < {N} rows)")
    return t.data_ptr(), S, N, stride_rows


def _check_tensor(t, dtype, name: str):
    """t must live on the current CUDA device and have the dtype the C ABI reads."""
    import torch

    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name}: expected a torch tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected dtype {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor, got one on {t.device}")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name}: on {t.device}, but the current device is "
                         f"cuda:{torch.cuda.current_device()}")


def _rows_view(t, H: int, row_elems: int, name: str, dtype):
    _check_tensor(t, dtype, name)
    return _rows_layout(t, H, row_elems, name)


def _table(t, S: int, H: int, d: int, name: str, dtype):
    _check_tensor(t, dtype, name)
    if tuple(t.shape) != (S, H, d) or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous [{S}, {H}, {d}], got {tuple(t.shape)}")
    return t.data_ptr()


def _dtypes():
    import torch

    return torch.float16, torch.uint8, torch.int8, torch.float32


def srftq_quantize(desc: SrftqDesc, x, signs, lam, codes, scales, stream=None) -> None:
    """x [S,N,H,d] fp16 -> codes [S,N,H,d*bits/8] uint8, scales [S,N,H,d/G] fp16."""
    lib = load_library()
    F16, U8, I8, F32 = _dtypes()
    H, d = desc.heads, desc.d
    px, S, N, xs = _rows_view(x, H, d, "x", F16)
    pc, S2, N2, os_ = _rows_view(codes, H, d * desc.bits // 8, "codes", U8)
    ps, S3, N3, os2 = _rows_view(scales, H, d // desc.group, "scales", F16)
    if (S2, N2) != (S, N) or (S3, N3) != (S, N) or os2 != os_:
        raise ValueError("codes/scales must match x's slices and rows and share a slice stride")
    st = lib.srftq_quantize(ctypes.byref(desc), S, N, px, xs, _table(signs, S, H, d, "signs", I8),
                            _table(lam, S, H, d, "lambda", F32), pc, ps, os_,
                            _stream_handle(stream))
    _check("srftq_quantize", st)


def srftq_dequantize(desc: SrftqDesc, codes, scales, signs, lam, xhat, stream=None) -> None:
    """codes, scales -> xhat [S,N,H,d] fp16 (the inverse of srftq_quantize)."""
    lib = load_library()
    F16, U8, I8, F32 = _dtypes()
    H, d = desc.heads, desc.d
    pc, S, N, is_ = _rows_view(codes, H, d * desc.bits // 8, "codes", U8)
    ps, S2, N2, is2 = _rows_view(scales, H, d // desc.group, "scales", F16)
    px, S3, N3, os_ = _rows_view(xhat, H, d, "xhat", F16)
    if (S2, N2) != (S, N) or (S3, N3) != (S, N) or is2 != is_:
        raise ValueError("codes/scales/xhat shapes disagree")
    st = lib.srftq_dequantize(ctypes.byref(desc), S, N, pc, ps, is_,
                              _table(signs, S, H, d, "signs", I8),
                              _table(lam, S, H, d, "lambda", F32), px, os_,
                              _stream_handle(stream))
    _check("srftq_dequantize", st)


def srftq_calibrate_lambda(desc: SrftqDesc, x, signs, lam_out, n_cal: int, stream=None) -> None:
    """lambda_out [S,H,d] float32 = RMS of the rotated first n_cal rows of x."""
    lib = load_library()
    F16, U8, I8, F32 = _dtypes()
    H, d = desc.heads, desc.d
    px, S, N, xs = _rows_view(x, H, d, "x", F16)
    if n_cal > N:
        raise ValueError("n_cal exceeds the rows of x")
    st = lib.srftq_calibrate_lambda(ctypes.byref(desc), S, int(n_cal), px, xs,
                                    _table(signs, S, H, d, "signs", I8),
                                    _table(lam_out, S, H, d, "lambda_out", F32),
                                    _stream_handle(stream))
    _check("srftq_calibrate_lambda", st)


def srftq_rotate(desc: SrftqDesc, x, signs, y_out, lam=None, stream=None) -> None:
    """y_out [S,N,H,d] float32 (contiguous) = R (s*x), divided by lambda if given."""
    lib = load_library()
    F16, U8, I8, F32 = _dtypes()
    H, d = desc.heads, desc.d
    px, S, N, xs = _rows_view(x, H, d, "x", F16)
    _check_tensor(y_out, F32, "y_out")
    if tuple(y_out.shape) != (S, N, H, d) or not y_out.is_contiguous():
        raise ValueError("y_out must be a contiguous [S, N, H, d] float32 tensor")
    pl = _table(lam, S, H, d, "lambda", F32) if lam is not None else None
    st = lib.srftq_rotate(ctypes.byref(desc), S, N, px, xs, _table(signs, S, H, d, "signs", I8),
                          pl, y_out.data_ptr(), _stream_handle(stream))
    _check("srftq_rotate", st)


def srftq_dequantize_rotated(desc: SrftqDesc, codes, scales, lam, out, stream=None) -> None:
    """codes, scales -> out [S,N,H,d] fp16 = lambda * sigma * q (the rotated domain)."""
    lib = load_library()
    F16, U8, I8, F32 = _dtypes()
    H, d = desc.heads, desc.d
    pc, S, N, is_ = _rows_view(codes, H, d * desc.bits // 8, "codes", U8)
    ps, S2, N2, is2 = _rows_view(scales, H, d // desc.group, "scales", F16)
    po, S3, N3, os_ = _rows_view(out, H, d, "out", F16)
    if (S2, N2) != (S, N) or (S3, N3) != (S, N) or is2 != is_:
        raise ValueError("codes/scales/out shapes disagree")
    st = lib.srftq_dequantize_rotated(ctypes.byref(desc), S, N, pc, ps, is_,
                                      _table(lam, S, H, d, "lambda", F32), po, os_,
                                      _stream_handle(stream))
    _check("srftq_dequantize_rotated", st)


def srftq_unrotate(desc: SrftqDesc, y, signs, x_out, stream=None) -> None:
    """x_out [S,N,H,d] float32 = s * R^T y for y [S,N,H,d] float32."""
    lib = load_library()
    F16, U8, I8, F32 = _dtypes()
    H, d = desc.heads, desc.d
    py, S, N, ys = _rows_view(y, H, d, "y", F32)
    px, S2, N2, xs = _rows_view(x_out, H, d, "x_out", F32)
    if (S2, N2) != (S, N):
        raise ValueError("y/x_out shapes disagree")
    st = lib.srftq_unrotate(ctypes.byref(desc), S, N, py, ys, _table(signs, S, H, d, "signs", I8),
                            px, xs, _stream_handle(stream))
    _check("srftq_unrotate", st)


def _cache_rows(t, H: int, row_elems: int, name: str, dtype):
    """(pointer, rows) of a contiguous [rows, H, e] cache tensor."""
    _check_tensor(t, dtype, name)
    if t.dim() != 3 or t.shape[1] != H or t.shape[2] != row_elems or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous [rows, {H}, {row_elems}], got "
                         f"{tuple(t.shape)}")
    return t.data_ptr(), t.shape[0]


def srftq_decode_attention(desc: SrftqDesc, q, k_codes, k_scales, k_signs, k_lambda, v_codes,
                           v_scales, v_signs, v_lambda, n_ctx: int, tok_stride_rows: int,
                           seq_stride_rows: int, scale: float, out, stream=None) -> None:
    """out [n_seq, H*q_per_kv, d] float32 = softmax(scale q . khat) vhat over n_ctx
    tokens of the quantised K and V caches ([rows, H, ...] tensors; token t of
    sequence b is row t*tok_stride_rows + b*seq_stride_rows). The call makes
    three launches on the stream and uses `out` as their scratch, so `out`
    holds the result once that work is complete."""
    lib = load_library()
    F16, U8, I8, F32 = _dtypes()
    H, d = desc.heads, desc.d
    _check_tensor(q, F16, "q")
    if q.dim() != 3 or q.shape[1] % H or q.shape[2] != d or not q.is_contiguous():
        raise ValueError(f"q: expected contiguous [n_seq, {H}*q_per_kv, {d}]")
    n_seq, q_per_kv = q.shape[0], q.shape[1] // H
    _check_tensor(out, F32, "out")
    if tuple(out.shape) != tuple(q.shape) or not out.is_contiguous():
        raise ValueError("out must be a contiguous float32 tensor shaped like q")
    cb, ng = d * desc.bits // 8, d // desc.group
    pk, rk = _cache_rows(k_codes, H, cb, "k_codes", U8)
    pks, rks = _cache_rows(k_scales, H, ng, "k_scales", F16)
    pv, rv = _cache_rows(v_codes, H, cb, "v_codes", U8)
    pvs, rvs = _cache_rows(v_scales, H, ng, "v_scales", F16)
    need = (n_ctx - 1) * tok_stride_rows + (n_seq - 1) * seq_stride_rows + 1 if n_seq else 0
    if min(rk, rks, rv, rvs) < need:
        raise ValueError(f"the caches hold fewer than the {need} rows addressed")
    for t, name, dt in ((k_signs, "k_signs", I8), (v_signs, "v_signs", I8),
                        (k_lambda, "k_lambda", F32), (v_lambda, "v_lambda", F32)):
        _check_tensor(t, dt, name)
        if tuple(t.shape) != (H, d) or not t.is_contiguous():
            raise ValueError(f"{name}: expected contiguous [{H}, {d}]")
    st = lib.srftq_decode_attention(ctypes.byref(desc), n_seq, int(n_ctx), q_per_kv, q.data_ptr(),
                                    pk, pks, k_signs.data_ptr(), k_lambda.data_ptr(), pv, pvs,
                                    v_signs.data_ptr(), v_lambda.data_ptr(), int(tok_stride_rows),
                                    int(seq_stride_rows), float(scale), out.data_ptr(),
                                    _stream_handle(stream))
    _check("srftq_decode_attention", st)


def _matrices(t, S: int, H: int, shape: tuple, name: str, dtype):
    _check_tensor(t, dtype, name)
    if tuple(t.shape) != (S, H) + tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {(S, H) + tuple(shape)}, "
                         f"got {tuple(t.shape)}")
    return t.data_ptr()


def srftq_householder_rotation(desc: SrftqDesc, reflectors, signs, rot_out, stream=None) -> None:
    """rot_out [S,H,d,d] float32 = H(v_1) ... H(v_k) B (B the signed SRFT/SRHT
    matrix of desc.rotation) for reflectors [S,H,k,d] float32 (None for k = 0)."""
    lib = load_library()
    F16, U8, I8, F32 = _dtypes()
    S, H, d = rot_out.shape[0], desc.heads, desc.d
    po = _matrices(rot_out, S, H, (d, d), "rot_out", F32)
    ps = _table(signs, S, H, d, "signs", I8)
    if reflectors is None:
        k, pr = 0, None
    else:
        if reflectors.dim() != 4:
            raise ValueError("reflectors: expected [S, H, k, d]")
        k = reflectors.shape[2]
        pr = _matrices(reflectors, S, H, (k, d), "reflectors", F32)
    st = lib.srftq_householder_rotation(ctypes.byref(desc), S, int(k), pr, ps, po,
                                        _stream_handle(stream))
    _check("srftq_householder_rotation", st)


def srftq_dense_operand(desc: SrftqDesc, rot, operand_out, stream=None) -> None:
    """operand_out [S,H,2,d,d] fp16 = (fp16(R), fp16(R - hi)) of rot [S,H,d,d] float32."""
    lib = load_library()
    F16, U8, I8, F32 = _dtypes()
    S, H, d = rot.shape[0], desc.heads, desc.d
    pr = _matrices(rot, S, H, (d, d), "rot", F32)
    po = _matrices(operand_out, S, H, (2, d, d), "operand_out", F16)
    st = lib.srftq_dense_operand(ctypes.byref(desc), S, pr, po, _stream_handle(stream))
    _check("srftq_dense_operand", st)


def srftq_calibrate_lambda_dense(desc: SrftqDesc, x, operand, lam_out, n_cal: int,
                                 stream=None) -> None:
    """lam_out [S,H,d] float32 = RMS of R x over the first n_cal rows of x."""
    lib = load_library()
    F16, U8, I8, F32 = _dtypes()
    H, d = desc.heads, desc.d
    px, S, N, xs = _rows_view(x, H, d, "x", F16)
    if n_cal > N:
        raise ValueError("n_cal exceeds the rows of x")
    st = lib.srftq_calibrate_lambda_dense(ctypes.byref(desc), S, int(n_cal), px, xs,
                                          _matrices(operand, S, H, (2, d, d), "operand", F16),
                                          _table(lam_out, S, H, d, "lambda_out", F32),
                                          _stream_handle(stream))
    _check("srftq_calibrate_lambda_dense", st)


def srftq_quantize_dense(desc: SrftqDesc, x, operand, lam, codes, scales, stream=None) -> None:
    """x [S,N,H,d] fp16 -> codes, scales with the dense rotation of `operand`."""
    lib = load_library()
    F16, U8, I8, F32 = _dtypes()
    H, d = desc.heads, desc.d
    px, S, N, xs = _rows_view(x, H, d, "x", F16)
    pc, S2, N2, os_ = _rows_view(codes, H, d * desc.bits // 8, "codes", U8)
    ps, S3, N3, os2 = _rows_view(scales, H, d // desc.group, "scales", F16)
    if (S2, N2) != (S, N) or (S3, N3) != (S, N) or os2 != os_:
        raise ValueError("codes/scales must match x's slices and rows and share a slice stride")
    st = lib.srftq_quantize_dense(ctypes.byref(desc), S, N, px, xs,
                                  _matrices(operand, S, H, (2, d, d), "operand", F16),
                                  _table(lam, S, H, d, "lambda", F32), pc, ps, os_,
                                  _stream_handle(stream))
    _check("srftq_quantize_dense", st)


def srftq_dequantize_dense(desc: SrftqDesc, codes, scales, operand, lam, xhat,
                           stream=None) -> None:
    """codes, scales -> xhat [S,N,H,d] fp16 = R^T (lambda sigma q)."""
    lib = load_library()
    F16, U8, I8, F32 = _dtypes()
    H, d = desc.heads, desc.d
    pc, S, N, is_ = _rows_view(codes, H, d * desc.bits // 8, "codes", U8)
    ps, S2, N2, is2 = _rows_view(scales, H, d // desc.group, "scales", F16)
    px, S3, N3, os_ = _rows_view(xhat, H, d, "xhat", F16)
    if (S2, N2) != (S, N) or (S3, N3) != (S, N) or is2 != is_:
        raise ValueError("codes/scales/xhat shapes disagree")
    st = lib.srftq_dequantize_dense(ctypes.byref(desc), S, N, pc, ps, is_,
                                    _matrices(operand, S, H, (2, d, d), "operand", F16),
                                    _table(lam, S, H, d, "lambda", F32), px, os_,
                                    _stream_handle(stream))
    _check("srftq_dequantize_dense", st)


def srftq_probe_wait_timeout(polls: int, stream=None) -> int:
    """Launches the device-side timeout probe (see include/srftq.h); returns the status."""
    return int(load_library().srftq_probe_wait_timeout(int(polls), _stream_handle(stream)))


def srftq_probe_index_check(index: int, limit: int, stream=None) -> int:
    """Launches the device-side index-check probe (see include/srftq.h); returns the status."""
    return int(load_library().srftq_probe_index_check(int(index), int(limit),
                                                      _stream_handle(stream)))


def srftq_debug_checks() -> bool:
    """Whether the active library was built with the device-side index checks."""
    return bool(load_library().srftq_debug_checks())


def srftq_check_device(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device guard status."""
    return int(load_library().srftq_check_device(_stream_handle(stream)))


def srftq_version() -> int:
    return int(load_library().srftq_version())


# ---------------------------------------------------------------------------
# Allocating conveniences (torch allocates; the library computes)
# ---------------------------------------------------------------------------

def quantize(x, signs, lam, group: int = 16, bits: int = 4, rotation: int = SRFT, stream=None):
    """Returns (codes, scales) for x [S,N,H,d] fp16 on a CUDA device."""
    import torch

    S, N, H, d = x.shape
    desc = make_desc(d, H, group, bits, rotation)
    codes = torch.empty((S, N, H, d * bits // 8), dtype=torch.uint8, device=x.device)
    scales = torch.empty((S, N, H, d // group), dtype=torch.float16, device=x.device)
    srftq_quantize(desc, x, signs, lam, codes, scales, stream)
    return codes, scales


def dequantize(codes, scales, signs, lam, d: int, group: int = 16, bits: int = 4,
               rotation: int = SRFT, stream=None):
    import torch

    S, N, H, _ = codes.shape
    desc = make_desc(d, H, group, bits, rotation)
    xhat = torch.empty((S, N, H, d), dtype=torch.float16, device=codes.device)
    srftq_dequantize(desc, codes, scales, signs, lam, xhat, stream)
    return xhat


def calibrate_lambda(x, signs, n_cal: int = 512, rotation: int = SRFT, stream=None):
    import torch

    S, N, H, d = x.shape
    desc = make_desc(d, H, 8, 4, rotation)
    lam = torch.empty((S, H, d), dtype=torch.float32, device=x.device)
    srftq_calibrate_lambda(desc, x, signs, lam, n_cal, stream)
    return lam


def rotate(x, signs, lam=None, rotation: int = SRFT, stream=None):
    import torch

    S, N, H, d = x.shape
    desc = make_desc(d, H, 8, 4, rotation)
    y = torch.empty((S, N, H, d), dtype=torch.float32, device=x.device)
    srftq_rotate(desc, x, signs, y, lam, stream)
    return y


def dequantize_rotated(codes, scales, lam, d: int, group: int = 16, bits: int = 4, stream=None):
    """Returns lambda * sigma * q [S,N,H,d] fp16: the cache in the rotated domain."""
    import torch

    S, N, H, _ = codes.shape
    desc = make_desc(d, H, group, bits, SRFT)
    out = torch.empty((S, N, H, d), dtype=torch.float16, device=codes.device)
    srftq_dequantize_rotated(desc, codes, scales, lam, out, stream)
    return out


def unrotate(y, signs, rotation: int = SRFT, stream=None):
    """Returns s * R^T y [S,N,H,d] float32 for y [S,N,H,d] float32."""
    import torch

    S, N, H, d = y.shape
    desc = make_desc(d, H, 8, 4, rotation)
    x = torch.empty((S, N, H, d), dtype=torch.float32, device=y.device)
    srftq_unrotate(desc, y, signs, x, stream)
    return x


def decode_attention(q, k_codes, k_scales, k_signs, k_lambda, v_codes, v_scales, v_signs,
                     v_lambda, group: int = 16, bits: int = 4, rotation: int = SRFT,
                     n_ctx: int = None, tok_stride_rows: int = None, seq_stride_rows: int = 1,
                     scale: float = None, stream=None):
    """Fused decode attention over quantised K/V caches (see srftq_decode_attention).
    Defaults follow the decode layout row = token * n_seq + sequence."""
    import math

    import torch

    n_seq, HQ, d = q.shape
    H = k_codes.shape[1]
    if tok_stride_rows is None:
        tok_stride_rows = n_seq
    if n_ctx is None:
        n_ctx = k_codes.shape[0] // tok_stride_rows
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    desc = make_desc(d, H, group, bits, rotation)
    out = torch.empty((n_seq, HQ, d), dtype=torch.float32, device=q.device)
    srftq_decode_attention(desc, q, k_codes, k_scales, k_signs, k_lambda, v_codes, v_scales,
                           v_signs, v_lambda, n_ctx, tok_stride_rows, seq_stride_rows, scale, out,
                           stream)
    return out


def householder_rotation(reflectors, signs, rotation: int = SRFT, stream=None):
    """Returns R [S,H,d,d] float32 = H(v_1) ... H(v_k) B for reflectors
    [S,H,k,d] float32 (or None) on top of the signed SRFT/SRHT base."""
    import torch

    S, H, d = signs.shape
    desc = make_desc(d, H, 8, 4, rotation)
    rot = torch.empty((S, H, d, d), dtype=torch.float32, device=signs.device)
    srftq_householder_rotation(desc, reflectors, signs, rot, stream)
    return rot


def dense_operand(rot, stream=None):
    """Returns the fp16 (hi, lo) operand [S,H,2,d,d] of rotations [S,H,d,d]."""
    import torch

    S, H, d, _ = rot.shape
    desc = make_desc(d, H, 8, 4)
    op = torch.empty((S, H, 2, d, d), dtype=torch.float16, device=rot.device)
    srftq_dense_operand(desc, rot, op, stream)
    return op


def calibrate_lambda_dense(x, operand, n_cal: int = 512, stream=None):
    import torch

    S, N, H, d = x.shape
    desc = make_desc(d, H, 8, 4)
    lam = torch.empty((S, H, d), dtype=torch.float32, device=x.device)
    srftq_calibrate_lambda_dense(desc, x, operand, lam, n_cal, stream)
    return lam


def quantize_dense(x, operand, lam, group: int = 16, bits: int = 4, stream=None):
    """Returns (codes, scales) for x [S,N,H,d] fp16 with the dense rotation."""
    import torch

    S, N, H, d = x.shape
    desc = make_desc(d, H, group, bits)
    codes = torch.empty((S, N, H, d * bits // 8), dtype=torch.uint8, device=x.device)
    scales = torch.empty((S, N, H, d // group), dtype=torch.float16, device=x.device)
    srftq_quantize_dense(desc, x, operand, lam, codes, scales, stream)
    return codes, scales


def dequantize_dense(codes, scales, operand, lam, d: int, group: int = 16, bits: int = 4,
                     stream=None):
    import torch

    S, N, H, _ = codes.shape
    desc = make_desc(d, H, group, bits)
    xhat = torch.empty((S, N, H, d), dtype=torch.float16, device=codes.device)
    srftq_dequantize_dense(desc, codes, scales, operand, lam, xhat, stream)
    return xhat
