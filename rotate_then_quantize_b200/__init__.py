"""B200-native rotate-then-quantize KV-cache codec (SRFT / SRHT, int4 / int8).

The codec runs in libsrftq.so (hand-written CUDA for sm_100a, C ABI declared
in include/srftq.h); this package holds its sources, the in-tree build and a
thin ctypes binding. Importing the package does not load the library; the
first call does, and fails loudly if it has not been built.
"""

from .binding import (  # noqa: F401
    EXPORTED,
    SRFT,
    SRHT,
    SrftqDesc,
    SrftqError,
    calibrate_lambda,
    calibrate_lambda_dense,
    debug_checks,
    decode_attention,
    dense_operand,
    dequantize,
    dequantize_dense,
    dequantize_rotated,
    householder_rotation,
    load_library,
    make_desc,
    quantize,
    quantize_dense,
    rotate,
    srftq_calibrate_lambda,
    srftq_calibrate_lambda_dense,
    srftq_check_device,
    srftq_decode_attention,
    srftq_dense_operand,
    srftq_dequantize,
    srftq_dequantize_dense,
    srftq_dequantize_rotated,
    srftq_householder_rotation,
    srftq_debug_checks,
    srftq_probe_index_check,
    srftq_probe_wait_timeout,
    srftq_quantize,
    srftq_quantize_dense,
    srftq_rotate,
    srftq_unrotate,
    srftq_version,
    status_string,
    unrotate,
)
