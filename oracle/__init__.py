"""CPU oracle for the rotate-then-quantize KV codec (test infrastructure only).

This package is the slow, plain, float64 statement of what the codec computes.
It exists so that the CUDA path can be checked against something written
independently of it. Only the test suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it; the
library itself never does, and it shares no code, tables or constants with the
CUDA sources.

Sources followed (cited by page title and section):

* "When Quantization Is Free" (technical summary), Methodology 1: the SRFT
  rotation SRFT(x) = pack(F . diag(s) . x) with F the unitary DFT and s a fixed
  random sign vector.
* same page, Methodology 2 (the fused kernel): the order of the stages -- sign
  multiply, FFT, Hermitian pack, per-channel lambda rescale, group absmax,
  round to signed int4/int8, nibble packing.
* same page, Methodology 3: per-channel scale (one per coordinate) combined
  with per-group absmax scaling over groups of 16.
* "HyperQuant" (technical summary), Methodology 1: the randomized Hadamard
  transform RHT(x) = H D x, used for the SRHT variant.
* "When Quantization Is Free", Methodology 3 (Householder rotations) and
  Key Results (lossless regime): the codec with a rotation given as an
  explicit matrix, in particular k Householder reflectors on top of the
  SRFT base (``dense_oracle``).

Every function is pinned by the ``-m "not gpu"`` tests in ``tests/`` against
closed forms, library special cases, brute force and hand-worked examples.
Nothing here is "parity unpinned" except the end-to-end model quality, which
needs trained models and is outside this codec.
"""

from .srft_oracle import (  # noqa: F401
    SRFT,
    SRHT,
    binary16_bits_to_float,
    calibrate_lambda,
    decode_attention,
    dequantize,
    dequantize_rotated,
    float_to_binary16_bits,
    pack_codes,
    qmax_for,
    quantize,
    quantize_vectors,
    rotate,
    rotation_matrix,
    srft_matrix,
    srht_matrix,
    unpack_codes,
    unrotate,
)
from .dense_oracle import (  # noqa: F401,E402
    calibrate_lambda_dense,
    dequantize_dense,
    householder_matrix,
    householder_rotations,
    quantize_dense,
    reflector,
    rotate_dense,
    split_operand,
    unrotate_dense,
)
