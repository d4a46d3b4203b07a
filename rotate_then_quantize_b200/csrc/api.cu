// C ABI of libsrftq.so: argument validation, dispatch on the head dimension,
// the device guard word and the tensor-map encoder. See include/srftq.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "../../include/srftq.h"
#include "common.cuh"
#include "launch.cuh"
#include "ptx.cuh"

// Library-wide device guard word (one per device that loads the module), and
// the word srftq_check_device reads it into.
__device__ unsigned g_srftq_guard;
__device__ unsigned g_srftq_guard_taken;

namespace srftq {
// One thread waits on a barrier that nothing arrives on, `polls` times at
// most, then records the timeout like the codec kernels' bounded waits.
__global__ void probe_wait_timeout_kernel(unsigned* guard, uint32_t polls) {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  fence_barrier_init();
  for (uint32_t i = 0; i < polls; ++i)
    if (mbar_try_wait(&bar, 0)) return;
  atomicOr(guard, kGuardWaitTimeout);
}

// The index check of the debug build, on a given index: records kGuardIndex
// when index is outside [0, limit) (the access it guards is never made).
__global__ void probe_index_check_kernel(unsigned* guard, int64_t index, int64_t limit) {
  (void)dbg_ok(index >= 0 && index < limit, guard);
}

// Reads and clears the guard word in one atomic step, so a bit that another
// stream's kernel sets meanwhile is either reported now or kept for the next
// check, never lost.
__global__ void take_guard_kernel(unsigned* guard, unsigned* taken) {
  *taken = atomicExch(guard, 0u);
}
}  // namespace srftq

namespace srftq {
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

constexpr int kMaxDevices = 64;
std::atomic<int> g_num_sms[kMaxDevices];
std::atomic<unsigned*> g_guard_ptr[kMaxDevices];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }

int check_desc(const srftq_desc* d) {
  if (!d) return SRFTQ_ERR_INVALID_ARG;
  if (d->heads < 1) return SRFTQ_ERR_INVALID_ARG;
  if (!(d->d == 16 || d->d == 32 || d->d == 64 || d->d == 128 || d->d == 256))
    return SRFTQ_ERR_UNSUPPORTED;
  if (d->bits != 4 && d->bits != 8) return SRFTQ_ERR_UNSUPPORTED;
  if (!is_pow2(d->group) || d->group < 8 || d->group > d->d) return SRFTQ_ERR_UNSUPPORTED;
  if (d->rotation != SRFTQ_ROT_SRFT && d->rotation != SRFTQ_ROT_SRHT) return SRFTQ_ERR_UNSUPPORTED;
  return SRFTQ_OK;
}

// The dense-rotation calls take d in {64, 128, 256}; the codec calls also
// check the group and code width.
int check_dense_shape(const srftq_desc* d, bool codec) {
  if (!d) return SRFTQ_ERR_INVALID_ARG;
  if (d->heads < 1) return SRFTQ_ERR_INVALID_ARG;
  if (d->d != 64 && d->d != 128 && d->d != 256) return SRFTQ_ERR_UNSUPPORTED;
  if (codec) {
    if (d->bits != 4 && d->bits != 8) return SRFTQ_ERR_UNSUPPORTED;
    if (!is_pow2(d->group) || d->group < 8 || d->group > d->d) return SRFTQ_ERR_UNSUPPORTED;
  }
  return SRFTQ_OK;
}

// Byte range [lo, hi) touched by rows 0..n_rows-1 of S slices with a stride
// of `stride` rows of `row_bytes` each.
struct Range {
  uintptr_t lo, hi;
};

Range extent(const void* p, int64_t S, int64_t stride, int64_t n_rows, int64_t row_bytes) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  const uint64_t rows = uint64_t(S - 1) * uint64_t(stride) + uint64_t(n_rows);
  return {lo, lo + uintptr_t(rows * uint64_t(row_bytes))};
}

bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

template <typename Fn>
int by_d(int d, Fn&& fn) {
  switch (d) {
    case 16: return fn(Int<16>{});
    case 32: return fn(Int<32>{});
    case 64: return fn(Int<64>{});
    case 128: return fn(Int<128>{});
    case 256: return fn(Int<256>{});
    default: return SRFTQ_ERR_UNSUPPORTED;
  }
}

}  // namespace

int Runtime::encode_4d(CUtensorMap* map, CUtensorMapDataType dtype, void* base,
                       const uint64_t dims[4], const uint64_t strides_bytes[3],
                       const uint32_t box[4], CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return -1;
  const cuuint64_t gd[4] = {dims[0], dims[1], dims[2], dims[3]};
  const cuuint64_t gs[3] = {strides_bytes[0], strides_bytes[1], strides_bytes[2]};
  const cuuint32_t bd[4] = {box[0], box[1], box[2], box[3]};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, dtype, 4, base, gd, gs, bd, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

int Runtime::num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 1;
  int n = g_num_sms[dev].load(std::memory_order_acquire);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
      n = 1;
    g_num_sms[dev].store(n, std::memory_order_release);
  }
  return n;
}

unsigned* Runtime::guard_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  unsigned* p = g_guard_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    void* q = nullptr;
    if (cudaGetSymbolAddress(&q, g_srftq_guard) != cudaSuccess) return nullptr;
    p = static_cast<unsigned*>(q);
    g_guard_ptr[dev].store(p, std::memory_order_release);
  }
  return p;
}

}  // namespace srftq

using namespace srftq;

extern "C" {

int srftq_quantize(const srftq_desc* desc, int64_t n_slices, int64_t n_rows, const uint16_t* x,
                   int64_t x_slice_stride_rows, const int8_t* signs, const float* lambda,
                   uint8_t* codes, uint16_t* scales, int64_t out_slice_stride_rows,
                   void* stream) {
  int rc = check_desc(desc);
  if (rc != SRFTQ_OK) return rc;
  if (n_slices < 0 || n_rows < 0) return SRFTQ_ERR_INVALID_ARG;
  if (n_slices == 0 || n_rows == 0) return SRFTQ_OK;
  if (x_slice_stride_rows < n_rows || out_slice_stride_rows < n_rows) return SRFTQ_ERR_INVALID_ARG;
  if (!x || !signs || !lambda || !codes || !scales) return SRFTQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(signs) || !aligned16(lambda) || !aligned16(codes) ||
      !aligned16(scales))
    return SRFTQ_ERR_MISALIGNED;
  const int64_t d = desc->d, H = desc->heads;
  const Range rx = extent(x, n_slices, x_slice_stride_rows, n_rows, H * d * 2);
  const Range rc_ = extent(codes, n_slices, out_slice_stride_rows, n_rows, H * d * desc->bits / 8);
  const Range rs = extent(scales, n_slices, out_slice_stride_rows, n_rows, H * (d / desc->group) * 2);
  const Range rsg = extent(signs, n_slices, H, H, d);
  const Range rl = extent(lambda, n_slices, H, H, d * 4);
  for (Range out : {rc_, rs})
    for (Range in : {rx, rsg, rl})
      if (overlap(out, in)) return SRFTQ_ERR_INVALID_ARG;
  if (overlap(rc_, rs)) return SRFTQ_ERR_INVALID_ARG;
  QuantCall c{desc->heads, desc->group, desc->bits, desc->rotation, n_slices, n_rows,
              x, x_slice_stride_rows, signs, lambda, codes, scales, out_slice_stride_rows,
              static_cast<cudaStream_t>(stream)};
  return by_d(desc->d, [&](auto d_) { return launch_quantize<decltype(d_)::value>(c); });
}

int srftq_dequantize(const srftq_desc* desc, int64_t n_slices, int64_t n_rows,
                     const uint8_t* codes, const uint16_t* scales, int64_t in_slice_stride_rows,
                     const int8_t* signs, const float* lambda, uint16_t* xhat,
                     int64_t out_slice_stride_rows, void* stream) {
  int rc = check_desc(desc);
  if (rc != SRFTQ_OK) return rc;
  if (n_slices < 0 || n_rows < 0) return SRFTQ_ERR_INVALID_ARG;
  if (n_slices == 0 || n_rows == 0) return SRFTQ_OK;
  if (in_slice_stride_rows < n_rows || out_slice_stride_rows < n_rows) return SRFTQ_ERR_INVALID_ARG;
  if (!codes || !scales || !signs || !lambda || !xhat) return SRFTQ_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(signs) || !aligned16(lambda) ||
      !aligned16(xhat))
    return SRFTQ_ERR_MISALIGNED;
  const int64_t d = desc->d, H = desc->heads;
  const Range rx = extent(xhat, n_slices, out_slice_stride_rows, n_rows, H * d * 2);
  const Range rc_ = extent(codes, n_slices, in_slice_stride_rows, n_rows, H * d * desc->bits / 8);
  const Range rs = extent(scales, n_slices, in_slice_stride_rows, n_rows, H * (d / desc->group) * 2);
  const Range rsg = extent(signs, n_slices, H, H, d);
  const Range rl = extent(lambda, n_slices, H, H, d * 4);
  for (Range in : {rc_, rs, rsg, rl})
    if (overlap(rx, in)) return SRFTQ_ERR_INVALID_ARG;
  DequantCall c{desc->heads, desc->group, desc->bits, desc->rotation, n_slices, n_rows,
                codes, scales, in_slice_stride_rows, signs, lambda, xhat, out_slice_stride_rows,
                static_cast<cudaStream_t>(stream)};
  return by_d(desc->d, [&](auto d_) { return launch_dequantize<decltype(d_)::value>(c); });
}

int srftq_calibrate_lambda(const srftq_desc* desc, int64_t n_slices, int64_t n_cal,
                           const uint16_t* x, int64_t x_slice_stride_rows, const int8_t* signs,
                           float* lambda_out, void* stream) {
  int rc = check_desc(desc);
  if (rc != SRFTQ_OK) return rc;
  if (n_slices < 0 || n_cal < 1) return SRFTQ_ERR_INVALID_ARG;
  if (n_slices == 0) return SRFTQ_OK;
  if (x_slice_stride_rows < n_cal) return SRFTQ_ERR_INVALID_ARG;
  if (!x || !signs || !lambda_out) return SRFTQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(signs) || !aligned16(lambda_out)) return SRFTQ_ERR_MISALIGNED;
  const int64_t d = desc->d, H = desc->heads;
  const Range rx = extent(x, n_slices, x_slice_stride_rows, n_cal, H * d * 2);
  const Range rsg = extent(signs, n_slices, H, H, d);
  const Range rl = extent(lambda_out, n_slices, H, H, d * 4);
  if (overlap(rl, rx) || overlap(rl, rsg)) return SRFTQ_ERR_INVALID_ARG;
  CalibCall c{desc->heads, desc->rotation, n_slices, n_cal, x, x_slice_stride_rows, signs,
              lambda_out, static_cast<cudaStream_t>(stream)};
  return by_d(desc->d, [&](auto d_) { return launch_calibrate<decltype(d_)::value>(c); });
}

int srftq_rotate(const srftq_desc* desc, int64_t n_slices, int64_t n_rows, const uint16_t* x,
                 int64_t x_slice_stride_rows, const int8_t* signs, const float* lambda_or_null,
                 float* y_out, void* stream) {
  int rc = check_desc(desc);
  if (rc != SRFTQ_OK) return rc;
  if (n_slices < 0 || n_rows < 0) return SRFTQ_ERR_INVALID_ARG;
  if (n_slices == 0 || n_rows == 0) return SRFTQ_OK;
  if (x_slice_stride_rows < n_rows) return SRFTQ_ERR_INVALID_ARG;
  if (!x || !signs || !y_out) return SRFTQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(signs) || !aligned16(y_out) ||
      (lambda_or_null && !aligned16(lambda_or_null)))
    return SRFTQ_ERR_MISALIGNED;
  const int64_t d = desc->d, H = desc->heads;
  const Range ry = extent(y_out, n_slices, n_rows, n_rows, H * d * 4);
  const Range rx = extent(x, n_slices, x_slice_stride_rows, n_rows, H * d * 2);
  const Range rsg = extent(signs, n_slices, H, H, d);
  if (overlap(ry, rx) || overlap(ry, rsg)) return SRFTQ_ERR_INVALID_ARG;
  if (lambda_or_null && overlap(ry, extent(lambda_or_null, n_slices, H, H, d * 4)))
    return SRFTQ_ERR_INVALID_ARG;
  RotateCall c{desc->heads, desc->rotation, n_slices, n_rows, x, x_slice_stride_rows, signs,
               lambda_or_null, y_out, static_cast<cudaStream_t>(stream)};
  return by_d(desc->d, [&](auto d_) { return launch_rotate<decltype(d_)::value>(c); });
}

const char* srftq_status_string(int status) {
  switch (status) {
    case SRFTQ_OK: return "ok";
    case SRFTQ_ERR_INVALID_ARG: return "invalid argument";
    case SRFTQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case SRFTQ_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case SRFTQ_ERR_CUDA: return "CUDA error";
    case SRFTQ_ERR_DEVICE_CHECK: return "device-side guard fired";
    default: return "unknown status";
  }
}

int srftq_check_device(void* stream) {
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* guard = srftq::Runtime::guard_word();
  void* taken = nullptr;
  if (!guard || cudaGetSymbolAddress(&taken, g_srftq_guard_taken) != cudaSuccess)
    return SRFTQ_ERR_CUDA;
  srftq::take_guard_kernel<<<1, 1, 0, st>>>(guard, static_cast<unsigned*>(taken));
  if (cudaGetLastError() != cudaSuccess) return SRFTQ_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyAsync(&v, taken, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return SRFTQ_ERR_CUDA;
  return v == 0 ? SRFTQ_OK : SRFTQ_ERR_DEVICE_CHECK;
}

int srftq_dequantize_rotated(const srftq_desc* desc, int64_t n_slices, int64_t n_rows,
                             const uint8_t* codes, const uint16_t* scales,
                             int64_t in_slice_stride_rows, const float* lambda, uint16_t* out,
                             int64_t out_slice_stride_rows, void* stream) {
  int rc = check_desc(desc);
  if (rc != SRFTQ_OK) return rc;
  if (n_slices < 0 || n_rows < 0) return SRFTQ_ERR_INVALID_ARG;
  if (n_slices == 0 || n_rows == 0) return SRFTQ_OK;
  if (in_slice_stride_rows < n_rows || out_slice_stride_rows < n_rows) return SRFTQ_ERR_INVALID_ARG;
  if (!codes || !scales || !lambda || !out) return SRFTQ_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(lambda) || !aligned16(out))
    return SRFTQ_ERR_MISALIGNED;
  const int64_t d = desc->d, H = desc->heads;
  const Range ro = extent(out, n_slices, out_slice_stride_rows, n_rows, H * d * 2);
  const Range rc_ = extent(codes, n_slices, in_slice_stride_rows, n_rows, H * d * desc->bits / 8);
  const Range rs = extent(scales, n_slices, in_slice_stride_rows, n_rows, H * (d / desc->group) * 2);
  const Range rl = extent(lambda, n_slices, H, H, d * 4);
  for (Range in : {rc_, rs, rl})
    if (overlap(ro, in)) return SRFTQ_ERR_INVALID_ARG;
  RotDequantCall c{desc->heads, desc->group, desc->bits, n_slices, n_rows, codes, scales,
                   in_slice_stride_rows, lambda, out, out_slice_stride_rows,
                   static_cast<cudaStream_t>(stream)};
  return by_d(desc->d, [&](auto d_) { return launch_dequantize_rotated<decltype(d_)::value>(c); });
}

int srftq_unrotate(const srftq_desc* desc, int64_t n_slices, int64_t n_rows, const float* y,
                   int64_t y_slice_stride_rows, const int8_t* signs, float* x,
                   int64_t x_slice_stride_rows, void* stream) {
  int rc = check_desc(desc);
  if (rc != SRFTQ_OK) return rc;
  if (n_slices < 0 || n_rows < 0) return SRFTQ_ERR_INVALID_ARG;
  if (n_slices == 0 || n_rows == 0) return SRFTQ_OK;
  if (y_slice_stride_rows < n_rows || x_slice_stride_rows < n_rows) return SRFTQ_ERR_INVALID_ARG;
  if (!y || !signs || !x) return SRFTQ_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(signs) || !aligned16(x)) return SRFTQ_ERR_MISALIGNED;
  const int64_t d = desc->d, H = desc->heads;
  const Range rx = extent(x, n_slices, x_slice_stride_rows, n_rows, H * d * 4);
  const Range ry = extent(y, n_slices, y_slice_stride_rows, n_rows, H * d * 4);
  const Range rsg = extent(signs, n_slices, H, H, d);
  if (overlap(rx, ry) || overlap(rx, rsg)) return SRFTQ_ERR_INVALID_ARG;
  UnrotateCall c{desc->heads, desc->rotation, n_slices, n_rows, y, y_slice_stride_rows, signs,
                 x, x_slice_stride_rows, static_cast<cudaStream_t>(stream)};
  return by_d(desc->d, [&](auto d_) { return launch_unrotate<decltype(d_)::value>(c); });
}

int srftq_decode_attention(const srftq_desc* desc, int64_t n_seq, int64_t n_ctx, int32_t q_per_kv,
                           const uint16_t* q, const uint8_t* k_codes, const uint16_t* k_scales,
                           const int8_t* k_signs, const float* k_lambda, const uint8_t* v_codes,
                           const uint16_t* v_scales, const int8_t* v_signs,
                           const float* v_lambda, int64_t tok_stride_rows,
                           int64_t seq_stride_rows, float softmax_scale, float* out,
                           void* stream) {
  int rc = check_desc(desc);
  if (rc != SRFTQ_OK) return rc;
  if (desc->d != 128) return SRFTQ_ERR_UNSUPPORTED;
  if (q_per_kv != 1 && q_per_kv != 2 && q_per_kv != 4 && q_per_kv != 8)
    return SRFTQ_ERR_UNSUPPORTED;
  if (n_seq < 0 || n_ctx < 1 || tok_stride_rows < 0 || seq_stride_rows < 0)
    return SRFTQ_ERR_INVALID_ARG;
  if (n_seq == 0) return SRFTQ_OK;
  if (!q || !k_codes || !k_scales || !k_signs || !k_lambda || !v_codes || !v_scales ||
      !v_signs || !v_lambda || !out)
    return SRFTQ_ERR_INVALID_ARG;
  for (const void* p : {static_cast<const void*>(q), static_cast<const void*>(k_codes),
                        static_cast<const void*>(k_scales), static_cast<const void*>(k_signs),
                        static_cast<const void*>(k_lambda), static_cast<const void*>(v_codes),
                        static_cast<const void*>(v_scales), static_cast<const void*>(v_signs),
                        static_cast<const void*>(v_lambda), static_cast<const void*>(out)})
    if (!aligned16(p)) return SRFTQ_ERR_MISALIGNED;
  const int64_t d = desc->d, H = desc->heads;
  const int64_t rows = (n_ctx - 1) * tok_stride_rows + (n_seq - 1) * seq_stride_rows + 1;
  const int64_t cb = H * d * desc->bits / 8, sb = H * (d / desc->group) * 2;
  const Range ro = extent(out, 1, 0, 1, n_seq * H * q_per_kv * d * 4);
  const Range rq_ = extent(q, 1, 0, 1, n_seq * H * q_per_kv * d * 2);
  for (Range in : {rq_, extent(k_codes, 1, 0, rows, cb), extent(k_scales, 1, 0, rows, sb),
                   extent(v_codes, 1, 0, rows, cb), extent(v_scales, 1, 0, rows, sb),
                   extent(k_signs, 1, 0, 1, H * d), extent(v_signs, 1, 0, 1, H * d),
                   extent(k_lambda, 1, 0, 1, H * d * 4), extent(v_lambda, 1, 0, 1, H * d * 4)})
    if (overlap(ro, in)) return SRFTQ_ERR_INVALID_ARG;
  AttnCall c{desc->heads, desc->group, desc->bits, desc->rotation, q_per_kv, n_seq, n_ctx,
             tok_stride_rows, seq_stride_rows, softmax_scale, q, k_codes, k_scales, k_signs,
             k_lambda, v_codes, v_scales, v_signs, v_lambda, out,
             static_cast<cudaStream_t>(stream)};
  return launch_decode_attention_d128(c);
}

// ---------------------------------------------------------------------------
// Dense-rotation codec
// ---------------------------------------------------------------------------

int srftq_householder_rotation(const srftq_desc* desc, int64_t n_slices, int32_t n_reflectors,
                               const float* reflectors, const int8_t* signs,
                               float* rotation_out, void* stream) {
  int rc = check_dense_shape(desc, false);
  if (rc != SRFTQ_OK) return rc;
  if (desc->rotation != SRFTQ_ROT_SRFT && desc->rotation != SRFTQ_ROT_SRHT)
    return SRFTQ_ERR_UNSUPPORTED;
  if (n_slices < 0 || n_reflectors < 0 || n_reflectors > 65536) return SRFTQ_ERR_INVALID_ARG;
  if (n_slices == 0) return SRFTQ_OK;
  if (!signs || !rotation_out || (n_reflectors > 0 && !reflectors)) return SRFTQ_ERR_INVALID_ARG;
  if (!aligned16(signs) || !aligned16(rotation_out) || (reflectors && !aligned16(reflectors)))
    return SRFTQ_ERR_MISALIGNED;
  const int64_t d = desc->d, H = desc->heads;
  const Range ro = extent(rotation_out, 1, 0, n_slices * H, d * d * 4);
  if (overlap(ro, extent(signs, 1, 0, n_slices * H, d))) return SRFTQ_ERR_INVALID_ARG;
  if (n_reflectors > 0 &&
      overlap(ro, extent(reflectors, 1, 0, n_slices * H * n_reflectors, d * 4)))
    return SRFTQ_ERR_INVALID_ARG;
  HouseholderCall c{desc->d, desc->heads, desc->rotation, n_reflectors, n_slices, reflectors,
                    signs, rotation_out, static_cast<cudaStream_t>(stream)};
  return launch_householder(c);
}

int srftq_dense_operand(const srftq_desc* desc, int64_t n_slices, const float* rotation,
                        uint16_t* operand_out, void* stream) {
  int rc = check_dense_shape(desc, false);
  if (rc != SRFTQ_OK) return rc;
  if (n_slices < 0) return SRFTQ_ERR_INVALID_ARG;
  if (n_slices == 0) return SRFTQ_OK;
  if (!rotation || !operand_out) return SRFTQ_ERR_INVALID_ARG;
  if (!aligned16(rotation) || !aligned16(operand_out)) return SRFTQ_ERR_MISALIGNED;
  const int64_t d = desc->d, H = desc->heads;
  if (overlap(extent(operand_out, 1, 0, n_slices * H, 2 * d * d * 2),
              extent(rotation, 1, 0, n_slices * H, d * d * 4)))
    return SRFTQ_ERR_INVALID_ARG;
  OperandCall c{desc->d, desc->heads, n_slices, rotation, operand_out,
                static_cast<cudaStream_t>(stream)};
  return launch_dense_operand(c);
}

int srftq_calibrate_lambda_dense(const srftq_desc* desc, int64_t n_slices, int64_t n_cal,
                                 const uint16_t* x, int64_t x_slice_stride_rows,
                                 const uint16_t* operand, float* lambda_out, void* stream) {
  int rc = check_dense_shape(desc, false);
  if (rc != SRFTQ_OK) return rc;
  if (n_slices < 0 || n_cal < 1) return SRFTQ_ERR_INVALID_ARG;
  if (n_slices == 0) return SRFTQ_OK;
  if (x_slice_stride_rows < n_cal) return SRFTQ_ERR_INVALID_ARG;
  if (!x || !operand || !lambda_out) return SRFTQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(operand) || !aligned16(lambda_out)) return SRFTQ_ERR_MISALIGNED;
  const int64_t d = desc->d, H = desc->heads;
  const Range rl = extent(lambda_out, 1, 0, n_slices * H, d * 4);
  if (overlap(rl, extent(x, n_slices, x_slice_stride_rows, n_cal, H * d * 2)) ||
      overlap(rl, extent(operand, 1, 0, n_slices * H, 2 * d * d * 2)))
    return SRFTQ_ERR_INVALID_ARG;
  DenseCalibCall c{desc->d, desc->heads, n_slices, n_cal, x_slice_stride_rows, x, operand,
                   lambda_out, static_cast<cudaStream_t>(stream)};
  return launch_calibrate_dense(c);
}

int srftq_quantize_dense(const srftq_desc* desc, int64_t n_slices, int64_t n_rows,
                         const uint16_t* x, int64_t x_slice_stride_rows, const uint16_t* operand,
                         const float* lambda, uint8_t* codes, uint16_t* scales,
                         int64_t out_slice_stride_rows, void* stream) {
  int rc = check_dense_shape(desc, true);
  if (rc != SRFTQ_OK) return rc;
  if (n_slices < 0 || n_rows < 0) return SRFTQ_ERR_INVALID_ARG;
  if (n_slices == 0 || n_rows == 0) return SRFTQ_OK;
  if (x_slice_stride_rows < n_rows || out_slice_stride_rows < n_rows) return SRFTQ_ERR_INVALID_ARG;
  if (!x || !operand || !lambda || !codes || !scales) return SRFTQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(operand) || !aligned16(lambda) || !aligned16(codes) ||
      !aligned16(scales))
    return SRFTQ_ERR_MISALIGNED;
  const int64_t d = desc->d, H = desc->heads;
  const Range rx = extent(x, n_slices, x_slice_stride_rows, n_rows, H * d * 2);
  const Range rc_ = extent(codes, n_slices, out_slice_stride_rows, n_rows, H * d * desc->bits / 8);
  const Range rs = extent(scales, n_slices, out_slice_stride_rows, n_rows, H * (d / desc->group) * 2);
  const Range rop = extent(operand, 1, 0, n_slices * H, 2 * d * d * 2);
  const Range rl = extent(lambda, 1, 0, n_slices * H, d * 4);
  for (Range out : {rc_, rs})
    for (Range in : {rx, rop, rl})
      if (overlap(out, in)) return SRFTQ_ERR_INVALID_ARG;
  if (overlap(rc_, rs)) return SRFTQ_ERR_INVALID_ARG;
  DenseCall c{desc->d, desc->heads, desc->group, desc->bits, n_slices, n_rows,
              x_slice_stride_rows, out_slice_stride_rows, x, nullptr, nullptr, codes, scales,
              nullptr, operand, lambda, static_cast<cudaStream_t>(stream)};
  return launch_quantize_dense(c);
}

int srftq_dequantize_dense(const srftq_desc* desc, int64_t n_slices, int64_t n_rows,
                           const uint8_t* codes, const uint16_t* scales,
                           int64_t in_slice_stride_rows, const uint16_t* operand,
                           const float* lambda, uint16_t* xhat, int64_t out_slice_stride_rows,
                           void* stream) {
  int rc = check_dense_shape(desc, true);
  if (rc != SRFTQ_OK) return rc;
  if (n_slices < 0 || n_rows < 0) return SRFTQ_ERR_INVALID_ARG;
  if (n_slices == 0 || n_rows == 0) return SRFTQ_OK;
  if (in_slice_stride_rows < n_rows || out_slice_stride_rows < n_rows) return SRFTQ_ERR_INVALID_ARG;
  if (!codes || !scales || !operand || !lambda || !xhat) return SRFTQ_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(operand) || !aligned16(lambda) ||
      !aligned16(xhat))
    return SRFTQ_ERR_MISALIGNED;
  const int64_t d = desc->d, H = desc->heads;
  const Range rx = extent(xhat, n_slices, out_slice_stride_rows, n_rows, H * d * 2);
  for (Range in : {extent(codes, n_slices, in_slice_stride_rows, n_rows, H * d * desc->bits / 8),
                   extent(scales, n_slices, in_slice_stride_rows, n_rows,
                          H * (d / desc->group) * 2),
                   extent(operand, 1, 0, n_slices * H, 2 * d * d * 2),
                   extent(lambda, 1, 0, n_slices * H, d * 4)})
    if (overlap(rx, in)) return SRFTQ_ERR_INVALID_ARG;
  DenseCall c{desc->d, desc->heads, desc->group, desc->bits, n_slices, n_rows,
              in_slice_stride_rows, out_slice_stride_rows, nullptr, codes, scales, nullptr,
              nullptr, xhat, operand, lambda, static_cast<cudaStream_t>(stream)};
  return launch_dequantize_dense(c);
}

int srftq_probe_wait_timeout(uint32_t polls, void* stream) {
  if (polls == 0 || polls > srftq::kWaitLimit) return SRFTQ_ERR_INVALID_ARG;
  unsigned* guard = srftq::Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  srftq::probe_wait_timeout_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(guard, polls);
  return cudaGetLastError() == cudaSuccess ? SRFTQ_OK : SRFTQ_ERR_CUDA;
}

int srftq_probe_index_check(int64_t index, int64_t limit, void* stream) {
  unsigned* guard = srftq::Runtime::guard_word();
  if (!guard) return SRFTQ_ERR_CUDA;
  srftq::probe_index_check_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(guard, index,
                                                                                 limit);
  return cudaGetLastError() == cudaSuccess ? SRFTQ_OK : SRFTQ_ERR_CUDA;
}

int srftq_debug_checks(void) { return srftq::kDebugChecks ? 1 : 0; }

int srftq_version(void) { return 200; }

}  // extern "C"
