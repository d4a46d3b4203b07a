// Compile-time helpers shared by the codec kernels: static loops, bit
// reversal and exact twiddle constants.
//
// Twiddles are cos/sin(2*pi*j/n) evaluated at compile time in double: the
// angle is reduced to [0, pi/4] exactly with integer octant arithmetic, then a
// Taylor series (terms up to x^23, truncation error < 1e-20 on [0, pi/4]) is
// summed in double and the result rounded once to float. No run-time
// trigonometry and no CUDA math-library internals are involved.
#pragma once

#include <cstdint>
#include <type_traits>

namespace srftq {

template <int I>
using Int = std::integral_constant<int, I>;

// static_for<B, E>(f): calls f(Int<i>{}) for i = B .. E-1 at compile time, so
// every index inside f is a constant expression (registers, twiddles).
template <int B, int E, typename F>
__host__ __device__ __forceinline__ void static_for(F&& f) {
  if constexpr (B < E) {
    f(Int<B>{});
    static_for<B + 1, E>(static_cast<F&&>(f));
  }
}

__host__ __device__ constexpr int ilog2(int x) {
  int r = 0;
  while ((1 << r) < x) ++r;
  return r;
}

__host__ __device__ constexpr int bitrev(int x, int bits) {
  int r = 0;
  for (int b = 0; b < bits; ++b) r = (r << 1) | ((x >> b) & 1);
  return r;
}

namespace ct {

constexpr double kPi = 3.14159265358979323846264338327950288;

// sin and cos on [0, pi/4] by their Maclaurin series.
__host__ __device__ constexpr double sin_small(double x) {
  double x2 = x * x, term = x, sum = x;
  for (int n = 1; n <= 11; ++n) {
    term *= -x2 / double((2 * n) * (2 * n + 1));
    sum += term;
  }
  return sum;
}

__host__ __device__ constexpr double cos_small(double x) {
  double x2 = x * x, term = 1.0, sum = 1.0;
  for (int n = 1; n <= 11; ++n) {
    term *= -x2 / double((2 * n - 1) * (2 * n));
    sum += term;
  }
  return sum;
}

struct CosSin {
  double c, s;
};

// cos and sin of 2*pi*j/n for integers j, n > 0. The angle is measured in
// units of 2*pi/(8n); its octant o and the offset inside the octant are
// found with integer arithmetic, so only an angle in [0, pi/4] ever reaches
// floating point.
__host__ __device__ constexpr CosSin cos_sin_2pi(long long j, long long n) {
  const long long m = 8 * n;
  long long J = (8 * j) % m;
  if (J < 0) J += m;
  const long long o = J / n;
  const long long rem = J - o * n;
  const bool odd = (o & 1) != 0;
  const double delta = 2.0 * kPi * double(odd ? (n - rem) : rem) / double(m);
  const double cd = cos_small(delta), sd = sin_small(delta);
  switch (o) {
    case 0: return {cd, sd};
    case 1: return {sd, cd};
    case 2: return {-sd, cd};
    case 3: return {-cd, sd};
    case 4: return {-cd, -sd};
    case 5: return {-sd, -cd};
    case 6: return {sd, -cd};
    default: return {cd, -sd};
  }
}

__host__ __device__ constexpr double cos2pi(long long j, long long n) { return cos_sin_2pi(j, n).c; }
__host__ __device__ constexpr double sin2pi(long long j, long long n) { return cos_sin_2pi(j, n).s; }
__host__ __device__ constexpr double dabs(double x) { return x < 0 ? -x : x; }

}  // namespace ct
}  // namespace srftq
