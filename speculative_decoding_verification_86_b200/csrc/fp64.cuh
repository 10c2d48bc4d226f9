// fp64 helpers of the refinement path.
//
// exp2_fast: 2^x for x <= ~0 in double precision, by the classic table-driven
// reduction (Tang, "Table-driven implementation of the exponential function in
// IEEE floating-point arithmetic", ACM TOMS 1989): x = k/32 + r with k an
// integer and |r| <= 1/64, 2^x = 2^(k>>5) * 2^((k&31)/32) * 2^r.  2^r is the
// Taylor series of exp(r ln 2) through degree 6 (truncation < 4e-18 relative
// on |r ln 2| <= 0.0109); the 32 table entries 2^(j/32) are computed once per
// CTA with exp2() into shared memory.  Error: a few ulp; the GPU tests compare
// it with exp2() over the whole argument range.
#pragma once
#include <cuda_runtime.h>
#include "common.cuh"

namespace sv {

constexpr int kExp2Table = 32;
constexpr double kLog2E = 1.4426950408889634074;
constexpr double kLn2d = 0.69314718055994530942;

// Every compute thread (warps 0 .. kWarps-1) must call this before the first
// exp2_fast.
__device__ __forceinline__ void exp2_table_init(double* tab) {
  for (int j = threadIdx.x; j < kExp2Table; j += kThreads) tab[j] = exp2(j / 32.0);
  sync_compute();
}

__device__ __forceinline__ double exp2_fast(double x, const double* tab) {
  if (!(x >= -1070.0)) return x != x ? x : 0.0;  // NaN stays NaN; below the range -> 0
  const double kMagic = 6755399441055744.0;      // 1.5 * 2^52: x*32 + magic rounds to an integer
  const double t = fma(x, 32.0, kMagic);
  const int k = __double2loint(t);                // the integer, in two's complement
  const double kd = t - kMagic;
  const double r = fma(kd, -0.03125, x);          // exact, |r| <= 1/64
  const double y = r * kLn2d;
  double p = 1.0 / 720.0;
  p = fma(p, y, 1.0 / 120.0);
  p = fma(p, y, 1.0 / 24.0);
  p = fma(p, y, 1.0 / 6.0);
  p = fma(p, y, 0.5);
  p = fma(p, y, 1.0);
  p = fma(p, y, 1.0);
  const double v = tab[k & 31] * p;
  const int n = k >> 5;                           // floor(k / 32)
  if (n >= -1021) return __hiloint2double(__double2hiint(v) + (n << 20), __double2loint(v));
  return ldexp(v, n);
}

// exp(l / T - m) with l a logit: 2^(l * s - m2) with s = log2(e) / T and
// m2 = m * log2(e) precomputed in fp64 (one fused multiply-add per logit).
__device__ __forceinline__ double exp_weight(float l, double s, double m2, const double* tab) {
  return exp2_fast(fma(static_cast<double>(l), s, -m2), tab);
}

}  // namespace sv
