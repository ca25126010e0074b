// Device side of the binary32 routing recipe: log-mean-exp pools and sigmoid gates.
//
// HLA summary page ("Overview": log-mean-exp pooled routing gates; "Methodology in
// Plain English": a sigmoid weight per historical chunk, thresholded without
// renormalisation).  Gates decide which chunks are skipped, so this file fixes the
// exact sequence of binary32 operations: only correctly rounded add, subtract,
// multiply, divide (the __f*_rn intrinsics, which are never fused into FMA),
// round-to-nearest-even to integer, and exact scaling by powers of two.
//
//   exp:  n = rint(x * log2e);  r = (x - n*ln2_hi) - n*ln2_lo  (ln2_hi has 16
//         significant bits so n*ln2_hi is exact);  p = Taylor series of e^r to r^7
//         in Horner form (p = p*r + 1/k!);  result = p * 2^n.  x > 88 -> +inf,
//         x < -86 -> 0.
//   log:  x = m 2^e with m in [sqrt(1/2), sqrt(2));  f = (m-1)/(m+1);
//         log m = 2 (f + f^3 p(f^2)), p = odd-reciprocal series 1/3 .. 1/15 in
//         Horner form;  result = e*ln2_hi + (log m + e*ln2_lo).
//   pool: y_t = x_t * (1/tau); m = max y_t; s = sum_t exp(y_t - m) in ascending t;
//         r = tau * (m + log(s / n)).
//   gate: dot = sum_c rq[c]*rk[c] in ascending c (product and sum rounded
//         separately); z = dot*c_d + b with c_d = 1/sqrt(d) rounded once from
//         double;  g = 1 / (1 + exp(-z)).
// All constants are derived from ln 2, 1/k! and 1/(2k+1), rounded once to binary32.
#pragma once

#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

namespace hla {
namespace route {

constexpr double kLn2 = 0.69314718055994530942;

struct Consts {
  float ln2_hi, ln2_lo, log2e, sqrt_half;
};

__device__ __forceinline__ Consts make_consts() {
  Consts k;
  const float ln2f = (float)kLn2;
  k.ln2_hi = __uint_as_float(__float_as_uint(ln2f) & 0xFFFFFF00u);
  k.ln2_lo = (float)(kLn2 - (double)k.ln2_hi);
  k.log2e = (float)(1.0 / kLn2);
  k.sqrt_half = (float)sqrt(0.5);
  return k;
}

__device__ __forceinline__ float rexp(float x, const Consts& k) {
  if (x > 88.0f) return CUDART_INF_F;
  if (x < -86.0f) return 0.0f;
  const float n = rintf(__fmul_rn(x, k.log2e));
  const float r = __fsub_rn(__fsub_rn(x, __fmul_rn(n, k.ln2_hi)), __fmul_rn(n, k.ln2_lo));
  float p = (float)(1.0 / 5040.0);
  p = __fadd_rn(__fmul_rn(p, r), (float)(1.0 / 720.0));
  p = __fadd_rn(__fmul_rn(p, r), (float)(1.0 / 120.0));
  p = __fadd_rn(__fmul_rn(p, r), (float)(1.0 / 24.0));
  p = __fadd_rn(__fmul_rn(p, r), (float)(1.0 / 6.0));
  p = __fadd_rn(__fmul_rn(p, r), (float)(1.0 / 2.0));
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  const int ni = (int)n;
  const float scale = __int_as_float((ni + 127) << 23);
  return __fmul_rn(p, scale);
}

// Natural log of a positive normal binary32 value.
__device__ __forceinline__ float rlog(float x, const Consts& k) {
  const unsigned int bits = __float_as_uint(x);
  int e = (int)((bits >> 23) & 0xFFu) - 126;
  float m = __uint_as_float((bits & 0x807FFFFFu) | (126u << 23));  // [0.5, 1)
  if (m < k.sqrt_half) {
    m = __fmul_rn(m, 2.0f);
    e -= 1;
  }
  const float f = __fdiv_rn(__fsub_rn(m, 1.0f), __fadd_rn(m, 1.0f));
  const float f2 = __fmul_rn(f, f);
  float p = (float)(1.0 / 15.0);
  p = __fadd_rn(__fmul_rn(p, f2), (float)(1.0 / 13.0));
  p = __fadd_rn(__fmul_rn(p, f2), (float)(1.0 / 11.0));
  p = __fadd_rn(__fmul_rn(p, f2), (float)(1.0 / 9.0));
  p = __fadd_rn(__fmul_rn(p, f2), (float)(1.0 / 7.0));
  p = __fadd_rn(__fmul_rn(p, f2), (float)(1.0 / 5.0));
  p = __fadd_rn(__fmul_rn(p, f2), (float)(1.0 / 3.0));
  const float t = __fmul_rn(__fmul_rn(f, f2), p);
  const float log_m = __fmul_rn(__fadd_rn(f, t), 2.0f);
  const float ef = (float)e;
  return __fadd_rn(__fmul_rn(ef, k.ln2_hi), __fadd_rn(log_m, __fmul_rn(ef, k.ln2_lo)));
}

// Sigmoid of the scaled score, from a finished dot product.
__device__ __forceinline__ float gate_from_dot(float dot, float c_d, float bias, const Consts& k) {
  const float z = __fadd_rn(__fmul_rn(dot, c_d), bias);
  return __fdiv_rn(1.0f, __fadd_rn(1.0f, rexp(-z, k)));
}

}  // namespace route
}  // namespace hla
