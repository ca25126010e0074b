// Device side of the binary32 routing recipe: log-mean-exp pools and sigmoid gates.
//
// HLA summary page ("Overview": log-mean-exp pooled routing gates; "Methodology in
// Plain English": a sigmoid weight per historical chunk, thresholded without
// renormalisation).  Gates decide which chunks are skipped, so this file fixes the
// exact sequence of binary32 operations: only correctly rounded add, subtract,
// multiply, divide, fused multiply-add (fma: a*b + c rounded once) and exact
// scaling by powers of two.  Products and sums written as separate operations use
// the __f*_rn intrinsics, which are never fused.
//
//   exp:  n = rint(x * log2e) of the exact product, as fma(x, log2e, 1.5 * 2^23)
//         - 1.5 * 2^23;  r = fma(-n, ln2_lo, fma(-n, ln2_hi, x));
//         p = Taylor series of e^r to r^7 in Horner form, p = fma(p, r, 1/k!);
//         result = p * 2^n.  x > 88 -> +inf, x < -86 -> 0.
//   log:  x = m 2^e with m in [sqrt(1/2), sqrt(2));  f = (m-1)/(m+1);
//         log m = 2 (f + f^3 p(f^2)), p = odd-reciprocal series 1/3 .. 1/15 in
//         Horner form with separate products and sums;
//         result = e*ln2_hi + (log m + e*ln2_lo).
//   pool: inv = 1/tau; m = max_t (x_t * inv); s = sum_t exp(fma(x_t, inv, -m)) in
//         ascending t;  r = tau * (m + log(s / n)).
//   gate: dot = fma(rq[c], rk[c], dot) over ascending c from 0;
//         z = fma(dot, c_d, b) with c_d = 1/sqrt(d) rounded once from double;
//         g = 1 / (1 + exp(-z)).
//   windowed gate (W window representatives per key chunk): t_u = dot_u * c_d;
//         m = max_u t_u; s = sum_u exp(t_u - m) ascending; z = (m + log s) + b;
//         g = 1 / (1 + exp(-z)).
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

// Round to nearest even of a product, |x * log2e| < 2^22: adding 1.5 * 2^23 inside
// one fma puts the sum in [2^23, 2^24), where the spacing is 1, so the rounded sum is
// 1.5 * 2^23 + rint(x * log2e) (ties go to the even integer, as 1.5 * 2^23 is even)
// and the subtraction is exact.  The integer n sits in the low bits of the sum:
// bits(sum) = 0x4B400000 + n.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr unsigned int kRoundMagicBits = 0x4B400000u;
constexpr unsigned int kScaleOffset = (127u - kRoundMagicBits) << 23;  // 2^n = bits(sum) << 23 + this

// e^x for -86 <= x <= 88 (no range checks).
__device__ __forceinline__ float rexp_core(float x, const Consts& k) {
  const float sum = __fmaf_rn(x, k.log2e, kRoundMagic);
  const float n = __fsub_rn(sum, kRoundMagic);
  const float r = __fmaf_rn(-n, k.ln2_lo, __fmaf_rn(-n, k.ln2_hi, x));
  float p = (float)(1.0 / 5040.0);
  p = __fmaf_rn(p, r, (float)(1.0 / 720.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 120.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 24.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 6.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 2.0));
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const float scale = __uint_as_float((__float_as_uint(sum) << 23) + kScaleOffset);
  return __fmul_rn(p, scale);
}

__device__ __forceinline__ float rexp(float x, const Consts& k) {
  if (x > 88.0f) return CUDART_INF_F;
  if (x < -86.0f) return 0.0f;
  return rexp_core(x, k);
}

// e^x for x <= 0 (the pool's shifted values).
__device__ __forceinline__ float rexp_nonpos(float x, const Consts& k) {
  const float e = rexp_core(fmaxf(x, -86.0f), k);
  return x < -86.0f ? 0.0f : e;
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

// The pool's shifted value fma(x, 1/tau, -m).
__device__ __forceinline__ float pool_shift(float x, float inv_tau, float m) { return __fmaf_rn(x, inv_tau, -m); }

// One step of the gate's dot product.
__device__ __forceinline__ float dot_step(float acc, float a, float b) { return __fmaf_rn(a, b, acc); }

// Sigmoid of the scaled score, from a finished dot product.
__device__ __forceinline__ float gate_from_dot(float dot, float c_d, float bias, const Consts& k) {
  const float z = __fmaf_rn(dot, c_d, bias);
  return __frcp_rn(__fadd_rn(1.0f, rexp(-z, k)));  // 1/x correctly rounded, as 1.0f / x
}

// Window scores of one key chunk: t_u = dot_u * c_d for u < W, where each dot_u is
// the gate's fma chain over ascending channels from 0.  The W chains are independent
// and advance together (four channels per step, 16-byte loads).  rq and rkj (W rows
// of d floats) are 16-byte aligned, d a multiple of 4.  Returns m = max_u t_u.
template <int kMax>
__device__ __forceinline__ float window_scores(const float* rq, const float* rkj, int W, int d, float c_d,
                                               float (&t)[kMax]) {
  float acc[kMax];
#pragma unroll
  for (int u = 0; u < kMax; ++u) acc[u] = 0.0f;
  for (int c = 0; c < d; c += 4) {
    const float4 q4 = *(const float4*)(rq + c);
#pragma unroll
    for (int u = 0; u < kMax; ++u)
      if (u < W) {
        const float4 r4 = *(const float4*)(rkj + (long)u * d + c);
        acc[u] = dot_step(acc[u], q4.x, r4.x);
        acc[u] = dot_step(acc[u], q4.y, r4.y);
        acc[u] = dot_step(acc[u], q4.z, r4.z);
        acc[u] = dot_step(acc[u], q4.w, r4.w);
      }
  }
  float m = -CUDART_INF_F;
#pragma unroll
  for (int u = 0; u < kMax; ++u) {
    t[u] = 0.0f;
    if (u < W) {
      t[u] = __fmul_rn(acc[u], c_d);
      m = fmaxf(m, t[u]);
    }
  }
  return m;
}

// Sigmoid of a log-sum-exp over a chunk's W window scores t_u = dot_u * c_d (each
// rounded once), m = max_u t_u:  s = sum_u exp(t_u - m) in ascending u from 0;
// z = (m + log s) + b;  g = 1 / (1 + exp(-z)).
template <int kMax>
__device__ __forceinline__ float gate_from_window_scores(const float (&t)[kMax], int W, float m, float bias,
                                                        const Consts& k) {
  float s = 0.0f;
#pragma unroll
  for (int u = 0; u < kMax; ++u)
    if (u < W) s = __fadd_rn(s, rexp_nonpos(__fsub_rn(t[u], m), k));
  const float z = __fadd_rn(__fadd_rn(m, rlog(s, k)), bias);
  return __frcp_rn(__fadd_rn(1.0f, rexp(-z, k)));
}

}  // namespace route
}  // namespace hla
