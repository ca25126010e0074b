// Thread layout shared by the token-rule kernels (transitions_token, readout_token).
//
// Under the token rule every row of the d x d state evolves on its own, and all rows
// read the same key, decay and query values at each token.  A CTA of 2 d threads
// splits the rows into d/4 groups of four rows, p, p + d/4, p + d/2, p + 3d/4, each
// handled by 8 threads; thread g of a group keeps the four rows on the d/8 columns
// 32 m + 4 g + u (u < 4) in registers, as two packed pairs (rows 0,1 and rows 2,3).
// Every 16-byte shared-memory read then feeds four rows; the 8 threads of a group
// read 8 adjacent 16-byte words (all 32 banks, no conflict).  Shared-memory data
// return (128 bytes per clock) is what bounds these kernels, so rows per loaded value
// is the figure that matters.
//
// Dot products over the row: each thread has partial sums for the four rows.  A
// reduce-scatter over the 8 threads (4 shuffles) leaves in thread g the total of row
// R(g) = 2 ((g >> 2) & 1) + ((g >> 1) & 1); an all-gather (3 shuffles) then hands every
// thread the four per-row scalars it needs for the update.
#pragma once

#include <cuda_runtime.h>

namespace hla {
namespace token_rows {

constexpr unsigned kFull = 0xFFFFFFFFu;

// The row (0..3 within the group) whose total thread g holds after rs_sum4.
__device__ __forceinline__ int owned_row(int g) { return 2 * ((g >> 2) & 1) + ((g >> 1) & 1); }

// Sum over the 8 threads of a group of the partials (p01 = rows 0,1; p23 = rows 2,3);
// returns the total of row owned_row(g).  Threads g and g ^ 1 get the same value.
__device__ __forceinline__ float rs_sum4(float2 p01, float2 p23, int g) {
  const bool hi = (g >> 2) & 1;
  const float k0 = hi ? p23.x : p01.x, k1 = hi ? p23.y : p01.y;
  const float s0 = hi ? p01.x : p23.x, s1 = hi ? p01.y : p23.y;
  const float q0 = k0 + __shfl_xor_sync(kFull, s0, 4);
  const float q1 = k1 + __shfl_xor_sync(kFull, s1, 4);
  const bool mid = (g >> 1) & 1;
  float s = (mid ? q1 : q0) + __shfl_xor_sync(kFull, mid ? q0 : q1, 2);
  s += __shfl_xor_sync(kFull, s, 1);
  return s;
}

// f holds the scalar of row owned_row(g); returns the scalars of rows 0..3.
__device__ __forceinline__ void ag_rows4(float f, int g, float2& f01, float2& f23) {
  const bool hi = (g >> 2) & 1, mid = (g >> 1) & 1;
  const float o = __shfl_xor_sync(kFull, f, 2);
  const float a0 = mid ? o : f, a1 = mid ? f : o;  // rows 2 hi, 2 hi + 1
  const float b0 = __shfl_xor_sync(kFull, a0, 4), b1 = __shfl_xor_sync(kFull, a1, 4);
  f01 = hi ? make_float2(b0, b1) : make_float2(a0, a1);
  f23 = hi ? make_float2(a0, a1) : make_float2(b0, b1);
}

__device__ __forceinline__ float2 dup(float v) { return make_float2(v, v); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }

}  // namespace token_rows
}  // namespace hla
