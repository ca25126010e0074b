// Routing diagnostics: mass and effective support of the gates per query chunk.
//
// HLA summary page, "Key Contributions" 3 and "Methodology in Plain English" para. 4:
// a budget penalty on the total routing mass and a support penalty on the effective
// number of accessed chunks, an order-2 effective number (inverse sum of squares),
// push routing toward few chunks so that low-weight chunks can be skipped.  Here
// they are measured, not trained: over the chunks j < i kept by the threshold,
//   mass_i = sum_j g_ij,   support_i = mass_i^2 / sum_j g_ij^2   (0 if none kept).
// One warp per query chunk reads its row of the gate matrix (coalesced), sums in
// float32 per lane and combines the lanes by a butterfly.
#include "common.cuh"
#include "kernels.cuh"

namespace hla {

namespace {

__global__ void __launch_bounds__(256) gate_support_kernel(const float* __restrict__ gates, int rows, int N,
                                                           float thr, float* __restrict__ mass_out,
                                                           float* __restrict__ support_out) {
  const long w = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= rows) return;
  const int i = (int)(w % N);
  const float* g = gates + w * N;
  float m = 0.0f, q = 0.0f;
  for (int j = lane; j < i; j += 32) {
    const float x = g[j];
    if (thr <= 0.0f || x >= thr) {
      m += x;
      q = fmaf(x, x, q);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    m += __shfl_xor_sync(0xFFFFFFFFu, m, o);
    q += __shfl_xor_sync(0xFFFFFFFFu, q, o);
  }
  if (lane == 0) {
    if (mass_out) mass_out[w] = m;
    if (support_out) support_out[w] = q > 0.0f ? __fdiv_rn(m * m, q) : 0.0f;
  }
}

}  // namespace

cudaError_t launch_gate_support(const float* gates, int B, int H, int N, float thr, float* mass_out,
                                float* support_out, cudaStream_t s) {
  const long rows = (long)B * H * N;
  if (rows <= 0) return cudaSuccess;
  const long blocks = (rows * 32 + 255) / 256;
  gate_support_kernel<<<(unsigned)blocks, 256, 0, s>>>(gates, (int)rows, N, thr, mass_out, support_out);
  return cudaGetLastError();
}

}  // namespace hla
