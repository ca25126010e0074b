// Gated composition on CUDA cores (float32), one CTA per query chunk (b, h, i).
//
// HLA summary page, "Methodology in Plain English" para. 3: a chunk's weight g
// interpolates its full transition with the identity, so for query chunk i
//   S <- 0;  for j in active(i), ascending:  S <- S + g_ij ((S A_j + B_j) - S)
// and para. 4: a chunk whose weight fell below the threshold is the identity and is
// not read at all (it is absent from the active list).  The result S_in(i) is
// written as float32 [d_v][d_k] for the read-out, into the slot of chunk i's first
// 64-token sub-chunk.
#include "common.cuh"
#include "kernels.cuh"

namespace hla {

template <int D, typename Tab>
__global__ void __launch_bounds__(256) compose_simt_kernel(ComposeArgs a) {
  constexpr int R = D / 16;  // each thread owns an R x R block of S
  constexpr int DP = D + 1;
  extern __shared__ float S[];  // [D][DP]
  const int i = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const long bh = (long)b * a.H + h;
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  for (int idx = tid; idx < D * DP; idx += blockDim.x) S[idx] = 0.0f;
  const long row = (bh * a.N + i);
  const int cnt = a.act_cnt[row];
  const int32_t* idx_list = a.act_idx + row * a.N;
  const float* g_list = a.act_g + row * a.N;
  __syncthreads();
  for (int p = 0; p < cnt; ++p) {
    const int j = idx_list[p];
    const float g = g_list[p];
    const Tab* A = (const Tab*)a.A + (bh * a.ab_chunk_stride + j) * (long)D * D;
    const Tab* Bm = (const Tab*)a.Bm + (bh * a.ab_chunk_stride + j) * (long)D * D;
    float acc[R][R];
#pragma unroll
    for (int u = 0; u < R; ++u)
#pragma unroll
      for (int w = 0; w < R; ++w) acc[u][w] = 0.0f;
    for (int r = 0; r < D; ++r) {
      float sv[R], av[R];
#pragma unroll
      for (int u = 0; u < R; ++u) sv[u] = S[(ty * R + u) * DP + r];
#pragma unroll
      for (int w = 0; w < R; ++w) av[w] = ldf(A + (long)r * D + tx * R + w);
#pragma unroll
      for (int u = 0; u < R; ++u)
#pragma unroll
        for (int w = 0; w < R; ++w) acc[u][w] = fmaf(sv[u], av[w], acc[u][w]);
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < R; ++u) {
      const int v = ty * R + u;
#pragma unroll
      for (int w = 0; w < R; ++w) {
        const int cc = tx * R + w;
        const float s_old = S[v * DP + cc];
        const float bval = ldf(Bm + (long)v * D + cc);
        S[v * DP + cc] = s_old + g * ((acc[u][w] + bval) - s_old);
      }
    }
    __syncthreads();
  }
  float* out = a.S_in + (bh * a.n_slots + (long)i * a.slot_mult) * (long)D * D;
  for (int idx = tid; idx < D * D; idx += blockDim.x) {
    const int v = idx / D, cc = idx - v * D;
    out[idx] = S[v * DP + cc];
  }
}

template <int D, typename Tab>
static cudaError_t launch_c(const ComposeArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)D * (D + 1) * sizeof(float);
  auto k = compose_simt_kernel<D, Tab>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.N, a.H, a.B);
  k<<<grid, 256, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_compose(const ComposeArgs& a, cudaStream_t s) {
  if (a.N <= 0) return cudaSuccess;
  if (a.d == 128)
    return a.dtype == HLA_BF16 ? launch_c<128, __nv_bfloat16>(a, s) : launch_c<128, float>(a, s);
  return a.dtype == HLA_BF16 ? launch_c<64, __nv_bfloat16>(a, s) : launch_c<64, float>(a, s);
}

}  // namespace hla
